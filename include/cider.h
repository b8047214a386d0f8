/*
 * cider.h -- C ABI of the B200 (sm_100a) W8A8 / W4A8 activation-quantized linear.
 *
 * The operation (sources: juejin post "在Mac上跑大模型，MLX 不是终点", sections
 * "W8A8 对称量化：Cider 的选择", "INT8 TensorOps 内核设计", "三种量化粒度的实现";
 * Cider README (WeHub translation), tables "模式" and "量化", sections
 * "Metal Kernel 流水线" and "底层 API"):
 *
 *   per token m:   scale_x[m] = max_k |x[m,k]| / 127                 (fp32)
 *                  q[m,k]     = clamp(round(x[m,k] / scale_x[m]), -128, 127)
 *   per-channel:   y[m,n] = (sum_k q[m,k] * w[n,k]) * scale_x[m] * scale_w[n]
 *   per-group:     y[m,n] = scale_x[m] * sum_g (sum_{k in g} q[m,k] * w[n,k]) * scale_w[g][n]
 *   W4A8:          w[n,k] = nibble(n,k) - 8, nibbles packed two per byte
 *
 * round() is round-half-away-from-zero; x / scale_x is one correctly rounded
 * fp32 division; an all-zero token has scale 0 and q = 0.  Products are
 * summed exactly in INT32.  The output is fp16 or bf16, round to nearest even.
 *
 * Conventions shared by every entry point below:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or synchronises on these calls.  Each call is
 *    enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream)
 *    and returns as soon as its kernels are launched.
 *  - Layouts are dense row-major: x [M][K], w [N][K] (nn.Linear convention:
 *    output channel n, input channel k), y [M][N], q [M][K]; only
 *    cider_quantize_act takes row strides.  A strided input goes through
 *    cider_quantize_act into a dense q and then a *_gemm_*_q entry point.  Per-group weight
 *    scales are GROUP-MAJOR, scale_w[K/gs][N], so that one group's scales for
 *    consecutive output channels are contiguous.  Packed INT4 weights are
 *    [N][K/2] bytes; byte j of row n holds k = 2j in its low nibble and
 *    k = 2j+1 in its high nibble, each as the offset-binary value q + 8.
 *  - Argument checks happen before any launch.  A call that fails them
 *    returns CIDER_ERR_INVALID_ARG and launches nothing; cider_last_error()
 *    then names the failed check.  Requirements: M >= 0 (M == 0 is a no-op),
 *    N, K >= 1; K % 16 == 0; N % 8 == 0; K <= 131072; tensor pointers and
 *    scale_w 16-byte aligned and non-NULL (scale_x 4-byte aligned); per-group
 *    gs is 64 or 128 and divides K; W4A8 also needs K % 32 == 0; y must not
 *    overlap any input or the workspace (checked by address range).
 *  - On a device that is not compute capability 10.x the calls return
 *    CIDER_ERR_UNSUPPORTED; there is no CPU fallback.
 *  - Launch failures return CIDER_ERR_CUDA.  Faults that happen later on the
 *    device surface at the caller's next synchronisation, as usual in CUDA.
 *  - Every wait inside the kernels is bounded in time.  A wait that runs out
 *    records CIDER_ERR_TIMEOUT in a device status word, which
 *    cider_device_status() reads back.
 */
#ifndef CIDER_H
#define CIDER_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CIDER_API __attribute__((visibility("default")))
#else
#define CIDER_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CIDER_OK = 0,
    CIDER_ERR_INVALID_ARG = 1, /* an argument check failed; nothing was launched */
    CIDER_ERR_UNSUPPORTED = 2, /* the current device is not sm_100-family */
    CIDER_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed */
    CIDER_ERR_TIMEOUT = 4      /* a bounded device-side wait ran out */
} cider_status_t;

typedef enum {
    CIDER_F16 = 0,  /* IEEE binary16 */
    CIDER_BF16 = 1  /* bfloat16 */
} cider_dtype_t;

/* ---- availability and diagnostics ------------------------------------- */

/* 1 iff the calling thread's current CUDA device is compute capability 10.x
 * (the hardware this library is built for), else 0.  Mirrors the pages'
 * is_available() (Cider README, section "条件编译（M4 / M5）"). */
CIDER_API int cider_is_available(void);

/* Static, NUL-terminated description of a status code. */
CIDER_API const char* cider_status_string(cider_status_t status);

/* Message of the last failing call on this host thread ("" if none).  The
 * string stays valid until the next call on the same thread. */
CIDER_API const char* cider_last_error(void);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device: CIDER_OK, or CIDER_ERR_TIMEOUT if a bounded wait in some
 * kernel ran out since the last read.  Not for the hot path. */
CIDER_API cider_status_t cider_device_status(void* stream);

/* Bytes of workspace the linear entry points need for M tokens of K inputs:
 * the quantized activations q [M][K] int8 and scale_x [M] fp32, each start
 * 256-byte aligned.  0 when M is small enough for the fused small-M kernel
 * (M <= cider_get_small_m_threshold()), which keeps q in shared memory. */
CIDER_API size_t cider_workspace_bytes(int64_t M, int64_t K);

/* Workspace that lets a linear of shape M x N x K take its fastest path on
 * the current device: cider_workspace_bytes(M, K), plus, for the per-group
 * linears when their 128 x 128 output tiles would leave at least half of the
 * SMs idle, room for split-K partial sums (fp32 [splits][M][N], 256-byte
 * aligned, after scale_x).  A per-group linear given less than this (but at
 * least cider_workspace_bytes(M, K)) runs without splitting K. */
CIDER_API size_t cider_workspace_bytes_mnk(int64_t M, int64_t N, int64_t K);

/* Workspace of cider_w4a8_linear_pc, which runs on the tensor cores at every
 * M: q [M][K] int8 and scale_x [M] fp32 (256-byte aligned) for any M >= 1,
 * plus room for its split-K partial sums as in cider_workspace_bytes_mnk.
 * Given only the first part, it runs without splitting K. */
CIDER_API size_t cider_workspace_bytes_w4a8_pc(int64_t M, int64_t N, int64_t K);

/* Calls with 1 <= M <= threshold use the fused small-M (decode-shaped) kernel;
 * larger M use quantize + the tcgen05 GEMM.  The threshold is process-wide;
 * 0 sends every call to the GEMM path.  Values above 16 are rejected.  The
 * pages pick a dedicated matrix-vector kernel for single-token decode (juejin
 * post, section "INT8 TensorOps 内核设计", "双路径自动切换"). */
CIDER_API cider_status_t cider_set_small_m_threshold(int64_t threshold);
CIDER_API int64_t cider_get_small_m_threshold(void);

/* ---- the four operations of the pages' interface ----------------------- */

/* Online per-token activation quantization (Cider README, section
 * "Metal Kernel 流水线", step quantize_per_token; juejin post, section
 * "W8A8 对称量化：Cider 的选择").
 * x: M rows of K fp16/bf16 values (xdt), row m at x + m * ldx elements;
 * q: M rows of K int8 codes out, row m at q + m * ldq bytes; scale_x: [M]
 * fp32 out.  The row strides let a caller quantize a strided view, such as
 * a slice of a fused buffer: ldx >= K, a multiple of 8 (16-byte rows);
 * ldq >= K, a multiple of 16.  The bytes between K and the stride are neither
 * read (x) nor written (q).  x, q and scale_x must not overlap. */
CIDER_API cider_status_t cider_quantize_act(const void* x, cider_dtype_t xdt, int64_t M, int64_t K, int64_t ldx,
                                  int8_t* q, int64_t ldq, float* scale_x, void* stream);

/* W8A8 linear, per-output-channel weight scales (Cider README, section
 * "底层 API" perchannel_linear; table "W8A8 量化粒度", Per-channel).
 * w: [N][K] int8; scale_w: [N] fp32; y: [M][N] (ydt).
 * workspace: device buffer of at least cider_workspace_bytes(M, K) bytes
 * (NULL allowed when that is 0); its contents on return are unspecified. */
CIDER_API cider_status_t cider_w8a8_linear_pc(const void* x, cider_dtype_t xdt, int64_t M, int64_t K,
                                    const int8_t* w, const float* scale_w, int64_t N,
                                    void* y, cider_dtype_t ydt,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* W8A16 decode matrix-vector product, per-output-channel weight scales: the
 * pages' decode kernel (Cider README, section "Metal Kernel 流水线", Decode:
 * a direct INT8 matrix-vector product, weights dequantized on the fly, no
 * activation quantization).  y[m,n] = round_ydt(scale_w[n] * sum_k x[m,k] *
 * w[n,k]), x widened to fp32 and the products summed in fp32; the activations
 * are NOT quantized, unlike cider_w8a8_linear_pc, whose small-M path keeps the
 * W8A8 semantics.  x: [M][K] (xdt), 1 <= M <= 4 and M * ceil(K / 512) * 2048
 * <= 160 KiB (the rows are staged in shared memory as fp32), K <= 32768; w: [N][K] int8;
 * scale_w: [N] fp32; y: [M][N] (ydt).  No workspace. */
CIDER_API cider_status_t cider_w8a16_mv_pc(const void* x, cider_dtype_t xdt, int64_t M, int64_t K,
                                 const int8_t* w, const float* scale_w, int64_t N,
                                 void* y, cider_dtype_t ydt, void* stream);

/* W8A16 decode matrix-vector product, per-group weight scales along K (gs =
 * 64 or 128): the pages' per-group INT8 MV decode kernel (Cider README,
 * section "Metal Kernel 流水线", Decode, and the per-group MV kernel of its
 * kernel list).  y[m,n] = round_ydt(sum_g scale_w[g][n] * sum_{k in g}
 * x[m,k] * w[n,k]) with x widened to fp32, each chunk of 16 products summed
 * in fp32, scaled by its group's scale and accumulated in fp32; the
 * activations are NOT quantized.  x: [M][K] (xdt), 1 <= M <= 4 and
 * M * ceil(K / 512) * 2048 <= 160 KiB (the rows are staged in shared memory
 * as fp32), K <= 32768; w: [N][K] int8; scale_w: [K/gs][N] fp32 (group-major,
 * as for the per-group linears); y: [M][N] (ydt).  No workspace.  Besides the
 * common checks, CIDER_ERR_INVALID_ARG when gs is not 64 or 128 or does not
 * divide K. */
CIDER_API cider_status_t cider_w8a16_mv_pg(const void* x, cider_dtype_t xdt, int64_t M, int64_t K,
                                 const int8_t* w, const float* scale_w, int64_t N, int64_t gs,
                                 void* y, cider_dtype_t ydt, void* stream);

/* W8A8 linear, per-group weight scales along K (gs = 64 or 128; Cider README,
 * table "W8A8 量化粒度"; juejin post, section "三种量化粒度的实现").
 * scale_w: [K/gs][N] fp32 (group-major).  The INT32 partial sum of each group
 * is rescaled by its scale in fp32 and the rescaled partials are summed.
 * With a workspace of cider_workspace_bytes_mnk(M, N, K) bytes, small tile
 * counts split K into pieces whose fp32 sums are added by a second kernel. */
CIDER_API cider_status_t cider_w8a8_linear_pg(const void* x, cider_dtype_t xdt, int64_t M, int64_t K,
                                    const int8_t* w, const float* scale_w, int64_t N, int64_t gs,
                                    void* y, cider_dtype_t ydt,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* W4A8 linear, per-group scales (Cider README, table "模式" W4A8, section
 * "Metal Kernel 流水线" (INT4 -> INT8 unpack in the load path), section
 * "底层 API" w4a8_linear).  w_packed: [N][K/2] bytes as described above;
 * scale_w: [K/gs][N] fp32. */
CIDER_API cider_status_t cider_w4a8_linear_pg(const void* x, cider_dtype_t xdt, int64_t M, int64_t K,
                                    const uint8_t* w_packed, const float* scale_w, int64_t N,
                                    int64_t gs, void* y, cider_dtype_t ydt,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* W4A8 linear, one scale per output channel (Cider README, table "量化",
 * W4A8 weights symmetric INT4, zero point 8, "per-column"; table "模式" and
 * section "Metal Kernel 流水线" for the on-chip INT4 -> INT8 unpack).
 * y[m,n] = round(acc[m,n] * scale_x[m] * scale_w[n]) with acc the INT32 sum
 * over all of K of the activation codes times the unpacked weights (nibble
 * - 8).  w_packed: [N][K/2] bytes as described above (from
 * cider_pack_weight_int4_pc); scale_w: [N] fp32.  Requires K % 32 == 0.
 * Every M runs on the tensor cores (there is no separate decode kernel for
 * this form), so the workspace is cider_workspace_bytes_w4a8_pc(M, N, K)
 * (at least its q and scale_x part, even for small M).  Errors as
 * cider_w4a8_linear_pg. */
CIDER_API cider_status_t cider_w4a8_linear_pc(const void* x, cider_dtype_t xdt, int64_t M, int64_t K,
                                    const uint8_t* w_packed, const float* scale_w, int64_t N,
                                    void* y, cider_dtype_t ydt,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* W8A8 per-channel linear for callers that cannot allocate device memory.
 * The pages have no counterpart: this is an addition of this library.
 *
 * Some callers cannot call cudaMalloc and so cannot pass a workspace: a host
 * application or framework that owns all of the GPU's memory through its own
 * pool and forbids outside allocations, or code that must stay inside a
 * memory budget fixed at start-up.  This entry point computes exactly what
 * cider_w8a8_linear_pc computes, but keeps the quantized activations and
 * their scales -- and, for shapes whose last round of output tiles is cut
 * along K, the fp32 partial sums of those tiles when they fit after them --
 * in a scratch array built into the library: 32 MiB of device memory, which
 * every GPU that loads the library holds until the process exits.  It
 * allocates nothing and calls no allocating routine.
 *  - Limit: cider_workspace_bytes(M, K) must not exceed 32 MiB (roughly
 *    M * K + 4 * M <= 32 MiB); larger calls return CIDER_ERR_INVALID_ARG with
 *    a message and launch nothing.  Calls that take the fused small-M kernel
 *    do not touch the scratch.
 *  - The first call on each device looks up the scratch's device address,
 *    with that device current; make that first call before any stream
 *    capture.  The address is kept for the life of the process: after a
 *    cudaDeviceReset() the array is reloaded elsewhere, so a process that
 *    resets a device must not call this entry point again on it.
 *  - All calls on a device share the one scratch array and it keeps the last
 *    call's contents.  Calls whose kernels overlap on the GPU (on different
 *    streams, or from different host threads) race on it and give wrong
 *    results; serialise them, e.g. on one stream.
 * Arguments, layouts and errors are as for cider_w8a8_linear_pc. */
CIDER_API cider_status_t cider_w8a8_linear_pc_noalloc(const void* x, cider_dtype_t xdt, int64_t M, int64_t K,
                                                      const int8_t* w, const float* scale_w, int64_t N,
                                                      void* y, cider_dtype_t ydt, void* stream);

/* ---- the GEMM stage on pre-quantized activations ------------------------ */
/* The same products and epilogues as the linears above, fed q [M][K] int8 and
 * scale_x [M] fp32 from cider_quantize_act or a fused producer.  Always the
 * tcgen05 tensor-core path. */
CIDER_API cider_status_t cider_w8a8_gemm_pc_q(const int8_t* q, const float* scale_x, int64_t M, int64_t K,
                                    const int8_t* w, const float* scale_w, int64_t N,
                                    void* y, cider_dtype_t ydt, void* stream);
CIDER_API cider_status_t cider_w8a8_gemm_pg_q(const int8_t* q, const float* scale_x, int64_t M, int64_t K,
                                    const int8_t* w, const float* scale_w, int64_t N, int64_t gs,
                                    void* y, cider_dtype_t ydt, void* stream);
CIDER_API cider_status_t cider_w4a8_gemm_pg_q(const int8_t* q, const float* scale_x, int64_t M, int64_t K,
                                    const uint8_t* w_packed, const float* scale_w, int64_t N,
                                    int64_t gs, void* y, cider_dtype_t ydt, void* stream);
CIDER_API cider_status_t cider_w4a8_gemm_pc_q(const int8_t* q, const float* scale_x, int64_t M, int64_t K,
                                    const uint8_t* w_packed, const float* scale_w, int64_t N,
                                    void* y, cider_dtype_t ydt, void* stream);

/* ---- decoder-MLP producer ------------------------------------------------ */
/* a = round_dt(silu(gate) * up) evaluated in fp32, then per-token quantized as
 * cider_quantize_act does, in one pass: the input of a down projection that
 * follows SiLU(gate) * up.  gate, up: [M][F] (dt); q: [M][F] int8 out;
 * scale_x: [M] fp32 out; a_out: optional [M][F] (dt) copy of a (NULL = skip).
 * Requires F % 16 == 0. */
CIDER_API cider_status_t cider_silu_mul_quantize(const void* gate, const void* up, cider_dtype_t dt,
                                       int64_t M, int64_t F, int8_t* q, float* scale_x,
                                       void* a_out, void* stream);

/* ---- offline weight quantization (Cider README, section "底层 API":
 * quantize_weight_int8, pack_weight_int4) -------------------------------- */
/* W: [N][K] fp32.  Per channel: scale_w[n] = max_k |W[n,k]| / 127,
 * w = clamp(round(W / scale_w), -128, 127). */
CIDER_API cider_status_t cider_quantize_weight_pc(const float* W, int64_t N, int64_t K,
                                        int8_t* w, float* scale_w, void* stream);
/* Per group of gs along K: scale_w[g][n] = max |W[n, g*gs:(g+1)*gs]| / 127 (group-major). */
CIDER_API cider_status_t cider_quantize_weight_pg(const float* W, int64_t N, int64_t K, int64_t gs,
                                        int8_t* w, float* scale_w, void* stream);
/* Percentile-clipped scales (Cider README, section "说明": the conversion's
 * scales come from min-max by default or from a percentile,
 * clip_percentile = 99.9).  Per slab -- an output row (_pc) or one group of
 * gs = 64 or 128 along K (_pg) -- c = the clip_percentile-th percentile of
 * |W| over the slab, linearly interpolated at position p/100 * (len - 1) of
 * the ascending order (the position in double; its fraction rounded once to
 * float; the interpolation in fp32); c = max|W| when that percentile is 0.
 * scale_w = c / 127 and w = clamp(round(W / scale_w), -127, 127): values
 * beyond the percentile saturate symmetrically.  clip_percentile = 100
 * gives exactly the min-max result above.  Same layouts as the min-max
 * versions (scale_w [N] or group-major [K/gs][N]); W, w and scale_w are
 * device pointers owned by the caller.  Errors: CIDER_ERR_INVALID_ARG for
 * clip_percentile outside [0, 100] (or NaN), bad sizes, gs, or NULL. */
CIDER_API cider_status_t cider_quantize_weight_pc_clip(const float* W, int64_t N, int64_t K, double clip_percentile,
                                             int8_t* w, float* scale_w, void* stream);
CIDER_API cider_status_t cider_quantize_weight_pg_clip(const float* W, int64_t N, int64_t K, int64_t gs,
                                             double clip_percentile, int8_t* w, float* scale_w, void* stream);
/* INT4 per group: scale_w[g][n] = max|W_group| / 7, q = clamp(round(W/scale), -8, 7),
 * packed as described above. */
CIDER_API cider_status_t cider_pack_weight_int4_pg(const float* W, int64_t N, int64_t K, int64_t gs,
                                         uint8_t* w_packed, float* scale_w, void* stream);
/* INT4 per output channel: scale_w[n] = max_k |W[n,k]| / 7, q = clamp(round(W/scale), -8, 7),
 * packed as described above; scale_w: [N].  Requires an even K. */
CIDER_API cider_status_t cider_pack_weight_int4_pc(const float* W, int64_t N, int64_t K,
                                         uint8_t* w_packed, float* scale_w, void* stream);

/* ---- decode attention (Cider README, section "优化 SDPA（解码注意力）") --------
 * Scaled dot-product attention for one query token per head with no mask:
 * for query head h and its KV head g = h / (H_q / H_kv),
 *   out[h] = sum_j softmax_j(q[h] . K[g][j] / sqrt(D)) V[g][j].
 * q [H_q][D], K and V [H_kv][N][D] (head-major cache), out [H_q][D]; all in
 * dt (fp16 or bf16), device memory owned by the caller, 16-byte aligned.
 * D must be 128; H_kv must divide H_q; 1 <= N <= 2^30.  The sequence is cut
 * into chunks whose fp32 partial results go to the workspace
 * (cider_sdpa_decode_workspace_bytes; it depends on the device's SM count);
 * a second kernel merges them.  Errors: CIDER_ERR_INVALID_ARG for the shape
 * rules, a short workspace, misalignment or out overlapping an input. */
CIDER_API size_t cider_sdpa_decode_workspace_bytes(int64_t H_q, int64_t H_kv, int64_t N, int64_t D);
CIDER_API cider_status_t cider_sdpa_decode(const void* q, const void* k, const void* v, cider_dtype_t dt,
                                 int64_t H_q, int64_t H_kv, int64_t N, int64_t D, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* ---- test exports (stable, but not part of the operation's interface) ---- */
/* The tcgen05 GEMM with an INT32 store epilogue: acc[m][n] = sum_k q[m,k]*w[n,k]. */
CIDER_API cider_status_t cider_test_gemm_i32(const int8_t* q, const int8_t* w, int64_t M, int64_t N,
                                   int64_t K, int32_t* acc, void* stream);
/* Per-group INT32 partials acc_g[g][m][n] = sum_{k in group g} q[m,k]*w[n,k]. */
CIDER_API cider_status_t cider_test_gemm_i32_grouped(const int8_t* q, const int8_t* w, int64_t M, int64_t N,
                                           int64_t K, int64_t gs, int32_t* acc_g, void* stream);
/* Forces the kernel variant of the per-channel and INT32 GEMM for later calls
 * (process-wide): 0 = automatic (default), 1 = single-CTA 128x128 tiles,
 * 2 = single-CTA 128x256 tiles, 3 = CTA-pair 256x256 tiles, 4 = single-CTA
 * 128x80 tiles, 5 = CTA-pair 256x192 tiles.  Lets tests cover every variant
 * on small shapes.  Outside [0, 5]: CIDER_ERR_INVALID_ARG, nothing changes. */
CIDER_API cider_status_t cider_test_set_gemm_variant(int variant);
/* Selects the decode-attention kernels for later calls (process-wide):
 * 0 = automatic (default: the tensor-core kernel when 2 <= H_q / H_kv <= 16,
 * the CUDA-core kernels otherwise), 1 = the CUDA-core kernels only, 2 = the
 * tensor-core kernel wherever it applies, 3 = the same with the two offset
 * fields of the V operand's shared-memory descriptor exchanged (a layout
 * probe for tests).  The workspace size follows the selection: query
 * cider_sdpa_decode_workspace_bytes after setting it. */
CIDER_API cider_status_t cider_test_set_sdpa_kernel(int kernel);
/* Selects the decode-shaped kernel of the small-M path for later calls
 * (process-wide): 0 = automatic (default: the one-shot kernel, which requests
 * all of a CTA's weights before using any, where its plan fits -- M <= 4 and
 * at most 12 passes of 512 weights per warp -- else the register-ring
 * kernel), 1 = the register-ring kernel, 2 = the bulk-staged kernel with the
 * whole shared memory, 3 = the bulk-staged kernel within half of it, 4 = the
 * one-shot kernel where its plan fits.  Shapes a selected kernel's plan
 * cannot hold take the register-ring kernel.  The W8A16 products: 0 takes
 * the one-shot form (x unquantized in shared memory) for the per-group
 * product and the register ring for the per-channel one, 4 the one-shot form
 * for both.  Lets tests and measurements compare the kernels on the same
 * shapes. */
CIDER_API cider_status_t cider_test_set_small_m_kernel(int kernel);
/* Selects, for later calls (process-wide), how the per-channel linear
 * (cider_w8a8_linear_pc and the workspace-free form) quantizes its
 * activations on the tensor-core path: 0 = automatic (default: the separate
 * quantize kernel, which measured faster), 1 = always the separate kernel,
 * 2 = always inside the GEMM launch.  Either way
 * the call leaves the codes q [M][K] at the start of the workspace and
 * scale_x [M] at byte offset align256(M * K), which lets tests check the
 * fused quantization bit for bit.  The fused launch synchronises its grid
 * once (one CTA per SM, all resident); it needs the GPU's SMs to itself for
 * that moment, and a barrier that cannot complete within 2 s records
 * CIDER_ERR_TIMEOUT for cider_device_status(). */
CIDER_API cider_status_t cider_test_set_fused_quantize(int mode);
/* Forces the split-K piece count of the per-group GEMM for later calls
 * (process-wide): 0 = automatic (default), 1 = never split, 2 .. 16 = that
 * many K pieces per tile (fewer when K has fewer 128-wide blocks).  The INT32
 * test export honours it without a workspace (it writes per-group partials);
 * the per-group linears need cider_workspace_bytes_mnk(M, N, K) bytes, read
 * after setting it, or they do not split. */
CIDER_API cider_status_t cider_test_set_split_k(int splits);
/* Exercises the bounded-wait path of the kernels without a fault: one warp
 * waits on an mbarrier that nothing arrives on and gives up after limit_ns
 * (1 .. 1e8).  The next cider_device_status() then returns CIDER_ERR_TIMEOUT
 * and clears the status word. */
CIDER_API cider_status_t cider_test_bounded_wait(int64_t limit_ns, void* stream);
/* The decode-attention cut for a device with num_sms SMs, without a device:
 * out4 = {query heads per CTA, head tiles per KV group, keys per chunk,
 * chunks}.  Same shape rules as cider_sdpa_decode. */
CIDER_API cider_status_t cider_test_sdpa_plan(int64_t H_q, int64_t H_kv, int64_t N, int64_t num_sms, int32_t* out4);
/* The W4A8 load path's unpack: w[n][k] = nibble(n, k) - 8. */
CIDER_API cider_status_t cider_test_unpack_int4(const uint8_t* w_packed, int64_t N, int64_t K, int8_t* w,
                                      void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CIDER_H */
