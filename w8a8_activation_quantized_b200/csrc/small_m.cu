// small_m.cu -- the fused decode-shaped linear (1 <= M <= 16 tokens): one
// launch that quantizes the few activation rows into shared memory and then
// streams every weight row once from HBM, taking INT8 dot products with dp4a
// and applying the per-channel or per-group dequant.
//
// The pages route single-token decode to a dedicated matrix-vector kernel
// instead of the GEMM (juejin post "在Mac上跑大模型，MLX 不是终点", section
// "INT8 TensorOps 内核设计", "双路径自动切换"; Cider README, section
// "Metal Kernel 流水线", Decode).  This kernel keeps the W8A8 semantics of the
// GEMM path (activations quantized per token, integer products), so one
// oracle covers every M.
//
// Work split.  The grid is persistent (two CTAs per SM): all warps of a CTA
// quantize the M activation rows into shared memory, then the CTA walks
// blocks of R output channels.  Its 8 warps form R rows x S K-slices
// (R*S = 8).  A weight row is read as 16-byte chunks (16 int8 weights, or 32
// packed int4 weights); 32 lanes read 32 consecutive chunks per "pass" (512 or
// 1024 k values), and a warp's slice is a whole number of passes, so a weight
// group (64 or 128 values) never straddles warps.  Each warp keeps a ring of
// three row blocks in registers -- all loads of a slice issued at once, two
// blocks ahead of the one being used -- and its first two blocks start
// loading before the activations are quantized.  Per-group: each lane scales
// its chunk's exact INT32 dot by the chunk's group scale scale_w[g][n] and
// adds it to an fp32 sum (scale_w[g] * acc_g, summed in another order); the
// warp's final shuffle reduction adds the lanes.  With one warp per row
// (S = 1) a warp writes its outputs directly; otherwise the slices combine
// through shared memory.
#include <algorithm>
#include <atomic>
#include <type_traits>

#include "cider_device.cuh"
#include "cider_kernels.h"

namespace cider {

constexpr int kSmallThreads = 256;
constexpr int kSmallWarps = kSmallThreads / 32;
// Row blocks per warp in the register ring: one being used and the rest
// loading; two for the widest slices (8 passes) to stay within registers.
template <int PPW>
struct RingDepth {
    static constexpr int value = PPW <= 5 ? 3 : 2;
};

__device__ __forceinline__ int dp4a(uint32_t a, uint32_t b, int c) {
    return __dp4a(static_cast<int>(a), static_cast<int>(b), c);
}

// INT32 dot of one 16-byte weight chunk with the matching activation codes.
template <bool W4>
__device__ __forceinline__ int chunk_dot(const uint4& wv, const int8_t* qrow, int k0) {
    if (!W4) {
        const uint4 qv = *reinterpret_cast<const uint4*>(qrow + k0);
        int a = dp4a(wv.x, qv.x, 0);
        a = dp4a(wv.y, qv.y, a);
        a = dp4a(wv.z, qv.z, a);
        return dp4a(wv.w, qv.w, a);
    } else {
        const uint4 q0 = *reinterpret_cast<const uint4*>(qrow + k0);
        const uint4 q1 = *reinterpret_cast<const uint4*>(qrow + k0 + 16);
        const uint2 u0 = unpack_int4x8(wv.x), u1 = unpack_int4x8(wv.y);
        const uint2 u2 = unpack_int4x8(wv.z), u3 = unpack_int4x8(wv.w);
        int a = dp4a(u0.x, q0.x, 0);
        a = dp4a(u0.y, q0.y, a);
        a = dp4a(u1.x, q0.z, a);
        a = dp4a(u1.y, q0.w, a);
        a = dp4a(u2.x, q1.x, a);
        a = dp4a(u2.y, q1.y, a);
        a = dp4a(u3.x, q1.z, a);
        return dp4a(u3.y, q1.w, a);
    }
}

struct SmallGeom {
    int S, R;     // K-slices per row, rows per block (R * S = 8)
    int ppw;      // passes (32 chunks) per warp slice
    int nblocks;  // row blocks
};

template <typename TX, bool PG, bool W4, int MAXM, int PPW>
__global__ void __launch_bounds__(kSmallThreads, 2) k_small_m(const TX* __restrict__ x, int M, int K,
                                                              const uint8_t* __restrict__ w,
                                                              const float* __restrict__ sw, int N, int gs,
                                                              void* __restrict__ y, int ydt, SmallGeom geo) {
    extern __shared__ __align__(16) int8_t s_q[];  // [M][K] codes
    __shared__ float s_sx[MAXM];
    __shared__ float s_red[MAXM][kSmallWarps];
    __shared__ float s_part[kSmallWarps][MAXM];
    constexpr int KC = W4 ? 32 : 16;  // weights per 16-byte chunk
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row_bytes = W4 ? K / 2 : K;
    const int nch = K / KC;
    const int r_in_blk = warp / geo.S, slice = warp % geo.S;
    const int pass0 = slice * geo.ppw;
    pdl_wait();
    pdl_trigger();

    // Ring slot: the block's weight chunks and the scales they need (per-channel:
    // scale_w[n]; per-group: this lane's group scale for each pass), all loaded
    // ahead so no scale load sits on the critical path.
    constexpr int kRing = RingDepth<PPW>::value;
    uint4 ring[kRing][PPW];
    float ring_s[kRing][PG ? PPW : 1];
    auto load = [&](uint4 (&dst)[PPW], float (&ds)[PG ? PPW : 1], int blk) {
        const int n = blk * geo.R + r_in_blk;
        const bool row_ok = blk < geo.nblocks && n < N;
        const uint4* wr = reinterpret_cast<const uint4*>(w + static_cast<int64_t>(n) * row_bytes);
#pragma unroll
        for (int p = 0; p < PPW; ++p) {
            const int c = (pass0 + p) * 32 + lane;
            const bool ok = p < geo.ppw && row_ok && c < nch;
            dst[p] = ok ? __ldcs(wr + c) : make_uint4(0, 0, 0, 0);
            if (PG) ds[p] = ok ? __ldg(sw + static_cast<int64_t>(c * KC / gs) * N + n) : 0.0f;
        }
        if (!PG) ds[0] = row_ok ? __ldg(sw + n) : 0.0f;
    };
    // weight traffic starts before the activations are quantized
#pragma unroll
    for (int i = 0; i < kRing - 1; ++i) load(ring[i], ring_s[i], blockIdx.x + i * gridDim.x);

    // Quantize the M activation rows into shared memory, all warps on every row.
    // (Quantizing per warp in registers at M = 1 -- each lane loading the x of
    // its own chunks, no CTA barrier -- measured slower: 12.9 against 10.7 us
    // per launch under ncu, with 4x the L2 reads of x and 122 registers.)
    const int nx = K / 8;  // 16-byte chunks of a row of x
    for (int m = 0; m < M; ++m) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K);
        typename Pack2<TX>::type m2 = {};
        for (int c = threadIdx.x; c < nx; c += kSmallThreads) m2 = absmax8<TX>(__ldg(xr + c), m2);
        float amax = absmax_to_f32<TX>(m2);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) s_red[m][warp] = amax;
    }
    __syncthreads();
    for (int m = 0; m < M; ++m) {
        float amax = s_red[m][0];
#pragma unroll
        for (int i = 1; i < kSmallWarps; ++i) amax = fmaxf(amax, s_red[m][i]);
        const float s = act_scale(amax);
        const float rs = act_rcp(s);
        if (threadIdx.x == 0) s_sx[m] = s;
        const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K);
        for (int c = threadIdx.x; c < nx; c += kSmallThreads) {
            float f[8];
            unpack8_f32<TX>(__ldg(xr + c), f);
            *reinterpret_cast<uint2*>(s_q + static_cast<int64_t>(m) * K + 8 * c) = quant8_codes(f, s, rs);
        }
    }
    __syncthreads();

    auto step = [&](const uint4 (&cur)[PPW], const float (&cs)[PG ? PPW : 1], int blk) {
        const int n = blk * geo.R + r_in_blk;
        int iacc[MAXM];
        float facc[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) { iacc[m] = 0; facc[m] = 0.0f; }
        if (n < N) {
#pragma unroll
            for (int p = 0; p < PPW; ++p) {
                if (p >= geo.ppw || (pass0 + p) * 32 >= nch) break;  // warp-uniform
                const int c = (pass0 + p) * 32 + lane;
                const bool valid = c < nch;
                const int k0 = c * KC;
                if (!PG) {
#pragma unroll
                    for (int m = 0; m < MAXM; ++m)
                        if (m < M && valid) iacc[m] = chunk_dot<W4>(cur[p], s_q + static_cast<int64_t>(m) * K, k0) + iacc[m];
                } else {
                    // Each lane scales its own chunk's exact INT32 dot by the chunk's
                    // group scale: summed over the group's lanes that is
                    // scale_w[g] * acc_g, with the fp32 additions in another order.
                    const float s = cs[p];  // this lane's group scale (0 for invalid chunks)
#pragma unroll
                    for (int m = 0; m < MAXM; ++m) {
                        if (m < M) {
                            const int pp = valid ? chunk_dot<W4>(cur[p], s_q + static_cast<int64_t>(m) * K, k0) : 0;
                            facc[m] = fmaf(static_cast<float>(pp), s, facc[m]);
                        }
                    }
                }
            }
        }
        // reduce over the warp; one warp per row (S == 1) stores directly,
        // otherwise the S slices of a row combine through shared memory
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
            if (m < M) {
                float v;
                if (!PG) {
                    int a = iacc[m];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                    v = __int_as_float(a);
                } else {
                    float a = facc[m];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                    v = a;
                }
                if (geo.S == 1) {
                    if (lane == 0 && n < N) {
                        const float out = PG ? v * s_sx[m] : static_cast<float>(__float_as_int(v)) * s_sx[m] * cs[0];
                        if (ydt == 1)
                            static_cast<__nv_bfloat16*>(y)[static_cast<int64_t>(m) * N + n] = __float2bfloat16_rn(out);
                        else
                            static_cast<__half*>(y)[static_cast<int64_t>(m) * N + n] = __float2half_rn(out);
                    }
                } else if (lane == 0) {
                    s_part[warp][m] = v;
                }
            }
        }
        if (geo.S > 1) {
            __syncthreads();
            for (int t = threadIdx.x; t < geo.R * M; t += kSmallThreads) {
                const int rr = t / M, m = t % M;
                const int nn = blk * geo.R + rr;
                if (nn < N) {
                    float out;
                    if (!PG) {
                        int a = 0;
                        for (int sl = 0; sl < geo.S; ++sl) a += __float_as_int(s_part[rr * geo.S + sl][m]);
                        out = static_cast<float>(a) * s_sx[m] * __ldg(sw + nn);
                    } else {
                        float a = 0.0f;
                        for (int sl = 0; sl < geo.S; ++sl) a += s_part[rr * geo.S + sl][m];
                        out = a * s_sx[m];
                    }
                    if (ydt == 1)
                        static_cast<__nv_bfloat16*>(y)[static_cast<int64_t>(m) * N + nn] = __float2bfloat16_rn(out);
                    else
                        static_cast<__half*>(y)[static_cast<int64_t>(m) * N + nn] = __float2half_rn(out);
                }
            }
            __syncthreads();
        }
    };
    // The ring is walked with compile-time slot indices (the loop is unrolled
    // by the ring depth) so that it stays in registers.
    int blk = blockIdx.x;
    while (blk < geo.nblocks) {
#pragma unroll
        for (int r = 0; r < kRing; ++r) {
            if (blk < geo.nblocks) {
                load(ring[(r + kRing - 1) % kRing], ring_s[(r + kRing - 1) % kRing], blk + (kRing - 1) * gridDim.x);
                step(ring[r], ring_s[r], blk);
            }
            blk += gridDim.x;
        }
    }
}

// ---- one-shot decode kernel (1 <= M <= 4) ----------------------------------
// The same quantize + dot + dequant, organised so that all of a CTA's weight
// bytes are requested at once, before any is used.  Measured on B200 (a 26 MB
// weight matrix, launches back to back in a CUDA graph): with each SM's whole
// share in flight at once the bytes land in about 4.2 us; loads issued in
// rounds (a ring of a few loads per thread) take 6-9 us, each round adding a
// DRAM round trip.  The weights come by bulk copies (the copy engine), not
// per-thread loads: as many per-thread loads as that needs fill the SM's
// load/store queue faster than DRAM drains it, and every later load, store
// or shared-memory access of the CTA then waits behind them (a global load
// issued behind them took ~3 us, the quantization of x ~2.4 us).  At most
// kShotWindow pieces are in flight per CTA: with every piece requested at
// once, all of an SM's pieces land within the last ~0.5 us and the dot
// products (bound by shared-memory bandwidth) start only then; with a window
// of a few 16 KB pieces the first lands after ~1.4 us, the rest follow at the
// SM's share of DRAM bandwidth, and the arithmetic overlaps the stream
// (measured on B200: 6.6 against 7.0 us per launch for the copies and the
// same shared-memory reads; windows of 2 to 8 pieces of 8 to 32 KB were
// within 0.4 us of each other on the decode shapes, 6 x 16 KB among the best).
//
// Work split.  One CTA of 1024 threads per SM; CTA b owns the contiguous
// weight rows [b N / G, (b+1) N / G), so the CTAs differ by at most one row.
// The last warp is the producer: one lane requests the activation rows (one
// bulk copy) and then the CTA's weight rows in pieces of at most 16 KB, each
// on its own mbarrier, issuing piece c once piece c - kShotWindow has landed.
// The other 31 warps (synchronising among themselves on a named barrier)
// stage the weight scales as 4-byte cp.async copies and quantize the
// activation rows as soon as they land.  The weight rows are cut into passes
// (32 consecutive 16-byte chunks of one row, the last pass of a row possibly
// partial) and the 31 warps take equal contiguous runs of passes, so a run
// may start and end inside a row; a warp waits only for the pieces its
// passes lie in.  A lane adds up the dot products of its chunks of one row;
// at the end of a row (or of its run) the warp reduces and lane 0 writes the
// row's partial sum into a per-row slot indexed by the warp's place among the
// warps that meet the row.  The output pass adds a row's slots in warp order,
// so results do not depend on timing.  Per group, each lane scales its
// chunk's exact INT32 dot by its group's scale (scale_w[g] * acc_g, summed in
// another order).
constexpr int kShotThreads = 1024;
constexpr int kShotWarps = kShotThreads / 32;
constexpr int kShotCompute = kShotWarps - 1;       // compute warps (the last warp is the producer)
constexpr int kShotComputeThreads = kShotCompute * 32;
constexpr int kShotWindow = 6;                     // weight pieces in flight per CTA
constexpr int kShotPieceBytes = 16 * 1024;  // weight bytes per bulk copy
constexpr int kShotMaxPieces = 15;          // 15 x 16 KB covers the shared memory
constexpr int kShotSmemBytes = 226 * 1024;  // dynamic shared memory (the static part stays below 1 KB)

struct ShotGeom {
    int ppr;       // passes per weight row
    int slots;     // per-row slots for the partial sums of the warps that meet the row
    int ngroups;   // per-group modes: K / gs
    int x_off;     // shared-memory byte offsets (the weight rows start at 0): activation rows, then their codes;
    int sw_off;    // weight scales;
    int part_off;  // row partial sums
};

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// fp32 dot of one 16-byte weight chunk with 16 activations of type TX read
// from shared memory (W8A16): each weight is widened exactly (its sign bit
// flipped, the byte placed under the exponent of 2^23 by one permute, 2^23 +
// 128 subtracted), each activation pair converted to an fp32 pair, and the
// products summed by packed FMAs, two per instruction.
template <typename TX>
__device__ __forceinline__ float chunk_dot_x16(const uint4& wv, const uint8_t* xs) {
    constexpr float kOff = 8388608.0f + 128.0f;  // 2^23 + 128
    const uint64_t neg_off = pack_f32x2(-kOff, -kOff);
    const uint4 xa = *reinterpret_cast<const uint4*>(xs);
    const uint4 xb = *reinterpret_cast<const uint4*>(xs + 16);
    const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
    const uint32_t wd[4] = {wv.x ^ 0x80808080u, wv.y ^ 0x80808080u, wv.z ^ 0x80808080u, wv.w ^ 0x80808080u};
    uint64_t acc = 0;  // two fp32 partial sums
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t v = wd[i];
        const uint64_t w01 = f32x2_add(
            (static_cast<uint64_t>(__byte_perm(v, 0x4B000000u, 0x7651)) << 32) | __byte_perm(v, 0x4B000000u, 0x7650),
            neg_off);
        const uint64_t w23 = f32x2_add(
            (static_cast<uint64_t>(__byte_perm(v, 0x4B000000u, 0x7653)) << 32) | __byte_perm(v, 0x4B000000u, 0x7652),
            neg_off);
        float2 x01, x23;
        if constexpr (std::is_same<TX, __half>::value) {
            x01 = __half22float2(*reinterpret_cast<const __half2*>(&xw[2 * i]));
            x23 = __half22float2(*reinterpret_cast<const __half2*>(&xw[2 * i + 1]));
        } else {
            x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[2 * i]));
            x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[2 * i + 1]));
        }
        acc = f32x2_fma(w01, pack_f32x2(x01.x, x01.y), acc);
        acc = f32x2_fma(w23, pack_f32x2(x23.x, x23.y), acc);
    }
    return lo_f32(acc) + hi_f32(acc);
}

// barrier of the compute warps only (the producer warp never joins it)
__device__ __forceinline__ void shot_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kShotComputeThreads) : "memory");
}

// A16: the W8A16 product (no activation quantization): the rows of x stay in
// shared memory as they arrive and the dot products are taken in fp32.
template <typename TX, bool PG, bool W4, int MAXM, bool A16 = false>
__global__ void __launch_bounds__(kShotThreads, 1) k_small_m_shot(const TX* __restrict__ x, int M, int K,
                                                                  const uint8_t* __restrict__ w,
                                                                  const float* __restrict__ sw, int N, int gs,
                                                                  void* __restrict__ y, int ydt, ShotGeom geo,
                                                                  unsigned* status) {
    extern __shared__ __align__(128) uint8_t s_raw[];
    const uint8_t* s_w = s_raw;                                      // [rows][row bytes]
    uint8_t* s_x = s_raw + geo.x_off;                                // [M][K] of TX, then [M][K] codes
    int8_t* s_q = reinterpret_cast<int8_t*>(s_x);
    float* s_sw = reinterpret_cast<float*>(s_raw + geo.sw_off);      // per group [rows][K / gs], per channel [rows]
    float* s_part = reinterpret_cast<float*>(s_raw + geo.part_off);  // [rows][slots][MAXM]
    __shared__ float s_sx[MAXM];
    __shared__ float s_red[MAXM][kShotCompute];
    __shared__ __align__(8) uint64_t s_bar[kShotMaxPieces + 1];      // the weight pieces, then the activation rows
    __shared__ int s_abort;
    volatile int* abort_flag = &s_abort;
    uint64_t* xbar = &s_bar[kShotMaxPieces];
    constexpr int KC = W4 ? 32 : 16;  // weights per 16-byte chunk
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_bytes = W4 ? K / 2 : K;
    const int nch = K / KC;
    const int ppr = geo.ppr;
    const int n0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * N / gridDim.x);
    const int n1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * N / gridDim.x);
    const int rows = n1 - n0;
    const int wbytes = rows * row_bytes;                             // < 226 KB, by the plan
    const int npieces = (wbytes + kShotPieceBytes - 1) / kShotPieceBytes;
    const int P = rows * ppr;                              // passes of this CTA
    const int pw = (P + kShotCompute - 1) / kShotCompute;  // passes per compute warp
    const int q0 = warp * pw;
    const int np = min(pw, P - q0);                    // this warp's passes (may be <= 0)
    const int r0 = np > 0 ? q0 / ppr : 0;              // the row, and the pass within it, where the run starts
    const int kp0 = np > 0 ? q0 - r0 * ppr : 0;
    const int nx = K / 8;  // 16-byte chunks of a row of x (M * nx <= 2 * compute threads, by the plan)
    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int i = 0; i <= kShotMaxPieces; ++i) mbar_init(&s_bar[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kShotCompute && lane == 0) {
        // The first window of weight pieces into L2 before the wait on the
        // previous kernel: a CTA that starts while the previous launch drains
        // streams meanwhile.  (Measured on B200 at M = 1: 7.72 -> 7.20 us per
        // channel, 8.67 -> 8.31 us per group; prefetching the whole range
        // instead made it slower, 8.3 us.)
        const uint8_t* src = w + static_cast<int64_t>(n0) * row_bytes;
        for (int off = 0; off < wbytes && off < kShotWindow * kShotPieceBytes; off += kShotPieceBytes)
            prefetch_l2_bulk(src + off, static_cast<uint32_t>(min(kShotPieceBytes, wbytes - off)));
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    if (warp == kShotCompute) {
        // the producer: the activation rows, then the weight pieces through the window
        if (lane == 0) {
            const uint32_t xbytes = static_cast<uint32_t>(M) * K * sizeof(TX);
            mbar_arrive_expect_tx(xbar, xbytes);
            bulk_load(s_x, x, xbytes, xbar);
            const uint8_t* src = w + static_cast<int64_t>(n0) * row_bytes;
            int issued = 0;
            for (int c = 0; c < npieces; ++c) {
                if (c >= kShotWindow && !mbar_wait(&s_bar[c - kShotWindow], 0, status, abort_flag)) break;
                const int off = c * kShotPieceBytes;
                const int sz = min(kShotPieceBytes, wbytes - off);
                mbar_arrive_expect_tx(&s_bar[c], sz);
                bulk_load(s_raw + off, src + off, sz, &s_bar[c]);
                issued = c + 1;
            }
            if (*abort_flag) {
                // a wait timed out (the status is flagged): let every issued
                // copy land, within a bound, before the CTA's shared memory
                // is released
                const unsigned long long t0 = global_timer_ns();
                for (int c = 0; c <= issued; ++c) {
                    uint64_t* bar = c < issued ? &s_bar[c] : xbar;
                    while (!mbar_try_wait(bar, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
                    }
                }
            }
        }
        return;
    }
    {
        const int ns = PG ? rows * geo.ngroups : rows;
        const uint32_t sw0 = smem_u32(s_sw);
        for (int i = threadIdx.x; i < ns; i += kShotComputeThreads) {
            if (PG) {
                const int g = i / rows, r = i - g * rows;  // read along n (contiguous)
                cp_async4(sw0 + (r * geo.ngroups + g) * 4u, sw + static_cast<int64_t>(g) * N + n0 + r);
            } else {
                cp_async4(sw0 + i * 4u, sw + n0 + i);
            }
        }
        cp_async_commit();
    }

    const bool x_ok = mbar_wait(xbar, 0, status, abort_flag);
    if constexpr (!A16) {
    // quantize the M activation rows: each thread takes (at most) two 16-byte
    // chunks into registers, so the codes can overwrite the rows afterwards
    uint4 xv[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
    float amax[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) amax[m] = 0.0f;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int i = threadIdx.x + j * kShotComputeThreads;  // chunk i % nx of row i / nx
        if (i < M * nx && x_ok) {
            xv[j] = *reinterpret_cast<const uint4*>(s_x + static_cast<int64_t>(i) * 16);
            const int m = i / nx;
            const float a = absmax_to_f32<TX>(absmax8<TX>(xv[j], typename Pack2<TX>::type{}));
#pragma unroll
            for (int mm = 0; mm < MAXM; ++mm)
                if (mm == m) amax[mm] = fmaxf(amax[mm], a);
        }
    }
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
        if (m < M) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax[m] = fmaxf(amax[m], __shfl_xor_sync(0xffffffffu, amax[m], o));
            if (lane == 0) s_red[m][warp] = amax[m];
        }
    }
    shot_sync();  // every read of the staged rows is done: the codes may overwrite them
    if (threadIdx.x < M) {
        float a = s_red[threadIdx.x][0];
        for (int i = 1; i < kShotCompute; ++i) a = fmaxf(a, s_red[threadIdx.x][i]);
        s_sx[threadIdx.x] = act_scale(a);
    }
    shot_sync();
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int i = threadIdx.x + j * kShotComputeThreads;
        if (i < M * nx) {
            const int m = i / nx, c = i - m * nx;
            const float sc = s_sx[m];
            float f[8];
            unpack8_f32<TX>(xv[j], f);
            *reinterpret_cast<uint2*>(s_q + static_cast<int64_t>(m) * K + 8 * c) = quant8_codes(f, sc, act_rcp(sc));
        }
    }
    }
    cp_async_wait_all();  // this thread's scale copies
    shot_sync();          // codes and every thread's scales visible to the compute warps

    // dot products, one row segment of the run at a time: wait for the pieces
    // the segment lies in, walk its passes, then reduce over the warp and
    // store the row's partial sum (every condition below is warp-uniform)
    if (np > 0) {
        const int r_last = (q0 + np - 1) / ppr;
        int ready = (r0 * row_bytes + kp0 * 512) / kShotPieceBytes;  // the first piece not yet waited for
        bool ok = true;
        for (int r = r0; r <= r_last; ++r) {
            const int kp_lo = max(q0, r * ppr) - r * ppr;
            const int kp_hi = min(q0 + np, (r + 1) * ppr) - r * ppr;
            const int seg_end = r * row_bytes + min(kp_hi * 512, row_bytes);  // one past the segment's last byte
            while (ok && ready <= (seg_end - 1) / kShotPieceBytes) ok = mbar_wait(&s_bar[ready++], 0, status, abort_flag);
            int iacc[MAXM];
            float facc[MAXM];
#pragma unroll
            for (int m = 0; m < MAXM; ++m) { iacc[m] = 0; facc[m] = 0.0f; }
            if (ok) {
                const uint8_t* wrow = s_w + r * row_bytes + lane * 16;
                const float* srow = s_sw + r * geo.ngroups;
#pragma unroll 4
                for (int kp = kp_lo; kp < kp_hi; ++kp) {
                    const int kc = kp * 32 + lane;
                    if (kc < nch) {
                        const uint4 wv = *reinterpret_cast<const uint4*>(wrow + kp * 512);
                        const int k0 = kc * KC;
                        const float gsc = PG ? srow[k0 / gs] : 0.0f;
#pragma unroll
                        for (int m = 0; m < MAXM; ++m) {
                            if (m < M) {
                                if constexpr (A16) {
                                    const float d = chunk_dot_x16<TX>(
                                        wv, s_x + (static_cast<int64_t>(m) * K + k0) * static_cast<int64_t>(sizeof(TX)));
                                    facc[m] = PG ? fmaf(d, gsc, facc[m]) : facc[m] + d;
                                } else {
                                    const int d = chunk_dot<W4>(wv, s_q + static_cast<int64_t>(m) * K, k0);
                                    if (PG)
                                        facc[m] = fmaf(static_cast<float>(d), gsc, facc[m]);
                                    else
                                        iacc[m] += d;
                                }
                            }
                        }
                    }
                }
            }
            const int slot = warp - (r * ppr) / pw;  // this warp's place among the row's warps
#pragma unroll
            for (int m = 0; m < MAXM; ++m) {
                if (m < M) {
                    float v;
                    if (PG || A16) {
                        float a = facc[m];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                        v = a;
                    } else {
                        v = __int_as_float(__reduce_add_sync(0xffffffffu, iacc[m]));
                    }
                    if (lane == 0) s_part[(r * geo.slots + slot) * MAXM + m] = v;
                }
            }
        }
    }
    shot_sync();

    // outputs: a row's partial sums in warp order, then the dequant
    for (int t = threadIdx.x; t < rows * M; t += kShotComputeThreads) {
        const int m = t / rows, r = t - m * rows;
        const int wa = (r * ppr) / pw, wb = ((r + 1) * ppr - 1) / pw;
        float out;
        if (A16) {
            float a = 0.0f;
            for (int wi = wa; wi <= wb; ++wi) a += s_part[(r * geo.slots + (wi - wa)) * MAXM + m];
            out = PG ? a : a * s_sw[r];
        } else if (PG) {
            float a = 0.0f;
            for (int wi = wa; wi <= wb; ++wi) a += s_part[(r * geo.slots + (wi - wa)) * MAXM + m];
            out = a * s_sx[m];
        } else {
            int a = 0;
            for (int wi = wa; wi <= wb; ++wi) a += __float_as_int(s_part[(r * geo.slots + (wi - wa)) * MAXM + m]);
            out = static_cast<float>(a) * s_sx[m] * s_sw[r];
        }
        const int64_t o = static_cast<int64_t>(m) * N + n0 + r;
        if (ydt == 1)
            static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(out);
        else
            static_cast<__half*>(y)[o] = __float2half_rn(out);
    }
}

// ---- bulk-staged decode kernel (1 <= M <= 4) --------------------------------
// The same fused quantize + dot + dequant as k_small_m, organised so that HBM
// sees as many bytes in flight as it can take.  One CTA per SM owns a
// contiguous, balanced range of weight rows [n0, n1) -- in the [N][K] layout a
// single contiguous byte range -- and a producer warp streams it through a
// ring of shared-memory stages with bulk asynchronous copies, one copy of R
// whole rows per stage, completion counted on the stage's mbarrier.  With ~20
// KB stages and the ring filling the rest of shared memory, ~150-200 KB per SM
// are requested before the first dot product is taken; at the decode shapes
// of the pages' tables (26 MB of weights over 148 SMs) that is almost the whole
// of each SM's share, so the copies keep HBM busy while the activations are
// quantized.  Eight consumer warps form R rows x S K-slices of each stage
// (R * S = 8); lane l of a slice takes its 16-byte chunks l, l + 32, ... from
// shared memory, so a warp reads 512 contiguous bytes per step.  Each (row,
// slice) partial goes to shared memory once; after the last stage the CTA
// adds the slices in order, dequantizes and writes its outputs, coalesced.
// With M = 1 the lane's activation codes sit in registers (the lane's chunk
// positions are the same for every row).  Every wait is bounded; a wait that
// runs out records the timeout, and the other warps leave their loops through
// the CTA's abort flag.
constexpr int kBulkConsumers = 8;                          // consumer warps
constexpr int kBulkThreads = (kBulkConsumers + 1) * 32;    // + one producer warp
constexpr int kBulkMaxStages = 16;

struct BulkGeom {
    int R, S;        // rows per stage, K-slices per row (R * S = 8)
    int cps, ppl;    // 16-byte chunks per slice, chunks per lane per slice
    int nstage;      // ring slots
    int rows_max;    // most rows of any CTA
    int slot_bytes;  // R * bytes per weight row
    int q_off, sw_off, part_off, ring_off, smem;  // dynamic shared memory layout
};

__device__ __forceinline__ void named_sync_consumers() {
    asm volatile("bar.sync 1, %0;" ::"n"(kBulkConsumers * 32) : "memory");
}

// The producer thread: stage j holds rows n0 + j*R .. of the CTA (the last
// stage possibly fewer), one bulk copy each; a slot is refilled once all eight
// consumer warps have released it.
__device__ __forceinline__ void bulk_produce(const uint8_t* __restrict__ w, int n0, int rows, int row_bytes,
                                             const BulkGeom& geo, uint8_t* ring, uint64_t* full, uint64_t* empty,
                                             unsigned* status, volatile int* abort_flag) {
    const uint8_t* src = w + static_cast<int64_t>(n0) * row_bytes;
    const int nst = (rows + geo.R - 1) / geo.R;
    for (int j = 0; j < nst; ++j) {
        const int slot = j % geo.nstage;
        if (j >= geo.nstage && !mbar_wait(&empty[slot], ((j / geo.nstage) - 1) & 1, status, abort_flag)) break;
        const int nr = min(geo.R, rows - j * geo.R);
        const uint32_t bytes = static_cast<uint32_t>(nr * row_bytes);
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_load(ring + slot * geo.slot_bytes, src + static_cast<int64_t>(j) * geo.R * row_bytes, bytes,
                  &full[slot]);
    }
}

template <typename TX, bool PG, bool W4, int MAXM, int PPL>
__global__ void __launch_bounds__(kBulkThreads, 1) k_small_m_bulk(const TX* __restrict__ x, int M, int K,
                                                                  const uint8_t* __restrict__ w,
                                                                  const float* __restrict__ sw, int N, int gs,
                                                                  void* __restrict__ y, int ydt, BulkGeom geo,
                                                                  unsigned* status) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t full[kBulkMaxStages], empty[kBulkMaxStages];
    __shared__ float s_sx[MAXM];
    __shared__ float s_red[MAXM][kBulkConsumers];
    __shared__ int s_abort;
    constexpr int KC = W4 ? 32 : 16;  // weights per 16-byte chunk
    int8_t* s_q = reinterpret_cast<int8_t*>(smem + geo.q_off);          // [M][K] codes
    float* s_sw = reinterpret_cast<float*>(smem + geo.sw_off);          // [K/gs][rows_max] group scales
    float* s_part = reinterpret_cast<float*>(smem + geo.part_off);      // [rows][S][M] partials
    uint8_t* ring = smem + geo.ring_off;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_bytes = W4 ? K / 2 : K;
    const int nch = row_bytes / 16;
    const int n0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * N / gridDim.x);
    const int n1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * N / gridDim.x);
    const int rows = n1 - n0;
    const int nst = (rows + geo.R - 1) / geo.R;
    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int i = 0; i < geo.nstage; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kBulkConsumers);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    volatile int* abort_flag = &s_abort;
    pdl_wait();
    pdl_trigger();

    if (warp == kBulkConsumers) {  // producer
        if (lane == 0) bulk_produce(w, n0, rows, row_bytes, geo, ring, full, empty, status, abort_flag);
        return;
    }

    // consumers: the CTA's group scales (group-major in HBM: one contiguous run
    // of the CTA's rows per group) and the M activation rows' codes
    if (PG) {
        const int G = K / gs;
        for (int t = threadIdx.x; t < G * rows; t += kBulkConsumers * 32) {
            const int g = t / rows, r = t - g * rows;
            s_sw[g * geo.rows_max + r] = __ldg(sw + static_cast<int64_t>(g) * N + n0 + r);
        }
    }
    const int nx = K / 8;  // 16-byte chunks of a row of x
    for (int m = 0; m < M; ++m) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K);
        typename Pack2<TX>::type m2 = {};
        for (int c = threadIdx.x; c < nx; c += kBulkConsumers * 32) m2 = absmax8<TX>(__ldg(xr + c), m2);
        float amax = absmax_to_f32<TX>(m2);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) s_red[m][warp] = amax;
    }
    named_sync_consumers();
    for (int m = 0; m < M; ++m) {
        float amax = s_red[m][0];
#pragma unroll
        for (int i = 1; i < kBulkConsumers; ++i) amax = fmaxf(amax, s_red[m][i]);
        const float s = act_scale(amax);
        const float rs = act_rcp(s);
        if (threadIdx.x == 0) s_sx[m] = s;
        const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K);
        for (int c = threadIdx.x; c < nx; c += kBulkConsumers * 32) {
            float f[8];
            unpack8_f32<TX>(__ldg(xr + c), f);
            *reinterpret_cast<uint2*>(s_q + static_cast<int64_t>(m) * K + 8 * c) = quant8_codes(f, s, rs);
        }
    }
    named_sync_consumers();

    const int r_in = warp / geo.S, sl = warp % geo.S;
    const int c_begin = sl * geo.cps, c_end = min(nch, c_begin + geo.cps);
    // M = 1: this lane's activation codes, the same chunk positions for every row
    constexpr int XQ = MAXM == 1 ? PPL : 1;
    uint4 xq[XQ][W4 ? 2 : 1];
    if constexpr (MAXM == 1) {
#pragma unroll
        for (int p = 0; p < PPL; ++p) {
            const int c = c_begin + 32 * p + lane;
            const bool ok = p < geo.ppl && c < c_end;
#pragma unroll
            for (int h = 0; h < (W4 ? 2 : 1); ++h)
                xq[p][h] = ok ? *reinterpret_cast<const uint4*>(s_q + c * KC + 16 * h) : make_uint4(0, 0, 0, 0);
        }
    }
    for (int j = 0; j < nst; ++j) {
        const int slot = j % geo.nstage;
        if (!mbar_wait(&full[slot], (j / geo.nstage) & 1, status, abort_flag)) break;
        const int rl = j * geo.R + r_in;  // the CTA-local row this warp takes
        int iacc[MAXM];
        float facc[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) { iacc[m] = 0; facc[m] = 0.0f; }
        if (rl < rows) {
            const uint8_t* wrow = ring + slot * geo.slot_bytes + r_in * row_bytes;
#pragma unroll
            for (int p = 0; p < PPL; ++p) {
                if (p >= geo.ppl) break;  // warp-uniform
                const int c = c_begin + 32 * p + lane;
                if (c < c_end) {
                    const uint4 wv = *reinterpret_cast<const uint4*>(wrow + 16 * c);
                    const int k0 = c * KC;
                    const float gsc = PG ? s_sw[(k0 / gs) * geo.rows_max + rl] : 0.0f;
#pragma unroll
                    for (int m = 0; m < MAXM; ++m) {
                        if (m < M) {
                            int d;
                            if constexpr (MAXM == 1) {
                                if constexpr (!W4) {
                                    d = dp4a(wv.x, xq[p][0].x, 0);
                                    d = dp4a(wv.y, xq[p][0].y, d);
                                    d = dp4a(wv.z, xq[p][0].z, d);
                                    d = dp4a(wv.w, xq[p][0].w, d);
                                } else {
                                    const uint2 u0 = unpack_int4x8(wv.x), u1 = unpack_int4x8(wv.y);
                                    const uint2 u2 = unpack_int4x8(wv.z), u3 = unpack_int4x8(wv.w);
                                    d = dp4a(u0.x, xq[p][0].x, 0);
                                    d = dp4a(u0.y, xq[p][0].y, d);
                                    d = dp4a(u1.x, xq[p][0].z, d);
                                    d = dp4a(u1.y, xq[p][0].w, d);
                                    d = dp4a(u2.x, xq[p][1].x, d);
                                    d = dp4a(u2.y, xq[p][1].y, d);
                                    d = dp4a(u3.x, xq[p][1].z, d);
                                    d = dp4a(u3.y, xq[p][1].w, d);
                                }
                            } else {
                                d = chunk_dot<W4>(wv, s_q + static_cast<int64_t>(m) * K, k0);
                            }
                            if (PG)
                                facc[m] = fmaf(static_cast<float>(d), gsc, facc[m]);
                            else
                                iacc[m] += d;
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);  // this warp's reads of the slot are done
        if (rl < rows) {
#pragma unroll
            for (int m = 0; m < MAXM; ++m) {
                if (m < M) {
                    float v;
                    if (PG) {
                        float a = facc[m];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                        v = a;
                    } else {
                        int a = iacc[m];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                        v = __int_as_float(a);
                    }
                    if (lane == 0) s_part[(rl * geo.S + sl) * M + m] = v;
                }
            }
        }
    }
    named_sync_consumers();
    if (*abort_flag) return;
    // add the slices in order, dequantize, write the CTA's outputs (row-major y)
    for (int t = threadIdx.x; t < rows * M; t += kBulkConsumers * 32) {
        const int m = t / rows, r = t - m * rows;
        float out;
        if (PG) {
            float a = 0.0f;
            for (int q = 0; q < geo.S; ++q) a += s_part[(r * geo.S + q) * M + m];
            out = a * s_sx[m];
        } else {
            int a = 0;
            for (int q = 0; q < geo.S; ++q) a += __float_as_int(s_part[(r * geo.S + q) * M + m]);
            out = static_cast<float>(a) * s_sx[m] * __ldg(sw + n0 + r);
        }
        const int64_t o = static_cast<int64_t>(m) * N + n0 + r;
        if (ydt == 1)
            static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(out);
        else
            static_cast<__half*>(y)[o] = __float2half_rn(out);
    }
}

// ---- W8A16 decode matrix-vector product ----------------------------------
// The pages' decode kernel (Cider README, section "Metal Kernel 流水线",
// Decode): a direct INT8 matrix-vector product with the weights dequantized
// on the fly and NO activation quantization.  y[m,n] = round(scale_w[n] *
// sum_k x[m,k] * w[n,k]) with x widened to fp32 (exact) and the products
// summed in fp32.  Same streaming layout as k_small_m (persistent grid, R rows
// x S K-slices, a register ring of 16-byte weight chunks); the M <= 4
// activation rows are staged once into shared memory as fp32 pairs laid out
// [pass][pair][lane], so that the lanes of a warp, each holding a different
// 16-weight chunk, read 32 consecutive pairs at a time (a row-major layout
// would put them 64 bytes apart: a 16-way bank conflict).
// fp32 dot of one 16-byte weight chunk with 16 activations.  Each weight is
// widened exactly without an int->float conversion: after flipping its sign
// bit the byte is u = w + 128, one byte permute places it under the exponent
// of 2^23 (the float 2^23 + u), and one packed subtract of 2^23 + 128 leaves
// w; the products then go through packed FMAs, two per instruction.
// xs: this lane's first activation pair of the chunk; pair j is at xs[32 * j]
// (the staging layout [pass][pair][lane] keeps a warp's loads conflict-free).
__device__ __forceinline__ float chunk_dot_f32(const uint4& wv, const uint64_t* xs) {
    constexpr float kOff = 8388608.0f + 128.0f;                          // 2^23 + 128
    const uint64_t neg_off = pack_f32x2(-kOff, -kOff);
    const uint32_t wd[4] = {wv.x ^ 0x80808080u, wv.y ^ 0x80808080u, wv.z ^ 0x80808080u, wv.w ^ 0x80808080u};
    uint64_t acc = 0;  // two fp32 partial sums
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t v = wd[i];
        const uint64_t w01 = f32x2_add(
            (static_cast<uint64_t>(__byte_perm(v, 0x4B000000u, 0x7651)) << 32) | __byte_perm(v, 0x4B000000u, 0x7650),
            neg_off);
        const uint64_t w23 = f32x2_add(
            (static_cast<uint64_t>(__byte_perm(v, 0x4B000000u, 0x7653)) << 32) | __byte_perm(v, 0x4B000000u, 0x7652),
            neg_off);
        acc = f32x2_fma(w01, xs[32 * (2 * i)], acc);
        acc = f32x2_fma(w23, xs[32 * (2 * i + 1)], acc);
    }
    return lo_f32(acc) + hi_f32(acc);
}

// PG: per-group scales scale_w[g][n] (group-major), applied per 16-weight
// chunk as its dot is accumulated; otherwise scale_w[n] on the row's sum.
template <typename TX, bool PG, int MAXM, int PPW>
__global__ void __launch_bounds__(kSmallThreads, 2) k_mv_w8a16(const TX* __restrict__ x, int M, int K,
                                                               const int8_t* __restrict__ w,
                                                               const float* __restrict__ sw, int N, int gs,
                                                               void* __restrict__ y, int ydt, SmallGeom geo) {
    extern __shared__ __align__(16) uint64_t s_x[];  // [M][pass][8 pairs][32 lanes] fp32 pairs
    __shared__ float s_part[kSmallWarps][MAXM];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = K / 16;
    const int npass = (nch + 31) / 32;
    const int r_in_blk = warp / geo.S, slice = warp % geo.S;
    const int pass0 = slice * geo.ppw;
    pdl_wait();
    pdl_trigger();

    constexpr int kRing = RingDepth<PPW>::value;
    uint4 ring[kRing][PPW];
    float ring_s[kRing][PG ? PPW : 1];
    auto load = [&](uint4 (&dst)[PPW], float (&ds)[PG ? PPW : 1], int blk) {
        const int n = blk * geo.R + r_in_blk;
        const bool row_ok = blk < geo.nblocks && n < N;
        const uint4* wr = reinterpret_cast<const uint4*>(w + static_cast<int64_t>(n) * K);
#pragma unroll
        for (int p = 0; p < PPW; ++p) {
            const int c = (pass0 + p) * 32 + lane;
            const bool ok = p < geo.ppw && row_ok && c < nch;
            dst[p] = ok ? __ldcs(wr + c) : make_uint4(0, 0, 0, 0);
            if (PG) ds[p] = ok ? __ldg(sw + static_cast<int64_t>(c * 16 / gs) * N + n) : 0.0f;
        }
        if (!PG) ds[0] = row_ok ? __ldg(sw + n) : 0.0f;
    };
#pragma unroll
    for (int i = 0; i < kRing - 1; ++i) load(ring[i], ring_s[i], blockIdx.x + i * gridDim.x);

    // stage the activations as fp32 pairs (exact widening): the 8 values at
    // k0 = 8t belong to chunk c = k0 / 16 (pass c / 32, lane c % 32), pairs
    // (k0 % 16) / 2 .. + 3
    const int nx = K / 8;
    for (int m = 0; m < M; ++m) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K);
        for (int t = threadIdx.x; t < nx; t += kSmallThreads) {
            float f[8];
            unpack8_f32<TX>(__ldg(xr + t), f);
            const int c = t >> 1, q = c >> 5, l = c & 31, j0 = (t & 1) * 4;
            uint64_t* dst = s_x + ((static_cast<int64_t>(m) * npass + q) * 8 + j0) * 32 + l;
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[32 * j] = pack_f32x2(f[2 * j], f[2 * j + 1]);
        }
    }
    __syncthreads();

    auto step = [&](const uint4 (&cur)[PPW], const float (&cs)[PG ? PPW : 1], int blk) {
        const int n = blk * geo.R + r_in_blk;
        float acc[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) acc[m] = 0.0f;
        if (n < N) {
#pragma unroll
            for (int p = 0; p < PPW; ++p) {
                if (p >= geo.ppw || (pass0 + p) * 32 >= nch) break;  // warp-uniform
                const int c = (pass0 + p) * 32 + lane;
                if (c < nch) {
#pragma unroll
                    for (int m = 0; m < MAXM; ++m)
                        if (m < M) {
                            const float d =
                                chunk_dot_f32(cur[p], s_x + ((static_cast<int64_t>(m) * npass + pass0 + p) * 8) * 32 + lane);
                            acc[m] = PG ? fmaf(d, cs[p], acc[m]) : acc[m] + d;
                        }
                }
            }
        }
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
            if (m < M) {
                float a = acc[m];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                if (geo.S == 1) {
                    if (lane == 0 && n < N) {
                        const float out = PG ? a : a * cs[0];
                        if (ydt == 1)
                            static_cast<__nv_bfloat16*>(y)[static_cast<int64_t>(m) * N + n] = __float2bfloat16_rn(out);
                        else
                            static_cast<__half*>(y)[static_cast<int64_t>(m) * N + n] = __float2half_rn(out);
                    }
                } else if (lane == 0) {
                    s_part[warp][m] = a;
                }
            }
        }
        if (geo.S > 1) {
            __syncthreads();
            for (int t = threadIdx.x; t < geo.R * M; t += kSmallThreads) {
                const int rr = t / M, m = t % M;
                const int nn = blk * geo.R + rr;
                if (nn < N) {
                    float a = 0.0f;
                    for (int sl = 0; sl < geo.S; ++sl) a += s_part[rr * geo.S + sl][m];
                    const float out = PG ? a : a * __ldg(sw + nn);
                    if (ydt == 1)
                        static_cast<__nv_bfloat16*>(y)[static_cast<int64_t>(m) * N + nn] = __float2bfloat16_rn(out);
                    else
                        static_cast<__half*>(y)[static_cast<int64_t>(m) * N + nn] = __float2half_rn(out);
                }
            }
            __syncthreads();
        }
    };
    int blk = blockIdx.x;
    while (blk < geo.nblocks) {
#pragma unroll
        for (int r = 0; r < kRing; ++r) {
            if (blk < geo.nblocks) {
                load(ring[(r + kRing - 1) % kRing], ring_s[(r + kRing - 1) % kRing], blk + (kRing - 1) * gridDim.x);
                step(ring[r], ring_s[r], blk);
            }
            blk += gridDim.x;
        }
    }
}

// W8A16 decode product on the bulk-staged layout of k_small_m_bulk (one CTA
// per SM, a contiguous range of weight rows streamed through a shared-memory
// ring by a producer warp), per output channel or per group of gs along K.
// The activation rows are staged once as fp32 pairs in the [pass][pair][lane]
// layout of k_mv_w8a16 (slices are whole 512-weight passes, so lane l always
// takes chunks l, l + 32, ... of a pass and its reads are conflict-free).  Per
// group, each lane multiplies its chunk's fp32 dot by the chunk's group scale
// scale_w[g][n] (staged per CTA) and accumulates; per channel the row's sum is
// scaled by scale_w[n] at the end.
template <typename TX, bool PG, int MAXM, int PPL>
__global__ void __launch_bounds__(kBulkThreads, 1) k_mv_w8a16_bulk(const TX* __restrict__ x, int M, int K,
                                                                   const int8_t* __restrict__ w,
                                                                   const float* __restrict__ sw, int N, int gs,
                                                                   void* __restrict__ y, int ydt, BulkGeom geo,
                                                                   unsigned* status) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t full[kBulkMaxStages], empty[kBulkMaxStages];
    __shared__ int s_abort;
    uint64_t* s_x = reinterpret_cast<uint64_t*>(smem + geo.q_off);  // [M][pass][8 pairs][32 lanes]
    float* s_sw = reinterpret_cast<float*>(smem + geo.sw_off);      // [K/gs][rows_max]
    float* s_part = reinterpret_cast<float*>(smem + geo.part_off);  // [rows][S][M]
    uint8_t* ring = smem + geo.ring_off;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = K / 16;
    const int npass = (nch + 31) / 32;
    const int n0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * N / gridDim.x);
    const int n1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * N / gridDim.x);
    const int rows = n1 - n0;
    const int nst = (rows + geo.R - 1) / geo.R;
    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int i = 0; i < geo.nstage; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kBulkConsumers);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    volatile int* abort_flag = &s_abort;
    pdl_wait();
    pdl_trigger();
    if (warp == kBulkConsumers) {
        if (lane == 0)
            bulk_produce(reinterpret_cast<const uint8_t*>(w), n0, rows, K, geo, ring, full, empty, status, abort_flag);
        return;
    }
    if (PG) {
        const int G = K / gs;
        for (int t = threadIdx.x; t < G * rows; t += kBulkConsumers * 32) {
            const int g = t / rows, r = t - g * rows;
            s_sw[g * geo.rows_max + r] = __ldg(sw + static_cast<int64_t>(g) * N + n0 + r);
        }
    }
    // the 8 values at k0 = 8t belong to chunk c = t / 2 (pass c / 32, lane
    // c % 32), pairs (t % 2) * 4 .. + 3
    const int nx = K / 8;
    for (int m = 0; m < M; ++m) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K);
        for (int t = threadIdx.x; t < nx; t += kBulkConsumers * 32) {
            float f[8];
            unpack8_f32<TX>(__ldg(xr + t), f);
            const int c = t >> 1, q = c >> 5, l = c & 31, j0 = (t & 1) * 4;
            uint64_t* dst = s_x + ((static_cast<int64_t>(m) * npass + q) * 8 + j0) * 32 + l;
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[32 * j] = pack_f32x2(f[2 * j], f[2 * j + 1]);
        }
    }
    named_sync_consumers();

    const int r_in = warp / geo.S, sl = warp % geo.S;
    const int pass0 = sl * (geo.cps / 32);
    for (int j = 0; j < nst; ++j) {
        const int slot = j % geo.nstage;
        if (!mbar_wait(&full[slot], (j / geo.nstage) & 1, status, abort_flag)) break;
        const int rl = j * geo.R + r_in;
        float acc[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) acc[m] = 0.0f;
        if (rl < rows) {
            const uint8_t* wrow = ring + slot * geo.slot_bytes + r_in * K;
#pragma unroll
            for (int p = 0; p < PPL; ++p) {
                if (p >= geo.ppl) break;  // warp-uniform
                const int c = (pass0 + p) * 32 + lane;
                if (c < nch) {
                    const uint4 wv = *reinterpret_cast<const uint4*>(wrow + 16 * c);
                    const float gsc = PG ? s_sw[((16 * c) / gs) * geo.rows_max + rl] : 1.0f;
#pragma unroll
                    for (int m = 0; m < MAXM; ++m) {
                        if (m < M) {
                            const float d =
                                chunk_dot_f32(wv, s_x + ((static_cast<int64_t>(m) * npass + pass0 + p) * 8) * 32 + lane);
                            acc[m] = PG ? fmaf(d, gsc, acc[m]) : acc[m] + d;
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (rl < rows) {
#pragma unroll
            for (int m = 0; m < MAXM; ++m) {
                if (m < M) {
                    float a = acc[m];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                    if (lane == 0) s_part[(rl * geo.S + sl) * M + m] = a;
                }
            }
        }
    }
    named_sync_consumers();
    if (*abort_flag) return;
    for (int t = threadIdx.x; t < rows * M; t += kBulkConsumers * 32) {
        const int m = t / rows, r = t - m * rows;
        float a = 0.0f;
        for (int q = 0; q < geo.S; ++q) a += s_part[(r * geo.S + q) * M + m];
        const float out = PG ? a : a * __ldg(sw + n0 + r);
        const int64_t o = static_cast<int64_t>(m) * N + n0 + r;
        if (ydt == 1)
            static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(out);
        else
            static_cast<__half*>(y)[o] = __float2half_rn(out);
    }
}

// Slices per row: as many as keep at least 4 passes per warp (at most 8).
static SmallGeom small_geom(int K, int N, bool w4) {
    SmallGeom g;
    const int kc = w4 ? 32 : 16;
    const int npass = (K / kc + 31) / 32;
    int S = 1;
    while (S < 8 && npass / (2 * S) >= 4) S *= 2;
    g.S = S;
    g.R = kSmallWarps / S;
    g.ppw = (npass + S - 1) / S;
    g.nblocks = (N + g.R - 1) / g.R;
    return g;
}

template <typename TX, bool PG, bool W4, int MAXM, int PPW>
static cudaError_t launch_small_t(const void* x, int M, int K, const void* w, const float* sw, int N, int gs,
                                  void* y, int ydt, const SmallGeom& geo, int num_sms, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(M) * K;
    auto kern = k_small_m<TX, PG, W4, MAXM, PPW>;
    // opt in above the default 48 KB: static shared memory counts against it too
    if (smem > 32 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int grid = geo.nblocks < 2 * num_sms ? geo.nblocks : 2 * num_sms;
    return launch_pdl(kern, grid, kSmallThreads, smem, st, static_cast<const TX*>(x), M, K,
                      static_cast<const uint8_t*>(w), sw, N, gs, y, ydt, geo);
}

template <typename TX, bool PG, bool W4, int MAXM>
static cudaError_t launch_small_ppw(const void* x, int M, int K, const void* w, const float* sw, int N, int gs,
                                   void* y, int ydt, int num_sms, cudaStream_t st) {
    const SmallGeom geo = small_geom(K, N, W4);
    if (geo.ppw <= 2) return launch_small_t<TX, PG, W4, MAXM, 2>(x, M, K, w, sw, N, gs, y, ydt, geo, num_sms, st);
    if (geo.ppw <= 4) return launch_small_t<TX, PG, W4, MAXM, 4>(x, M, K, w, sw, N, gs, y, ydt, geo, num_sms, st);
    if (geo.ppw <= 5) return launch_small_t<TX, PG, W4, MAXM, 5>(x, M, K, w, sw, N, gs, y, ydt, geo, num_sms, st);
    if (geo.ppw <= 8) return launch_small_t<TX, PG, W4, MAXM, 8>(x, M, K, w, sw, N, gs, y, ydt, geo, num_sms, st);
    return cudaErrorInvalidValue;  // K beyond the small-M kernel: the host sends such calls to the GEMM path
}

template <typename TX, bool PG, bool W4>
static cudaError_t launch_small_m_t(const void* x, int M, int K, const void* w, const float* sw, int N, int gs,
                                    void* y, int ydt, int num_sms, cudaStream_t st) {
    if (M <= 1) return launch_small_ppw<TX, PG, W4, 1>(x, M, K, w, sw, N, gs, y, ydt, num_sms, st);
    if (M <= 4) return launch_small_ppw<TX, PG, W4, 4>(x, M, K, w, sw, N, gs, y, ydt, num_sms, st);
    if (M <= 8) return launch_small_ppw<TX, PG, W4, 8>(x, M, K, w, sw, N, gs, y, ydt, num_sms, st);
    return launch_small_ppw<TX, PG, W4, 16>(x, M, K, w, sw, N, gs, y, ydt, num_sms, st);
}

// Shared-memory plan of k_small_m_bulk: R rows per stage with R * row bytes
// <= 24 KB (R = 8, 4, 2 or 1), the codes, the CTA's group scales and the
// partials first, the ring of stages in the rest (at most 16 stages).  Returns
// false when fewer than three stages fit, or a slice needs more than 8 chunks
// per lane; those calls take k_small_m.
constexpr int kBulkSmemBytes = 225 * 1024;
// test override of the decode kernel: 0 automatic (one-shot where its plan
// fits, else the register ring), 1 register ring, 2 bulk with the whole shared
// memory, 3 bulk within half of it, 4 one-shot where its plan fits
static std::atomic<int> g_small_kernel{0};
static int bulk_smem_budget() { return g_small_kernel.load() == 3 ? 110 * 1024 : kBulkSmemBytes; }
// With a16 (the W8A16 product) the activation rows are staged as fp32 pairs,
// M * (whole 512-weight passes) * 2048 bytes, and slices are whole passes.
static bool bulk_plan(int M, int K, int N, bool pg, bool w4, int gs, int num_sms, BulkGeom& g, int& grid,
                      bool a16 = false) {
    const int budget = bulk_smem_budget();
    const int row_bytes = w4 ? K / 2 : K;
    int R = 8;
    while (R > 1 && R * row_bytes > 24 * 1024) R >>= 1;
    g.R = R;
    g.S = kBulkConsumers / R;
    const int nch = row_bytes / 16;
    g.cps = (nch + g.S - 1) / g.S;
    if (a16) g.cps = (g.cps + 31) / 32 * 32;
    g.ppl = (g.cps + 31) / 32;
    if (g.ppl > 8) return false;
    g.slot_bytes = R * row_bytes;
    grid = N / R < num_sms ? (N / R > 0 ? N / R : 1) : num_sms;
    g.rows_max = (N + grid - 1) / grid;
    auto al = [](int64_t v) { return static_cast<int>((v + 127) & ~int64_t(127)); };
    int off = 0;
    g.q_off = off;
    off += a16 ? al(static_cast<int64_t>(M) * ((nch + 31) / 32) * 2048) : al(static_cast<int64_t>(M) * K);
    g.sw_off = off;
    off += pg ? al(static_cast<int64_t>(K / gs) * g.rows_max * 4) : 0;
    g.part_off = off;
    off += al(static_cast<int64_t>(g.rows_max) * g.S * M * 4);
    g.ring_off = off;
    if (off >= budget) return false;
    g.nstage = (budget - off) / g.slot_bytes;
    if (g.nstage > kBulkMaxStages) g.nstage = kBulkMaxStages;
    if (g.nstage < 3) return false;
    g.smem = off + g.nstage * g.slot_bytes;
    return true;
}

template <typename TX, bool PG, bool W4, int MAXM, int PPL>
static cudaError_t launch_bulk_t(const void* x, int M, int K, const void* w, const float* sw, int N, int gs, void* y,
                                 int ydt, const BulkGeom& geo, int grid, unsigned* status, cudaStream_t st) {
    auto kern = k_small_m_bulk<TX, PG, W4, MAXM, PPL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, geo.smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, grid, kBulkThreads, geo.smem, st, static_cast<const TX*>(x), M, K,
                      static_cast<const uint8_t*>(w), sw, N, gs, y, ydt, geo, status);
}

template <typename TX, bool PG, bool W4, int MAXM>
static cudaError_t launch_bulk_ppl(const void* x, int M, int K, const void* w, const float* sw, int N, int gs,
                                   void* y, int ydt, const BulkGeom& geo, int grid, unsigned* status,
                                   cudaStream_t st) {
    if (geo.ppl <= 2) return launch_bulk_t<TX, PG, W4, MAXM, 2>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
    if (geo.ppl <= 4) return launch_bulk_t<TX, PG, W4, MAXM, 4>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
    if (geo.ppl <= 6) return launch_bulk_t<TX, PG, W4, MAXM, 6>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
    return launch_bulk_t<TX, PG, W4, MAXM, 8>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
}

// Plan of k_small_m_shot: one CTA per SM (at most one per row), at most two
// 16-byte chunks of x per thread, and the CTA's weight rows, activation rows,
// weight scales and row partial sums within one CTA's shared memory; false
// otherwise (those calls take the register-ring kernel).
static bool shot_plan(int M, int K, int N, bool pg, bool w4, int gs, int num_sms, ShotGeom& g, int& grid,
                      int& smem, bool a16 = false) {
    if (M < 1 || M > 4 || N < 1) return false;
    if (!a16 && M * (K / 8) > 2 * kShotComputeThreads) return false;  // the quantizer's two chunks a thread
    const int64_t row_bytes = w4 ? K / 2 : K;
    const int nch = K / (w4 ? 32 : 16);
    g.ppr = (nch + 31) / 32;
    grid = std::min(num_sms, N);
    const int64_t rows_max = (N + grid - 1) / grid, rows_min = N / grid;
    const int64_t wbytes = rows_max * row_bytes;
    if (wbytes > static_cast<int64_t>(kShotMaxPieces) * kShotPieceBytes) return false;
    const int64_t pw_min = std::max<int64_t>(1, (rows_min * g.ppr + kShotCompute - 1) / kShotCompute);
    // a row's ppr passes meet at most ceil(ppr / pw) + 1 warps' runs
    g.slots = static_cast<int>(std::min<int64_t>(kShotCompute, (g.ppr + pw_min - 1) / pw_min + 1));
    g.ngroups = pg ? K / gs : 0;
    auto al = [](int64_t v) { return (v + 127) & ~int64_t(127); };
    int64_t off = al(wbytes);
    g.x_off = static_cast<int>(off);
    off += al(static_cast<int64_t>(M) * K * 2);  // the activation rows (16-bit), then their codes
    g.sw_off = static_cast<int>(off);
    off += al(rows_max * (pg ? g.ngroups : 1) * 4);
    g.part_off = static_cast<int>(off);
    off += al(rows_max * g.slots * 4 * 4);  // MAXM <= 4 partial sums per slot
    if (off > kShotSmemBytes) return false;
    smem = static_cast<int>(off);
    return true;
}

template <typename TX, bool PG, bool W4, int MAXM, bool A16 = false>
static cudaError_t launch_shot_t(const void* x, int M, int K, const void* w, const float* sw, int N, int gs, void* y,
                                 int ydt, const ShotGeom& geo, int grid, int smem, unsigned* status,
                                 cudaStream_t st) {
    auto kern = k_small_m_shot<TX, PG, W4, MAXM, A16>;
    if (smem > 32 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(kern, grid, kShotThreads, smem, st, static_cast<const TX*>(x), M, K,
                      static_cast<const uint8_t*>(w), sw, N, gs, y, ydt, geo, status);
}

template <typename TX, bool PG, bool W4>
static cudaError_t launch_shot_m(const void* x, int M, int K, const void* w, const float* sw, int N, int gs, void* y,
                                 int ydt, const ShotGeom& geo, int grid, int smem, unsigned* status,
                                 cudaStream_t st) {
    if (M == 1) return launch_shot_t<TX, PG, W4, 1>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, smem, status, st);
    return launch_shot_t<TX, PG, W4, 4>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, smem, status, st);
}

template <bool PG, bool W4>
static cudaError_t launch_small_m_v(const void* x, int xdt, int M, int K, const void* w, const float* sw, int N,
                                    int gs, void* y, int ydt, int num_sms, unsigned* status, cudaStream_t st) {
    BulkGeom geo;
    int grid = 0;
    // the register-ring kernel is the default: the bulk-staged one measured
    // slower on B200 (M = 1, N = 10240, K = 2560: 11.3 / 10.0 us with the
    // whole / half of shared memory against 8.8 us); it stays selectable
    const int sel = g_small_kernel.load();
    ShotGeom sg;
    int sgrid = 0, ssmem = 0;
    if (((sel == 0 && gs > 0) || sel == 4) && shot_plan(M, K, N, PG, W4, gs, num_sms, sg, sgrid, ssmem)) {
        if (xdt == 1)
            return launch_shot_m<__nv_bfloat16, PG, W4>(x, M, K, w, sw, N, gs, y, ydt, sg, sgrid, ssmem, status, st);
        return launch_shot_m<__half, PG, W4>(x, M, K, w, sw, N, gs, y, ydt, sg, sgrid, ssmem, status, st);
    }
    if (M <= 4 && (sel == 2 || sel == 3) && bulk_plan(M, K, N, PG, W4, gs, num_sms, geo, grid)) {
        if (xdt == 1) {
            if (M == 1)
                return launch_bulk_ppl<__nv_bfloat16, PG, W4, 1>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
            return launch_bulk_ppl<__nv_bfloat16, PG, W4, 4>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
        }
        if (M == 1) return launch_bulk_ppl<__half, PG, W4, 1>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
        return launch_bulk_ppl<__half, PG, W4, 4>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
    }
    if (xdt == 1) return launch_small_m_t<__nv_bfloat16, PG, W4>(x, M, K, w, sw, N, gs, y, ydt, num_sms, st);
    return launch_small_m_t<__half, PG, W4>(x, M, K, w, sw, N, gs, y, ydt, num_sms, st);
}

template <typename TX, bool PG, int MAXM, int PPW>
static cudaError_t launch_mv_t(const void* x, int M, int K, const int8_t* w, const float* sw, int N, int gs, void* y,
                               int ydt, const SmallGeom& geo, int num_sms, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(M) * ((K / 16 + 31) / 32) * 2048;  // whole passes of pairs
    auto kern = k_mv_w8a16<TX, PG, MAXM, PPW>;
    // opt in above the default 48 KB: static shared memory counts against it too
    if (smem > 32 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int grid = geo.nblocks < 2 * num_sms ? geo.nblocks : 2 * num_sms;
    return launch_pdl(kern, grid, kSmallThreads, smem, st, static_cast<const TX*>(x), M, K, w, sw, N, gs, y, ydt, geo);
}

template <typename TX, bool PG, int MAXM>
static cudaError_t launch_mv_ppw(const void* x, int M, int K, const int8_t* w, const float* sw, int N, int gs,
                                 void* y, int ydt, int num_sms, cudaStream_t st) {
    const SmallGeom geo = small_geom(K, N, false);
    if (geo.ppw <= 2) return launch_mv_t<TX, PG, MAXM, 2>(x, M, K, w, sw, N, gs, y, ydt, geo, num_sms, st);
    if (geo.ppw <= 4) return launch_mv_t<TX, PG, MAXM, 4>(x, M, K, w, sw, N, gs, y, ydt, geo, num_sms, st);
    if (geo.ppw <= 5) return launch_mv_t<TX, PG, MAXM, 5>(x, M, K, w, sw, N, gs, y, ydt, geo, num_sms, st);
    if (geo.ppw <= 8) return launch_mv_t<TX, PG, MAXM, 8>(x, M, K, w, sw, N, gs, y, ydt, geo, num_sms, st);
    return cudaErrorInvalidValue;  // K beyond the kernel: rejected by the host checks first
}

template <typename TX, bool PG>
static cudaError_t launch_mv_reg(const void* x, int M, int K, const int8_t* w, const float* sw, int N, int gs,
                                 void* y, int ydt, int num_sms, cudaStream_t st) {
    if (M <= 1) return launch_mv_ppw<TX, PG, 1>(x, M, K, w, sw, N, gs, y, ydt, num_sms, st);
    return launch_mv_ppw<TX, PG, 4>(x, M, K, w, sw, N, gs, y, ydt, num_sms, st);
}

template <typename TX, bool PG, int MAXM, int PPL>
static cudaError_t launch_mv_bulk_t(const void* x, int M, int K, const int8_t* w, const float* sw, int N, int gs,
                                    void* y, int ydt, const BulkGeom& geo, int grid, unsigned* status,
                                    cudaStream_t st) {
    auto kern = k_mv_w8a16_bulk<TX, PG, MAXM, PPL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, geo.smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, grid, kBulkThreads, geo.smem, st, static_cast<const TX*>(x), M, K, w, sw, N, gs, y, ydt,
                      geo, status);
}

template <typename TX, bool PG, int MAXM>
static cudaError_t launch_mv_bulk_ppl(const void* x, int M, int K, const int8_t* w, const float* sw, int N, int gs,
                                      void* y, int ydt, const BulkGeom& geo, int grid, unsigned* status,
                                      cudaStream_t st) {
    if (geo.ppl <= 2) return launch_mv_bulk_t<TX, PG, MAXM, 2>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
    if (geo.ppl <= 4) return launch_mv_bulk_t<TX, PG, MAXM, 4>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
    if (geo.ppl <= 6) return launch_mv_bulk_t<TX, PG, MAXM, 6>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
    return launch_mv_bulk_t<TX, PG, MAXM, 8>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
}

template <typename TX, bool PG>
static cudaError_t launch_mv_bulk_m(const void* x, int M, int K, const int8_t* w, const float* sw, int N, int gs,
                                    void* y, int ydt, const BulkGeom& geo, int grid, unsigned* status,
                                    cudaStream_t st) {
    if (M <= 1) return launch_mv_bulk_ppl<TX, PG, 1>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
    return launch_mv_bulk_ppl<TX, PG, 4>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
}


template <typename TX, bool PG>
static cudaError_t launch_mv_shot(const void* x, int M, int K, const int8_t* w, const float* sw, int N, int gs, void* y,
                                  int ydt, const ShotGeom& geo, int grid, int smem, unsigned* status, cudaStream_t st) {
    if (M == 1) return launch_shot_t<TX, PG, false, 1, true>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, smem, status, st);
    return launch_shot_t<TX, PG, false, 4, true>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, smem, status, st);
}

cudaError_t launch_mv_w8a16(const void* x, int xdt, int M, int K, const int8_t* w, const float* sw, int N, int gs,
                            void* y, int ydt, int num_sms, unsigned* status, cudaStream_t st) {
    // Per group, the one-shot kernel (A16 mode) where its plan fits (M = 1,
    // N = 2560, K = 10240 on B200: 11.1 / 11.7 us at gs = 128 / 64 against
    // 14.7 / 15.0 us for the register ring); per channel the register ring,
    // whose fp32 activation pairs are staged once (N = 10240, K = 2560: the
    // one-shot kernel, which widens the activations for every chunk, was
    // 1% faster timed alone but 10% slower within the full set of bench
    // rows, 10.5 against 9.6 us).  The test switch's 1 forces the ring, 4
    // the one-shot kernel for both; the bulk-staged kernel (11.3 us per
    // channel) runs when the switch selects it and its plan fits.
    BulkGeom geo;
    int grid = 0;
    const int sel = g_small_kernel.load();
    ShotGeom sg;
    int sgrid = 0, ssmem = 0;
    if ((sel == 0 || sel == 4) &&
        shot_plan(M, K, N, gs > 0, false, gs > 0 ? gs : 64, num_sms, sg, sgrid, ssmem, true)) {
        if (gs > 0) {
            if (xdt == 1) return launch_mv_shot<__nv_bfloat16, true>(x, M, K, w, sw, N, gs, y, ydt, sg, sgrid, ssmem, status, st);
            return launch_mv_shot<__half, true>(x, M, K, w, sw, N, gs, y, ydt, sg, sgrid, ssmem, status, st);
        }
        if (xdt == 1) return launch_mv_shot<__nv_bfloat16, false>(x, M, K, w, sw, N, 0, y, ydt, sg, sgrid, ssmem, status, st);
        return launch_mv_shot<__half, false>(x, M, K, w, sw, N, 0, y, ydt, sg, sgrid, ssmem, status, st);
    }
    if ((sel == 2 || sel == 3) && bulk_plan(M, K, N, gs > 0, false, gs, num_sms, geo, grid, true)) {
        if (gs > 0) {
            if (xdt == 1) return launch_mv_bulk_m<__nv_bfloat16, true>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
            return launch_mv_bulk_m<__half, true>(x, M, K, w, sw, N, gs, y, ydt, geo, grid, status, st);
        }
        if (xdt == 1) return launch_mv_bulk_m<__nv_bfloat16, false>(x, M, K, w, sw, N, 0, y, ydt, geo, grid, status, st);
        return launch_mv_bulk_m<__half, false>(x, M, K, w, sw, N, 0, y, ydt, geo, grid, status, st);
    }
    if (gs > 0) {
        if (xdt == 1) return launch_mv_reg<__nv_bfloat16, true>(x, M, K, w, sw, N, gs, y, ydt, num_sms, st);
        return launch_mv_reg<__half, true>(x, M, K, w, sw, N, gs, y, ydt, num_sms, st);
    }
    if (xdt == 1) return launch_mv_reg<__nv_bfloat16, false>(x, M, K, w, sw, N, 0, y, ydt, num_sms, st);
    return launch_mv_reg<__half, false>(x, M, K, w, sw, N, 0, y, ydt, num_sms, st);
}

cudaError_t set_small_m_kernel(int k) {
    if (k < 0 || k > 4) return cudaErrorInvalidValue;
    g_small_kernel.store(k);
    return cudaSuccess;
}

cudaError_t launch_small_m(int mode, const void* x, int xdt, int M, int K, const void* w,
                           const float* sw, int N, int gs, void* y, int ydt, int num_sms,
                           unsigned* status, cudaStream_t st) {
    switch (mode) {
        case kModePC: return launch_small_m_v<false, false>(x, xdt, M, K, w, sw, N, gs, y, ydt, num_sms, status, st);
        case kModePG: return launch_small_m_v<true, false>(x, xdt, M, K, w, sw, N, gs, y, ydt, num_sms, status, st);
        case kModeW4: return launch_small_m_v<true, true>(x, xdt, M, K, w, sw, N, gs, y, ydt, num_sms, status, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace cider
