// quantize.cu -- memory-bound kernels around the GEMM:
//  * per-token activation quantization (one pass over x: absmax, scale, codes);
//  * the fused SiLU(gate) * up -> quantize producer of a decoder MLP;
//  * offline weight quantization (per channel, per group, INT4 packed);
//  * the INT4 unpack of the W4A8 load path, as a standalone test kernel.
//
// Activation quantization follows the juejin post "在Mac上跑大模型，MLX 不是终点",
// section "W8A8 对称量化：Cider 的选择" (scale = max|x|/127, codes
// round(x/scale) clamped to [-128,127]); weight quantization the Cider README,
// section "底层 API" (quantize_weight_int8, pack_weight_int4) and table "量化".
//
// Layout: a token row is read with 16-byte vector loads (8 fp16/bf16 values),
// thread-strided so that each warp load covers 512 contiguous bytes; codes are
// written as 8-byte vectors.  Rows up to 12288 wide are spread over 32 to 256
// threads and stay in registers between the max and the quantize pass; wider
// rows go to one 256-thread CTA that re-reads the row.
#include "cider_device.cuh"
#include "cider_kernels.h"

namespace cider {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Quantize eight values with `scale` (reciprocal `rcp`) and store them as 8 bytes.
__device__ __forceinline__ void quant_store8(const float (&f)[8], float scale, float rcp, int8_t* dst) {
    *reinterpret_cast<uint2*>(dst) = quant8_codes(f, scale, rcp);
}

// ---- tpr threads per token row, row kept in registers -------------------
// A 256-thread CTA holds 256 / tpr rows (tpr = 32, 64, 128 or 256); thread j
// of a row loads the row's 16-byte chunks j, j + tpr, ... (at most NV of
// them), so each warp load still covers 512 contiguous bytes.  The row max
// is a warp shuffle reduction, then (tpr > 32) a shared-memory max over the
// row's warps.  The per-thread chain (loads, max, codes, stores) is short:
// the launcher picks tpr so that NV <= 6 and, for few rows, so that the grid
// still fills the GPU -- one row per warp with long chains was bound by the
// latency of that chain, not by memory.  (A persistent, software-pipelined
// version -- four CTAs per SM walking row groups, the next group's loads in
// flight while the current one is stored -- measured slower on B200: 10.7
// against 9.3 us at 4096 x 2560 and 60.1 against 49.9 us at 8192 x 10240;
// with every CTA resident at once the whole input is requested up front.)
template <typename T, int NV>
__global__ void __launch_bounds__(256) k_quantize_rows(const T* __restrict__ x, int64_t M, int K, int64_t ldx,
                                                       int tpr, int8_t* __restrict__ q, int64_t ldq,
                                                       float* __restrict__ sx) {
    __shared__ float red[8];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (256 / tpr) + tid / tpr;
    const int j = tid % tpr;
    const bool live = row < M;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (live ? row : 0) * ldx);
    const int nch = K >> 3;
    uint4 v[NV];
    // all loads of the thread in flight before any of them is used
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = j + tpr * i;
        v[i] = (live && c < nch) ? __ldcs(xr + c) : make_uint4(0, 0, 0, 0);
    }
    typename Pack2<T>::type m2 = {};
#pragma unroll
    for (int i = 0; i < NV; ++i) m2 = absmax8<T>(v[i], m2);
    float amax = warp_max(absmax_to_f32<T>(m2));
    if (tpr > 32) {  // uniform across the CTA
        if ((tid & 31) == 0) red[tid >> 5] = amax;
        __syncthreads();
        const int w0 = (tid / tpr) * (tpr >> 5);
        amax = red[w0];
        for (int w = 1; w < (tpr >> 5); ++w) amax = fmaxf(amax, red[w0 + w]);
    }
    if (!live) return;
    const float s = act_scale(amax);
    const float rs = act_rcp(s);
    if (j == 0) sx[row] = s;
    int8_t* qr = q + row * ldq;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = j + tpr * i;
        if (c < nch) {
            float f[8];
            unpack8_f32<T>(v[i], f);
            quant_store8(f, s, rs, qr + 8 * c);
        }
    }
}

// ---- one CTA (256 threads) per token row, any width -------------------------
// NV > 0: up to NV 16-byte chunks per thread stay in registers; NV == 0:
// any width, the quantize pass re-reads the row (L1/L2 hits).
template <typename T, int NV>
__global__ void __launch_bounds__(256) k_quantize_cta(const T* __restrict__ x, int K, int64_t ldx,
                                                      int8_t* __restrict__ q, int64_t ldq,
                                                      float* __restrict__ sx) {
    __shared__ float red[8];
    pdl_wait();
    pdl_trigger();
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x;
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * ldx);
    const int nch = K >> 3;
    constexpr int R = NV > 0 ? NV : 1;
    uint4 v[R];
    float amax = 0.0f;
    if (NV > 0) {
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int c = tid + 256 * i;
            v[i] = c < nch ? __ldcs(xr + c) : make_uint4(0, 0, 0, 0);
        }
        typename Pack2<T>::type m2 = {};
#pragma unroll
        for (int i = 0; i < R; ++i) m2 = absmax8<T>(v[i], m2);
        amax = absmax_to_f32<T>(m2);
    } else {
        for (int c = tid; c < nch; c += 256) {
            float f[8];
            unpack8_f32<T>(__ldg(xr + c), f);
#pragma unroll
            for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
        }
    }
    amax = warp_max(amax);
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float s = act_scale(amax);
    const float rs = act_rcp(s);
    if (tid == 0) sx[row] = s;
    int8_t* qr = q + row * ldq;
    if (NV > 0) {
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int c = tid + 256 * i;
            if (c < nch) {
                float f[8];
                unpack8_f32<T>(v[i], f);
                quant_store8(f, s, rs, qr + 8 * c);
            }
        }
    } else {
        for (int c = tid; c < nch; c += 256) {
            float f[8];
            unpack8_f32<T>(__ldg(xr + c), f);
            quant_store8(f, s, rs, qr + 8 * c);
        }
    }
}

template <typename T>
static cudaError_t launch_quantize_t(const void* x, int64_t M, int K, int64_t ldx, int8_t* q, int64_t ldq, float* sx,
                                     int num_sms, cudaStream_t st) {
    const T* xt = static_cast<const T*>(x);
    if (M == 0) return cudaSuccess;
    const int nch = K / 8;
    if (nch > 6 * 256) {  // wider than 12288: one CTA per row, re-reading the row
        return launch_pdl(k_quantize_cta<T, 0>, static_cast<unsigned>(M), 256, 0, st, xt, K, ldx, q, ldq, sx);
    }
    // threads per row: the fewest with <= 6 chunks each, then more while the
    // rows would give fewer than ~4 warps per SM sub-partition
    int tpr = 32;
    while (tpr < 256 && (nch + tpr - 1) / tpr > 6) tpr *= 2;
    while (tpr < 256 && M * tpr < 148LL * 512 && nch >= 2 * tpr) tpr *= 2;
    const int nv = (nch + tpr - 1) / tpr;
    (void)num_sms;
    const unsigned grid = static_cast<unsigned>((M * tpr + 255) / 256);
    switch (nv) {
        case 1: return launch_pdl(k_quantize_rows<T, 1>, grid, 256, 0, st, xt, M, K, ldx, tpr, q, ldq, sx);
        case 2: return launch_pdl(k_quantize_rows<T, 2>, grid, 256, 0, st, xt, M, K, ldx, tpr, q, ldq, sx);
        case 3: return launch_pdl(k_quantize_rows<T, 3>, grid, 256, 0, st, xt, M, K, ldx, tpr, q, ldq, sx);
        case 4: return launch_pdl(k_quantize_rows<T, 4>, grid, 256, 0, st, xt, M, K, ldx, tpr, q, ldq, sx);
        case 5: return launch_pdl(k_quantize_rows<T, 5>, grid, 256, 0, st, xt, M, K, ldx, tpr, q, ldq, sx);
        default: return launch_pdl(k_quantize_rows<T, 6>, grid, 256, 0, st, xt, M, K, ldx, tpr, q, ldq, sx);
    }
}

cudaError_t launch_quantize_act(const void* x, int xdt, int64_t M, int K, int64_t ldx, int8_t* q, int64_t ldq,
                                float* sx, int num_sms, cudaStream_t st) {
    return xdt == 1 ? launch_quantize_t<__nv_bfloat16>(x, M, K, ldx, q, ldq, sx, num_sms, st)
                    : launch_quantize_t<__half>(x, M, K, ldx, q, ldq, sx, num_sms, st);
}

// ---- SiLU(gate) * up -> quantize, one CTA per token row ---------------------
// a = round_T(silu(g) * u) in fp32 with silu(g) = g * sigmoid(g); the codes
// are taken from the rounded a, exactly as quantizing a stored `a` would.
template <typename T, int NV>
__global__ void __launch_bounds__(256) k_silu_mul_quantize(const T* __restrict__ gate,
                                                           const T* __restrict__ up, int F,
                                                           int8_t* __restrict__ q,
                                                           float* __restrict__ sx,
                                                           T* __restrict__ a_out) {
    __shared__ float red[8];
    pdl_wait();
    pdl_trigger();
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x;
    const uint4* gr = reinterpret_cast<const uint4*>(gate + row * F);
    const uint4* ur = reinterpret_cast<const uint4*>(up + row * F);
    const int nch = F >> 3;
    uint4 av[NV];
    float amax = 0.0f;
    uint4 gv[NV], uv[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = tid + 256 * i;
        gv[i] = c < nch ? __ldcs(gr + c) : make_uint4(0, 0, 0, 0);
        uv[i] = c < nch ? __ldcs(ur + c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = tid + 256 * i;
        if (c < nch) {
            float g[8], u[8];
            unpack8_f32<T>(gv[i], g);
            unpack8_f32<T>(uv[i], u);
            T* ah = reinterpret_cast<T*>(&av[i]);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                // sigmoid(g) = 1/(1+e^-g) for g >= 0 and e^g/(1+e^g) for g < 0:
                // e^-|g| never overflows, so large negative g keep their tiny value.
                // The quotient's denominator lies in [1, 2], where __fdividef is
                // within 2 ulp of fp32: far below the one unit of fp16/bf16 that
                // a is rounded to (the IEEE division cost more than the rest of
                // the element's work).
                const float e = expf(-fabsf(g[j]));
                const float sig = __fdividef(g[j] >= 0.0f ? 1.0f : e, 1.0f + e);
                ah[j] = from_f32<T>((g[j] * sig) * u[j]);
                amax = fmaxf(amax, fabsf(to_f32<T>(ah[j])));
            }
            if (a_out) reinterpret_cast<uint4*>(a_out + row * F)[c] = av[i];
        }
    }
    amax = warp_max(amax);
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float s = act_scale(amax);
    const float rs = act_rcp(s);
    if (tid == 0) sx[row] = s;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = tid + 256 * i;
        if (c < nch) {
            float f[8];
            unpack8_f32<T>(av[i], f);
            quant_store8(f, s, rs, q + row * F + 8 * c);
        }
    }
}

template <typename T>
static cudaError_t launch_silu_t(const void* g, const void* u, int64_t M, int F, int8_t* q,
                                 float* sx, void* a_out, cudaStream_t st) {
    if (M == 0) return cudaSuccess;
    const int nv = (F / 8 + 255) / 256;
    const T* gt = static_cast<const T*>(g);
    const T* ut = static_cast<const T*>(u);
    T* at = static_cast<T*>(a_out);
    const unsigned grid = static_cast<unsigned>(M);
    if (nv <= 2) return launch_pdl(k_silu_mul_quantize<T, 2>, grid, 256, 0, st, gt, ut, F, q, sx, at);
    else if (nv <= 4) return launch_pdl(k_silu_mul_quantize<T, 4>, grid, 256, 0, st, gt, ut, F, q, sx, at);
    else if (nv <= 6) return launch_pdl(k_silu_mul_quantize<T, 6>, grid, 256, 0, st, gt, ut, F, q, sx, at);
    else if (nv <= 8) return launch_pdl(k_silu_mul_quantize<T, 8>, grid, 256, 0, st, gt, ut, F, q, sx, at);
    else if (nv <= 16) return launch_pdl(k_silu_mul_quantize<T, 16>, grid, 256, 0, st, gt, ut, F, q, sx, at);
    return cudaErrorInvalidValue;  // F > 32768: rejected by the host checks first
}

cudaError_t launch_silu_mul_quantize(const void* g, const void* u, int dt, int64_t M, int F,
                                     int8_t* q, float* sx, void* a_out, cudaStream_t st) {
    return dt == 1 ? launch_silu_t<__nv_bfloat16>(g, u, M, F, q, sx, a_out, st)
                   : launch_silu_t<__half>(g, u, M, F, q, sx, a_out, st);
}

// ---- offline weight quantization --------------------------------------------
// Per channel: one CTA per output row, two passes (max, then codes).
__global__ void __launch_bounds__(256) k_quantize_weight_pc(const float* __restrict__ W, int K,
                                                            int8_t* __restrict__ w,
                                                            float* __restrict__ sw) {
    __shared__ float red[8];
    pdl_wait();
    pdl_trigger();
    const int64_t n = blockIdx.x;
    const float* wr = W + n * K;
    float amax = 0.0f;
    for (int k = threadIdx.x; k < K; k += 256) amax = fmaxf(amax, fabsf(wr[k]));
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    const float s = act_scale(amax);
    if (threadIdx.x == 0) sw[n] = s;
    for (int k = threadIdx.x; k < K; k += 256) w[n * K + k] = static_cast<int8_t>(quant_code(wr[k], s));
}

// INT4 per output channel: one CTA per row; scale = max|W[n,:]| / 7, codes
// clamp(round(W / scale), -8, 7) stored as q + 8, even k in the low nibble.
__global__ void __launch_bounds__(256) k_pack_weight_int4_pc(const float* __restrict__ W, int K,
                                                             uint8_t* __restrict__ out, float* __restrict__ sw) {
    __shared__ float red[8];
    pdl_wait();
    pdl_trigger();
    const int64_t n = blockIdx.x;
    const float* wr = W + n * K;
    float amax = 0.0f;
    for (int k = threadIdx.x; k < K; k += 256) amax = fmaxf(amax, fabsf(wr[k]));
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    const float s = __fdiv_rn(amax, 7.0f);
    if (threadIdx.x == 0) sw[n] = s;
    uint8_t* p = out + n * (K / 2);
    for (int j = threadIdx.x; j < K / 2; j += 256) {
        int c0 = 0, c1 = 0;
        if (s != 0.0f) {
            c0 = static_cast<int>(fminf(fmaxf(roundf(__fdiv_rn(wr[2 * j], s)), -8.0f), 7.0f));
            c1 = static_cast<int>(fminf(fmaxf(roundf(__fdiv_rn(wr[2 * j + 1], s)), -8.0f), 7.0f));
        }
        p[j] = static_cast<uint8_t>((c0 + 8) | ((c1 + 8) << 4));
    }
}

// Per group (INT8 or INT4): one warp per kWeightGroupsPerWarp consecutive
// groups of a row.  Lane l holds elements 2l and 2l + 1 of every 64-wide part
// of a group (2 * PPL values, gs = 64 * PPL), so its INT4 byte packs its own
// pair; all the groups' loads go out before the first maximum, so a warp has
// a few KB in flight.  Scales group-major [G][N].
constexpr int kWeightGroupsPerWarp = 4;
template <bool INT4, int PPL>
__global__ void __launch_bounds__(256) k_quantize_weight_group(const float* __restrict__ W,
                                                               int64_t N, int K,
                                                               void* __restrict__ out,
                                                               float* __restrict__ sw) {
    pdl_wait();
    pdl_trigger();
    constexpr int GS = 64 * PPL;
    constexpr int GPW = kWeightGroupsPerWarp;
    const int64_t item = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int G = K / GS;
    const int wpr = (G + GPW - 1) / GPW;  // warps per row
    if (item >= N * wpr) return;  // whole warps
    const int64_t n = item / wpr;
    const int g0 = static_cast<int>(item % wpr) * GPW;
    float x[GPW][2 * PPL];
#pragma unroll
    for (int h = 0; h < GPW; ++h)
        if (g0 + h < G) {
            const float* wg = W + n * K + static_cast<int64_t>(g0 + h) * GS;
#pragma unroll
            for (int i = 0; i < PPL; ++i) {
                x[h][2 * i] = wg[2 * lane + 64 * i];
                x[h][2 * i + 1] = wg[2 * lane + 1 + 64 * i];
            }
        }
#pragma unroll
    for (int h = 0; h < GPW; ++h) {
        const int g = g0 + h;
        if (g >= G) break;  // warp-uniform
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 2 * PPL; ++i) amax = fmaxf(amax, fabsf(x[h][i]));
        amax = warp_max(amax);
        const float s = INT4 ? __fdiv_rn(amax, 7.0f) : act_scale(amax);
        if (lane == 0) sw[static_cast<int64_t>(g) * N + n] = s;
        if (!INT4) {
            int8_t* w = static_cast<int8_t*>(out) + n * K + static_cast<int64_t>(g) * GS;
#pragma unroll
            for (int i = 0; i < PPL; ++i) {
                w[2 * lane + 64 * i] = static_cast<int8_t>(quant_code(x[h][2 * i], s));
                w[2 * lane + 1 + 64 * i] = static_cast<int8_t>(quant_code(x[h][2 * i + 1], s));
            }
        } else {
            uint8_t* p = static_cast<uint8_t*>(out) + n * (K / 2) + static_cast<int64_t>(g) * (GS / 2);
#pragma unroll
            for (int i = 0; i < PPL; ++i) {
                int c0 = 0, c1 = 0;
                if (s != 0.0f) {
                    c0 = static_cast<int>(fminf(fmaxf(roundf(__fdiv_rn(x[h][2 * i], s)), -8.0f), 7.0f));
                    c1 = static_cast<int>(fminf(fmaxf(roundf(__fdiv_rn(x[h][2 * i + 1], s)), -8.0f), 7.0f));
                }
                p[lane + 32 * i] = static_cast<uint8_t>((c0 + 8) | ((c1 + 8) << 4));
            }
        }
    }
}

cudaError_t launch_quantize_weight(int mode, const float* W, int64_t N, int K, int gs, void* out,
                                   float* sw, cudaStream_t st) {
    if (mode == 0)
        return launch_pdl(k_quantize_weight_pc, static_cast<unsigned>(N), 256, 0, st, W, K, static_cast<int8_t*>(out), sw);
    if (mode == 3)
        return launch_pdl(k_pack_weight_int4_pc, static_cast<unsigned>(N), 256, 0, st, W, K, static_cast<uint8_t*>(out), sw);
    const int64_t warps = N * ((K / gs + kWeightGroupsPerWarp - 1) / kWeightGroupsPerWarp);
    const unsigned grid = static_cast<unsigned>((warps + 7) / 8);
    if (gs != 64 && gs != 128) return cudaErrorInvalidValue;  // rejected by the host checks first
    if (mode == 1)
        return gs == 64 ? launch_pdl(k_quantize_weight_group<false, 1>, grid, 256, 0, st, W, N, K, out, sw)
                        : launch_pdl(k_quantize_weight_group<false, 2>, grid, 256, 0, st, W, N, K, out, sw);
    return gs == 64 ? launch_pdl(k_quantize_weight_group<true, 1>, grid, 256, 0, st, W, N, K, out, sw)
                    : launch_pdl(k_quantize_weight_group<true, 2>, grid, 256, 0, st, W, N, K, out, sw);
}

// ---- percentile-clipped weight scales (clip_percentile) ----------------------
// Cider README, section "说明": besides min-max, the conversion can take its
// scales from a percentile of the weights (clip_percentile = 99.9).  Per slab
// (an output row, or one group of gs along K): c = the p-th percentile of
// |w|, linearly interpolated between the order statistics k0 and k0 + 1 with
// weight t (k0 and t come from the host); scale = c / 127; codes
// clamp(round(w / scale), -127, 127).  A zero percentile takes c = max|w|.
//
// The order statistics are found bit by bit from the top: the k-th smallest
// magnitude is the largest pattern r with at most k magnitudes below it
// (|x| as an unsigned bit pattern orders like |x|).  Each of the 31 counting
// passes (bit 31 of |x| is 0) counts for both statistics at once.  Exact for
// any slab length.  A row of up to 4096 weights is held in registers for the
// passes; a longer one is read through L1 each pass.

__device__ __forceinline__ float clip_value(uint32_t r0, uint32_t r1, bool two, float t, float amax) {
    const float a = __uint_as_float(r0);
    const float v = two ? __fadd_rn(a, __fmul_rn(t, __fsub_rn(__uint_as_float(r1), a))) : a;
    return v == 0.0f ? amax : v;
}
__device__ __forceinline__ int8_t clip_code(float x, float s) {
    return static_cast<int8_t>(max(quant_code(x, s), -127));
}
// clip_code without the division.  With r = 1/s correctly rounded, t = x * r
// lies within a relative 1.5 * 2^-23 of the correctly rounded quotient (three
// roundings of at most 2^-24 each), i.e. within 2^-15 of it below 128.  So
// wherever t is more than 2^-14 from a halfway point k + 1/2 below 127.5,
// rint(t) (taken by adding 1.5 * 2^23, as in quant8_codes) is the code, and
// halfway points never reach this path, so ties-to-even and round-half-away
// cannot differ.  Beyond 127.5 + 2^-14 every rounding of the quotient
// saturates at +-127.  Anything else -- a near tie, s = 0, a NaN -- takes the
// exact clip_code.
__device__ __forceinline__ int8_t clip_code_fast(float x, float s, float r) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    constexpr float kMargin = 0x1p-14f;
    const float t = __fmul_rn(x, r);
    const float at = fabsf(t);
    if (at < 127.5f - kMargin) {
        const float v = __fadd_rn(t, kMagic);
        const float d = __fsub_rn(t, __fsub_rn(v, kMagic));
        if (fabsf(d) < 0.5f - kMargin) return static_cast<int8_t>(static_cast<int>(__fsub_rn(v, kMagic)));
    } else if (at > 127.5f + kMargin && s != 0.0f) {
        return static_cast<int8_t>(t > 0.0f ? 127 : -127);
    }
    return clip_code(x, s);
}

// High percentiles (the pages' 99.9) sit a few ranks below the maximum.  With
// j = len - 1 - k0 the rank of the first statistic counted from the top, a
// slab with j <= kClipTop is walked down through its distinct magnitudes
// instead: the largest magnitude below the previous one, then how many
// elements equal it, until the run of equal values that holds rank j.  That
// takes at most j + 1 steps of two reductions (every step passes at least
// one element) and gives the same order statistics, ties included; rank
// j - 1 (the second statistic) is in the same run or is the previous value.
constexpr int kClipTop = 12;

// 256-thread block reductions: warp redux, then the 8 warps' values through
// shared memory.  Two buffers alternate, so a call's writes never meet the
// previous call's reads (the barrier of the call between them orders them).
__device__ __forceinline__ uint32_t clip_block_max(uint32_t v, uint32_t (&buf)[2][8], int& par) {
    v = __reduce_max_sync(0xffffffffu, v);
    if ((threadIdx.x & 31) == 0) buf[par][threadIdx.x >> 5] = v;
    __syncthreads();
    uint32_t r = buf[par][0];
#pragma unroll
    for (int i = 1; i < 8; ++i) r = max(r, buf[par][i]);
    par ^= 1;
    return r;
}
__device__ __forceinline__ uint32_t clip_block_sum(uint32_t v, uint32_t (&buf)[2][8], int& par) {
    v = __reduce_add_sync(0xffffffffu, v);
    if ((threadIdx.x & 31) == 0) buf[par][threadIdx.x >> 5] = v;
    __syncthreads();
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) r += buf[par][i];
    par ^= 1;
    return r;
}
__device__ __forceinline__ uint32_t mag_bits(float x) { return __float_as_uint(x) & 0x7FFFFFFFu; }

// The order statistics r0 = k0-th and r1 = (k0+1)-th smallest magnitude of a
// slab of `len` values held by one warp.  `each(f)` calls f(u, q) for every
// valid magnitude pattern u the lane holds, q in [0, 4) spreading them over
// four independent accumulators (one chain of dependent max / add operations
// per accumulator instead of one for the whole lane).
template <typename Each>
__device__ __forceinline__ void warp_select2(int len, int k0, Each&& each, uint32_t& r0, uint32_t& r1) {
    r0 = r1 = 0;
    const int j = len - 1 - k0;
    if (j <= kClipTop) {
        // the maximum, then per step one pass for both the count of the
        // current value m and the largest magnitude below it
        uint32_t lm[4] = {0, 0, 0, 0};
        each([&](uint32_t u, int q) { lm[q] = max(lm[q], u); });
        uint32_t m = __reduce_max_sync(0xffffffffu, max(max(lm[0], lm[1]), max(lm[2], lm[3])));
        int above = 0;  // elements above m
        uint32_t prev = 0;
        for (int it = 0; it <= kClipTop; ++it) {
            uint32_t lc[4] = {0, 0, 0, 0}, lb[4] = {0, 0, 0, 0};
            each([&](uint32_t u, int q) {
                lc[q] += u == m;
                if (u < m) lb[q] = max(lb[q], u);
            });
            const int c = static_cast<int>(__reduce_add_sync(0xffffffffu, (lc[0] + lc[1]) + (lc[2] + lc[3])));
            const uint32_t below = __reduce_max_sync(0xffffffffu, max(max(lb[0], lb[1]), max(lb[2], lb[3])));
            if (j < above + c) {
                r0 = m;
                r1 = (j >= 1 && j - 1 < above) ? prev : m;
                return;
            }
            above += c;
            prev = m;
            m = below;
        }
    } else {
        for (int b = 30; b >= 0; --b) {
            const uint32_t t0 = r0 | (1u << b), t1 = r1 | (1u << b);
            uint32_t c0[4] = {0, 0, 0, 0}, c1[4] = {0, 0, 0, 0};
            each([&](uint32_t u, int q) {
                c0[q] += u < t0;
                c1[q] += u < t1;
            });
            const uint32_t n0 = __reduce_add_sync(0xffffffffu, (c0[0] + c0[1]) + (c0[2] + c0[3]));
            const uint32_t n1 = __reduce_add_sync(0xffffffffu, (c1[0] + c1[1]) + (c1[2] + c1[3]));
            if (static_cast<int>(n0) <= k0) r0 = t0;
            if (static_cast<int>(n1) <= k0 + 1) r1 = t1;
        }
    }
}

// Per channel, rows of K <= 32 * VPL weights with K % 4 == 0 (16-byte aligned
// rows): one warp per output row, the row in registers (lane l holds the
// 16-byte chunks l, l + 32, ...), every reduction a warp redux -- no block
// barriers, and eight rows per 256-thread CTA in flight at once.
template <int VPL>
__global__ void __launch_bounds__(256) k_quantize_weight_pc_clip_warp(const float* __restrict__ W, int64_t N, int K,
                                                                      int k0, float t, int8_t* __restrict__ w,
                                                                      float* __restrict__ sw) {
    static_assert(VPL % 4 == 0, "whole 16-byte chunks per lane");
    pdl_wait();
    pdl_trigger();
    const int64_t n = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (n >= N) return;  // whole warps
    const float* wr = W + n * K;
    float x[VPL];
#pragma unroll
    for (int i = 0; i < VPL / 4; ++i) {
        const int k = 4 * (lane + 32 * i);
        float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (k < K) v = __ldg(reinterpret_cast<const float4*>(wr + k));
        x[4 * i] = v.x;
        x[4 * i + 1] = v.y;
        x[4 * i + 2] = v.z;
        x[4 * i + 3] = v.w;
    }
    float am[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < VPL / 4; ++i)
        if (4 * (lane + 32 * i) < K)
#pragma unroll
            for (int c = 0; c < 4; ++c) am[c] = fmaxf(am[c], fabsf(x[4 * i + c]));
    const float amax = warp_max(fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3])));
    auto each = [&](auto&& f) {
#pragma unroll
        for (int i = 0; i < VPL / 4; ++i)
            if (4 * (lane + 32 * i) < K)  // K % 4 == 0: a chunk is wholly inside the row or wholly past it
#pragma unroll
                for (int c = 0; c < 4; ++c) f(mag_bits(x[4 * i + c]), c);
    };
    uint32_t r0, r1;
    warp_select2(K, k0, each, r0, r1);
    const float c = clip_value(r0, r1, t != 0.0f && k0 + 1 < K, t, amax);
    const float s = act_scale(c);
    const float r = __frcp_rn(s);
    if (lane == 0) sw[n] = s;
#pragma unroll
    for (int i = 0; i < VPL / 4; ++i) {
        const int k = 4 * (lane + 32 * i);
        if (k < K) {
            const uint32_t b0 = static_cast<uint8_t>(clip_code_fast(x[4 * i], s, r));
            const uint32_t b1 = static_cast<uint8_t>(clip_code_fast(x[4 * i + 1], s, r));
            const uint32_t b2 = static_cast<uint8_t>(clip_code_fast(x[4 * i + 2], s, r));
            const uint32_t b3 = static_cast<uint8_t>(clip_code_fast(x[4 * i + 3], s, r));
            *reinterpret_cast<uint32_t*>(w + n * K + k) = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
        }
    }
}

// This thread's elements of a row (k = tid, tid + 256, ...): held in
// registers when VPT > 0 (K <= 256 * VPT), else read through L1 each time.
template <int VPT, typename F>
__device__ __forceinline__ void clip_each(const float* wr, int K, const float (&x)[VPT > 0 ? VPT : 1], F&& f) {
    if constexpr (VPT > 0) {
#pragma unroll
        for (int i = 0; i < VPT; ++i)
            if (static_cast<int>(threadIdx.x) + 256 * i < K) f(x[i]);
    } else {
        for (int k = threadIdx.x; k < K; k += 256) f(__ldg(wr + k));
    }
}

// Per channel: one CTA of 256 threads per output row.
template <int VPT>
__global__ void __launch_bounds__(256) k_quantize_weight_pc_clip(const float* __restrict__ W, int K, int k0,
                                                                 float t, int8_t* __restrict__ w,
                                                                 float* __restrict__ sw) {
    __shared__ uint32_t buf[2][8];
    __shared__ int red[2][8][2];
    __shared__ float redm[8];
    pdl_wait();
    pdl_trigger();
    const int64_t n = blockIdx.x;
    const float* wr = W + n * K;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    float x[VPT > 0 ? VPT : 1];
    if constexpr (VPT > 0) {
#pragma unroll
        for (int i = 0; i < VPT; ++i) x[i] = tid + 256 * i < K ? wr[tid + 256 * i] : 0.0f;
    }
    float amax = 0.0f;
    clip_each<VPT>(wr, K, x, [&](float v) { amax = fmaxf(amax, fabsf(v)); });
    amax = warp_max(amax);
    if (lane == 0) redm[wp] = amax;
    __syncthreads();
    amax = redm[0];
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, redm[i]);
    uint32_t r0 = 0, r1 = 0;
    const int j = K - 1 - k0;
    if (j <= kClipTop) {
        int par = 0, above = 0;  // elements at or above the current value
        uint32_t thr = 0xFFFFFFFFu, prev = 0;
        for (int it = 0; it <= kClipTop; ++it) {
            uint32_t lm = 0;
            clip_each<VPT>(wr, K, x, [&](float v) {
                const uint32_t u = mag_bits(v);
                if (u < thr) lm = max(lm, u);
            });
            const uint32_t m = clip_block_max(lm, buf, par);
            uint32_t lc = 0;
            clip_each<VPT>(wr, K, x, [&](float v) { lc += mag_bits(v) == m; });
            const int c = static_cast<int>(clip_block_sum(lc, buf, par));
            if (j < above + c) {
                r0 = m;
                r1 = (j >= 1 && j - 1 < above) ? prev : m;
                break;
            }
            above += c;
            prev = m;
            thr = m;
        }
    } else {
        for (int b = 30; b >= 0; --b) {
            const uint32_t t0 = r0 | (1u << b), t1 = r1 | (1u << b);
            int c0 = 0, c1 = 0;
            clip_each<VPT>(wr, K, x, [&](float v) {
                const uint32_t u = mag_bits(v);
                c0 += u < t0;
                c1 += u < t1;
            });
            c0 = __reduce_add_sync(0xffffffffu, c0);
            c1 = __reduce_add_sync(0xffffffffu, c1);
            // two buffers: a pass's writes never meet the previous pass's reads
            int(*rb)[2] = red[b & 1];
            if (lane == 0) {
                rb[wp][0] = c0;
                rb[wp][1] = c1;
            }
            __syncthreads();
            c0 = c1 = 0;
            for (int i = 0; i < 8; ++i) {
                c0 += rb[i][0];
                c1 += rb[i][1];
            }
            if (c0 <= k0) r0 = t0;
            if (c1 <= k0 + 1) r1 = t1;
        }
    }
    const float c = clip_value(r0, r1, t != 0.0f && k0 + 1 < K, t, amax);
    const float s = act_scale(c);
    const float rs = __frcp_rn(s);
    if (tid == 0) sw[n] = s;
    if constexpr (VPT > 0) {
#pragma unroll
        for (int i = 0; i < VPT; ++i)
            if (tid + 256 * i < K) w[n * K + tid + 256 * i] = clip_code_fast(x[i], s, rs);
    } else {
        for (int k = tid; k < K; k += 256) w[n * K + k] = clip_code_fast(wr[k], s, rs);
    }
}

// Per group: one warp per GPW consecutive groups of a row (group g of row n
// and the next ones), each group's gs = 32 * VPL magnitudes held in
// registers; all the groups' loads go out before the first selection, so a
// warp has GPW * gs * 4 bytes in flight.  Scales group-major [G][N].
constexpr int kClipGroupsPerWarp = 4;
template <int VPL>
__global__ void __launch_bounds__(256) k_quantize_weight_pg_clip(const float* __restrict__ W, int64_t N, int K,
                                                                 int k0, float t, int8_t* __restrict__ out,
                                                                 float* __restrict__ sw) {
    pdl_wait();
    pdl_trigger();
    constexpr int GS = 32 * VPL;
    constexpr int GPW = kClipGroupsPerWarp;
    const int64_t item = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int G = K / GS;
    const int wpr = (G + GPW - 1) / GPW;  // warps per row
    if (item >= N * wpr) return;  // whole warps
    const int64_t n = item / wpr;
    const int g0 = static_cast<int>(item % wpr) * GPW;
    float x[GPW][VPL];
#pragma unroll
    for (int h = 0; h < GPW; ++h)
        if (g0 + h < G) {
            const float* wg = W + n * K + static_cast<int64_t>(g0 + h) * GS;
#pragma unroll
            for (int i = 0; i < VPL; ++i) x[h][i] = wg[lane + 32 * i];
        }
#pragma unroll
    for (int h = 0; h < GPW; ++h) {
        const int g = g0 + h;
        if (g >= G) break;  // warp-uniform
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < VPL; ++i) amax = fmaxf(amax, fabsf(x[h][i]));
        amax = warp_max(amax);
        auto each = [&](auto&& f) {
#pragma unroll
            for (int i = 0; i < VPL; ++i) f(mag_bits(x[h][i]), i & 3);
        };
        uint32_t r0, r1;
        warp_select2(GS, k0, each, r0, r1);
        const float c = clip_value(r0, r1, t != 0.0f && k0 + 1 < GS, t, amax);
        const float s = act_scale(c);
        const float rs = __frcp_rn(s);
        if (lane == 0) sw[static_cast<int64_t>(g) * N + n] = s;
        int8_t* w = out + n * K + static_cast<int64_t>(g) * GS;
#pragma unroll
        for (int i = 0; i < VPL; ++i) w[lane + 32 * i] = clip_code_fast(x[h][i], s, rs);
    }
}

cudaError_t launch_quantize_weight_clip(const float* W, int64_t N, int K, int gs, int k0, float t, int8_t* out,
                                        float* sw, cudaStream_t st) {
    const bool vec = K % 4 == 0 && (reinterpret_cast<uintptr_t>(W) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(out) & 3) == 0;
    if (gs == 0 && vec && K <= 32 * 128) {
        const unsigned grid = static_cast<unsigned>((N + 7) / 8);  // a warp per row
        if (K <= 32 * 64)
            return launch_pdl(k_quantize_weight_pc_clip_warp<64>, grid, 256, 0, st, W, N, K, k0, t, out, sw);
        if (K <= 32 * 80)
            return launch_pdl(k_quantize_weight_pc_clip_warp<80>, grid, 256, 0, st, W, N, K, k0, t, out, sw);
        return launch_pdl(k_quantize_weight_pc_clip_warp<128>, grid, 256, 0, st, W, N, K, k0, t, out, sw);
    }
    if (gs == 0 && K <= 256 * 16)
        return launch_pdl(k_quantize_weight_pc_clip<16>, static_cast<unsigned>(N), 256, 0, st, W, K, k0, t, out, sw);
    if (gs == 0)
        return launch_pdl(k_quantize_weight_pc_clip<0>, static_cast<unsigned>(N), 256, 0, st, W, K, k0, t, out, sw);
    const int64_t items = N * ((K / gs + kClipGroupsPerWarp - 1) / kClipGroupsPerWarp);  // warps
    const unsigned grid = static_cast<unsigned>((items + 7) / 8);
    if (gs == 64) return launch_pdl(k_quantize_weight_pg_clip<2>, grid, 256, 0, st, W, N, K, k0, t, out, sw);
    if (gs == 128) return launch_pdl(k_quantize_weight_pg_clip<4>, grid, 256, 0, st, W, N, K, k0, t, out, sw);
    return cudaErrorInvalidValue;  // rejected by the host checks first
}

// ---- INT4 unpack (the W4A8 load path's conversion), standalone ---------------
__global__ void k_unpack_int4(const uint32_t* __restrict__ packed, int64_t words, uint2* __restrict__ w) {
    pdl_wait();
    pdl_trigger();
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < words) w[i] = unpack_int4x8(packed[i]);
}

cudaError_t launch_unpack_int4(const uint8_t* packed, int64_t N, int K, int8_t* w, cudaStream_t st) {
    const int64_t words = N * (K / 8);  // K % 32 == 0 keeps rows whole words
    if (words == 0) return cudaSuccess;
    return launch_pdl(k_unpack_int4, static_cast<unsigned>((words + 255) / 256), 256, 0, st,
                      reinterpret_cast<const uint32_t*>(packed), words, reinterpret_cast<uint2*>(w));
}

// ---- self-test of the bounded wait ------------------------------------------
// One warp waits on an mbarrier that nothing ever arrives on; the wait must
// give up after limit_ns and record the timeout in the status word.
__global__ void k_wait_selftest(unsigned* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait_for(&bar, 0, status, &abort_flag, limit_ns);
}

cudaError_t launch_wait_selftest(unsigned* status, unsigned long long limit_ns, cudaStream_t st) {
    k_wait_selftest<<<1, 32, 0, st>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace cider
