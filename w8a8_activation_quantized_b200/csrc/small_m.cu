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
// Work split.  The grid is persistent (two CTAs per SM): each CTA quantizes
// the M activation rows once into shared memory, then walks blocks of R
// output channels.  Its 8 warps form R rows x S K-slices (R*S = 8).  A weight
// row is read as 16-byte chunks (16 int8 weights, or 32 packed int4 weights);
// 32 lanes read 32 consecutive chunks per "pass" (512 or 1024 k values), and
// a warp's slice is a whole number of passes, so a weight group (64 or 128
// values) never straddles warps.  Each warp issues all loads of its slice
// before using any (up to kMaxPass passes), and loads the next block's slice
// while it computes the current one.  Per-group: the lanes of one group reduce
// its INT32 partial with shuffles and one lane rescales it by scale_w[g][n]
// in fp32.  Slices combine through shared memory.
#include "cider_device.cuh"
#include "cider_kernels.h"

namespace cider {

constexpr int kSmallThreads = 256;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kMaxPass = 8;  // passes of 32 chunks a warp keeps in flight

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
    int S, R;          // K-slices per row, rows per block (R * S = 8)
    int ppw;           // passes per warp slice
    int nblocks;       // row blocks
};

template <typename TX, typename TY, bool PG, bool W4, int MAXM>
__global__ void __launch_bounds__(kSmallThreads) k_small_m(const TX* __restrict__ x, int M, int K,
                                                           const uint8_t* __restrict__ w,
                                                           const float* __restrict__ sw, int N,
                                                           int gs, TY* __restrict__ y, SmallGeom geo) {
    extern __shared__ __align__(16) int8_t s_q[];  // [M][K] codes
    __shared__ float s_sx[MAXM];
    __shared__ float s_part[kSmallWarps][MAXM];  // per-warp partials (int32 bits for per-channel)
    constexpr int KC = W4 ? 32 : 16;            // weights per 16-byte chunk
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row_bytes = W4 ? K / 2 : K;
    const int nch = K / KC;
    const int r_in_blk = warp / geo.S, slice = warp % geo.S;
    const int pass0 = slice * geo.ppw;

    uint4 cur[kMaxPass], nxt[kMaxPass];
    auto load = [&](uint4 (&dst)[kMaxPass], int blk) {
        const int n = blk * geo.R + r_in_blk;
        const uint4* wr = reinterpret_cast<const uint4*>(w + static_cast<int64_t>(n) * row_bytes);
#pragma unroll
        for (int p = 0; p < kMaxPass; ++p) {
            const int c = (pass0 + p) * 32 + lane;
            dst[p] = (p < geo.ppw && blk < geo.nblocks && n < N && c < nch) ? __ldcs(wr + c) : make_uint4(0, 0, 0, 0);
        }
    };
    int blk = blockIdx.x;
    load(cur, blk);

    // Quantize the M activation rows into shared memory (one warp per row).
    for (int m = warp; m < M; m += kSmallWarps) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K);
        float amax = 0.0f;
        for (int c = lane; c < K / 8; c += 32) {
            float f[8];
            unpack8_f32<TX>(__ldg(xr + c), f);
#pragma unroll
            for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = act_scale(amax);
        const float rs = act_rcp(s);
        if (lane == 0) s_sx[m] = s;
        for (int c = lane; c < K / 8; c += 32) {
            float f[8];
            unpack8_f32<TX>(__ldg(xr + c), f);
            *reinterpret_cast<uint2*>(s_q + static_cast<int64_t>(m) * K + 8 * c) = quant8_codes(f, s, rs);
        }
    }
    __syncthreads();

    const int lpg = PG ? gs / KC : 32;  // lanes per group: 2, 4 or 8
    for (; blk < geo.nblocks; blk += gridDim.x) {
        load(nxt, blk + gridDim.x);
        const int n = blk * geo.R + r_in_blk;
        int iacc[MAXM];
        float facc[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) { iacc[m] = 0; facc[m] = 0.0f; }
        if (n < N) {
#pragma unroll
            for (int p = 0; p < kMaxPass; ++p) {
                if (p >= geo.ppw) break;  // warp-uniform
                const int c = (pass0 + p) * 32 + lane;
                if ((pass0 + p) * 32 >= nch) break;  // warp-uniform
                const bool valid = c < nch;
                const int k0 = c * KC;
                if (!PG) {
#pragma unroll
                    for (int m = 0; m < MAXM; ++m)
                        if (m < M && valid) iacc[m] = chunk_dot<W4>(cur[p], s_q + static_cast<int64_t>(m) * K, k0) + iacc[m];
                } else {
                    const int g = valid ? k0 / gs : 0;
                    const float s = valid ? __ldg(sw + static_cast<int64_t>(g) * N + n) : 0.0f;
#pragma unroll
                    for (int m = 0; m < MAXM; ++m) {
                        if (m < M) {
                            int pp = valid ? chunk_dot<W4>(cur[p], s_q + static_cast<int64_t>(m) * K, k0) : 0;
                            for (int o = 1; o < lpg; o <<= 1) pp += __shfl_xor_sync(0xffffffffu, pp, o);
                            if ((lane & (lpg - 1)) == 0) facc[m] = fmaf(static_cast<float>(pp), s, facc[m]);
                        }
                    }
                }
            }
        }
        // warp reduction, then across the S slices of each row
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
            if (m < M) {
                if (!PG) {
                    int a = iacc[m];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                    if (lane == 0) s_part[warp][m] = __int_as_float(a);
                } else {
                    float a = facc[m];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                    if (lane == 0) s_part[warp][m] = a;
                }
            }
        }
        __syncthreads();
        for (int t = threadIdx.x; t < geo.R * M; t += kSmallThreads) {
            const int rr = t / M, m = t % M;
            const int nn = blk * geo.R + rr;
            if (nn < N) {
                float v;
                if (!PG) {
                    int a = 0;
                    for (int sl = 0; sl < geo.S; ++sl) a += __float_as_int(s_part[rr * geo.S + sl][m]);
                    v = static_cast<float>(a) * s_sx[m] * __ldg(sw + nn);
                } else {
                    float a = 0.0f;
                    for (int sl = 0; sl < geo.S; ++sl) a += s_part[rr * geo.S + sl][m];
                    v = a * s_sx[m];
                }
                y[static_cast<int64_t>(m) * N + nn] = from_f32<TY>(v);
            }
        }
        __syncthreads();
#pragma unroll
        for (int p = 0; p < kMaxPass; ++p) cur[p] = nxt[p];
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

template <typename TX, typename TY, bool PG, bool W4, int MAXM>
static cudaError_t launch_small_t(const void* x, int M, int K, const void* w, const float* sw,
                                  int N, int gs, void* y, int num_sms, cudaStream_t st) {
    const SmallGeom geo = small_geom(K, N, W4);
    if (geo.ppw > kMaxPass) return cudaErrorInvalidValue;  // K too large for this kernel
    const size_t smem = static_cast<size_t>(M) * K;
    auto kern = k_small_m<TX, TY, PG, W4, MAXM>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int grid = geo.nblocks < 2 * num_sms ? geo.nblocks : 2 * num_sms;
    kern<<<grid, kSmallThreads, smem, st>>>(static_cast<const TX*>(x), M, K, static_cast<const uint8_t*>(w), sw, N,
                                             gs, static_cast<TY*>(y), geo);
    return cudaGetLastError();
}

bool small_m_supported(int K, bool w4) { return small_geom(K, 8, w4).ppw <= kMaxPass; }

template <typename TX, typename TY, bool PG, bool W4>
static cudaError_t launch_small_m_tt(const void* x, int M, int K, const void* w, const float* sw,
                                     int N, int gs, void* y, int num_sms, cudaStream_t st) {
    if (M <= 1) return launch_small_t<TX, TY, PG, W4, 1>(x, M, K, w, sw, N, gs, y, num_sms, st);
    if (M <= 4) return launch_small_t<TX, TY, PG, W4, 4>(x, M, K, w, sw, N, gs, y, num_sms, st);
    if (M <= 8) return launch_small_t<TX, TY, PG, W4, 8>(x, M, K, w, sw, N, gs, y, num_sms, st);
    return launch_small_t<TX, TY, PG, W4, 16>(x, M, K, w, sw, N, gs, y, num_sms, st);
}

template <bool PG, bool W4>
static cudaError_t launch_small_m_v(const void* x, int xdt, int M, int K, const void* w,
                                    const float* sw, int N, int gs, void* y, int ydt, int num_sms,
                                    cudaStream_t st) {
    if (xdt == 0 && ydt == 0)
        return launch_small_m_tt<__half, __half, PG, W4>(x, M, K, w, sw, N, gs, y, num_sms, st);
    if (xdt == 0 && ydt == 1)
        return launch_small_m_tt<__half, __nv_bfloat16, PG, W4>(x, M, K, w, sw, N, gs, y, num_sms, st);
    if (xdt == 1 && ydt == 0)
        return launch_small_m_tt<__nv_bfloat16, __half, PG, W4>(x, M, K, w, sw, N, gs, y, num_sms, st);
    return launch_small_m_tt<__nv_bfloat16, __nv_bfloat16, PG, W4>(x, M, K, w, sw, N, gs, y, num_sms, st);
}

cudaError_t launch_small_m(int mode, const void* x, int xdt, int M, int K, const void* w,
                           const float* sw, int N, int gs, void* y, int ydt, int num_sms,
                           cudaStream_t st) {
    switch (mode) {
        case kModePC: return launch_small_m_v<false, false>(x, xdt, M, K, w, sw, N, gs, y, ydt, num_sms, st);
        case kModePG: return launch_small_m_v<true, false>(x, xdt, M, K, w, sw, N, gs, y, ydt, num_sms, st);
        case kModeW4: return launch_small_m_v<true, true>(x, xdt, M, K, w, sw, N, gs, y, ydt, num_sms, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace cider
