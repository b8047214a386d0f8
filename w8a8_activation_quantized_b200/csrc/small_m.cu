// small_m.cu -- the fused decode-shaped linear (1 <= M <= 16 tokens): one
// launch that quantizes the few activation rows into shared memory and then
// streams every weight row once from HBM, taking INT8 dot products with
// dp4a and applying the per-channel or per-group dequant.
//
// The pages route single-token decode to a dedicated matrix-vector kernel
// instead of the GEMM (juejin post "在Mac上跑大模型，MLX 不是终点", section
// "INT8 TensorOps 内核设计", "双路径自动切换"; Cider README, section
// "Metal Kernel 流水线", Decode).  This kernel keeps the W8A8 semantics of the
// GEMM path (activations quantized per token, integer products), so the same
// oracle covers every M.
//
// Work split: each CTA quantizes all M rows redundantly (x is a few KB and
// sits in L2), then each warp owns whole output channels n.  A weight row is
// streamed in 16-byte lane-strided chunks; each chunk holds 16 int8 weights
// (W8) or 32 packed int4 weights (W4).  Segments of SEG chunks per lane are
// double-buffered in registers, and a warp loads its first segment before
// the quantize phase, so weight traffic starts at once.
//
// Per-group: the lanes covering one group of gs weights reduce their INT32
// partial with shuffles; one lane rescales it by scale_w[g][n] in fp32.
#include "cider_device.cuh"
#include "cider_kernels.h"

namespace cider {

constexpr int kSmallThreads = 256;
constexpr int kSeg = 4;  // 16-byte chunks per lane per segment

template <bool W4>
struct ChunkGeom {
    static constexpr int kk = W4 ? 32 : 16;  // weights per 16-byte chunk
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
        uint2 u0 = unpack_int4x8(wv.x), u1 = unpack_int4x8(wv.y);
        uint2 u2 = unpack_int4x8(wv.z), u3 = unpack_int4x8(wv.w);
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

template <typename TX, typename TY, bool PG, bool W4, int MAXM>
__global__ void __launch_bounds__(kSmallThreads) k_small_m(const TX* __restrict__ x, int M, int K,
                                                           const uint8_t* __restrict__ w,
                                                           const float* __restrict__ sw, int N,
                                                           int gs, TY* __restrict__ y) {
    extern __shared__ __align__(16) int8_t s_q[];  // [M][K] codes
    __shared__ float s_sx[MAXM];
    constexpr int KC = ChunkGeom<W4>::kk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = kSmallThreads / 32;
    const int64_t row_bytes = W4 ? K / 2 : K;
    const int nch = K / KC;            // chunks per weight row
    const int nseg = (nch + 32 * kSeg - 1) / (32 * kSeg);
    const int gwarp = blockIdx.x * nwarps + warp;
    const int stride = gridDim.x * nwarps;

    // Load the first segment of this warp's first row before quantizing.
    uint4 cur[kSeg], nxt[kSeg];
    int n = gwarp, seg = 0;
    auto load_seg = [&](uint4 (&dst)[kSeg], int nn, int sg) {
        const uint4* wr = reinterpret_cast<const uint4*>(w + static_cast<int64_t>(nn) * row_bytes);
#pragma unroll
        for (int i = 0; i < kSeg; ++i) {
            const int c = sg * 32 * kSeg + i * 32 + lane;
            dst[i] = (nn < N && c < nch) ? __ldcs(wr + c) : make_uint4(0, 0, 0, 0);
        }
    };
    load_seg(cur, n, 0);

    // Quantize the M activation rows into shared memory (warp per row).
    for (int m = warp; m < M; m += nwarps) {
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
        if (lane == 0) s_sx[m] = s;
        for (int c = lane; c < K / 8; c += 32) {
            float f[8];
            unpack8_f32<TX>(__ldg(xr + c), f);
            int cc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) cc[j] = quant_code(f[j], s);
            *reinterpret_cast<uint2*>(s_q + static_cast<int64_t>(m) * K + 8 * c) = pack8_i8(cc);
        }
    }
    __syncthreads();

    const int lanes_per_group = PG ? gs / KC : 32;  // 2, 4 or 8 for PG
    int iacc[MAXM];
    float facc[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) { iacc[m] = 0; facc[m] = 0.0f; }

    while (n < N) {
        // prefetch the next segment (of this row, or of the warp's next row)
        const bool last_seg = (seg + 1 == nseg);
        const int n_next = last_seg ? n + stride : n;
        const int seg_next = last_seg ? 0 : seg + 1;
        load_seg(nxt, n_next, seg_next);

#pragma unroll
        for (int i = 0; i < kSeg; ++i) {
            const int cbase = seg * 32 * kSeg + i * 32;  // first chunk of this 32-chunk pass
            if (cbase >= nch) break;                     // warp-uniform
            const int c = cbase + lane;
            const bool valid = c < nch;
            const int k0 = c * KC;
            if (!PG) {
#pragma unroll
                for (int m = 0; m < MAXM; ++m)
                    if (m < M && valid) iacc[m] = chunk_dot<W4>(cur[i], s_q + static_cast<int64_t>(m) * K, k0) + iacc[m];
            } else {
                // group of this lane's chunk; lanes_per_group lanes share a group
                const int g = valid ? k0 / gs : 0;
                const float s = valid ? __ldg(sw + static_cast<int64_t>(g) * N + n) : 0.0f;
#pragma unroll
                for (int m = 0; m < MAXM; ++m) {
                    if (m < M) {
                        int p = valid ? chunk_dot<W4>(cur[i], s_q + static_cast<int64_t>(m) * K, k0) : 0;
                        for (int o = 1; o < lanes_per_group; o <<= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
                        if ((lane & (lanes_per_group - 1)) == 0) facc[m] = fmaf(static_cast<float>(p), s, facc[m]);
                    }
                }
            }
        }

        if (last_seg) {
            // finish output channel n
#pragma unroll
            for (int m = 0; m < MAXM; ++m) {
                if (m < M) {
                    if (!PG) {
                        int a = iacc[m];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                        if (lane == 0)
                            y[static_cast<int64_t>(m) * N + n] =
                                from_f32<TY>(static_cast<float>(a) * s_sx[m] * __ldg(sw + n));
                    } else {
                        float a = facc[m];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                        if (lane == 0) y[static_cast<int64_t>(m) * N + n] = from_f32<TY>(a * s_sx[m]);
                    }
                }
                iacc[m] = 0;
                facc[m] = 0.0f;
            }
        }
        n = n_next;
        seg = seg_next;
#pragma unroll
        for (int i = 0; i < kSeg; ++i) cur[i] = nxt[i];
    }
}

template <typename TX, typename TY, bool PG, bool W4, int MAXM>
static cudaError_t launch_small_t(const void* x, int M, int K, const void* w, const float* sw,
                                  int N, int gs, void* y, int num_sms, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(M) * K;
    auto kern = k_small_m<TX, TY, PG, W4, MAXM>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int warps_needed = N;
    int grid = (warps_needed + (kSmallThreads / 32) - 1) / (kSmallThreads / 32);
    const int max_grid = num_sms * 2;
    if (grid > max_grid) grid = max_grid;
    kern<<<grid, kSmallThreads, smem, st>>>(static_cast<const TX*>(x), M, K,
                                             static_cast<const uint8_t*>(w), sw, N, gs,
                                             static_cast<TY*>(y));
    return cudaGetLastError();
}

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
