// sdpa_decode.cu -- decode attention: scaled dot-product attention for one
// query token per head, no mask, several query heads per KV head.
//
// What it computes (Cider README, section "优化 SDPA（解码注意力）"): for query
// head h and its KV head g = h / (H_q / H_kv),
//   out_h = sum_j softmax_j(q_h . k_{g,j} / sqrt(D)) v_{g,j},   D = 128,
// with q [H_q][D], K and V [H_kv][N][D] (head-major cache) in fp16 or bf16,
// out [H_q][D] in the same format.
//
// The pages' three techniques, B200 form:
//  * one CTA serves a tile of up to four query heads of one KV group, so the
//    group's K and V stream from HBM once per tile (the pages' contiguous-chunk
//    GQA scheduling; four heads per thread is their register tiling);
//  * the sequence is cut into chunks, one CTA per (chunk, KV head, head tile),
//    about four CTAs per SM, and a second kernel merges the chunks (their
//    two-pass split of the KV sequence);
//  * inside a CTA, each half-warp streams every 16th key of the chunk: lane l
//    holds dims 8l .. 8l+7 of the row (one 16-byte load of K and of V), the
//    score is a 4-step shuffle reduction within the half-warp, and the
//    softmax runs online in the log2 domain (q pre-scaled by log2(e)/sqrt(D)).
// Partial results are fp32: the unnormalised output, the running maximum and
// the running sum of exponentials, per (head, chunk).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <type_traits>

#include "cider_device.cuh"
#include "cider_kernels.h"
#include "sdpa_decode.h"

namespace cider {
namespace {

constexpr int kSdpaThreads = 256;  // 8 warps = 16 half-warp key streams
constexpr int kStreams = kSdpaThreads / 16;
constexpr int kMaxChunks = 1024;   // chunk scales of one head fit in shared memory

// 2^x by the hardware approximation (PTX ex2.approx: relative error near
// 2^-22, 2^-inf = +0); the softmax weights need no more.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float warp_reduce_max(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_reduce_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename T>
__device__ __forceinline__ void cvt8(const uint4& raw, float (&f)[8]) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t;
        if constexpr (sizeof(T) == 2 && std::is_same<T, __half>::value)
            t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
        else
            t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]) {
    cvt8<T>(__ldg(reinterpret_cast<const uint4*>(p)), f);
}

// Merge online-softmax state (m2, l2, a2) into (m, l, a); m = -inf means empty.
template <int ND>
__device__ __forceinline__ void merge_state(float& m, float& l, float (&a)[ND], float m2, float l2, const float (&a2)[ND]) {
    const float M = fmaxf(m, m2);
    if (M == -INFINITY) return;  // both empty
    const float s1 = ex2(m - M), s2 = ex2(m2 - M);
    l = l * s1 + l2 * s2;
#pragma unroll
    for (int d = 0; d < ND; ++d) a[d] = a[d] * s1 + a2[d] * s2;
    m = M;
}

// One CTA: KV head hk, head tile `tile` (query heads h0 .. h0+TH-1), chunk c.
template <int TH, typename T>
__global__ void __launch_bounds__(kSdpaThreads) k_sdpa_decode_split(const T* __restrict__ q, const T* __restrict__ k,
                                                                     const T* __restrict__ v, int G, int tiles, int N,
                                                                     int chunk, int chunks, float qscale,
                                                                     float* __restrict__ part) {
    constexpr int D = kSdpaD;
    __shared__ float s_m[kSdpaThreads / 32][TH], s_l[kSdpaThreads / 32][TH];
    __shared__ float s_o[kSdpaThreads / 32][TH][D];
    pdl_wait();
    pdl_trigger();
    const int c = blockIdx.x;
    const int hk = blockIdx.y / tiles;
    const int h0 = hk * G + (blockIdx.y % tiles) * TH;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hl = lane & 15;                       // dims 8 hl .. 8 hl + 7
    const int stream = warp * 2 + (lane >> 4);      // 0 .. 15
    float qr[TH][8];
#pragma unroll
    for (int i = 0; i < TH; ++i) {
        load8(q + static_cast<int64_t>(h0 + i) * D + 8 * hl, qr[i]);
#pragma unroll
        for (int d = 0; d < 8; ++d) qr[i][d] *= qscale;
    }
    float m[TH], l[TH], acc[TH][8];
#pragma unroll
    for (int i = 0; i < TH; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.0f;
#pragma unroll
        for (int d = 0; d < 8; ++d) acc[i][d] = 0.0f;
    }
    const int j0 = c * chunk, j1 = min(N, j0 + chunk);
    const T* kb = k + static_cast<int64_t>(hk) * N * D + 8 * hl;
    const T* vb = v + static_cast<int64_t>(hk) * N * D + 8 * hl;
    // The trip count is the same for every lane of the CTA: the shuffles below
    // always run with the whole warp; keys past the chunk only skip the update.
    // With two or four heads per thread the next key's K and V rows are loaded
    // while the current key is used (measured: GQA4 / GQA8 at N = 32K 65.0 /
    // 59.7 -> 50.6 / 46.6 us); with one head the direct loads measured faster
    // (MHA at N = 32K: 102.6 us against 152.6 us with the prefetch).
    constexpr bool kPrefetch = TH > 1;
    const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
    uint4 knext = zero4, vnext = zero4;
    if (kPrefetch && j0 + stream < j1) {
        knext = __ldg(reinterpret_cast<const uint4*>(kb + static_cast<int64_t>(j0 + stream) * D));
        vnext = __ldg(reinterpret_cast<const uint4*>(vb + static_cast<int64_t>(j0 + stream) * D));
    }
    for (int base = j0; base < j1; base += kStreams) {
        const int j = base + stream;
        const bool valid = j < j1;
        float kf[8], vf[8];
        if constexpr (kPrefetch) {
            const uint4 kraw = knext, vraw = vnext;
            const int jn = j + kStreams;
            knext = vnext = zero4;
            if (jn < j1) {
                knext = __ldg(reinterpret_cast<const uint4*>(kb + static_cast<int64_t>(jn) * D));
                vnext = __ldg(reinterpret_cast<const uint4*>(vb + static_cast<int64_t>(jn) * D));
            }
            cvt8<T>(kraw, kf);  // zeros past the chunk
            cvt8<T>(vraw, vf);
        } else if (valid) {
            load8(kb + static_cast<int64_t>(j) * D, kf);
            load8(vb + static_cast<int64_t>(j) * D, vf);
        } else {
#pragma unroll
            for (int d = 0; d < 8; ++d) kf[d] = vf[d] = 0.0f;
        }
        float s[TH];
#pragma unroll
        for (int i = 0; i < TH; ++i) {
            float t = 0.0f;
#pragma unroll
            for (int d = 0; d < 8; ++d) t = fmaf(qr[i][d], kf[d], t);
            s[i] = t;
        }
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
            for (int i = 0; i < TH; ++i) s[i] += __shfl_xor_sync(0xffffffffu, s[i], off);
        if (valid) {
#pragma unroll
            for (int i = 0; i < TH; ++i) {
                // rescale only when the key raises the running maximum (the same
                // decision in the whole half-warp; rare after the first keys)
                if (s[i] > m[i]) {
                    const float corr = ex2(m[i] - s[i]);  // 0 for the first key (m = -inf)
                    l[i] *= corr;
#pragma unroll
                    for (int d = 0; d < 8; ++d) acc[i][d] *= corr;
                    m[i] = s[i];
                }
                const float p = ex2(s[i] - m[i]);
                l[i] += p;
#pragma unroll
                for (int d = 0; d < 8; ++d) acc[i][d] = fmaf(p, vf[d], acc[i][d]);
            }
        }
    }
    // the two half-warps of a warp hold the same dims: merge them
#pragma unroll
    for (int i = 0; i < TH; ++i) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m[i], 16);
        const float l2 = __shfl_xor_sync(0xffffffffu, l[i], 16);
        float a2[8];
#pragma unroll
        for (int d = 0; d < 8; ++d) a2[d] = __shfl_xor_sync(0xffffffffu, acc[i][d], 16);
        merge_state<8>(m[i], l[i], acc[i], m2, l2, a2);
    }
    if (lane < 16) {
#pragma unroll
        for (int i = 0; i < TH; ++i) {
            if (lane == 0) {
                s_m[warp][i] = m[i];
                s_l[warp][i] = l[i];
            }
#pragma unroll
            for (int d = 0; d < 8; ++d) s_o[warp][i][8 * hl + d] = acc[i][d];
        }
    }
    __syncthreads();
    // merge the 8 warps: thread t owns (head t / D, dim t % D)
    for (int t = threadIdx.x; t < TH * D; t += kSdpaThreads) {
        const int i = t / D, d = t % D;
        float M = -INFINITY;
        for (int w = 0; w < kSdpaThreads / 32; ++w) M = fmaxf(M, s_m[w][i]);
        float L = 0.0f, O = 0.0f;
        for (int w = 0; w < kSdpaThreads / 32; ++w) {
            const float sc = s_m[w][i] == -INFINITY ? 0.0f : ex2(s_m[w][i] - M);
            L = fmaf(s_l[w][i], sc, L);
            O = fmaf(s_o[w][i][d], sc, O);
        }
        float* pp = part + (static_cast<int64_t>(h0 + i) * chunks + c) * kSdpaPartStride;
        pp[d] = O;
        if (d == 0) {
            pp[D] = M;
            pp[D + 1] = L;
        }
    }
}

// out[h][d] = sum_c o_c[d] 2^(m_c - M) / sum_c l_c 2^(m_c - M): one CTA per
// query head, 256 threads.  The maximum and the sum run across the block and
// the chunk scales wait in shared memory; then warp w adds chunks w, w + 8, ...
// with each lane holding four dims (one 16-byte load per chunk, all of a
// lane's loads in flight together), and the eight warps' partial sums meet in
// shared memory.  (The first version had one thread per dim walking every
// chunk: ~9 us per launch at 64 chunks, as long as the split kernel.)
constexpr int kMergeThreads = 256;
constexpr int kMergeWarps = kMergeThreads / 32;
template <typename T>
__global__ void __launch_bounds__(kMergeThreads) k_sdpa_decode_merge(const float* __restrict__ part, int chunks,
                                                                    T* __restrict__ out) {
    constexpr int D = kSdpaD;
    __shared__ float s_sc[kMaxChunks];
    __shared__ float s_red[2][kMergeWarps];
    __shared__ float4 s_acc[kMergeWarps][D / 4];
    pdl_wait();
    pdl_trigger();
    const int h = blockIdx.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const float* ph = part + static_cast<int64_t>(h) * chunks * kSdpaPartStride;
    // The o vectors of each warp's first four chunks are requested now, beside
    // the chunk maxima, so the weighted sum below does not wait for another
    // L2 round trip once the maximum is known (the sums keep their order).
    float4 o_first[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int cj = w + j * kMergeWarps;
        o_first[j] = cj < chunks ? __ldg(reinterpret_cast<const float4*>(ph + cj * kSdpaPartStride) + lane)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float M = -INFINITY;
    for (int c = t; c < chunks; c += kMergeThreads) M = fmaxf(M, __ldg(ph + c * kSdpaPartStride + D));
    M = warp_reduce_max(M);
    if (lane == 0) s_red[0][w] = M;
    __syncthreads();
    M = s_red[0][0];
#pragma unroll
    for (int i = 1; i < kMergeWarps; ++i) M = fmaxf(M, s_red[0][i]);
    float L = 0.0f;
    for (int c = t; c < chunks; c += kMergeThreads) {
        const float sc = ex2(__ldg(ph + c * kSdpaPartStride + D) - M);
        s_sc[c] = sc;
        L = fmaf(__ldg(ph + c * kSdpaPartStride + D + 1), sc, L);
    }
    L = warp_reduce_sum(L);
    if (lane == 0) s_red[1][w] = L;
    __syncthreads();  // s_sc and the partial sums are complete
    L = 0.0f;
#pragma unroll
    for (int i = 0; i < kMergeWarps; ++i) L += s_red[1][i];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int c = w;
    if (c + 3 * kMergeWarps < chunks) {  // the first four chunks, already in registers
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float sc = s_sc[c + j * kMergeWarps];
            acc.x = fmaf(o_first[j].x, sc, acc.x);
            acc.y = fmaf(o_first[j].y, sc, acc.y);
            acc.z = fmaf(o_first[j].z, sc, acc.z);
            acc.w = fmaf(o_first[j].w, sc, acc.w);
        }
        c += 4 * kMergeWarps;
    } else {  // fewer than four chunks for this warp: the tail loop below, from registers
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (c + j * kMergeWarps < chunks) {
                const float sc = s_sc[c + j * kMergeWarps];
                acc.x = fmaf(o_first[j].x, sc, acc.x);
                acc.y = fmaf(o_first[j].y, sc, acc.y);
                acc.z = fmaf(o_first[j].z, sc, acc.z);
                acc.w = fmaf(o_first[j].w, sc, acc.w);
            }
        }
        c = chunks;  // all of this warp's chunks are added
    }
    for (; c + 3 * kMergeWarps < chunks; c += 4 * kMergeWarps) {  // four chunks' loads in flight
        float4 o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = __ldg(reinterpret_cast<const float4*>(ph + (c + j * kMergeWarps) * kSdpaPartStride) + lane);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float sc = s_sc[c + j * kMergeWarps];
            acc.x = fmaf(o[j].x, sc, acc.x);
            acc.y = fmaf(o[j].y, sc, acc.y);
            acc.z = fmaf(o[j].z, sc, acc.z);
            acc.w = fmaf(o[j].w, sc, acc.w);
        }
    }
    for (; c < chunks; c += kMergeWarps) {
        const float4 o = __ldg(reinterpret_cast<const float4*>(ph + c * kSdpaPartStride) + lane);
        const float sc = s_sc[c];
        acc.x = fmaf(o.x, sc, acc.x);
        acc.y = fmaf(o.y, sc, acc.y);
        acc.z = fmaf(o.z, sc, acc.z);
        acc.w = fmaf(o.w, sc, acc.w);
    }
    s_acc[w][lane] = acc;
    __syncthreads();
    if (t < D) {
        const float* sa = reinterpret_cast<const float*>(&s_acc[0][0]);
        float y = 0.0f;
#pragma unroll
        for (int i = 0; i < kMergeWarps; ++i) y += sa[i * D + t];
        y /= L;
        if constexpr (std::is_same<T, __half>::value)
            out[static_cast<int64_t>(h) * D + t] = __float2half_rn(y);
        else
            out[static_cast<int64_t>(h) * D + t] = __float2bfloat16_rn(y);
    }
}

template <int TH, typename T>
cudaError_t launch_t(const void* q, const void* k, const void* v, int H_q, int H_kv, int N, const SdpaPlan& p,
                     float* part, void* out, cudaStream_t st) {
    const int G = H_q / H_kv;
    const float qscale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kSdpaD)));
    const dim3 grid(static_cast<unsigned>(p.chunks), static_cast<unsigned>(H_kv * p.tiles));
    cudaError_t e = launch_pdl(k_sdpa_decode_split<TH, T>, grid, kSdpaThreads, 0, st, static_cast<const T*>(q),
                               static_cast<const T*>(k), static_cast<const T*>(v), G, p.tiles, N, p.chunk, p.chunks,
                               qscale, part);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_sdpa_decode_merge<T>, static_cast<unsigned>(H_q), kMergeThreads, 0, st,
                      static_cast<const float*>(part), p.chunks, static_cast<T*>(out));
}

template <typename T>
cudaError_t launch_dt(const void* q, const void* k, const void* v, int H_q, int H_kv, int N, const SdpaPlan& p,
                      float* part, void* out, cudaStream_t st) {
    switch (p.th) {
        case 4: return launch_t<4, T>(q, k, v, H_q, H_kv, N, p, part, out, st);
        case 2: return launch_t<2, T>(q, k, v, H_q, H_kv, N, p, part, out, st);
        default: return launch_t<1, T>(q, k, v, H_q, H_kv, N, p, part, out, st);
    }
}

}  // namespace

SdpaPlan sdpa_plan(int64_t H_q, int64_t H_kv, int64_t N, int num_sms) {
    if (sdpa_tc_applies(H_q, H_kv, N)) return sdpa_tc_plan(H_q, H_kv, N, num_sms);
    SdpaPlan p{};
    const int64_t G = H_q / H_kv;
    p.th = G % 4 == 0 ? 4 : (G % 2 == 0 ? 2 : 1);
    p.tiles = static_cast<int>(G / p.th);
    const int64_t rows = H_kv * p.tiles;                  // CTAs per chunk index
    const int64_t target = 4 * static_cast<int64_t>(num_sms);
    int64_t chunks = std::max<int64_t>(1, (target + rows - 1) / rows);
    chunks = std::min<int64_t>(chunks, (N + kStreams - 1) / kStreams);  // at least 16 keys per chunk
    chunks = std::min<int64_t>(chunks, kMaxChunks);                      // the merge keeps one scale per chunk
    int64_t chunk = (N + chunks - 1) / chunks;
    chunk = (chunk + kStreams - 1) / kStreams * kStreams;
    p.chunk = static_cast<int>(chunk);
    p.chunks = static_cast<int>((N + chunk - 1) / chunk);
    return p;
}

size_t sdpa_part_bytes(int64_t H_q, const SdpaPlan& p) {
    return static_cast<size_t>(H_q) * p.chunks * kSdpaPartStride * sizeof(float);
}

cudaError_t launch_sdpa_decode(const void* q, const void* k, const void* v, int dt, int H_q, int H_kv, int N,
                               const SdpaPlan& plan, float* part, void* out, unsigned* status, cudaStream_t st) {
    if (plan.tc) return launch_sdpa_tc(q, k, v, dt, H_q, H_kv, N, plan, part, out, status, st);
    return dt == 1 ? launch_dt<__nv_bfloat16>(q, k, v, H_q, H_kv, N, plan, part, out, st)
                   : launch_dt<__half>(q, k, v, H_q, H_kv, N, plan, part, out, st);
}

cudaError_t launch_sdpa_merge(const float* part, int chunks, void* out, int H_q, int dt, cudaStream_t st) {
    if (dt == 1)
        return launch_pdl(k_sdpa_decode_merge<__nv_bfloat16>, static_cast<unsigned>(H_q), kMergeThreads, 0, st, part,
                          chunks, static_cast<__nv_bfloat16*>(out));
    return launch_pdl(k_sdpa_decode_merge<__half>, static_cast<unsigned>(H_q), kMergeThreads, 0, st, part, chunks,
                      static_cast<__half*>(out));
}

}  // namespace cider
