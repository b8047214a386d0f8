// sdpa_tc.cu -- decode attention for grouped KV heads on the tensor cores.
//
// What it computes is what sdpa_decode.cu computes (Cider README, section
// "优化 SDPA（解码注意力）": one query token per head, no mask, query head h
// reads KV head h / G, G = H_q / H_kv query heads per KV head, D = 128):
//   out_h = sum_j softmax_j(q_h . k_j / sqrt(D)) v_j.
// The CUDA-core kernel spends ~16 fp32 operations per key, head and lane plus
// shuffles and an exponential per key and head; with four heads per thread
// it is bound by instruction issue, not HBM (ncu at G = 8, N = 32K: issue
// slots 65% busy, DRAM 18%).  Here the two products run on tcgen05.mma
// (kind::f16, fp32 accumulation in TMEM) and the CUDA cores keep only the
// softmax:
//  * one CTA per (KV head, chunk of up to 512 keys), two CTAs per SM;
//  * warp 0 streams 128-key tiles of K, then of V, through a two-stage ring
//    (TMA, 128-byte swizzle: each tile is two boxes of 64 dims x 128 keys);
//  * warp 1 issues S^T = K . Q^T per K tile (M = 128 keys, N = 16 query
//    heads -- the group padded with zero rows -- K = 128 dims in 8 steps),
//    into TMEM columns 16 t .. 16 t + 15;
//  * four softmax warps read S^T (thread = key), take the chunk maximum per
//    head in the log2 domain, p = 2^(s log2(e)/sqrt(D) - m), the sum l per
//    head, and write P to shared memory as a sum of 16-bit parts in the
//    input format (fp16: p = hi + lo, bf16: three parts), exact to ~2^-22 of
//    p, so that P . V keeps the precision of an fp32 product;
//  * warp 1 then issues O^T = V^T . P^T per V tile and part (M = 128 dims,
//    V read in its natural [key][dim] layout as an MN-major operand, N = 16
//    heads, K = 16 keys per step) into TMEM;
//  * the softmax warps write the unnormalised O, m and l of the chunk in the
//    partial-result format of sdpa_decode.cu, whose merge kernel combines the
//    chunks.
// Every wait is bounded (mbar_wait).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include "gemm_common.cuh"
#include "sdpa_decode.h"

namespace cider {
namespace {

constexpr int kTcKeys = 128;       // keys per K / V tile
constexpr int kTcHeads = 16;       // MMA N: the query heads of one KV group, padded
constexpr int kTcMaxTiles = 4;     // keys per CTA <= 512: S^T is 4 x 16 TMEM columns
constexpr int kTcThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2..5 softmax / output
constexpr int kTcStages = 2;       // ring of K / V tiles
constexpr int kTcTileBytes = kTcKeys * kSdpaD * 2;                    // 32 KB: two 16 KB boxes
constexpr int kTcQBytes = 2 * kTcHeads * 128;                         // Q: 2 atoms x 16 rows x 128 B
constexpr int kTcPPartBytes = kTcMaxTiles * (kTcKeys / 64) * kTcHeads * 128;  // one part of P: 16 KB
constexpr int kTcOCol = kTcMaxTiles * kTcHeads;                       // TMEM column of O^T
constexpr int kTcTmemCols = 128;

std::atomic<int> g_sdpa_kernel{0};  // test override: 0 automatic, 1 CUDA cores, 2/3 tensor cores (V descriptor order)

// K-major operand, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t addr) { return umma_desc_sw128(addr); }

// MN-major operand with the 128-byte swizzle: rows of 128 bytes run along
// MN (64 16-bit elements), 8-row groups along K.  `lbo` and `sbo` are the
// byte offsets between 64-element atoms along MN and between 8-row groups
// along K, in the descriptor's order.
__device__ __forceinline__ uint64_t desc_mn(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;  // version
    d |= static_cast<uint64_t>(2u) << 61;  // SWIZZLE_128B
    return d;
}

// kind::f16 instruction descriptor: D = F32, A = B = fp16 (bf = 0) or bf16
// (bf = 1); a_mn: A is MN-major (transposed).
__host__ __device__ constexpr uint32_t idesc_16(int M, int N, int bf, int a_mn) {
    return (1u << 4) | (static_cast<uint32_t>(bf) << 7) | (static_cast<uint32_t>(bf) << 10) |
           (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// Byte offset of element (row, k) in a K-major, 128-byte-swizzled tile of
// `rows` rows whose K runs over 64-element atoms `rows * 128` bytes apart.
__device__ __forceinline__ uint32_t kmaj_offset(int row, int k, int rows) {
    const int atom = k >> 6, kk = k & 63;
    const int r8 = row & 7;
    return atom * rows * 128 + (row >> 3) * 1024 + r8 * 128 + ((((kk >> 3) ^ r8) & 7) << 4) + (kk & 7) * 2;
}

// 2^x by the hardware approximation (PTX ex2.approx: relative error near
// 2^-22, 2^-inf = +0), as in the CUDA-core kernels.
__device__ __forceinline__ float ex2_tc(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <typename T>
__device__ __forceinline__ uint16_t to_bits(T v) {
    return *reinterpret_cast<uint16_t*>(&v);
}

// p = sum of NP 16-bit parts, each the rounding of what the previous ones
// leave (fp16: 2 parts, 22 bits; bf16: 3 parts, 24 bits).
template <typename T, int NP>
__device__ __forceinline__ void split_parts(float p, uint16_t (&part)[NP]) {
    float r = p;
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const T h = from_f32<T>(r);
        part[i] = to_bits(h);
        r -= to_f32<T>(h);
    }
}

template <typename T>
__global__ void __launch_bounds__(kTcThreads) k_sdpa_tc(const __grid_constant__ CUtensorMap tmK,
                                                        const __grid_constant__ CUtensorMap tmV,
                                                        const T* __restrict__ q, int G, int N, int chunk,
                                                        int chunks, float qscale, float* __restrict__ part,
                                                        uint32_t v_lbo, uint32_t v_sbo, unsigned* status) {
    constexpr bool BF = std::is_same<T, __nv_bfloat16>::value;
    constexpr int NP = BF ? 3 : 2;  // 16-bit parts of P
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                                   // 4 KB
    uint8_t* sRing = sQ + kTcQBytes;                      // kTcStages x 32 KB
    uint8_t* sP = sRing + kTcStages * kTcTileBytes;       // NP x 16 KB
    __shared__ uint64_t full[kTcStages], empty[kTcStages], sdone, pready, odone;
    __shared__ uint32_t tmem_slot;
    __shared__ float s_red[4][kTcHeads];
    __shared__ int s_abort;
    volatile int* abort_flag = &s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, hk = blockIdx.y;
    const int j0 = c * chunk, j1 = min(N, j0 + chunk);
    const int nt = (j1 - j0 + kTcKeys - 1) / kTcKeys;  // K / V tiles of this chunk
    const int row0 = hk * N + j0;                      // first key row in the [H_kv * N][D] view

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&sdone, 1);
        mbar_init(&pready, 128);
        mbar_init(&odone, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
    }
    if (warp == 1) tmem_alloc(&tmem_slot, kTcTmemCols);
    pdl_wait();
    pdl_trigger();
    // Q of the group, zero rows beyond G, K-major with the 128-byte swizzle:
    // 16 rows x 2 atoms x 8 chunks of 8 dims
    for (int i = threadIdx.x; i < kTcHeads * 16; i += kTcThreads) {
        const int h = i >> 4, d8 = (i & 15) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (h < G) v = __ldg(reinterpret_cast<const uint4*>(q + static_cast<int64_t>(hk * G + h) * kSdpaD + d8));
        *reinterpret_cast<uint4*>(sQ + kmaj_offset(h, d8, kTcHeads)) = v;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            for (int i = 0; i < 2 * nt; ++i) {
                const int s = i % kTcStages;
                const uint32_t ph = (i / kTcStages) & 1u;
                if (i >= kTcStages && !mbar_wait(&empty[s], ph ^ 1u, status, abort_flag)) break;
                const CUtensorMap* map = i < nt ? &tmK : &tmV;
                const int row = row0 + (i % nt) * kTcKeys;
                mbar_arrive_expect_tx(&full[s], kTcTileBytes);
                tma_load_2d(sRing + s * kTcTileBytes, map, &full[s], 0, row);
                tma_load_2d(sRing + s * kTcTileBytes + kTcTileBytes / 2, map, &full[s], 128, row);
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_16(128, kTcHeads, BF ? 1 : 0, 0);
            constexpr uint32_t idesc_o = idesc_16(128, kTcHeads, BF ? 1 : 0, 1);
            bool ok = true;
            for (int i = 0; i < nt && ok; ++i) {  // S^T of K tile i
                const int s = i % kTcStages;
                if (!mbar_wait(&full[s], (i / kTcStages) & 1u, status, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(sRing + s * kTcTileBytes), b0 = smem_u32(sQ);
#pragma unroll
                for (int kk = 0; kk < kSdpaD / 16; ++kk) {
                    const uint32_t off_a = (kk >> 2) * (kTcTileBytes / 2) + (kk & 3) * 32;
                    const uint32_t off_b = (kk >> 2) * (kTcHeads * 128) + (kk & 3) * 32;
                    mma16(tmem + i * kTcHeads, desc_k(a0 + off_a), desc_k(b0 + off_b), idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&empty[s]);
            }
            if (ok) umma_commit(&sdone);
            if (ok && !mbar_wait(&pready, 0, status, abort_flag)) ok = false;
            tc_fence_after();
            for (int t = 0; t < nt && ok; ++t) {  // O^T += V^T . P^T of V tile t
                const int i = nt + t, s = i % kTcStages;
                if (!mbar_wait(&full[s], (i / kTcStages) & 1u, status, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(sRing + s * kTcTileBytes);
#pragma unroll
                for (int kk = 0; kk < kTcKeys / 16; ++kk) {
                    const uint64_t a = desc_mn(a0 + kk * 2048, v_lbo, v_sbo);  // keys 16 kk .. of the tile
                    const int key = t * kTcKeys + kk * 16;                    // of the chunk
                    const uint32_t off_b = (key >> 6) * (kTcHeads * 128) + ((key & 63) >> 3) * 16;
#pragma unroll
                    for (int pp = 0; pp < NP; ++pp)
                        mma16(tmem + kTcOCol, a, desc_k(smem_u32(sP + pp * kTcPPartBytes) + off_b), idesc_o,
                              (t > 0 || kk > 0 || pp > 0) ? 1u : 0u);
                }
                umma_commit(&empty[s]);
            }
            if (ok) umma_commit(&odone);
        }
        __syncwarp();
    } else {
        // ------------------------- softmax and output warps ------------------------
        const int wq = warp & 3;  // TMEM lane quarter: keys (and dims) 32 wq .. 32 wq + 31
        const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
        bool ok = mbar_wait(&sdone, 0, status, abort_flag);
        tc_fence_after();
        float sv[kTcMaxTiles][kTcHeads];
        float m[kTcHeads], l[kTcHeads];
#pragma unroll
        for (int h = 0; h < kTcHeads; ++h) { m[h] = -INFINITY; l[h] = 0.0f; }
#pragma unroll
        for (int t = 0; t < kTcMaxTiles; ++t) {
            const int j = j0 + t * kTcKeys + wq * 32 + lane;
            uint32_t r[16];
            if (t < nt) {
                tmem_ld_32x32b_x16(tmem + lane_addr + t * kTcHeads, r);
                tmem_ld_wait();
            }
#pragma unroll
            for (int h = 0; h < kTcHeads; ++h) {
                sv[t][h] = (t < nt && j < j1) ? __uint_as_float(r[h]) * qscale : -INFINITY;
                m[h] = fmaxf(m[h], sv[t][h]);
            }
        }
        // the chunk's maximum per head, over the 128 threads (heads beyond the
        // group are padding: no reductions, no weights)
#pragma unroll
        for (int h = 0; h < kTcHeads; ++h) {
            if (h < G) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], o));
            }
        }
        if (lane < kTcHeads) {
            float v = m[0];
#pragma unroll
            for (int h = 1; h < kTcHeads; ++h) v = lane == h ? m[h] : v;
            s_red[wq][lane] = v;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
        for (int h = 0; h < kTcHeads; ++h)
            m[h] = fmaxf(fmaxf(s_red[0][h], s_red[1][h]), fmaxf(s_red[2][h], s_red[3][h]));
        asm volatile("bar.sync 1, 128;" ::: "memory");  // s_red is reused for the sums below
        // weights, their sum, and P as 16-bit parts in shared memory
#pragma unroll
        for (int t = 0; t < kTcMaxTiles; ++t) {
            const int key = t * kTcKeys + wq * 32 + lane;  // within the chunk
#pragma unroll
            for (int h = 0; h < kTcHeads; ++h) {
                if (h < G && t < nt) {
                    const float p = ex2_tc(sv[t][h] - m[h]);  // 0 for keys past the chunk (-inf)
                    l[h] += p;
                    uint16_t pt[NP];
                    split_parts<T, NP>(p, pt);
                    const uint32_t off = kmaj_offset(h, key, kTcHeads);
#pragma unroll
                    for (int pp = 0; pp < NP; ++pp) *reinterpret_cast<uint16_t*>(sP + pp * kTcPPartBytes + off) = pt[pp];
                }
            }
        }
        fence_async_smem();
        mbar_arrive(&pready);
        // the chunk's sum of weights per head
#pragma unroll
        for (int h = 0; h < kTcHeads; ++h) {
            if (h < G) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
            }
        }
        if (lane < kTcHeads) {
            float v = l[0];
#pragma unroll
            for (int h = 1; h < kTcHeads; ++h) v = lane == h ? l[h] : v;
            s_red[wq][lane] = v;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // O^T: thread = dim 32 wq + lane, columns = heads
        ok = ok && mbar_wait(&odone, 0, status, abort_flag);
        tc_fence_after();
        if (ok) {
            uint32_t o[16];
            tmem_ld_32x32b_x16(tmem + lane_addr + kTcOCol, o);
            tmem_ld_wait();
            const int d = wq * 32 + lane;
            for (int h = 0; h < G; ++h) {
                float* pp = part + (static_cast<int64_t>(hk * G + h) * chunks + c) * kSdpaPartStride;
                pp[d] = __uint_as_float(o[h]);
                if (d == 0) {
                    pp[kSdpaD] = m[h];
                    pp[kSdpaD + 1] = (s_red[0][h] + s_red[1][h]) + (s_red[2][h] + s_red[3][h]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
    }
}

template <typename T>
cudaError_t launch_tc(const void* q, const void* k, const void* v, int H_q, int H_kv, int N, const SdpaPlan& p,
                      float* part, void* out, unsigned* status, cudaStream_t st) {
    CUtensorMap tmK, tmV;
    const uint64_t rows = static_cast<uint64_t>(H_kv) * N;
    if (!make_map_2d(&tmK, k, kSdpaD * 2, rows, 128, kTcKeys, true)) return cudaErrorInvalidValue;
    if (!make_map_2d(&tmV, v, kSdpaD * 2, rows, 128, kTcKeys, true)) return cudaErrorInvalidValue;
    const int np = std::is_same<T, __nv_bfloat16>::value ? 3 : 2;
    const int smem = 1024 + kTcQBytes + kTcStages * kTcTileBytes + np * kTcPPartBytes;
    auto kern = k_sdpa_tc<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const float qscale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kSdpaD)));
    // V as an MN-major operand: 64-dim atoms 16 KB apart (the two TMA boxes),
    // 8-key groups 1 KB apart; mode 3 of the test switch swaps the two fields
    const bool swap = g_sdpa_kernel.load() == 3;
    const uint32_t lbo = swap ? 1024u : static_cast<uint32_t>(kTcTileBytes / 2);
    const uint32_t sbo = swap ? static_cast<uint32_t>(kTcTileBytes / 2) : 1024u;
    const dim3 grid(static_cast<unsigned>(p.chunks), static_cast<unsigned>(H_kv));
    e = launch_pdl(kern, grid, kTcThreads, smem, st, tmK, tmV, static_cast<const T*>(q), H_q / H_kv, N, p.chunk,
                   p.chunks, qscale, part, lbo, sbo, status);
    if (e != cudaSuccess) return e;
    return launch_sdpa_merge(part, p.chunks, out, H_q, std::is_same<T, __nv_bfloat16>::value ? 1 : 0, st);
}

}  // namespace

bool sdpa_tc_applies(int64_t H_q, int64_t H_kv, int64_t N) {
    const int sel = g_sdpa_kernel.load();
    if (sel == 1) return false;
    const int64_t G = H_q / H_kv;
    if (G < 2 || G > kTcHeads) return false;
    if (H_kv * N >= (int64_t(1) << 31)) return false;
    return (N + kTcMaxTiles * kTcKeys - 1) / (kTcMaxTiles * kTcKeys) <= 1024;  // the merge's chunk limit
}

// Chunks of 128 .. 512 keys, as many as give about two CTAs per SM.
SdpaPlan sdpa_tc_plan(int64_t H_q, int64_t H_kv, int64_t N, int num_sms) {
    SdpaPlan p{};
    p.th = static_cast<int>(H_q / H_kv);
    p.tiles = 1;
    const int64_t target = std::max<int64_t>(1, (2 * static_cast<int64_t>(num_sms) + H_kv - 1) / H_kv);
    int64_t chunk = (N + target - 1) / target;
    chunk = (chunk + kTcKeys - 1) / kTcKeys * kTcKeys;
    chunk = std::min<int64_t>(std::max<int64_t>(chunk, kTcKeys), kTcMaxTiles * kTcKeys);
    p.chunk = static_cast<int>(chunk);
    p.chunks = static_cast<int>((N + chunk - 1) / chunk);
    p.tc = 1;
    return p;
}

cudaError_t launch_sdpa_tc(const void* q, const void* k, const void* v, int dt, int H_q, int H_kv, int N,
                           const SdpaPlan& plan, float* part, void* out, unsigned* status, cudaStream_t st) {
    return dt == 1 ? launch_tc<__nv_bfloat16>(q, k, v, H_q, H_kv, N, plan, part, out, status, st)
                   : launch_tc<__half>(q, k, v, H_q, H_kv, N, plan, part, out, status, st);
}

cudaError_t set_sdpa_kernel(int k) {
    if (k < 0 || k > 3) return cudaErrorInvalidValue;
    g_sdpa_kernel.store(k);
    return cudaSuccess;
}

}  // namespace cider
