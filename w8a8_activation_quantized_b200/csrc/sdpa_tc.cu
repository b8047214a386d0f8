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
//  * one CTA per (KV head, chunk of 1 .. 15 tiles of 128 keys), one CTA per
//    SM: the plan takes the fewest tiles per chunk that put every chunk in
//    one wave, so the SMs get equal shares of the K/V bytes;
//  * warp 0 streams the chunk's 128-key tiles of K, then of V, through a
//    six-stage ring (TMA, 128-byte swizzle: each tile is two boxes of 64 dims
//    x 128 keys), up to ~192 KB in flight;
//  * warp 1 issues S^T = K . Q^T per K tile (M = 128 keys, N = 16 query
//    heads -- the group padded with zero rows -- K = 128 dims in 8 steps),
//    into TMEM columns 16 t .. 16 t + 15;
//  * eight softmax warps (two per TMEM lane quarter, each with half of the
//    query heads) read S^T (thread = key) twice: first each tile as soon as
//    its scores are made, for the chunk maximum per head in the log2 domain,
//    then, tile by tile, for
//    p = 2^(s log2(e)/sqrt(D) - m) and the sum l per head, writing each
//    tile's P into one of two shared-memory buffers as a sum of 16-bit parts
//    in the input format (fp16: p = hi + lo, bf16: three parts), exact to
//    ~2^-22 of p, so that P . V keeps the precision of an fp32 product;
//  * warp 1 issues O^T = V^T . P^T per V tile and part as soon as that
//    tile's P is written (M = 128 dims, V read in its natural [key][dim]
//    layout as an MN-major operand, N = 16 heads, K = 16 keys per step), so
//    the V tiles stream on while the softmax writes the later tiles' P.
//    The parts of P are stacked along the MMA's N (16 rows per part: N = 32
//    for fp16, 48 for bf16), so one MMA per 16 keys makes every part's
//    product, and the two tile parities accumulate into separate TMEM
//    columns; the output pass adds parts and parities.  (With one MMA per
//    part into one accumulator a tile took 16 MMAs, ~1 us on B200, and the P
//    buffer of tile t + 2 waited for them: that set the pace of the kernel.)
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
constexpr int kTcMaxTiles = 15;    // tiles per chunk: S^T takes 15 x 16 TMEM columns
constexpr int kTcSlices = 2;       // softmax warps per TMEM lane quarter (head slices)
constexpr int kTcSmxThreads = kTcSlices * 128;
constexpr int kTcThreads = 64 + kTcSmxThreads;  // warp 0 TMA, warp 1 MMA, the rest softmax / output
constexpr int kTcStages = 6;       // ring of K / V tiles
constexpr int kTcTileBytes = kTcKeys * kSdpaD * 2;                    // 32 KB: two 16 KB boxes
constexpr int kTcQBytes = 2 * kTcHeads * 128;                         // Q: 2 atoms x 16 rows x 128 B
constexpr int kTcPPartBytes = (kTcKeys / 64) * kTcHeads * 128;        // one part of one tile's P: 4 KB (as bytes)
constexpr int kTcOCol = kTcMaxTiles * kTcHeads;                       // TMEM column of the O^T accumulators
constexpr int kTcTmemCols = 512;  // S^T 240 columns + two O^T accumulators of 16 x parts (at most 48) columns

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
__global__ void __launch_bounds__(kTcThreads, 1) k_sdpa_tc(const __grid_constant__ CUtensorMap tmK,
                                                           const __grid_constant__ CUtensorMap tmV,
                                                           const T* __restrict__ q, int G, int N, int chunk,
                                                           int chunks, float qscale, float* __restrict__ part,
                                                           uint32_t v_lbo, uint32_t v_sbo, int npre,
                                                           unsigned* status) {
    constexpr bool BF = std::is_same<T, __nv_bfloat16>::value;
    constexpr int NP = BF ? 3 : 2;  // 16-bit parts of P
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                                   // 4 KB
    uint8_t* sRing = sQ + kTcQBytes;                      // kTcStages x 32 KB
    uint8_t* sP = sRing + kTcStages * kTcTileBytes;       // 2 buffers of P^T: 16 NP rows x 128 keys
    __shared__ uint64_t full[kTcStages], empty[kTcStages], sfull[kTcMaxTiles], pfull[2], pempty[2], odone;
    __shared__ uint32_t tmem_slot;
    __shared__ float s_red[4][kTcHeads];  // [lane quarter][head]
    __shared__ int s_abort;
    volatile int* abort_flag = &s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, hk = blockIdx.y;
    const int j0 = c * chunk, j1 = min(N, j0 + chunk);
    const int nt = (j1 - j0 + kTcKeys - 1) / kTcKeys;  // K / V tiles of this chunk (<= kTcMaxTiles, by the plan)
    const int row0 = hk * N + j0;                      // first key row in the [H_kv * N][D] view

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&pfull[b], kTcSmxThreads);
            mbar_init(&pempty[b], 1);
        }
        for (int t = 0; t < kTcMaxTiles; ++t) mbar_init(&sfull[t], 1);
        mbar_init(&odone, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
        // The ring's first npre tiles into L2 before the wait on the previous
        // kernel (a prefetch writes no shared memory, and the loads after the
        // wait still see that kernel's writes): a CTA that starts while the
        // previous launch drains streams meanwhile.
        for (int i = 0; i < 2 * nt && i < npre; ++i) {
            const CUtensorMap* map = i < nt ? &tmK : &tmV;
            const int row = row0 + (i % nt) * kTcKeys;
            tma_prefetch_l2_2d(map, 0, row);
            tma_prefetch_l2_2d(map, 128, row);
        }
    }
    if (warp == 1) tmem_alloc(&tmem_slot, kTcTmemCols);
    pdl_wait();
    pdl_trigger();
    // The thread that initialised the barriers fills the ring at once (no
    // stage is in use yet), before the CTA-wide setup below.
    const int first = min(kTcStages, 2 * nt);
    if (threadIdx.x == 0) {
        for (int i = 0; i < first; ++i) {
            const CUtensorMap* map = i < nt ? &tmK : &tmV;
            const int row = row0 + (i % nt) * kTcKeys;
            mbar_arrive_expect_tx(&full[i], kTcTileBytes);
            tma_load_2d(sRing + i * kTcTileBytes, map, &full[i], 0, row);
            tma_load_2d(sRing + i * kTcTileBytes + kTcTileBytes / 2, map, &full[i], 128, row);
        }
    }
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
            for (int i = first; i < 2 * nt; ++i) {  // the rest, as stages free up
                const int s = i % kTcStages;
                const uint32_t ph = (i / kTcStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, status, abort_flag)) break;
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
            constexpr uint32_t idesc_o = idesc_16(128, NP * kTcHeads, BF ? 1 : 0, 1);
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
                umma_commit(&sfull[i]);  // tile i's scores are in TMEM
            }
            for (int t = 0; t < nt && ok; ++t) {  // O^T += V^T . P^T of V tile t, once its P is written
                const int i = nt + t, s = i % kTcStages, b = t & 1;
                if (!mbar_wait(&full[s], (i / kTcStages) & 1u, status, abort_flag)) { ok = false; break; }
                if (!mbar_wait(&pfull[b], (t >> 1) & 1u, status, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(sRing + s * kTcTileBytes);
                const uint32_t p0 = smem_u32(sP + b * NP * kTcPPartBytes);
#pragma unroll
                for (int kk = 0; kk < kTcKeys / 16; ++kk) {
                    const uint64_t a = desc_mn(a0 + kk * 2048, v_lbo, v_sbo);  // keys 16 kk .. of the tile
                    const int key = kk * 16;
                    const uint32_t off_b = (key >> 6) * (NP * kTcHeads * 128) + ((key & 63) >> 3) * 16;
                    // accumulator t & 1 starts at tile t & 1
                    mma16(tmem + kTcOCol + b * NP * kTcHeads, a, desc_k(p0 + off_b), idesc_o,
                          (t >= 2 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&empty[s]);
                umma_commit(&pempty[b]);
            }
            if (ok) umma_commit(&odone);
        }
        __syncwarp();
    } else {
        // ------------------------- softmax and output warps ------------------------
        const int wq = warp & 3;  // TMEM lane quarter: keys (and dims) 32 wq .. 32 wq + 31
        const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
        const int key = wq * 32 + lane;  // this thread's key within a tile
        // this warp's slice of the query heads: [h0, h1)
        const int per = (G + kTcSlices - 1) / kTcSlices;
        const int h0 = min(G, ((warp - 2) >> 2) * per), h1 = min(G, h0 + per);
        bool ok = true;
        float m[kTcHeads], l[kTcHeads];
#pragma unroll
        for (int h = 0; h < kTcHeads; ++h) { m[h] = -INFINITY; l[h] = 0.0f; }
        // the chunk's maximum per head (heads beyond the group are padding),
        // each tile as soon as its scores are made
        for (int t = 0; t < nt && ok; ++t) {
            ok = mbar_wait(&sfull[t], 0, status, abort_flag);
            tc_fence_after();
            if (!ok) break;
            uint32_t r[16];
            tmem_ld_32x32b_x16(tmem + lane_addr + t * kTcHeads, r);
            tmem_ld_wait();
            if (j0 + t * kTcKeys + key < j1) {
#pragma unroll
                for (int h = 0; h < kTcHeads; ++h)
                    if (h >= h0 && h < h1) m[h] = fmaxf(m[h], __uint_as_float(r[h]) * qscale);
            }
        }
#pragma unroll
        for (int h = 0; h < kTcHeads; ++h) {
            if (h >= h0 && h < h1) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], o));
                if (lane == 0) s_red[wq][h] = m[h];
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kTcSmxThreads) : "memory");
#pragma unroll
        for (int h = 0; h < kTcHeads; ++h)
            if (h >= h0 && h < h1) m[h] = fmaxf(fmaxf(s_red[0][h], s_red[1][h]), fmaxf(s_red[2][h], s_red[3][h]));
        asm volatile("bar.sync 1, %0;" ::"n"(kTcSmxThreads) : "memory");  // s_red is reused for the sums below
        // tile by tile: the weights, their sum, and the tile's P as 16-bit parts
        // in buffer t % 2, once the products of tile t - 2 are done with it
        for (int t = 0; t < nt; ++t) {
            const int b = t & 1;
            if (t >= 2 && ok) ok = mbar_wait(&pempty[b], ((t - 2) >> 1) & 1u, status, abort_flag);
            if (ok) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(tmem + lane_addr + t * kTcHeads, r);
                tmem_ld_wait();
                const bool live = j0 + t * kTcKeys + key < j1;
                uint8_t* pb = sP + b * NP * kTcPPartBytes;
#pragma unroll
                for (int h = 0; h < kTcHeads; ++h) {
                    if (h >= h0 && h < h1) {
                        const float sv = live ? __uint_as_float(r[h]) * qscale : -INFINITY;
                        const float p = ex2_tc(sv - m[h]);  // 0 for keys past the chunk
                        l[h] += p;
                        uint16_t pt[NP];
                        split_parts<T, NP>(p, pt);
#pragma unroll
                        for (int pp = 0; pp < NP; ++pp)
                            *reinterpret_cast<uint16_t*>(pb + kmaj_offset(pp * kTcHeads + h, key, NP * kTcHeads)) = pt[pp];
                    }
                }
                fence_async_smem();
            }
            mbar_arrive(&pfull[b]);
        }
        // the chunk's sum of weights per head
#pragma unroll
        for (int h = 0; h < kTcHeads; ++h) {
            if (h >= h0 && h < h1) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
                if (lane == 0) s_red[wq][h] = l[h];
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kTcSmxThreads) : "memory");
        // O^T: thread = dim 32 wq + lane, columns = heads
        ok = ok && mbar_wait(&odone, 0, status, abort_flag);
        tc_fence_after();
        if (ok) {
            // O^T = the sum of the accumulators written (tile parity 1 only if nt > 1)
            float o[kTcHeads];
#pragma unroll
            for (int h = 0; h < kTcHeads; ++h) o[h] = 0.0f;
#pragma unroll
            for (int pp = 0; pp < NP; ++pp) {
                uint32_t r0[16], r1[16];
                tmem_ld_32x32b_x16(tmem + lane_addr + kTcOCol + pp * kTcHeads, r0);
                tmem_ld_32x32b_x16(tmem + lane_addr + kTcOCol + (NP + pp) * kTcHeads, r1);
                tmem_ld_wait();
#pragma unroll
                for (int h = 0; h < kTcHeads; ++h)
                    o[h] += nt > 1 ? __uint_as_float(r0[h]) + __uint_as_float(r1[h]) : __uint_as_float(r0[h]);
            }
            const int d = wq * 32 + lane;
#pragma unroll
            for (int h = 0; h < kTcHeads; ++h) {
                if (h >= h0 && h < h1) {
                    float* pp = part + (static_cast<int64_t>(hk * G + h) * chunks + c) * kSdpaPartStride;
                    pp[d] = o[h];
                    if (d == 0) {
                        pp[kSdpaD] = m[h];
                        pp[kSdpaD + 1] = (s_red[0][h] + s_red[1][h]) + (s_red[2][h] + s_red[3][h]);
                    }
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
    const int smem = 1024 + kTcQBytes + kTcStages * kTcTileBytes + 2 * np * kTcPPartBytes;
    auto kern = k_sdpa_tc<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const float qscale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kSdpaD)));
    // V as an MN-major operand: 64-dim atoms 16 KB apart (the two TMA boxes),
    // 8-key groups 1 KB apart; mode 3 of the test switch swaps the two fields
    const bool swap = g_sdpa_kernel.load() == 3;
    const uint32_t lbo = swap ? 1024u : static_cast<uint32_t>(kTcTileBytes / 2);
    const uint32_t sbo = swap ? static_cast<uint32_t>(kTcTileBytes / 2) : 1024u;
    // Prefetch the ring's first stages before the grid-dependency wait only
    // when all of K and V fit in L2.  Measured on B200 (32 query heads,
    // D = 128): GQA8 19.9 -> 19.4 us at N = 32K (67 MB) and 9.6 -> 9.0 us at
    // 4K; GQA4 at 32K (134 MB, more than L2) 29.7 -> 30.4 us, so not there.
    int dev = 0, l2 = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev)) != cudaSuccess) return e;
    const int npre = 2 * rows * kSdpaD * 2 <= static_cast<uint64_t>(l2) ? kTcStages : 0;
    const dim3 grid(static_cast<unsigned>(p.chunks), static_cast<unsigned>(H_kv));
    e = launch_pdl(kern, grid, kTcThreads, smem, st, tmK, tmV, static_cast<const T*>(q), H_q / H_kv, N, p.chunk,
                   p.chunks, qscale, part, lbo, sbo, npre, status);
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

// Chunks of whole 128-key tiles: the fewest tiles per chunk (at most
// kTcMaxTiles) that put every (KV head, chunk) CTA in one wave of one CTA per
// SM, so the SMs get equal shares of the K/V bytes.
SdpaPlan sdpa_tc_plan(int64_t H_q, int64_t H_kv, int64_t N, int num_sms) {
    SdpaPlan p{};
    p.th = static_cast<int>(H_q / H_kv);
    p.tiles = 1;
    const int64_t tiles = (N + kTcKeys - 1) / kTcKeys;  // per KV head
    int64_t t = 1;
    while (t < kTcMaxTiles && H_kv * ((tiles + t - 1) / t) > num_sms) ++t;
    p.chunk = static_cast<int>(t * kTcKeys);
    p.chunks = static_cast<int>((N + p.chunk - 1) / p.chunk);
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
