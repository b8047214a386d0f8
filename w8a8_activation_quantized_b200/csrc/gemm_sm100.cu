// gemm_sm100.cu -- INT8 x INT8 -> INT32 GEMM on the 5th-generation tensor
// cores (tcgen05.mma kind::i8), fused with the dequant epilogue.
//
// What it computes (juejin post "在Mac上跑大模型，MLX 不是终点", sections
// "INT8 TensorOps 内核设计" and "W8A8 对称量化"; Cider README, table "量化"):
//   per-channel  y[m,n] = acc[m,n] * scale_x[m] * scale_w[n],
//   acc = sum_k q[m,k] * w[n,k] in INT32, exact.
// (The per-group and W4A8 forms are in gemm_grouped.cu.)
//
// Two kernels, one CTA (or CTA pair) per SM, persistent over output tiles:
//  * k_gemm_pair -- the large-M kernel: a 256 x 256 tile per cluster of two
//    CTAs with tcgen05.mma.cta_group::2 (see its comment);
//  * k_gemm_sm100 -- single-CTA 128 x BN tiles (BN 256 or 128) for shapes with
//    too few 256 x 256 tiles to fill the GPU.
// Common to both: A = q [M][K] and B = w [N][K] are K-major and land in shared
// memory through TMA with the 128-byte swizzle the UMMA descriptors expect;
// warp 0 (one lane) issues the TMA loads into a ring of mbarrier-guarded
// stages of 128 K values; warp 1 (one lane) issues the MMAs into INT32 TMEM
// accumulators and releases stages with tcgen05.commit; two accumulators let
// the epilogue of one tile overlap the main loop of the next.  Every mbarrier
// wait is bounded (mbar_wait).
//
// The pages' own tiles (BM128 BN128 BK512 on Apple TensorOps) are prior art;
// the sizes here follow from TMEM (512 columns x 128 lanes x 32 bit per SM),
// the 256x256x32 kind::i8 pair MMA shape and 227 KB of shared memory.
#include <algorithm>

#include "gemm_common.cuh"

namespace cider {

// Single-CTA per-channel (and INT32 test) kernel: 128 x BN tiles.
template <int BN_, int MODE_>
struct GemmCfg {
    static constexpr int BN = BN_;
    static constexpr int MODE = MODE_;
    static constexpr int EPI_WARPS = 4;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS);
    static constexpr int A_BYTES = kBM * kBK;
    static constexpr int B_BYTES = BN * kBK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (kSmemBudget / STAGE_BYTES) > 8 ? 8 : (kSmemBudget / STAGE_BYTES);
    static constexpr int ACC_BUFS = 2;
    // two accumulators of BN columns, allocated as a power of two (256 or 512)
    static constexpr int TMEM_COLS = ACC_BUFS * BN <= 256 ? 256 : 512;
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * ACC_BUFS) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
    static_assert(BN % 16 == 0 && BN <= 256, "BN: a multiple of 16 (the M = 128 MMA shape rule), at most 256");
    static_assert(ACC_BUFS * BN <= TMEM_COLS, "TMEM");
};

template <typename TY>
__device__ __forceinline__ void store_row8(TY* dst, const float (&v)[8]) {
    uint4 o;
    o.x = pack2_out<TY>(v[0], v[1]);
    o.y = pack2_out<TY>(v[2], v[3]);
    o.z = pack2_out<TY>(v[4], v[5]);
    o.w = pack2_out<TY>(v[6], v[7]);
    *reinterpret_cast<uint4*>(dst) = o;
}

// 16 accumulator columns of one row m (the tail chunk of a BN that is not a
// multiple of 32): the same expression as store_chunk_pc.
template <int MODE, typename TY>
__device__ __forceinline__ void store_chunk16_pc(const GemmArgs& p, const uint32_t (&r)[16], int m, int n0,
                                                 float sxm) {
    if (MODE == kModeI32) {
        int32_t* out = static_cast<int32_t*>(p.y) + static_cast<int64_t>(m) * p.N;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (n0 + 4 * j < p.N)
                *reinterpret_cast<uint4*>(out + n0 + 4 * j) = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
    } else {
        TY* out = static_cast<TY*>(p.y) + static_cast<int64_t>(m) * p.N;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (n0 + 8 * j < p.N) {
                const float4 w0 = __ldg(reinterpret_cast<const float4*>(p.sw + n0 + 8 * j));
                const float4 w1 = __ldg(reinterpret_cast<const float4*>(p.sw + n0 + 8 * j + 4));
                const float ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    v[e] = (static_cast<float>(static_cast<int32_t>(r[8 * j + e])) * sxm) * ws[e];
                store_row8<TY>(out + n0 + 8 * j, v);
            }
        }
    }
}

// Per-channel (or INT32) epilogue for 32 accumulator columns of one row m:
// y[m, n0..n0+31] = acc * scale_x[m] * scale_w[n], or the raw INT32 values.
template <int MODE, typename TY>
__device__ __forceinline__ void store_chunk_pc(const GemmArgs& p, const uint32_t (&r)[32], int m, int n0, float sxm) {
    if (MODE == kModeI32) {
        int32_t* out = static_cast<int32_t*>(p.y) + static_cast<int64_t>(m) * p.N;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (n0 + 4 * j < p.N)
                *reinterpret_cast<uint4*>(out + n0 + 4 * j) = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
    } else {
        TY* out = static_cast<TY*>(p.y) + static_cast<int64_t>(m) * p.N;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (n0 + 8 * j < p.N) {
                const float4 w0 = __ldg(reinterpret_cast<const float4*>(p.sw + n0 + 8 * j));
                const float4 w1 = __ldg(reinterpret_cast<const float4*>(p.sw + n0 + 8 * j + 4));
                const float ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    v[e] = (static_cast<float>(static_cast<int32_t>(r[8 * j + e])) * sxm) * ws[e];
                store_row8<TY>(out + n0 + 8 * j, v);
            }
        }
    }
}

template <typename Cfg, typename TY>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    k_gemm_sm100(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 GemmArgs p) {
    constexpr int BN = Cfg::BN;
    constexpr int S = Cfg::STAGES;
    constexpr int NB = Cfg::ACC_BUFS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + S * Cfg::A_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + S * Cfg::B_BYTES);
    uint64_t* empty = full + S;
    uint64_t* accf = empty + S;
    uint64_t* acce = accf + NB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + NB);
    __shared__ int s_abort;
    __shared__ uint64_t qready;  // fused launches: the grid's codes are written

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.num_m_blocks * p.num_n_blocks;

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], Cfg::EPI_WARPS * 32);
        }
        mbar_init(&qready, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        // With one block row of A (M <= 128: the weights are nearly all the
        // bytes), the first tile's weight tiles go into L2 before the wait on
        // the previous kernel (the quantizer that writes A), so they stream
        // while it runs (see prefetch_l2_bulk for why this is safe).
        // Measured on B200, N = 10240, K = 2560: M = 128 15.2 -> 14.4 us; at
        // M = 1024 and 4096 (the quantizer already streaming at full rate)
        // it cost 0.7-0.9%, so larger M does not prefetch.
        if (p.num_m_blocks == 1 && blockIdx.x < num_tiles) {
            int mb, nb;
            tile_coords(blockIdx.x, p.num_m_blocks, p.num_n_blocks, mb, nb);
            for (int kb = 0; kb < p.num_k_blocks && kb < kPrefetchKBlocks; ++kb) tma_prefetch_l2_2d(&tmB, kb * kBK, nb * BN);
        }
    }
    if (warp == 1) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    volatile int* abort_flag = &s_abort;
    pdl_wait();  // inputs of the previous kernel on the stream are complete
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            // Fused launch: the weights do not depend on the quantization, so
            // the first ring's B tiles go out while the grid quantizes x; their
            // A tiles follow once the codes are written (qready).
            int pre = 0;
            if (p.x != nullptr) {
                for (int t = blockIdx.x; t < num_tiles && pre < S; t += gridDim.x) {
                    int mb, nb;
                    tile_coords(t, p.num_m_blocks, p.num_n_blocks, mb, nb);
                    for (int kb = 0; kb < p.num_k_blocks && pre < S; ++kb, ++pre) {
                        mbar_arrive_expect_tx(&full[pre], Cfg::STAGE_BYTES);
                        tma_load_2d(sB + pre * Cfg::B_BYTES, &tmB, &full[pre], kb * kBK, nb * BN);
                    }
                }
                ok = mbar_wait(&qready, 0, p.status, abort_flag);
                asm volatile("fence.proxy.async.global;" ::: "memory");  // the codes, for the TMA reads below
            }
            int j = 0;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, p.num_m_blocks, p.num_n_blocks, mb, nb);
                for (int kb = 0; kb < p.num_k_blocks; ++kb, ++j) {
                    if (j < pre) {  // B already in flight on this stage's first use
                        tma_load_2d(sA + stage * Cfg::A_BYTES, &tmA, &full[stage], kb * kBK, mb * kBM);
                    } else {
                        if (!mbar_wait(&empty[stage], phase ^ 1u, p.status, abort_flag)) { ok = false; break; }
                        mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
                        tma_load_2d(sA + stage * Cfg::A_BYTES, &tmA, &full[stage], kb * kBK, mb * kBM);
                        tma_load_2d(sB + stage * Cfg::B_BYTES, &tmB, &full[stage], kb * kBK, nb * BN);
                    }
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_i8(kBM, BN);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t acc_i = 0;  // accumulator-buffer uses so far
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                const uint32_t b = acc_i % NB;
                if (!mbar_wait(&acce[b], ((acc_i / NB) & 1u) ^ 1u, p.status, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + b * BN;
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, p.status, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = umma_desc_sw128(smem_u32(sA + stage * Cfg::A_BYTES));
                    const uint64_t bdesc = umma_desc_sw128(smem_u32(sB + stage * Cfg::B_BYTES));
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk)
                        umma_i8(d, adesc + (kk * kUmmaK >> 4), bdesc + (kk * kUmmaK >> 4), idesc,
                                (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[stage]);
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&accf[b]);
                ++acc_i;
            }
        }
        __syncwarp();
    } else {
        // ------------------------------ epilogue ----------------------------------
        if (p.x != nullptr) {
            // fused launch: quantize this CTA's share of the token rows first
            fused_quantize(p, warp - 2, Cfg::EPI_WARPS);
            asm volatile("bar.sync 2, %0;" ::"n"(Cfg::EPI_WARPS * 32) : "memory");
            if (warp == 2 && lane == 0) {
                // a barrier that runs out leaves the status word set; the
                // kernel still runs to completion
                fused_grid_barrier(p.fuse_slot, p.status, abort_flag);
                mbar_arrive(&qready);
            }
            // scale_x was written in this launch by other CTAs: wait for the
            // barrier's release, and read it from L2 (__ldcg) below
            mbar_wait(&qready, 0, p.status, abort_flag);
        }
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t acc_i = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            int mb, nb;
            tile_coords(t, p.num_m_blocks, p.num_n_blocks, mb, nb);
            const int m = mb * kBM + row;
            const bool mvalid = m < p.M;
            const uint32_t b = acc_i % NB;
            if (!mbar_wait(&accf[b], (acc_i / NB) & 1u, p.status, abort_flag)) { ok = false; break; }
            tc_fence_after();
            // coherent load: a fused launch writes scale_x itself
            const float sxm = (Cfg::MODE == kModePC && mvalid) ? __ldcg(p.sx + m) : 0.0f;
            constexpr int NC = BN / 32;               // whole 32-column chunks
            constexpr bool TAIL = (BN % 32) != 0;     // and one 16-column chunk
#pragma unroll 1
            for (int c = 0; c < NC; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + lane_addr + b * BN + c * 32, r);
                tmem_ld_wait();
                if (!TAIL && c == NC - 1) {
                    tc_fence_before();
                    mbar_arrive(&acce[b]);
                }
                if (mvalid) store_chunk_pc<Cfg::MODE, TY>(p, r, m, nb * BN + c * 32, sxm);
            }
            if constexpr (TAIL) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(tmem_base + lane_addr + b * BN + NC * 32, r);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&acce[b]);
                if (mvalid) store_chunk16_pc<Cfg::MODE, TY>(p, r, m, nb * BN + NC * 32, sxm);
            }
            ++acc_i;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// CTA-pair kernel (per-channel and INT32 modes): one 256 x BN output tile per
// cluster of two CTAs with tcgen05.mma.cta_group::2 (BN = 256, or 192 where
// the narrower tile fills the SM pairs' last round better).  Each CTA stages
// its own 128 rows of A and its half (BN / 2 rows) of B, so per multiply-add
// a CTA moves two thirds of the bytes of the single-CTA 128 x 256 tile.  The
// even CTA (the pair's leader) issues the MMAs; its full barrier counts the
// TMA bytes of both CTAs, the MMA commits arrive on both CTAs' barriers, and
// the epilogue warps of both CTAs report to the leader's accumulator-empty
// barriers.  Each CTA's TMEM holds the accumulator rows of its own 128 rows of A.
// ---------------------------------------------------------------------------
template <int BN_>
struct PairCfgN {
    static constexpr int BM = 256;                   // rows of the pair tile
    static constexpr int BN = BN_;                   // columns of the pair tile
    static constexpr int A_BYTES = 128 * kBK;        // this CTA's rows of A
    static constexpr int B_BYTES = (BN / 2) * kBK;   // this CTA's half of B
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = kSmemBudget / STAGE_BYTES;  // 6 (BN 256), 7 (BN 192)
    static constexpr int ACC_BUFS = 2;
    static constexpr int TMEM_COLS = 512;
    static constexpr int EPI_WARPS = 8;                 // two per TMEM lane quarter
    static constexpr int EPI_COLS = BN / 2;             // columns per epilogue warp
    static constexpr int THREADS = 32 * (2 + EPI_WARPS);
    static constexpr int STG_BYTES = 32 * 32 * 2;       // one 32 x 32 fp16 output box
    static constexpr int STG_PER_WARP = 2;              // double-buffered
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * ACC_BUFS) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_WARPS * STG_PER_WARP * STG_BYTES + BAR_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    // 32-column epilogue chunks per warp; the cta_group::2 M = 256 shape takes N % 16 == 0, N <= 256
    static_assert(BN % 64 == 0 && BN <= 256, "pair tile width");
    static_assert(ACC_BUFS * BN <= TMEM_COLS, "TMEM");
    static_assert(B_BYTES % 1024 == 0, "stage bases on the 1024-byte swizzle atom");
};
using PairCfg = PairCfgN<256>;  // the split-K tail and its reduce use the square tile

// 32 accumulators of one row -> 32 outputs, written as 4 swizzled 16-byte
// chunks into row `r` of a 32 x 32 staging box laid out for the TMA 64-byte
// swizzle (16-byte chunk j of row r lands at chunk j ^ ((r >> 1) & 3)).
template <typename TY>
__device__ __forceinline__ void stage_row32(uint8_t* box, int r, const uint32_t (&acc)[32], const float (&ws)[32],
                                            float sxm) {
    uint8_t* row = box + r * 64;
    const int sw = (r >> 1) & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            v[e] = (static_cast<float>(static_cast<int32_t>(acc[8 * j + e])) * sxm) * ws[8 * j + e];
        uint4 o;
        o.x = pack2_out<TY>(v[0], v[1]);
        o.y = pack2_out<TY>(v[2], v[3]);
        o.z = pack2_out<TY>(v[4], v[5]);
        o.w = pack2_out<TY>(v[6], v[7]);
        *reinterpret_cast<uint4*>(row + ((j ^ sw) << 4)) = o;
    }
}

__device__ __forceinline__ void load_scales32(const float* sw, int n0, int N, float (&ws)[32]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (n0 + 4 * j < N) v = __ldg(reinterpret_cast<const float4*>(sw + n0 + 4 * j));
        ws[4 * j] = v.x;
        ws[4 * j + 1] = v.y;
        ws[4 * j + 2] = v.z;
        ws[4 * j + 3] = v.w;
    }
}

template <int MODE, typename TY, int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfgN<BN>::THREADS, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmP, GemmArgs p) {
    using C = PairCfgN<BN>;
    constexpr int S = C::STAGES;
    constexpr int NB = C::ACC_BUFS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + S * C::A_BYTES;
    uint8_t* sStg = sB + S * C::B_BYTES;  // [EPI_WARPS][2][32 x 32 outputs]
    uint64_t* full = reinterpret_cast<uint64_t*>(sStg + C::EPI_WARPS * C::STG_PER_WARP * C::STG_BYTES);
    uint64_t* empty = full + S;
    uint64_t* accf = empty + S;
    uint64_t* acce = accf + NB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + NB);
    __shared__ int s_abort;
    __shared__ uint64_t qready;  // fused launches: the grid's codes are written

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = (rank == 0);
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(cluster_count_x());
    const int nunits = num_units(p);  // whole tiles, then K pieces of the tail tiles

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 2 * C::EPI_WARPS);  // one arrival per epilogue warp of either CTA
        }
        mbar_init(&qready, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (MODE == kModePC) tma_prefetch_desc(&tmY);
    }
    if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    volatile int* abort_flag = &s_abort;
    pdl_wait();  // inputs of the previous kernel on the stream are complete
    pdl_trigger();

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs): own A rows, own half of B ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            // Fused launch: the first ring's B tiles go out while the grid
            // quantizes x, their A tiles once this CTA's qready has fired.
            int pre = 0;
            if (p.x != nullptr) {
                for (int u = cid; u < nunits && pre < S; u += ncl) {
                    const TileUnit w = tile_unit(p, u);
                    for (int kb = w.kb0; kb < w.kb1 && pre < S; ++kb, ++pre) {
                        if (leader) mbar_arrive_expect_tx(&full[pre], 2 * C::STAGE_BYTES);
                        const uint32_t bar = map_to_rank(&full[pre], 0);
                        tma_load_2d_pair(sB + pre * C::B_BYTES, &tmB, bar, kb * kBK,
                                         w.nb * C::BN + static_cast<int>(rank) * (C::BN / 2));
                    }
                }
                ok = mbar_wait(&qready, 0, p.status, abort_flag);
                asm volatile("fence.proxy.async.global;" ::: "memory");  // the codes, for the TMA reads below
            }
            int j = 0;
            for (int u = cid; u < nunits && ok; u += ncl) {
                const TileUnit w = tile_unit(p, u);
                for (int kb = w.kb0; kb < w.kb1; ++kb, ++j) {
                    const uint32_t bar = map_to_rank(&full[stage], 0);
                    if (j >= pre) {
                        if (!mbar_wait_cluster(&empty[stage], phase ^ 1u, p.status, abort_flag)) { ok = false; break; }
                        if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
                    }
                    tma_load_2d_pair(sA + stage * C::A_BYTES, &tmA, bar, kb * kBK, w.mb * C::BM + static_cast<int>(rank) * 128);
                    if (j >= pre)
                        tma_load_2d_pair(sB + stage * C::B_BYTES, &tmB, bar, kb * kBK,
                                         w.nb * C::BN + static_cast<int>(rank) * (C::BN / 2));
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader CTA only) ----------------
        if (leader && lane == 0) {
            constexpr uint32_t idesc = umma_idesc_i8(C::BM, C::BN);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t acc_i = 0;
            bool ok = true;
            for (int u = cid; u < nunits && ok; u += ncl) {
                const TileUnit w = tile_unit(p, u);
                const uint32_t b = acc_i % NB;
                if (!mbar_wait_cluster(&acce[b], ((acc_i / NB) & 1u) ^ 1u, p.status, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + b * C::BN;
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
                    if (!mbar_wait_cluster(&full[stage], phase, p.status, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = umma_desc_sw128(smem_u32(sA + stage * C::A_BYTES));
                    const uint64_t bdesc = umma_desc_sw128(smem_u32(sB + stage * C::B_BYTES));
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk)
                        umma_i8_pair(d, adesc + (kk * kUmmaK >> 4), bdesc + (kk * kUmmaK >> 4), idesc,
                                     (kb > w.kb0 || kk > 0) ? 1u : 0u);
                    umma_commit_pair(&empty[stage]);
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit_pair(&accf[b]);
                ++acc_i;
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (both CTAs): this CTA's 128 rows x BN columns ----------------
        // Warp w reads TMEM lanes 32*(w%4).. and columns [half*BN/2, (half+1)*BN/2) in
        // chunks of 32, loading chunk c+1 (and its scales) before converting chunk c.
        // Per-channel outputs go through a swizzled shared-memory box and a TMA store.
        if (p.x != nullptr) {
            // fused launch: quantize this CTA's share of the token rows first
            fused_quantize(p, warp - 2, C::EPI_WARPS);
            asm volatile("bar.sync 2, %0;" ::"n"(C::EPI_WARPS * 32) : "memory");
            if (warp == 2 && lane == 0) {
                fused_grid_barrier(p.fuse_slot, p.status, abort_flag);
                mbar_arrive(&qready);
            }
            mbar_wait(&qready, 0, p.status, abort_flag);  // as in k_gemm_sm100: scale_x of this launch
        }
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int half = ew / 4;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint8_t* stg = sStg + ew * C::STG_PER_WARP * C::STG_BYTES;
        constexpr int NCH = C::EPI_COLS / 32;
        uint32_t acc_i = 0, nstore = 0;
        bool ok = true;
        for (int u = cid; u < nunits && ok; u += ncl) {
            const TileUnit w = tile_unit(p, u);
            const int m0 = w.mb * C::BM + static_cast<int>(rank) * 128 + quarter * 32;  // first row of this warp
            const int m = m0 + lane;
            const bool mvalid = m < p.M;
            const int nw = w.nb * C::BN + half * C::EPI_COLS;  // first column of this warp
            const uint32_t b = acc_i % NB;
            const bool piece = w.slot >= 0;  // K piece of a tail tile: INT32 partial sums out
            // coherent load: a fused launch writes scale_x itself
            const float sxm = (MODE == kModePC && mvalid) ? __ldcg(p.sx + m) : 0.0f;
            float ws[2][32];
            if (MODE == kModePC && !piece) load_scales32(p.sw, nw, p.N, ws[0]);
            if (!mbar_wait_cluster(&accf[b], (acc_i / NB) & 1u, p.status, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t r[2][32];
            const uint32_t tbase = tmem_base + lane_addr + b * C::BN + half * C::EPI_COLS;
            tmem_ld_32x32b_x32(tbase, r[0]);
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                tmem_ld_wait();
                if (c + 1 < NCH) {
                    tmem_ld_32x32b_x32(tbase + (c + 1) * 32, r[(c + 1) & 1]);
                    if (MODE == kModePC && !piece) load_scales32(p.sw, nw + (c + 1) * 32, p.N, ws[(c + 1) & 1]);
                } else {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(map_to_rank(&acce[b], 0));
                }
                const int n0 = nw + c * 32;
                if (MODE == kModeI32) {
                    if (mvalid) store_chunk_pc<MODE, TY>(p, r[c & 1], m, n0, sxm);
                } else if (piece) {
                    // this piece's INT32 sums, two 32 x 16 boxes into the tile-local slot
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint8_t* box = stg + (nstore & 1) * C::STG_BYTES;
                        if (lane == 0) bulk_wait_read<1>();
                        __syncwarp();
                        float v[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(r[c & 1][16 * h + e]);
                        stage_row16_f32(box, lane, v);
                        fence_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_3d(&tmP, box, half * C::EPI_COLS + c * 32 + 16 * h,
                                         static_cast<int>(rank) * 128 + quarter * 32, w.slot);
                            bulk_commit();
                        }
                        ++nstore;
                    }
                } else {
                    uint8_t* box = stg + (nstore & 1) * C::STG_BYTES;
                    if (lane == 0) bulk_wait_read<1>();  // the store issued two boxes ago has read `box`
                    __syncwarp();
                    stage_row32<TY>(box, lane, r[c & 1], ws[c & 1], sxm);
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0 && n0 < p.N && m0 < p.M) {
                        tma_store_2d(&tmY, box, n0, m0);
                        bulk_commit();
                    }
                    ++nstore;
                }
            }
            ++acc_i;
        }
        if (MODE == kModePC && lane == 0) bulk_wait<0>();
    }

    tc_fence_before();
    cluster_sync();  // all MMAs of the pair consumed, no peer arrivals in flight
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Host side: launch.
// ---------------------------------------------------------------------------
template <typename Cfg, typename TY>
static cudaError_t launch_gemm_cfg(const GemmLaunch& L, cudaStream_t st) {
    CUtensorMap tmA, tmB;
    if (!make_map_2d(&tmA, L.q, L.K, L.M, kBK, kBM, true)) return cudaErrorInvalidValue;
    if (!make_map_2d(&tmB, L.w, L.K, L.N, kBK, Cfg::BN, true)) return cudaErrorInvalidValue;
    GemmArgs a;
    a.M = L.M;
    a.N = L.N;
    a.K = L.K;
    a.gs = L.gs;
    a.num_m_blocks = (L.M + kBM - 1) / kBM;
    a.num_n_blocks = (L.N + Cfg::BN - 1) / Cfg::BN;
    a.num_k_blocks = (L.K + kBK - 1) / kBK;
    a.sx = L.sx;
    a.sw = L.sw;
    a.y = L.y;
    a.status = L.status;
    a.full_tiles = a.num_m_blocks * a.num_n_blocks;
    a.splits = 1;
    a.kb_per_split = a.num_k_blocks;
    a.x = L.x;
    a.xdt = L.xdt;
    a.qout = const_cast<int8_t*>(L.q);
    a.sxout = const_cast<float*>(L.sx);
    a.fuse_slot = L.fuse_slot;
    const int tiles = a.num_m_blocks * a.num_n_blocks;
    const int grid = tiles < L.num_sms ? tiles : L.num_sms;
    auto kern = k_gemm_sm100<Cfg, TY>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, grid, Cfg::THREADS, Cfg::SMEM_BYTES, st, tmA, tmB, a);
}

// The end of a split tail tile of the per-channel pair GEMM: the pieces'
// INT32 sums add exactly, then y = fp16/bf16((acc * scale_x[m]) * scale_w[n])
// -- the same expression as the fused epilogue, so split and unsplit results
// are equal bit for bit.  32 CTAs per 256 x 256 tail tile (8 rows each), eight
// outputs per thread.
template <typename TY>
__global__ void __launch_bounds__(256) k_splitk_reduce_pc(const int32_t* __restrict__ part, GemmArgs p,
                                                          TY* __restrict__ y) {
    pdl_wait();  // the partial sums of the GEMM before it are complete
    pdl_trigger();
    constexpr int T = PairCfg::BM;  // 256 x 256 tiles
    static_assert(PairCfg::BM == PairCfg::BN, "square pair tiles");
    const int ti = blockIdx.x / (T / 8);
    const int r = (blockIdx.x % (T / 8)) * 8 + threadIdx.x / 32;
    const int c = (threadIdx.x % 32) * 8;
    int mb, nb;
    tile_coords(p.full_tiles + ti, p.num_m_blocks, p.num_n_blocks, mb, nb);
    const int m = mb * T + r, n = nb * T + c;
    if (m >= p.M || n >= p.N) return;
    const int32_t* src = part + (static_cast<int64_t>(ti) * p.splits * T + r) * T + c;
    int acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    constexpr int64_t piece = static_cast<int64_t>(T) * T;
    int s = 0;
    for (; s + 4 <= p.splits; s += 4) {  // four pieces' loads in flight, then the adds
        int4 x[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x[2 * j] = __ldg(reinterpret_cast<const int4*>(src + (s + j) * piece));
            x[2 * j + 1] = __ldg(reinterpret_cast<const int4*>(src + (s + j) * piece) + 1);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[0] += x[2 * j].x; acc[1] += x[2 * j].y; acc[2] += x[2 * j].z; acc[3] += x[2 * j].w;
            acc[4] += x[2 * j + 1].x; acc[5] += x[2 * j + 1].y; acc[6] += x[2 * j + 1].z; acc[7] += x[2 * j + 1].w;
        }
    }
    for (; s < p.splits; ++s) {
        const int4 a = __ldg(reinterpret_cast<const int4*>(src + s * piece));
        const int4 b = __ldg(reinterpret_cast<const int4*>(src + s * piece) + 1);
        acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
        acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
    const float sxm = __ldg(p.sx + m);
    const float4 w0 = __ldg(reinterpret_cast<const float4*>(p.sw + n));
    const float4 w1 = __ldg(reinterpret_cast<const float4*>(p.sw + n) + 1);
    const float ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = (static_cast<float>(acc[e]) * sxm) * ws[e];
    store_row8<TY>(y + static_cast<int64_t>(m) * p.N + n, v);
}

template <int MODE, typename TY, int BN>
static cudaError_t launch_gemm_pair(const GemmLaunch& L, cudaStream_t st) {
    using C = PairCfgN<BN>;
    CUtensorMap tmA, tmB, tmY, tmP;
    if (!make_map_2d(&tmA, L.q, L.K, L.M, kBK, 128, true)) return cudaErrorInvalidValue;
    if (!make_map_2d(&tmB, L.w, L.K, L.N, kBK, C::BN / 2, true)) return cudaErrorInvalidValue;
    if (MODE == kModePC) {
        if (!make_map_out(&tmY, L.y, L.M, L.N, L.ydt)) return cudaErrorInvalidValue;
    } else {
        tmY = tmA;  // unused by the INT32 epilogue
    }
    GemmArgs a;
    a.M = L.M;
    a.N = L.N;
    a.K = L.K;
    a.gs = 0;
    a.num_m_blocks = (L.M + C::BM - 1) / C::BM;
    a.num_n_blocks = (L.N + C::BN - 1) / C::BN;
    a.num_k_blocks = (L.K + kBK - 1) / kBK;
    a.sx = L.sx;
    a.sw = L.sw;
    a.y = L.y;
    a.status = L.status;
    a.x = L.x;
    a.xdt = L.xdt;
    a.qout = const_cast<int8_t*>(L.q);
    a.sxout = const_cast<float*>(L.sx);
    a.fuse_slot = L.fuse_slot;
    const int tiles = a.num_m_blocks * a.num_n_blocks;
    // split K of the tail tiles (per-channel square tiles with a partial-sum buffer only)
    int splits = (MODE == kModePC && BN == PairCfg::BN && L.part != nullptr && L.splits > 1) ? L.splits : 1;
    const int full = splits > 1 ? std::min(std::max(L.full_tiles, 0), tiles) : tiles;
    a.kb_per_split = (a.num_k_blocks + splits - 1) / splits;
    a.splits = (a.num_k_blocks + a.kb_per_split - 1) / a.kb_per_split;
    a.full_tiles = a.splits > 1 ? full : tiles;
    if (a.splits > 1 && a.full_tiles < tiles) {
        if (!make_map_part(&tmP, L.part, PairCfg::BM, PairCfg::BN, (tiles - full) * splits)) return cudaErrorInvalidValue;
    } else {
        a.splits = 1;
        a.full_tiles = tiles;
        tmP = tmA;  // unused without split partial sums
    }
    const int units = a.full_tiles + (tiles - a.full_tiles) * a.splits;
    const int clusters = units < L.num_sms / 2 ? units : L.num_sms / 2;
    auto kern = k_gemm_pair<MODE, TY, BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, 2 * clusters, C::THREADS, C::SMEM_BYTES, st, tmA, tmB, tmY, tmP, a);
    if (e != cudaSuccess || a.splits == 1) return e;
    return launch_pdl(k_splitk_reduce_pc<TY>, (tiles - a.full_tiles) * (PairCfg::BM / 8), 256, 0, st,
                      reinterpret_cast<const int32_t*>(L.part), a, static_cast<TY*>(L.y));
}

template <int MODE, typename TY>
static cudaError_t launch_gemm_mode(const GemmLaunch& L, cudaStream_t st) {
    if (L.variant == kGemmPair) return launch_gemm_pair<MODE, TY, 256>(L, st);
    if (L.variant == kGemmPair192) return launch_gemm_pair<MODE, TY, 192>(L, st);
    if (L.variant == kGemmSingle128) return launch_gemm_cfg<GemmCfg<128, MODE>, TY>(L, st);
    if (L.variant == kGemmSingle80) return launch_gemm_cfg<GemmCfg<80, MODE>, TY>(L, st);
    return launch_gemm_cfg<GemmCfg<256, MODE>, TY>(L, st);
}

cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t st) {
    const bool bf = (L.ydt == 1);
    switch (L.mode) {
        case kModePC: return bf ? launch_gemm_mode<kModePC, __nv_bfloat16>(L, st) : launch_gemm_mode<kModePC, __half>(L, st);
        case kModeI32: return launch_gemm_mode<kModeI32, __half>(L, st);
        case kModePG:
        case kModeW4:
        case kModeI32G:
        case kModeW4PC: return launch_gemm_grouped(L, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace cider
