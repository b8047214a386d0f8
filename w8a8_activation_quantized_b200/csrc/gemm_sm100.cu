// gemm_sm100.cu -- INT8 x INT8 -> INT32 GEMM on the 5th-generation tensor
// cores (tcgen05.mma kind::i8), fused with the dequant epilogue.
//
// What it computes (juejin post "在Mac上跑大模型，MLX 不是终点", sections
// "INT8 TensorOps 内核设计" and "三种量化粒度的实现"; Cider README, table "量化"):
//   per-channel  y[m,n] = acc[m,n] * scale_x[m] * scale_w[n]
//   per-group    y[m,n] = scale_x[m] * sum_g acc_g[m,n] * scale_w[g][n]
//   W4A8         the per-group form with INT4 weights unpacked to INT8 on chip
// acc = sum_k q[m,k] * w[n,k] in INT32, exact.
//
// Design (sm_100a, one CTA per SM, persistent over output tiles):
//  * tile BM=128 x BN (256 per-channel, 128 per-group) x BK=128 int8 per stage;
//    A = q [M][K] and B = w [N][K] are both K-major and land in shared
//    memory through TMA with the 128-byte swizzle the UMMA descriptors expect;
//  * warp 0 (one lane) issues the TMA loads into a ring of mbarrier-guarded
//    stages; warp 1 (one lane) issues tcgen05.mma into tensor-memory (TMEM)
//    INT32 accumulators and releases stages with tcgen05.commit;
//  * per-channel: two TMEM accumulators of BN columns, so the epilogue of
//    tile i overlaps the main loop of tile i+1;
//  * per-group: every group of gs (64 or 128) K values gets its own INT32
//    partial in a ring of TMEM buffers; the epilogue warps read each partial
//    (tcgen05.ld), rescale it by its group's weight scale in fp32 and keep the
//    running sums in registers -- the "piecewise multiply" of the pages;
//  * W4A8: packed [N][K/2] tiles arrive by TMA unswizzled; four converter warps
//    expand each nibble to int8 (nibble - 8) into the swizzled B stage, fence
//    the writes to the async proxy, and hand the stage to the MMA warp;
//  * every mbarrier wait is bounded (see mbar_wait).
//
// The pages' own tiles (BM128 BN128 BK512 on Apple TensorOps) are prior art;
// the sizes here follow from TMEM (512 columns x 128 lanes x 32 bit per SM),
// the 128x256x32 kind::i8 MMA shape and 227 KB of shared memory.
#include "cider_device.cuh"
#include "cider_kernels.h"

namespace cider {

constexpr int kBM = 128;
constexpr int kBK = 128;      // int8 K values per stage = one 128-byte swizzle row
constexpr int kUmmaK = 32;    // K per kind::i8 MMA
constexpr int kGroupM = 8;    // tile raster: 8 M-blocks share each N-block in turn
constexpr int kSmemBudget = 196608;

template <int BN_, int MODE_>
struct GemmCfg {
    static constexpr int BN = BN_;
    static constexpr int MODE = MODE_;
    static constexpr bool GROUPED = (MODE == kModePG || MODE == kModeW4 || MODE == kModeI32G);
    static constexpr bool W4 = (MODE == kModeW4);
    static constexpr int EPI_WARPS = GROUPED ? 8 : 4;
    static constexpr int CONV_WARPS = W4 ? 4 : 0;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS + CONV_WARPS);
    static constexpr int A_BYTES = kBM * kBK;
    static constexpr int B_BYTES = BN * kBK;
    static constexpr int BP_BYTES = W4 ? BN * kBK / 2 : 0;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + BP_BYTES;
    static constexpr int STAGES = (kSmemBudget / STAGE_BYTES) > 8 ? 8 : (kSmemBudget / STAGE_BYTES);
    static constexpr int ACC_BUFS = GROUPED ? 512 / BN : 2;
    static constexpr int TMEM_COLS = ACC_BUFS * BN;  // 256 or 512
    static constexpr int EPI_COLS = GROUPED ? BN / 2 : BN;  // columns per epilogue thread
    static constexpr int BAR_BYTES = 8 * (3 * STAGES + 2 * ACC_BUFS) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
    static_assert(BN % 32 == 0 && BN <= 256, "BN");
    static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of two");
    static_assert(STAGES >= 2, "stages");
};

struct GemmArgs {
    int M, N, K;
    int gs;             // group size (grouped modes)
    int num_m_blocks, num_n_blocks, num_k_blocks;
    const float* sx;    // [M]
    const float* sw;    // [N] or [G][N]
    void* y;            // [M][N] output (fp16/bf16), or int32 acc / acc_g in test modes
    unsigned* status;   // device status word
};

__device__ __forceinline__ void tile_coords(int t, int nm, int nn, int& mb, int& nb) {
    const int per_group = kGroupM * nn;
    const int grp = t / per_group;
    const int first_m = grp * kGroupM;
    const int gm = min(nm - first_m, kGroupM);
    const int r = t % per_group;
    mb = first_m + r % gm;
    nb = r / gm;
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <typename TY>
__device__ __forceinline__ void store_row8(TY* dst, const float (&v)[8]) {
    uint4 o;
    o.x = pack2_out<TY>(v[0], v[1]);
    o.y = pack2_out<TY>(v[2], v[3]);
    o.z = pack2_out<TY>(v[4], v[5]);
    o.w = pack2_out<TY>(v[6], v[7]);
    *reinterpret_cast<uint4*>(dst) = o;
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
    uint8_t* sBP = sB + S * Cfg::B_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sBP + S * Cfg::BP_BYTES);
    uint64_t* empty = full + S;
    uint64_t* conv = empty + S;
    uint64_t* accf = conv + S;
    uint64_t* acce = accf + NB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + NB);
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.num_m_blocks * p.num_n_blocks;

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&conv[s], Cfg::CONV_WARPS * 32);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], Cfg::EPI_WARPS * 32);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    volatile int* abort_flag = &s_abort;

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            const uint32_t tx = Cfg::A_BYTES + (Cfg::W4 ? Cfg::BP_BYTES : Cfg::B_BYTES);
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, p.num_m_blocks, p.num_n_blocks, mb, nb);
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.status, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[stage], tx);
                    tma_load_2d(sA + stage * Cfg::A_BYTES, &tmA, &full[stage], kb * kBK, mb * kBM);
                    if (Cfg::W4)
                        tma_load_2d(sBP + stage * Cfg::BP_BYTES, &tmB, &full[stage], kb * (kBK / 2), nb * BN);
                    else
                        tma_load_2d(sB + stage * Cfg::B_BYTES, &tmB, &full[stage], kb * kBK, nb * BN);
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
            const int G = Cfg::GROUPED ? p.K / p.gs : 0;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                int g = 0;  // next group of this tile (grouped modes)
                if (!Cfg::GROUPED) {
                    const uint32_t b = acc_i % NB;
                    if (!mbar_wait(&acce[b], ((acc_i / NB) & 1u) ^ 1u, p.status, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                }
                for (int kb = 0; kb < p.num_k_blocks && ok; ++kb) {
                    if (!mbar_wait(&full[stage], phase, p.status, abort_flag)) { ok = false; break; }
                    if (Cfg::W4 && !mbar_wait(&conv[stage], phase, p.status, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = umma_desc_sw128(smem_u32(sA + stage * Cfg::A_BYTES));
                    const uint64_t bdesc = umma_desc_sw128(smem_u32(sB + stage * Cfg::B_BYTES));
                    if (!Cfg::GROUPED) {
                        const uint32_t d = tmem_base + (acc_i % NB) * BN;
#pragma unroll
                        for (int kk = 0; kk < kBK / kUmmaK; ++kk)
                            umma_i8(d, adesc + (kk * kUmmaK >> 4), bdesc + (kk * kUmmaK >> 4), idesc,
                                    (kb > 0 || kk > 0) ? 1u : 0u);
                    } else {
                        const int gpk = kBK / p.gs;  // groups per stage: 1 or 2
                        const int steps = p.gs / kUmmaK;
                        for (int j = 0; j < gpk && g < G; ++j, ++g) {
                            const uint32_t b = acc_i % NB;
                            if (!mbar_wait(&acce[b], ((acc_i / NB) & 1u) ^ 1u, p.status, abort_flag)) { ok = false; break; }
                            tc_fence_after();
                            const uint32_t d = tmem_base + b * BN;
                            for (int kk = 0; kk < steps; ++kk) {
                                const int off = (j * steps + kk) * kUmmaK;
                                umma_i8(d, adesc + (off >> 4), bdesc + (off >> 4), idesc, kk > 0 ? 1u : 0u);
                            }
                            umma_commit(&accf[b]);
                            ++acc_i;
                        }
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
                if (!Cfg::GROUPED && ok) {
                    umma_commit(&accf[acc_i % NB]);
                    ++acc_i;
                }
            }
        }
        __syncwarp();
    } else if (warp < 2 + Cfg::EPI_WARPS) {
        // ------------------------------ epilogue ----------------------------------
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int colhalf = Cfg::GROUPED ? (warp - 2) / 4 : 0;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t acc_i = 0;
        bool ok = true;
        const int G = Cfg::GROUPED ? p.K / p.gs : 0;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            int mb, nb;
            tile_coords(t, p.num_m_blocks, p.num_n_blocks, mb, nb);
            const int m = mb * kBM + row;
            const bool mvalid = m < p.M;
            const int n_base = nb * BN + colhalf * Cfg::EPI_COLS;
            if (!Cfg::GROUPED) {
                const uint32_t b = acc_i % NB;
                if (!mbar_wait(&accf[b], (acc_i / NB) & 1u, p.status, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const float sxm = (Cfg::MODE == kModePC && mvalid) ? __ldg(p.sx + m) : 0.0f;
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem_base + lane_addr + b * BN + c * 32, r);
                    tmem_ld_wait();
                    if (c == BN / 32 - 1) {
                        tc_fence_before();
                        mbar_arrive(&acce[b]);
                    }
                    if (mvalid) store_chunk_pc<Cfg::MODE, TY>(p, r, m, n_base + c * 32, sxm);
                }
                ++acc_i;
            } else {
                float sum[Cfg::EPI_COLS];
#pragma unroll
                for (int j = 0; j < Cfg::EPI_COLS; ++j) sum[j] = 0.0f;
                for (int g = 0; g < G; ++g) {
                    const uint32_t b = acc_i % NB;
                    if (!mbar_wait(&accf[b], (acc_i / NB) & 1u, p.status, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const float* swg = p.sw + static_cast<int64_t>(g) * p.N;
#pragma unroll
                    for (int c = 0; c < Cfg::EPI_COLS / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(tmem_base + lane_addr + b * BN + colhalf * Cfg::EPI_COLS + c * 32, r);
                        tmem_ld_wait();
                        if (c == Cfg::EPI_COLS / 32 - 1) {
                            tc_fence_before();
                            mbar_arrive(&acce[b]);
                        }
                        const int n0 = n_base + c * 32;
                        if (Cfg::MODE == kModeI32G) {
                            if (mvalid) {
                                int32_t* out = static_cast<int32_t*>(p.y) +
                                               (static_cast<int64_t>(g) * p.M + m) * p.N;
#pragma unroll
                                for (int j = 0; j < 8; ++j)
                                    if (n0 + 4 * j < p.N)
                                        *reinterpret_cast<uint4*>(out + n0 + 4 * j) = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
                                if (n0 + 4 * j < p.N) w4 = __ldg(reinterpret_cast<const float4*>(swg + n0 + 4 * j));
                                sum[c * 32 + 4 * j + 0] = fmaf(static_cast<float>(static_cast<int32_t>(r[4 * j + 0])), w4.x, sum[c * 32 + 4 * j + 0]);
                                sum[c * 32 + 4 * j + 1] = fmaf(static_cast<float>(static_cast<int32_t>(r[4 * j + 1])), w4.y, sum[c * 32 + 4 * j + 1]);
                                sum[c * 32 + 4 * j + 2] = fmaf(static_cast<float>(static_cast<int32_t>(r[4 * j + 2])), w4.z, sum[c * 32 + 4 * j + 2]);
                                sum[c * 32 + 4 * j + 3] = fmaf(static_cast<float>(static_cast<int32_t>(r[4 * j + 3])), w4.w, sum[c * 32 + 4 * j + 3]);
                            }
                        }
                    }
                    ++acc_i;
                }
                if (!ok) break;
                if (Cfg::MODE != kModeI32G && mvalid) {
                    const float sxm = __ldg(p.sx + m);
                    TY* out = static_cast<TY*>(p.y) + static_cast<int64_t>(m) * p.N;
#pragma unroll
                    for (int j = 0; j < Cfg::EPI_COLS / 8; ++j) {
                        if (n_base + 8 * j < p.N) {
                            float v[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) v[e] = sum[8 * j + e] * sxm;
                            store_row8<TY>(out + n_base + 8 * j, v);
                        }
                    }
                }
            }
        }
    } else {
        // --------------------- W4A8 converter warps: INT4 -> INT8 ------------------
        if (Cfg::W4) {
            const int ct = threadIdx.x - 32 * (2 + Cfg::EPI_WARPS);  // 0..127
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, p.status, abort_flag)) { ok = false; break; }
                    const uint8_t* src = sBP + stage * Cfg::BP_BYTES;  // [BN][64] packed, row-major
                    uint8_t* dst = sB + stage * Cfg::B_BYTES;          // [BN][128] int8, 128B swizzle
#pragma unroll
                    for (int it = 0; it < BN * 4 / 128; ++it) {
                        const int item = ct + 128 * it;
                        const int r = item >> 2, j = item & 3;  // row, 16-byte packed chunk
                        const uint4 pk = *reinterpret_cast<const uint4*>(src + r * 64 + j * 16);
                        const uint2 u0 = unpack_int4x8(pk.x), u1 = unpack_int4x8(pk.y);
                        const uint2 u2 = unpack_int4x8(pk.z), u3 = unpack_int4x8(pk.w);
                        uint8_t* row = dst + r * 128;
                        const int sw = r & 7;
                        *reinterpret_cast<uint4*>(row + (((2 * j) ^ sw) << 4)) = make_uint4(u0.x, u0.y, u1.x, u1.y);
                        *reinterpret_cast<uint4*>(row + (((2 * j + 1) ^ sw) << 4)) = make_uint4(u2.x, u2.y, u3.x, u3.y);
                    }
                    fence_async_smem();
                    mbar_arrive(&conv[stage]);
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            }
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
// CTA-pair kernel (per-channel and INT32 modes): one 256 x 256 output tile per
// cluster of two CTAs with tcgen05.mma.cta_group::2.  Each CTA stages its own
// 128 rows of A and its half (128 rows) of B, so per multiply-add a CTA moves
// two thirds of the bytes of the single-CTA 128 x 256 tile.  The even CTA
// (the pair's leader) issues the MMAs; its full barrier counts the TMA bytes of
// both CTAs, the MMA commits arrive on both CTAs' barriers, and the epilogue
// warps of both CTAs report to the leader's accumulator-empty barriers.
// Each CTA's TMEM holds the accumulator rows of its own 128 rows of A.
// ---------------------------------------------------------------------------
struct PairCfg {
    static constexpr int BM = 256;                   // rows of the pair tile
    static constexpr int BN = 256;                   // columns of the pair tile
    static constexpr int A_BYTES = 128 * kBK;        // this CTA's rows of A
    static constexpr int B_BYTES = (BN / 2) * kBK;   // this CTA's half of B
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = kSmemBudget / STAGE_BYTES;  // 6
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
};

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

template <int MODE, typename TY>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg::THREADS, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, GemmArgs p) {
    using C = PairCfg;
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

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = (rank == 0);
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(cluster_count_x());
    const int num_tiles = p.num_m_blocks * p.num_n_blocks;

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

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs): own A rows, own half of B ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = cid; t < num_tiles && ok; t += ncl) {
                int mb, nb;
                tile_coords(t, p.num_m_blocks, p.num_n_blocks, mb, nb);
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait_cluster(&empty[stage], phase ^ 1u, p.status, abort_flag)) { ok = false; break; }
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
                    const uint32_t bar = map_to_rank(&full[stage], 0);
                    tma_load_2d_pair(sA + stage * C::A_BYTES, &tmA, bar, kb * kBK, mb * C::BM + static_cast<int>(rank) * 128);
                    tma_load_2d_pair(sB + stage * C::B_BYTES, &tmB, bar, kb * kBK, nb * C::BN + static_cast<int>(rank) * (C::BN / 2));
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
            for (int t = cid; t < num_tiles && ok; t += ncl) {
                const uint32_t b = acc_i % NB;
                if (!mbar_wait_cluster(&acce[b], ((acc_i / NB) & 1u) ^ 1u, p.status, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + b * C::BN;
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait_cluster(&full[stage], phase, p.status, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = umma_desc_sw128(smem_u32(sA + stage * C::A_BYTES));
                    const uint64_t bdesc = umma_desc_sw128(smem_u32(sB + stage * C::B_BYTES));
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk)
                        umma_i8_pair(d, adesc + (kk * kUmmaK >> 4), bdesc + (kk * kUmmaK >> 4), idesc,
                                     (kb > 0 || kk > 0) ? 1u : 0u);
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
        // ---------------- epilogue (both CTAs): this CTA's 128 rows x 256 columns ----------------
        // Warp w reads TMEM lanes 32*(w%4).. and columns [half*128, half*128+128) in
        // chunks of 32, loading chunk c+1 (and its scales) before converting chunk c.
        // Per-channel outputs go through a swizzled shared-memory box and a TMA store.
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int half = ew / 4;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint8_t* stg = sStg + ew * C::STG_PER_WARP * C::STG_BYTES;
        constexpr int NCH = C::EPI_COLS / 32;
        uint32_t acc_i = 0, nstore = 0;
        bool ok = true;
        for (int t = cid; t < num_tiles && ok; t += ncl) {
            int mb, nb;
            tile_coords(t, p.num_m_blocks, p.num_n_blocks, mb, nb);
            const int m0 = mb * C::BM + static_cast<int>(rank) * 128 + quarter * 32;  // first row of this warp
            const int m = m0 + lane;
            const bool mvalid = m < p.M;
            const int nw = nb * C::BN + half * C::EPI_COLS;  // first column of this warp
            const uint32_t b = acc_i % NB;
            const float sxm = (MODE == kModePC && mvalid) ? __ldg(p.sx + m) : 0.0f;
            float ws[2][32];
            if (MODE == kModePC) load_scales32(p.sw, nw, p.N, ws[0]);
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
                    if (MODE == kModePC) load_scales32(p.sw, nw + (c + 1) * 32, p.N, ws[(c + 1) & 1]);
                } else {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(map_to_rank(&acce[b], 0));
                }
                const int n0 = nw + c * 32;
                if (MODE == kModeI32) {
                    if (mvalid) store_chunk_pc<MODE, TY>(p, r[c & 1], m, n0, sxm);
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
// Host side: tensor maps and launch.
// ---------------------------------------------------------------------------
static bool make_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                        uint32_t box_inner, uint32_t box_rows, bool swizzle128) {
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner};  // bytes (uint8 elements)
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return encode_tensor_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                             strides, box, estr,
                             swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <typename Cfg, typename TY>
static cudaError_t launch_gemm_cfg(const GemmLaunch& L, cudaStream_t st) {
    CUtensorMap tmA, tmB;
    if (!make_map_2d(&tmA, L.q, L.K, L.M, kBK, kBM, true)) return cudaErrorInvalidValue;
    if (Cfg::W4) {
        if (!make_map_2d(&tmB, L.w, L.K / 2, L.N, kBK / 2, Cfg::BN, false)) return cudaErrorInvalidValue;
    } else {
        if (!make_map_2d(&tmB, L.w, L.K, L.N, kBK, Cfg::BN, true)) return cudaErrorInvalidValue;
    }
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
    const int tiles = a.num_m_blocks * a.num_n_blocks;
    const int grid = tiles < L.num_sms ? tiles : L.num_sms;
    auto kern = k_gemm_sm100<Cfg, TY>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, st>>>(tmA, tmB, a);
    return cudaGetLastError();
}

// Output map for the TMA stores of the epilogue: [M][N] 16-bit values, 32 x 32
// boxes, 64-byte swizzle.
static bool make_map_out(CUtensorMap* map, void* y, int M, int N, int ydt) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    return encode_tensor_map(map, ydt == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, y,
                             dims, strides, box, estr, CU_TENSOR_MAP_SWIZZLE_64B);
}

template <int MODE, typename TY>
static cudaError_t launch_gemm_pair(const GemmLaunch& L, cudaStream_t st) {
    CUtensorMap tmA, tmB, tmY;
    if (!make_map_2d(&tmA, L.q, L.K, L.M, kBK, 128, true)) return cudaErrorInvalidValue;
    if (!make_map_2d(&tmB, L.w, L.K, L.N, kBK, PairCfg::BN / 2, true)) return cudaErrorInvalidValue;
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
    a.num_m_blocks = (L.M + PairCfg::BM - 1) / PairCfg::BM;
    a.num_n_blocks = (L.N + PairCfg::BN - 1) / PairCfg::BN;
    a.num_k_blocks = (L.K + kBK - 1) / kBK;
    a.sx = L.sx;
    a.sw = L.sw;
    a.y = L.y;
    a.status = L.status;
    const int tiles = a.num_m_blocks * a.num_n_blocks;
    const int clusters = tiles < L.num_sms / 2 ? tiles : L.num_sms / 2;
    auto kern = k_gemm_pair<MODE, TY>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<2 * clusters, PairCfg::THREADS, PairCfg::SMEM_BYTES, st>>>(tmA, tmB, tmY, a);
    return cudaGetLastError();
}

template <int MODE, typename TY>
static cudaError_t launch_gemm_mode(const GemmLaunch& L, cudaStream_t st) {
    if constexpr (MODE == kModePC || MODE == kModeI32) {
        if (L.variant == kGemmPair) return launch_gemm_pair<MODE, TY>(L, st);
        if (L.variant == kGemmSingle128) return launch_gemm_cfg<GemmCfg<128, MODE>, TY>(L, st);
        return launch_gemm_cfg<GemmCfg<256, MODE>, TY>(L, st);
    } else {
        return launch_gemm_cfg<GemmCfg<128, MODE>, TY>(L, st);
    }
}

cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t st) {
    const bool bf = (L.ydt == 1);
    switch (L.mode) {
        case kModePC: return bf ? launch_gemm_mode<kModePC, __nv_bfloat16>(L, st) : launch_gemm_mode<kModePC, __half>(L, st);
        case kModePG: return bf ? launch_gemm_mode<kModePG, __nv_bfloat16>(L, st) : launch_gemm_mode<kModePG, __half>(L, st);
        case kModeW4: return bf ? launch_gemm_mode<kModeW4, __nv_bfloat16>(L, st) : launch_gemm_mode<kModeW4, __half>(L, st);
        case kModeI32: return launch_gemm_mode<kModeI32, __half>(L, st);
        case kModeI32G: return launch_gemm_mode<kModeI32G, __half>(L, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace cider
