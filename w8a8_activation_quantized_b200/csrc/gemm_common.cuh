// gemm_common.cuh -- pieces shared by the tcgen05 GEMM kernels: tile sizes,
// kernel arguments, the tile raster, tensor maps and the output staging.
#pragma once

#include "cider_device.cuh"
#include "cider_kernels.h"

namespace cider {

constexpr int kBM = 128;          // rows of A per CTA tile
constexpr int kBK = 128;          // int8 K values per stage = one 128-byte swizzle row
constexpr int kUmmaK = 32;        // K per kind::i8 MMA
constexpr int kGroupM = 8;        // tile raster: 8 M-blocks share each N-block in turn
constexpr int kSmemBudget = 196608;
// k-blocks of a CTA's first weight tile requested into L2 before its
// grid-dependency wait (one 128-wide k-block per request).
constexpr int kPrefetchKBlocks = 32;
constexpr int kSmemMax = 232448;  // dynamic shared memory per CTA on sm_100

struct GemmArgs {
    int M, N, K;
    int gs;             // group size (grouped modes)
    int num_m_blocks, num_n_blocks, num_k_blocks;
    // grouped modes: tiles [0, full_tiles) run over all of K; every later tile
    // is cut into `splits` K pieces of kb_per_split k-blocks
    int full_tiles, splits, kb_per_split;
    const float* sx;    // [M]
    const float* sw;    // [N] or [G][N]
    void* y;            // [M][N] output (fp16/bf16), or int32 acc / acc_g in test modes
    unsigned* status;   // device status word
    // Fused activation quantization (per-channel kernels): with x set, the
    // kernel itself quantizes x [M][K] (xdt) into qout [M][K] and sxout [M] --
    // the buffers its A tensor map and sx point at -- before its first A load,
    // synchronising the grid on barrier slot fuse_slot.
    const void* x = nullptr;
    int xdt = 0;
    int8_t* qout = nullptr;
    float* sxout = nullptr;
    int fuse_slot = 0;
};

// ---- fused activation quantization -----------------------------------------
// Barrier slots of the fused launches (kFuseSlots, cider_kernels.h),
// {arrivals, generation} each.  Zero at load; every launch leaves its slot's
// arrival count at zero again.  Only the per-channel kernels' translation
// unit uses them.
static __device__ unsigned g_fuse_bar[kFuseSlots][2];

__device__ __forceinline__ float fuse_warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Quantizer warp wq of nwq in every CTA: rows r = blockIdx.x + gridDim.x * (wq
// + nwq * i), one warp per row -- the row's absmax over all of K, then its
// codes -- with the same arithmetic as cider_quantize_act (act_scale,
// quant8_codes), so the codes are those of the separate quantize kernel.
// Rows of up to 32 * kFuseNV 16-byte chunks (K <= 6144) are loaded once, all
// loads in flight together, and quantized from registers: one memory round
// trip per row.  Wider rows take two passes over x (the second from L2).
constexpr int kFuseNV = 12;
template <typename TX>
__device__ __forceinline__ void fused_quantize_rows(const GemmArgs& p, int wq, int nwq) {
    const int lane = threadIdx.x & 31;
    const int nch = p.K / 8;
    for (int64_t r = blockIdx.x + static_cast<int64_t>(gridDim.x) * wq; r < p.M;
         r += static_cast<int64_t>(gridDim.x) * nwq) {
        const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const TX*>(p.x) + r * p.K);
        int8_t* qr = p.qout + r * p.K;
        typename Pack2<TX>::type m2 = {};
        if (nch <= 32 * kFuseNV) {
            uint4 v[kFuseNV];
#pragma unroll
            for (int i = 0; i < kFuseNV; ++i) {
                const int c = lane + 32 * i;
                v[i] = c < nch ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < kFuseNV; ++i) m2 = absmax8<TX>(v[i], m2);
            const float amax = fuse_warp_max(absmax_to_f32<TX>(m2));
            const float s = act_scale(amax);
            const float rs = act_rcp(s);
            if (lane == 0) p.sxout[r] = s;
#pragma unroll
            for (int i = 0; i < kFuseNV; ++i) {
                const int c = lane + 32 * i;
                if (c < nch) {
                    float f[8];
                    unpack8_f32<TX>(v[i], f);
                    *reinterpret_cast<uint2*>(qr + 8 * c) = quant8_codes(f, s, rs);
                }
            }
        } else {
#pragma unroll 4
            for (int c = lane; c < nch; c += 32) m2 = absmax8<TX>(__ldg(xr + c), m2);
            const float amax = fuse_warp_max(absmax_to_f32<TX>(m2));
            const float s = act_scale(amax);
            const float rs = act_rcp(s);
            if (lane == 0) p.sxout[r] = s;
#pragma unroll 4
            for (int c = lane; c < nch; c += 32) {
                float f[8];
                unpack8_f32<TX>(__ldg(xr + c), f);
                *reinterpret_cast<uint2*>(qr + 8 * c) = quant8_codes(f, s, rs);
            }
        }
    }
    // these generic-proxy writes are read by other CTAs' TMA (async proxy)
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void fused_quantize(const GemmArgs& p, int wq, int nwq) {
    if (p.xdt == 1)
        fused_quantize_rows<__nv_bfloat16>(p, wq, nwq);
    else
        fused_quantize_rows<__half>(p, wq, nwq);
}

// Grid-wide barrier of a fused launch, called by one thread per CTA after its
// CTA's quantizer warps have synchronised.  Every CTA of the grid is resident
// (one per SM, grid <= SMs).  Sense-reversing on the launch's slot: read the
// generation, arrive; the last arrival resets the count and bumps the
// generation, the others wait for that bump -- bounded in time like every
// other wait.  On timeout it records CIDER_ERR_TIMEOUT in the status word and
// returns false without aborting the CTA: the kernel then runs to completion
// on whatever codes are in place, and the caller learns of the failure from
// cider_device_status().
__device__ __forceinline__ bool fused_grid_barrier(int slot, unsigned* status, volatile int* abort_flag) {
    unsigned* cnt = &g_fuse_bar[slot][0];
    unsigned* gen = &g_fuse_bar[slot][1];
    unsigned g0;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(g0) : "l"(gen) : "memory");
    __threadfence();
    const unsigned arrived = atomicAdd(cnt, 1u) + 1u;
    if (arrived == gridDim.x) {
        atomicExch(cnt, 0u);
        __threadfence();
        asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(gen), "r"(g0 + 1u) : "memory");
        return true;
    }
    const unsigned long long t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        unsigned g;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(g) : "l"(gen) : "memory");
        if (g != g0) return true;
        if ((it & 63u) == 0u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicOr(status, kStatusTimeout);
                return false;
            }
        }
        __nanosleep(64);
    }
}

// Raster: kGroupM consecutive M-blocks walk the N-blocks together, so the
// CTAs running at the same time share B tiles in L2.
__device__ __forceinline__ void tile_coords(int t, int nm, int nn, int& mb, int& nb) {
    const int per_group = kGroupM * nn;
    const int grp = t / per_group;
    const int first_m = grp * kGroupM;
    const int gm = min(nm - first_m, kGroupM);
    const int r = t % per_group;
    mb = first_m + r % gm;
    nb = r / gm;
}

// Work unit u of a GEMM with a split tail: a whole tile (u < full_tiles) or
// one K piece of a tail tile.  Tile coordinates, k-blocks [kb0, kb1) and, for
// a piece, the slot of its partial sums (-1 for a whole tile).
struct TileUnit {
    int mb, nb, kb0, kb1, slot;
};
__device__ __forceinline__ TileUnit tile_unit(const GemmArgs& p, int u) {
    TileUnit w;
    int t, piece;
    if (u < p.full_tiles) {
        t = u;
        piece = -1;
    } else {
        const int v = u - p.full_tiles;
        t = p.full_tiles + v / p.splits;
        piece = v % p.splits;
    }
    tile_coords(t, p.num_m_blocks, p.num_n_blocks, w.mb, w.nb);
    w.slot = piece < 0 ? -1 : (t - p.full_tiles) * p.splits + piece;
    w.kb0 = piece < 0 ? 0 : piece * p.kb_per_split;
    w.kb1 = piece < 0 ? p.num_k_blocks : min(w.kb0 + p.kb_per_split, p.num_k_blocks);
    return w;
}
__device__ __forceinline__ int num_units(const GemmArgs& p) {
    return p.full_tiles + (p.num_m_blocks * p.num_n_blocks - p.full_tiles) * p.splits;
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Eight outputs of one row packed into a 16-byte vector.
template <typename TY>
__device__ __forceinline__ uint4 pack8_out(const float* v) {
    uint4 o;
    o.x = pack2_out<TY>(v[0], v[1]);
    o.y = pack2_out<TY>(v[2], v[3]);
    o.z = pack2_out<TY>(v[4], v[5]);
    o.w = pack2_out<TY>(v[6], v[7]);
    return o;
}

// Row `r` of a 32 x 32 staging box of 16-bit outputs, laid out for the TMA
// 64-byte swizzle: 16-byte chunk j of row r lands at chunk j ^ ((r >> 1) & 3),
// so the 32 lanes writing 32 rows hit distinct banks.
template <typename TY>
__device__ __forceinline__ void stage_row32_f(uint8_t* box, int r, const float (&v)[32]) {
    uint8_t* row = box + r * 64;
    const int sw = (r >> 1) & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4*>(row + ((j ^ sw) << 4)) = pack8_out<TY>(v + 8 * j);
}

// Row `r` of a 32 x 16 staging box of fp32 values, in the same 64-byte swizzle
// (a row is 64 bytes either way).
__device__ __forceinline__ void stage_row16_f32(uint8_t* box, int r, const float* v) {
    uint8_t* row = box + r * 64;
    const int sw = (r >> 1) & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<float4*>(row + ((j ^ sw) << 4)) = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

// ---------------------------------------------------------------------------
// Host-side tensor maps
// ---------------------------------------------------------------------------
// 2-D uint8 map over a row-major [rows][inner] byte matrix.
inline bool make_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                        uint32_t box_rows, bool swizzle128) {
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return encode_tensor_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                             swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Output map for the epilogues' TMA stores: [M][N] 16-bit values, 32 x 32
// boxes, 64-byte swizzle.
inline bool make_map_out(CUtensorMap* map, void* y, int M, int N, int ydt) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    return encode_tensor_map(map, ydt == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, y,
                             dims, strides, box, estr, CU_TENSOR_MAP_SWIZZLE_64B);
}

// Map of split-K partial sums: `slots` tile-local blocks of rows x cols fp32,
// for TMA stores of 32-row x 16-column boxes.
inline bool make_map_part(CUtensorMap* map, float* part, int rows, int cols, int slots) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(slots)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 4, static_cast<cuuint64_t>(rows) * cols * 4};
    cuuint32_t box[3] = {16, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return encode_tensor_map(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, part, dims, strides, box, estr,
                             CU_TENSOR_MAP_SWIZZLE_64B);
}

}  // namespace cider
