// grouped_common.cuh -- pieces of the per-group GEMM kernel: the bias-removing
// rescale of INT32 partials, the cp.async scale ring and the INT32 test store.
#pragma once

#include "gemm_common.cuh"

namespace cider {

constexpr uint32_t kPartialBias = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr int kScaleSlots = 4;                   // per-warp scale ring depth

__device__ __forceinline__ uint64_t pack_u32x2(uint32_t lo, uint32_t hi) {
    return (static_cast<uint64_t>(hi) << 32) | lo;
}
// 16 bytes global -> shared, zero-filled when `bytes` is 0.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Scales of 4 consecutive columns as two packed pairs; the load is ordered
// (volatile) so the compiler keeps scale registers short-lived.
__device__ __forceinline__ void lds_scale4(const uint8_t* p, uint64_t& a, uint64_t& b) {
    asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(smem_u32(p)) : "memory");
}

// sum += (partial - preset) * scale for 16 columns, two per instruction; the
// next 16 bytes of scales are loaded while the current ones are used.
__device__ __forceinline__ void rescale16(uint64_t* sum2, const uint32_t (&r)[16], const uint8_t* scales,
                                          uint64_t neg_bias2) {
    uint64_t a0, a1, b0, b1;
    lds_scale4(scales, a0, a1);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j + 1 < 4) lds_scale4(scales + 16 * (j + 1), b0, b1);
        sum2[2 * j] = f32x2_fma(f32x2_add(pack_u32x2(r[4 * j], r[4 * j + 1]), neg_bias2), a0, sum2[2 * j]);
        sum2[2 * j + 1] = f32x2_fma(f32x2_add(pack_u32x2(r[4 * j + 2], r[4 * j + 3]), neg_bias2), a1, sum2[2 * j + 1]);
        a0 = b0;
        a1 = b1;
    }
}

// Test mode: 16 per-group INT32 partials of one row (preset removed).
__device__ __forceinline__ void store_partial16(const GemmArgs& p, const uint32_t (&r)[16], int g, int m, bool mvalid,
                                                int n0) {
    if (!mvalid) return;
    int32_t* out = static_cast<int32_t*>(p.y) + (static_cast<int64_t>(g) * p.M + m) * p.N;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if (n0 + 4 * j < p.N)
            *reinterpret_cast<int4*>(out + n0 + 4 * j) =
                make_int4(static_cast<int>(r[4 * j] - kPartialBias), static_cast<int>(r[4 * j + 1] - kPartialBias),
                          static_cast<int>(r[4 * j + 2] - kPartialBias), static_cast<int>(r[4 * j + 3] - kPartialBias));
}

}  // namespace cider
