// cider_device.cuh -- device-side building blocks for sm_100a: bounded
// mbarrier waits, TMA tile loads, tcgen05 (UMMA) descriptors, issue and
// tensor-memory access, and the activation quantization step.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "cider_kernels.h"

namespace cider {

// A bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned long long global_timer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Programmatic dependent launch: every kernel of this library is launched so
// that it may start while the previous kernel on the stream finishes.  It
// must call pdl_wait() before its first read of global memory another kernel
// may have written; pdl_trigger() lets the next kernel begin its own launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete.  Gives up (returns
// false, sets the status word) after limit_ns, or as soon as another thread
// has recorded a failure in *abort_flag.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, unsigned* status,
                                              volatile int* abort_flag, unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    unsigned long long t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                atomicOr(status, kStatusTimeout);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* status,
                                          volatile int* abort_flag) {
    return mbar_wait_for(bar, parity, status, abort_flag, kWaitLimitNs);
}

// ---------------------------------------------------------------------------
// Thread-block clusters (pairs of CTAs sharing one tcgen05 MMA)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// All threads of both CTAs of the cluster (convergent code only).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared::cluster address of the variable at the same offset in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
    uint32_t d;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(smem_u32(p)), "r"(rank));
    return d;
}
// Arrive on an mbarrier given by a shared::cluster address (possibly the peer's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Arrive without release semantics.  For a reader that only signals "my
// tcgen05.ld reads of this TMEM buffer are complete" (after tcgen05.wait::ld):
// the reads are finished when the arrive executes, and the arrive publishes
// no memory, so a release fence buys nothing.
__device__ __forceinline__ void mbar_arrive_relaxed(uint64_t* bar) {
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait on a barrier that threads of the peer CTA also arrive on.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, unsigned* status,
                                                  volatile int* abort_flag) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    unsigned long long t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if ((it & 255u) == 0u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicOr(status, kStatusTimeout);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), no multicast
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tile load; c0 is the innermost coordinate (elements), c1 the row.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// 2-D tile load into this CTA's shared memory whose completion is counted on
// an mbarrier given by a shared::cluster address (the pair leader's barrier).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}

// 2-D tile store from this CTA's shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(smem_src)), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* smem_src, int32_t c0, int32_t c1,
                                             int32_t c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
// Untiled bulk copy of `bytes` contiguous bytes from this GPU's global memory
// into this CTA's shared memory (no multicast), counted on `bar` by
// complete_tx.  Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// L2 prefetches.  They write neither shared memory nor registers, only bring
// global lines into the L2, which every SM reads through (the point of
// coherence), so a kernel may issue them before its grid-dependency wait: a
// load after the wait still sees every write of the kernel before it.  Used
// for the streamed operands of the HBM-bound kernels, so the next launch's
// CTAs start pulling their bytes while the previous launch drains.
// Untiled: `gsrc` 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void prefetch_l2_bulk(const void* gsrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gsrc), "r"(bytes) : "memory");
}
// One box of a 2-D tensor map (no multicast; c0 innermost, as in tma_load_2d).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, UMMA descriptors, MMA issue, commit, loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// CTA-pair variants: both CTAs of the pair execute alloc/relinquish/dealloc
// from the same warp with the same destination offset.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row swizzle atoms 1024 bytes apart.
// Fields: start address >> 4 (bits 0-13), leading byte offset >> 4 (16-29,
// unused for swizzled K-major), stride byte offset >> 4 (32-45), descriptor
// version 1 (46-47), base offset 0 (49-51), layout type 2 = 128B swizzle (61-63).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;             // LBO (ignored)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;     // SBO = 1024 B
    d |= static_cast<uint64_t>(1u) << 46;             // version
    d |= static_cast<uint64_t>(2u) << 61;             // SWIZZLE_128B
    return d;
}

// Shared-memory matrix descriptor for an unswizzled K-major tile: core
// matrices of 8 rows x 16 bytes, `lbo` bytes apart along K and `sbo` bytes
// apart along M/N.
__device__ __forceinline__ uint64_t umma_desc_plain(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;             // version
    return d;                                         // layout type 0: no swizzle
}

// Instruction descriptor, kind::f16: D = F32, A = B = f16, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
    return (1u << 4)                                 // D format F32
           | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

// Instruction descriptor, kind::i8: D = S32, A = B = signed 8-bit, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_i8(int M, int N) {
    return (2u << 4)                                 // D format S32
           | (1u << 7)                               // A signed int8
           | (1u << 10)                              // B signed int8
           | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, one 128 x N x 32 int8 step.
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] = A[smem] * B[smem]^T with f16 operands, no accumulate: one
// 128 x N x 16 step.
__device__ __forceinline__ void umma_f16_overwrite(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                   uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(0u)
        : "memory");
}

// D[tmem of both CTAs] (+)= A[smem of both] * B[smem of both]^T: one
// 256 x N x 32 int8 step of a CTA pair, issued by the even CTA only.
__device__ __forceinline__ void umma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the barrier at `bar`'s offset in every CTA of the pair when
// the pair's previously issued tcgen05 ops complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\t"
        "mov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05 ops of this thread complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 lanes x 32 columns of 32-bit tensor memory -> 32 registers per thread
// (thread i of the warp gets lane base+i, columns col..col+31).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Activation quantization step, shared by every kernel that quantizes tokens.
// scale = amax / 127 (fp32, correctly rounded); q = clamp(round(x / scale),
// -128, 127) with round = roundf (halfway cases away from zero) applied to
// the correctly rounded fp32 quotient; amax == 0 gives scale 0 and q = 0.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float act_scale(float amax) { return __fdiv_rn(amax, 127.0f); }

__device__ __forceinline__ int quant_code(float x, float scale) {
    if (scale == 0.0f) return 0;
    float r = roundf(__fdiv_rn(x, scale));
    r = fminf(fmaxf(r, -128.0f), 127.0f);
    return static_cast<int>(r);
}

// Packed fp32 arithmetic: two IEEE operations (round to nearest) per instruction.
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float lo_f32(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi_f32(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Eight codes at once, bit-identical to quant_code but mostly without a
// division.  With r = 1/scale correctly rounded (__frcp_rn) and |x/scale| <= 127
// (+ one ulp), the product t = x * r lies within 2^-15 of the correctly rounded
// quotient fl(x/scale): each of the two roundings adds at most 2^-24 relative
// error on a value below 128.  Whenever t is more than 2^-14 away from the
// nearest halfway point k + 1/2, both t and fl(x/scale) round to the same
// integer, so rint(t) is the code.  rint is taken by adding 1.5 * 2^23: the sum
// has spacing 1, so it rounds t to an integer, and its low byte is that
// integer's two's-complement byte; d = t - (sum - 1.5 * 2^23) is exact and
// measures the distance to that integer.  The eight values go two per packed
// instruction and are checked together: if any of them is within the margin
// of a halfway point (or r is not finite, which makes d NaN), all eight are
// recomputed exactly with quant_code -- one rarely taken branch per eight
// codes.  Returns the eight code bytes.
__device__ __forceinline__ uint2 quant8_codes(const float (&f)[8], float scale, float rcp) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    constexpr float kMargin = 0.5f - 0x1p-14f;
    const uint64_t r2 = pack_f32x2(rcp, rcp);
    const uint64_t m2 = pack_f32x2(kMagic, kMagic), nm2 = pack_f32x2(-kMagic, -kMagic);
    const uint64_t neg1 = pack_f32x2(-1.0f, -1.0f);
    uint32_t b[8];
    bool near_tie = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint64_t t2 = f32x2_mul(pack_f32x2(f[2 * i], f[2 * i + 1]), r2);
        const uint64_t v2 = f32x2_add(t2, m2);
        const uint64_t d2 = f32x2_fma(f32x2_add(v2, nm2), neg1, t2);  // t - (v - 1.5 * 2^23)
        near_tie |= !(fabsf(lo_f32(d2)) < kMargin);
        near_tie |= !(fabsf(hi_f32(d2)) < kMargin);
        b[2 * i] = static_cast<uint32_t>(v2);
        b[2 * i + 1] = static_cast<uint32_t>(v2 >> 32);
    }
    if (near_tie) {
#pragma unroll
        for (int i = 0; i < 8; ++i) b[i] = __float_as_uint(static_cast<float>(quant_code(f[i], scale)) + kMagic);
    }
    uint2 o;
    o.x = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    o.y = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
    return o;
}

// Reciprocal used by quant8_codes; a zero scale gives +inf, which sends every
// element of an all-zero token to the exact path (code 0).
__device__ __forceinline__ float act_rcp(float scale) { return __frcp_rn(scale); }

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) {
    return __half2float(v);
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

// Running max of |v| over 16-bit values, two at a time (exact: max and abs
// do not round).
template <typename T>
struct Pack2;
template <>
struct Pack2<__half> {
    using type = __half2;
};
template <>
struct Pack2<__nv_bfloat16> {
    using type = __nv_bfloat162;
};

template <typename T>
__device__ __forceinline__ typename Pack2<T>::type absmax8(const uint4& v, typename Pack2<T>::type m) {
    using P = typename Pack2<T>::type;
    const P* h = reinterpret_cast<const P*>(&v);
    m = __hmax2(m, __habs2(h[0]));
    m = __hmax2(m, __habs2(h[1]));
    m = __hmax2(m, __habs2(h[2]));
    return __hmax2(m, __habs2(h[3]));
}

template <typename T>
__device__ __forceinline__ float absmax_to_f32(typename Pack2<T>::type m) {
    return fmaxf(to_f32<T>(m.x), to_f32<T>(m.y));
}

// Eight 16-bit values packed in a uint4 -> eight floats (exact widening).
template <typename T>
__device__ __forceinline__ void unpack8_f32(const uint4& v, float (&f)[8]) {
    const T* h = reinterpret_cast<const T*>(&v);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = to_f32<T>(h[i]);
}

// Eight codes -> two 32-bit words of int8 (byte i = code i).
__device__ __forceinline__ uint2 pack8_i8(const int (&c)[8]) {
    uint2 o;
    o.x = (c[0] & 0xFF) | ((c[1] & 0xFF) << 8) | ((c[2] & 0xFF) << 16) | ((uint32_t)(c[3] & 0xFF) << 24);
    o.y = (c[4] & 0xFF) | ((c[5] & 0xFF) << 8) | ((c[6] & 0xFF) << 16) | ((uint32_t)(c[7] & 0xFF) << 24);
    return o;
}

// Output conversion, round to nearest even.
template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) {
    return __float2half_rn(v);
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Two output values packed into one 32-bit word (element 0 in the low half).
template <typename T>
__device__ __forceinline__ uint32_t pack2_out(float a, float b) {
    T lo = from_f32<T>(a), hi = from_f32<T>(b);
    return static_cast<uint32_t>(*reinterpret_cast<uint16_t*>(&lo)) |
           (static_cast<uint32_t>(*reinterpret_cast<uint16_t*>(&hi)) << 16);
}

// ---------------------------------------------------------------------------
// INT4 -> INT8 unpack (W4A8 load path).  Four packed bytes hold eight nibbles
// n0..n7 in k order (byte j: k=2j low, k=2j+1 high).  Output: eight int8
// values nibble - 8 in k order, as two 32-bit words.  Per byte, u - 8 for a
// 4-bit u is ((u + 0x78) ^ 0x80) with no carry out of the byte.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint2 unpack_int4x8(uint32_t p) {
    uint32_t lo = p & 0x0F0F0F0Fu;         // even k, bytes 0..3
    uint32_t hi = (p >> 4) & 0x0F0F0F0Fu;  // odd k, bytes 0..3
    uint2 o;
    o.x = __byte_perm(lo, hi, 0x5140);  // lo0 hi0 lo1 hi1
    o.y = __byte_perm(lo, hi, 0x7362);  // lo2 hi2 lo3 hi3
    o.x = (o.x + 0x78787878u) ^ 0x80808080u;
    o.y = (o.y + 0x78787878u) ^ 0x80808080u;
    return o;
}

}  // namespace cider
