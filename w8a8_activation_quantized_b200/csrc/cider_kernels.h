// cider_kernels.h -- host-side launchers shared between the library's
// translation units (not part of the public C ABI; see include/cider.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/cider.h"

namespace cider {

// Device status word bits (read back by cider_device_status()).
constexpr unsigned kStatusTimeout = 1u;

enum : int {
    kModePC = 0,    // per-channel dequant epilogue
    kModePG = 1,    // per-group dequant epilogue
    kModeW4 = 2,    // per-group epilogue, INT4 packed weights unpacked on chip
    kModeI32 = 3,   // test: store the INT32 accumulator
    kModeI32G = 4,  // test: store every per-group INT32 partial
    kModeW4PC = 5,  // per-channel epilogue, INT4 packed weights unpacked on chip
};

// Kernel variants of the per-channel GEMM (the grouped modes always use the
// single-CTA kernel with 128-wide N tiles).
enum : int { kGemmAuto = 0, kGemmSingle128 = 1, kGemmSingle256 = 2, kGemmPair = 3, kGemmSingle80 = 4, kGemmPair192 = 5 };

// Grid-barrier slots of the launches that quantize inside the GEMM: the host
// hands out slots in turn, so launches that run at the same time (up to this
// many in flight) never share one.
constexpr int kFuseSlots = 256;

struct GemmLaunch {
    int mode;
    const int8_t* q;   // [M][K]
    const void* w;     // [N][K] int8, or [N][K/2] packed int4
    const float* sx;   // [M]
    const float* sw;   // [N] or [K/gs][N]
    void* y;           // output
    int M, N, K, gs;
    int ydt;           // 0 fp16, 1 bf16
    int variant;       // per-channel modes: one of the kGemm* kernel variants above
    int full_tiles;    // grouped modes: tiles that run over all of K (the rest are split)
    int splits;        // grouped modes: K pieces of each later tile (1 = no split)
    float* part;       // grouped modes with splits > 1: fp32 partial sums, [piece slot][128][128]
    int num_sms;
    unsigned* status;  // device status word
    // per-channel kernels: quantize x into q / sx inside the GEMM launch
    // (x == nullptr: q / sx are inputs written by an earlier kernel)
    const void* x = nullptr;
    int xdt = 0;
    int fuse_slot = 0;
};

// Launches `kern` with programmatic stream serialisation allowed, so that its
// setup overlaps the tail of the previous kernel on the stream (each kernel
// waits with griddepcontrol.wait before reading global memory).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Records a message for cider_last_error() on this thread and returns `s`.
cider_status_t set_error(cider_status_t s, const char* fmt, ...);

// Encodes a TMA descriptor through the driver entry point (no libcuda link).
bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, cuuint32_t rank, void* base,
                       const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                       const cuuint32_t* elem_strides, CUtensorMapSwizzle swizzle);

cudaError_t launch_quantize_act(const void* x, int xdt, int64_t M, int K, int64_t ldx, int8_t* q, int64_t ldq,
                                float* sx, int num_sms, cudaStream_t st);
cudaError_t launch_silu_mul_quantize(const void* g, const void* u, int dt, int64_t M, int F,
                                     int8_t* q, float* sx, void* a_out, cudaStream_t st);
// mode 0: per channel (out = int8 [N][K]); 1: per group int8; 2: per group int4 packed;
// 3: per channel int4 packed
cudaError_t launch_quantize_weight(int mode, const float* W, int64_t N, int K, int gs, void* out,
                                   float* sw, cudaStream_t st);
// percentile-clipped weights: gs = 0 per channel, else per group of gs (64 or 128);
// k0, t: the percentile's position within a slab (order statistic k0, fraction t)
cudaError_t launch_quantize_weight_clip(const float* W, int64_t N, int K, int gs, int k0, float t, int8_t* out,
                                        float* sw, cudaStream_t st);
cudaError_t launch_wait_selftest(unsigned* status, unsigned long long limit_ns, cudaStream_t st);
cudaError_t launch_unpack_int4(const uint8_t* packed, int64_t N, int K, int8_t* w, cudaStream_t st);
cudaError_t launch_small_m(int mode, const void* x, int xdt, int M, int K, const void* w,
                           const float* sw, int N, int gs, void* y, int ydt, int num_sms,
                           unsigned* status, cudaStream_t st);
cudaError_t launch_mv_w8a16(const void* x, int xdt, int M, int K, const int8_t* w, const float* sw, int N, int gs,
                            void* y, int ydt, int num_sms, unsigned* status, cudaStream_t st);
// Test override of the decode-shaped kernel (0 automatic, 1 register ring,
// 2 bulk-staged, 3 bulk-staged within half of shared memory).
cudaError_t set_small_m_kernel(int k);

cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t st);
cudaError_t launch_gemm_grouped(const GemmLaunch& L, cudaStream_t st);

}  // namespace cider
