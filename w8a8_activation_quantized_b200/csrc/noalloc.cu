// noalloc.cu -- cider_w8a8_linear_pc_noalloc: the per-channel W8A8 linear for
// callers that cannot allocate device memory and so cannot hand the library a
// workspace.  Typical cases: a host application or framework that owns all of
// the GPU's memory through its own pool and forbids any other cudaMalloc, or
// code that must run within a memory budget fixed at start-up.  Instead of a
// caller workspace, the quantized activations and their scales live in one
// file-scope device array of fixed size, which every GPU that loads this
// library holds until the process exits.
#include <cstdarg>
#include <mutex>

#include "../../include/cider.h"
#include "cider_kernels.h"

namespace cider {
namespace {

// Room for q [M][K] int8 plus scale_x [M] fp32, each 256-byte aligned, and,
// when they fit after those, the fp32 partial sums of tiles cut along K.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB

// Shared by every call on a device: it keeps whatever the last call wrote.
// Nothing in it needs to start at zero: each call writes the M rows of codes
// and the M scales it reads, and the GEMM never reads rows beyond M (its tile
// loads fill those with zeros); every K piece of a split tile stores its whole
// partial-sum slot before the reduce kernel reads it.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// The array's name is only a host-side stand-in for it; the kernels need its
// device address, which is looked up once per device, with that device current.
cider_status_t scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_error(CIDER_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return set_error(CIDER_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return set_error(CIDER_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return CIDER_OK;
}

}  // namespace
}  // namespace cider

extern "C" cider_status_t cider_w8a8_linear_pc_noalloc(const void* x, cider_dtype_t xdt, int64_t M, int64_t K,
                                                       const int8_t* w, const float* scale_w, int64_t N, void* y,
                                                       cider_dtype_t ydt, void* stream) {
    using namespace cider;
    const size_t need = cider_workspace_bytes(M, K);
    if (need == 0)  // M <= 0, or the fused small-M kernel, which keeps its codes in shared memory
        return cider_w8a8_linear_pc(x, xdt, M, K, w, scale_w, N, y, ydt, nullptr, 0, stream);
    if (need > kNoAllocScratchBytes)
        return set_error(CIDER_ERR_INVALID_ARG,
                         "M = %lld, K = %lld need %zu bytes of scratch; the built-in scratch holds %zu bytes "
                         "(M * K + 4 * M must stay within about 32 MiB); use cider_w8a8_linear_pc with a workspace",
                         (long long)M, (long long)K, need, kNoAllocScratchBytes);
    if (!cider_is_available())
        return set_error(CIDER_ERR_UNSUPPORTED, "the current device is not compute capability 10.x");
    void* scratch = nullptr;
    cider_status_t s = scratch_address(&scratch);
    if (s != CIDER_OK) return s;
    return cider_w8a8_linear_pc(x, xdt, M, K, w, scale_w, N, y, ydt, scratch, kNoAllocScratchBytes, stream);
}
