// cider_api.cu -- the extern "C" entry points declared in include/cider.h:
// argument checks, device checks, path selection and launches.  No entry
// point allocates, frees or synchronises (cider_device_status excepted).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/cider.h"
#include "cider_kernels.h"
#include "sdpa_decode.h"

namespace cider {

// Device status word: bit 0 = a bounded wait ran out (kStatusTimeout).
__device__ unsigned g_status_word;

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxK = 131072;            // 127 * 128 * K < 2^31 keeps INT32 exact
constexpr int64_t kMaxSmallM = 16;
constexpr int64_t kSmallSmemLimit = 160 * 1024;  // q rows of the small-M kernel in shared memory
constexpr int64_t kSmallMaxK = 32768;
constexpr int kMaxMvM = 4;                        // rows of the W8A16 decode kernel
constexpr int kMaxSmallXBytes = 160 * 1024;       // its fp32 activation rows in shared memory

struct DeviceInfo {
    int ready = 0;     // 1 = filled in
    int cc_major = 0;
    int num_sms = 0;
    unsigned* status = nullptr;  // device address of g_status_word on this device
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;
std::atomic<int64_t> g_small_m_threshold{4};
thread_local char t_last_error[512] = "";

cider_status_t fail(cider_status_t s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_error, sizeof t_last_error, fmt, ap);
    va_end(ap);
    return s;
}

cider_status_t cuda_fail(cudaError_t e, const char* what) {
    return fail(CIDER_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Fills in (once per device, with that device current) the compute
// capability, SM count and the device address of the status word.
cider_status_t device_info(DeviceInfo** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(CIDER_ERR_UNSUPPORTED, "device index %d out of range", dev);
    DeviceInfo& d = g_dev[dev];
    if (!__atomic_load_n(&d.ready, __ATOMIC_ACQUIRE)) {
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        if (!d.ready) {
            int major = 0, sms = 0;
            if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
                return cuda_fail(e, "cudaDeviceGetAttribute");
            if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
                return cuda_fail(e, "cudaDeviceGetAttribute");
            void* addr = nullptr;
            if (major == 10) {
                if ((e = cudaGetSymbolAddress(&addr, g_status_word)) != cudaSuccess)
                    return cuda_fail(e, "cudaGetSymbolAddress(status word)");
            }
            d.cc_major = major;
            d.num_sms = sms;
            d.status = static_cast<unsigned*>(addr);
            __atomic_store_n(&d.ready, 1, __ATOMIC_RELEASE);
        }
    }
    if (d.cc_major != 10)
        return fail(CIDER_ERR_UNSUPPORTED, "device %d is compute capability %d.x; this library needs 10.x (sm_100a)",
                    dev, d.cc_major);
    *out = &d;
    return CIDER_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
    uintptr_t lo, hi;
};
Range rng(const void* p, size_t bytes) {
    uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return {a, a + bytes};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// The fused small-M kernel keeps the M code rows in shared memory and at most
// 8 passes of 512 weights per warp in registers (K <= 32768).
// q [M][K] int8 and scale_x [M] fp32 of the quantize + tensor-core path
size_t tensor_path_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0) return 0;
    return align256(static_cast<size_t>(M) * K) + align256(static_cast<size_t>(M) * 4);
}

bool small_m_path(int64_t M, int64_t K) {
    return M >= 1 && M <= g_small_m_threshold.load() && M * K <= kSmallSmemLimit && K <= kSmallMaxK;
}

// Common checks of the linear / GEMM entry points.
cider_status_t check_common(const void* x, int64_t M, int64_t K, const void* w, const float* sw,
                            int64_t N, const void* y, int dt_in, int dt_out) {
    if (M < 0) return fail(CIDER_ERR_INVALID_ARG, "M = %lld must be >= 0", (long long)M);
    if (N < 1 || K < 1) return fail(CIDER_ERR_INVALID_ARG, "N = %lld and K = %lld must be >= 1", (long long)N, (long long)K);
    if (K % 16) return fail(CIDER_ERR_INVALID_ARG, "K = %lld must be a multiple of 16", (long long)K);
    if (N % 8) return fail(CIDER_ERR_INVALID_ARG, "N = %lld must be a multiple of 8", (long long)N);
    if (K > kMaxK) return fail(CIDER_ERR_INVALID_ARG, "K = %lld exceeds %lld", (long long)K, (long long)kMaxK);
    if (M > INT32_MAX || N > INT32_MAX) return fail(CIDER_ERR_INVALID_ARG, "M and N must be < 2^31");
    if (dt_in != CIDER_F16 && dt_in != CIDER_BF16) return fail(CIDER_ERR_INVALID_ARG, "input dtype %d unknown", dt_in);
    if (dt_out != CIDER_F16 && dt_out != CIDER_BF16) return fail(CIDER_ERR_INVALID_ARG, "output dtype %d unknown", dt_out);
    if (M == 0) return CIDER_OK;
    if (!x || !w || !sw || !y) return fail(CIDER_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(x) || !aligned16(w) || !aligned16(sw) || !aligned16(y))
        return fail(CIDER_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    return CIDER_OK;
}

cider_status_t check_gs(int64_t K, int64_t gs, bool w4) {
    if (gs != 64 && gs != 128) return fail(CIDER_ERR_INVALID_ARG, "gs = %lld must be 64 or 128", (long long)gs);
    if (K % gs) return fail(CIDER_ERR_INVALID_ARG, "gs = %lld must divide K = %lld", (long long)gs, (long long)K);
    if (w4 && K % 32) return fail(CIDER_ERR_INVALID_ARG, "W4A8 needs K %% 32 == 0 (K = %lld)", (long long)K);
    return CIDER_OK;
}

// gs and K rules of a linear mode: per group needs gs in {64, 128} dividing K;
// packed INT4 weights need K % 32 == 0 (16-byte rows of K/2 bytes).
cider_status_t check_mode_k(int mode, int64_t K, int64_t gs) {
    if (mode == kModePG || mode == kModeW4) return check_gs(K, gs, mode == kModeW4);
    if (mode == kModeW4PC && K % 32) return fail(CIDER_ERR_INVALID_ARG, "W4A8 needs K %% 32 == 0 (K = %lld)", (long long)K);
    return CIDER_OK;
}

std::atomic<int> g_gemm_variant{kGemmAuto};  // test override
std::atomic<int> g_split_override{0};         // test override of the split-K piece count (0 = automatic)
std::atomic<int> g_fuse_override{0};          // test override of the fused quantize: 0 auto, 1 never, 2 always
std::atomic<unsigned> g_fuse_next{0};         // next grid-barrier slot of a fused launch

// Whether the per-channel linear quantizes its activations inside the GEMM
// launch.  Automatic: never -- measured on B200 the fused launch was slower
// at every M tried (N = 10240, K = 2560: M = 128 19.3 us against 15.4 us for
// quantize kernel + GEMM, M = 1024 35.0 against 31.2, M = 4096 90.7 against
// 82.6): the grid barrier and the quantizing warps cost more than the
// separate launch they replace.  The fused path stays selectable.
bool use_fused_quantize(int mode, int64_t M) {
    (void)M;
    if (mode != kModePC) return false;
    return g_fuse_override.load() == 2;
}
constexpr int kMaxSplits = 16;

int pick_variant(int64_t M, int64_t N, int64_t K, int num_sms);

// Split-K plan of a persistent GEMM with `slots` resident tiles (SMs, or SM
// pairs): the tiles that fill whole rounds run over all of K; the R tiles of
// the last, partial round are cut into S K pieces so that their R * S units
// fill that round (S <= slots / R, >= 4 k-blocks per piece, <= 16), provided
// the cut saves at least min_saved k-blocks on the critical path (the partial
// sums and the reduce kernel cost a few microseconds).  A forced piece count
// (test override) splits every tile.  Partial sums take one tile-sized slot
// of 32-bit values per piece.
struct SplitPlan {
    int full_tiles, splits;
    int64_t tail_tiles, tile_elems;
};
SplitPlan split_plan(int64_t tiles, int64_t tile_elems, int slots, int64_t K, int64_t min_saved) {
    const int forced = g_split_override.load();
    if (forced > 1) return {0, forced, tiles, tile_elems};
    if (forced == 1 || slots <= 0) return {static_cast<int>(tiles), 1, 0, tile_elems};
    const int64_t full = tiles / slots * slots, tail = tiles - full;
    if (tail == 0) return {static_cast<int>(tiles), 1, 0, tile_elems};
    const int64_t nkb = (K + 127) / 128;
    int64_t s = std::min<int64_t>(slots / tail, nkb / 4);
    s = std::min<int64_t>(s, kMaxSplits);
    if (s < 2 || nkb - (nkb + s - 1) / s < min_saved) return {static_cast<int>(tiles), 1, 0, tile_elems};
    return {static_cast<int>(full), static_cast<int>(s), tail, tile_elems};
}
// Per-group GEMM: 128 x 128 tiles, one CTA per SM; a k-block costs ~0.5-1 us
// of epilogue time, so any cut of >= 4 k-blocks pays.
SplitPlan grouped_split_plan(int64_t M, int64_t N, int64_t K, int num_sms) {
    return split_plan(((M + 127) / 128) * ((N + 127) / 128), 128 * 128, num_sms, K, 4);
}
// Per-channel GEMM: only on the CTA-pair 256 x 256 tile, whose k-block takes
// ~0.27 us; measured at K = 2560 (M = 1024 and 8192) the split does not pay,
// so it needs >= 32 saved k-blocks (K of roughly 5120 and more).
SplitPlan pair_split_plan(int64_t M, int64_t N, int64_t K, int num_sms) {
    return split_plan(((M + 255) / 256) * ((N + 255) / 256), 256 * 256, num_sms / 2, K, 32);
}
SplitPlan pc_split_plan(int64_t M, int64_t N, int64_t K, int num_sms) {
    if (pick_variant(M, N, K, num_sms) != kGemmPair) return {0, 1, 0, 0};
    return pair_split_plan(M, N, K, num_sms);
}

// Bytes of 32-bit partial sums: one tile-sized slot per K piece of a tail tile.
size_t part_bytes(const SplitPlan& sp) {
    return sp.splits > 1 ? align256(static_cast<size_t>(sp.tail_tiles) * sp.splits * sp.tile_elems * 4) : 0;
}

// Per-channel GEMM variant: the CTA-pair 256x256 tile when it still gives
// every pair of SMs a tile, else single-CTA tiles of 128x256, or -- when those
// leave SMs idle -- 128x128 or 128x80, whichever gives the busiest SM fewer
// weight rows to stream (rounds of the persistent grid x tile width; at
// M <= 128, N = 10240 that is one round of 128 tiles of 80 rows instead of
// 80 tiles of 128 rows on 80 SMs).  Among the pair tiles, 256x192 replaces
// 256x256 when the square tile's tail is not split along K and the busiest
// pair streams fewer operand bytes: rounds x (128 rows of A + BN / 2 rows of B)
// per k-block and CTA.  Measured on B200 (N = 10240, K = 2560) the time per
// round follows those bytes: M = 512 and 1024 (2 and 3 rounds either way)
// gain 3.7% and 2.0% with 192 columns, M = 2048 (5 rounds of 256 against 6 of
// 192) loses 10% and M = 4096 (9 against 12) 16% -- which this rule avoids.
int pick_variant(int64_t M, int64_t N, int64_t K, int num_sms) {
    const int forced = g_gemm_variant.load();
    if (forced != kGemmAuto) return forced;
    const int64_t pair_tiles = ((M + 255) / 256) * ((N + 255) / 256);
    if (M > 128 && pair_tiles >= num_sms / 2) {
        const int64_t pairs = num_sms / 2, mbp = (M + 255) / 256;
        auto bytes_per_pair = [&](int64_t bn) { return (mbp * ((N + bn - 1) / bn) + pairs - 1) / pairs * (128 + bn / 2); };
        if (pair_split_plan(M, N, K, num_sms).splits == 1 && bytes_per_pair(192) < bytes_per_pair(256)) return kGemmPair192;
        return kGemmPair;
    }
    const int64_t mb = (M + 127) / 128;
    const int64_t tiles256 = mb * ((N + 255) / 256);
    if (tiles256 >= num_sms) return kGemmSingle256;
    auto rows_per_sm = [&](int64_t bn) { return (mb * ((N + bn - 1) / bn) + num_sms - 1) / num_sms * bn; };
    return rows_per_sm(80) < rows_per_sm(128) ? kGemmSingle80 : kGemmSingle128;
}

cider_status_t run_gemm(int mode, const int8_t* q, const float* sx, int64_t M, int64_t K,
                        const void* w, const float* sw, int64_t N, int64_t gs, void* y, int ydt,
                        const DeviceInfo* d, cudaStream_t st, SplitPlan sp = {0, 1, 0, 0}, float* part = nullptr,
                        const void* x = nullptr, int xdt = 0) {
    GemmLaunch L;
    L.x = x;
    L.xdt = xdt;
    L.fuse_slot = x ? static_cast<int>(g_fuse_next.fetch_add(1u) % kFuseSlots) : 0;
    L.mode = mode;
    L.q = q;
    L.w = w;
    L.sx = sx;
    L.sw = sw;
    L.y = y;
    L.M = static_cast<int>(M);
    L.N = static_cast<int>(N);
    L.K = static_cast<int>(K);
    L.gs = static_cast<int>(gs);
    L.ydt = ydt;
    L.variant = (mode == kModePC || mode == kModeI32) ? pick_variant(M, N, K, d->num_sms) : kGemmSingle128;
    L.full_tiles = sp.full_tiles;
    L.splits = sp.splits;
    L.part = part;
    L.num_sms = d->num_sms;
    L.status = d->status;
    cudaError_t e = launch_gemm(L, st);
    if (e != cudaSuccess) return cuda_fail(e, "tcgen05 GEMM launch");
    return CIDER_OK;
}

// The three linears share this body: quantize + tensor-core GEMM, or the
// fused small-M kernel.
cider_status_t linear(int mode, const void* x, int xdt, int64_t M, int64_t K, const void* w,
                      const float* sw, int64_t N, int64_t gs, void* y, int ydt, void* ws,
                      size_t ws_bytes, void* stream) {
    t_last_error[0] = '\0';
    cider_status_t s = check_common(x, M, K, w, sw, N, y, xdt, ydt);
    if (s != CIDER_OK) return s;
    if ((s = check_mode_k(mode, K, gs)) != CIDER_OK) return s;
    if (M == 0) return CIDER_OK;
    const size_t ysz = static_cast<size_t>(M) * N * 2;
    const bool packed = mode == kModeW4 || mode == kModeW4PC;
    const size_t wbytes = packed ? static_cast<size_t>(N) * K / 2 : static_cast<size_t>(N) * K;
    const size_t swbytes = (mode == kModePC || mode == kModeW4PC) ? N * 4 : static_cast<size_t>(K / gs) * N * 4;
    const Range ry = rng(y, ysz);
    if (overlap(ry, rng(x, static_cast<size_t>(M) * K * 2)) || overlap(ry, rng(w, wbytes)) ||
        overlap(ry, rng(sw, swbytes)))
        return fail(CIDER_ERR_INVALID_ARG, "y overlaps an input");
    DeviceInfo* d = nullptr;
    if ((s = device_info(&d)) != CIDER_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (mode != kModeW4PC && small_m_path(M, K)) {  // per-channel INT4: tensor-core path at every M
        cudaError_t e = launch_small_m(mode, x, xdt, static_cast<int>(M), static_cast<int>(K), w, sw,
                                       static_cast<int>(N), static_cast<int>(gs), y, ydt, d->num_sms, d->status, st);
        if (e != cudaSuccess) return cuda_fail(e, "small-M kernel launch");
        return CIDER_OK;
    }
    const size_t need = mode == kModeW4PC ? tensor_path_bytes(M, K) : cider_workspace_bytes(M, K);
    if (!ws || ws_bytes < need)
        return fail(CIDER_ERR_INVALID_ARG, "workspace of %zu bytes needed (got %zu)", need, ws ? ws_bytes : 0);
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(CIDER_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    // split-K partial sums of the per-group GEMM, when the workspace holds them
    SplitPlan plan{0, 1, 0, 0};
    float* part = nullptr;
    size_t used = need;
    {
        const SplitPlan sp = mode == kModePC ? pc_split_plan(M, N, K, d->num_sms)
                                             : grouped_split_plan(M, N, K, d->num_sms);
        const size_t pb = part_bytes(sp);
        if (sp.splits > 1 && ws_bytes >= need + pb) {
            plan = sp;
            part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + need);
            used = need + pb;
        }
    }
    if (overlap(ry, rng(ws, used))) return fail(CIDER_ERR_INVALID_ARG, "y overlaps the workspace");
    int8_t* q = static_cast<int8_t*>(ws);
    float* sx = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + align256(static_cast<size_t>(M) * K));
    if (use_fused_quantize(mode, M))  // one launch: the GEMM quantizes x into q / sx itself
        return run_gemm(mode, q, sx, M, K, w, sw, N, gs, y, ydt, d, st, plan, part, x, xdt);
    cudaError_t e = launch_quantize_act(x, xdt, M, static_cast<int>(K), K, q, K, sx, d->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
    return run_gemm(mode, q, sx, M, K, w, sw, N, gs, y, ydt, d, st, plan, part);
}

cider_status_t gemm_q(int mode, const int8_t* q, const float* sx, int64_t M, int64_t K, const void* w,
                      const float* sw, int64_t N, int64_t gs, void* y, int ydt, void* stream) {
    t_last_error[0] = '\0';
    cider_status_t s = check_common(q, M, K, w, sw, N, y, CIDER_F16, ydt);
    if (s != CIDER_OK) return s;
    if ((s = check_mode_k(mode, K, gs)) != CIDER_OK) return s;
    if (M == 0) return CIDER_OK;
    if (!sx || (reinterpret_cast<uintptr_t>(sx) & 3u)) return fail(CIDER_ERR_INVALID_ARG, "scale_x must be non-NULL and 4-byte aligned");
    const Range ry = rng(y, static_cast<size_t>(M) * N * 2);
    if (overlap(ry, rng(q, static_cast<size_t>(M) * K)) || overlap(ry, rng(sx, M * 4)))
        return fail(CIDER_ERR_INVALID_ARG, "y overlaps an input");
    DeviceInfo* d = nullptr;
    if ((s = device_info(&d)) != CIDER_OK) return s;
    return run_gemm(mode, q, sx, M, K, w, sw, N, gs, y, ydt, d, static_cast<cudaStream_t>(stream));
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

}  // namespace

cider_status_t set_error(cider_status_t s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_error, sizeof t_last_error, fmt, ap);
    va_end(ap);
    return s;
}

bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, cuuint32_t rank, void* base,
                       const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                       const cuuint32_t* elem_strides, CUtensorMapSwizzle swizzle) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return false;
    return g_encode(map, dtype, rank, base, dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace cider

using namespace cider;

extern "C" {

int cider_is_available(void) {
    int dev = -1, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return major == 10 ? 1 : 0;
}

const char* cider_status_string(cider_status_t s) {
    switch (s) {
        case CIDER_OK: return "ok";
        case CIDER_ERR_INVALID_ARG: return "invalid argument";
        case CIDER_ERR_UNSUPPORTED: return "unsupported device (needs compute capability 10.x)";
        case CIDER_ERR_CUDA: return "CUDA error";
        case CIDER_ERR_TIMEOUT: return "a bounded device wait ran out";
    }
    return "unknown status";
}

const char* cider_last_error(void) { return t_last_error; }

cider_status_t cider_device_status(void* stream) {
    t_last_error[0] = '\0';
    DeviceInfo* d = nullptr;
    cider_status_t s = device_info(&d);
    if (s != CIDER_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned v = 0;
    if ((e = cudaMemcpy(&v, d->status, sizeof v, cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "reading the status word");
    if (v != 0) {
        unsigned zero = 0;
        if ((e = cudaMemcpy(d->status, &zero, sizeof zero, cudaMemcpyHostToDevice)) != cudaSuccess)
            return cuda_fail(e, "clearing the status word");
        if (v & kStatusTimeout) return fail(CIDER_ERR_TIMEOUT, "a bounded device-side wait ran out");
    }
    return CIDER_OK;
}

size_t cider_workspace_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0 || small_m_path(M, K)) return 0;
    return tensor_path_bytes(M, K);
}

size_t cider_workspace_bytes_w4a8_pc(int64_t M, int64_t N, int64_t K) {
    const size_t need = tensor_path_bytes(M, K);
    if (need == 0 || N <= 0) return need;
    DeviceInfo* d = nullptr;
    if (device_info(&d) != CIDER_OK) return need;
    return need + part_bytes(grouped_split_plan(M, N, K, d->num_sms));
}

size_t cider_workspace_bytes_mnk(int64_t M, int64_t N, int64_t K) {
    const size_t need = cider_workspace_bytes(M, K);
    if (need == 0 || N <= 0) return need;
    DeviceInfo* d = nullptr;
    if (device_info(&d) != CIDER_OK) return need;
    return need + std::max(part_bytes(grouped_split_plan(M, N, K, d->num_sms)),
                           part_bytes(pc_split_plan(M, N, K, d->num_sms)));
}

cider_status_t cider_test_set_split_k(int splits) {
    if (splits < 0 || splits > kMaxSplits)
        return fail(CIDER_ERR_INVALID_ARG, "splits %d outside [0, %d]", splits, kMaxSplits);
    g_split_override.store(splits);
    return CIDER_OK;
}

cider_status_t cider_set_small_m_threshold(int64_t threshold) {
    if (threshold < 0 || threshold > kMaxSmallM)
        return fail(CIDER_ERR_INVALID_ARG, "threshold %lld outside [0, %lld]", (long long)threshold, (long long)kMaxSmallM);
    g_small_m_threshold.store(threshold);
    return CIDER_OK;
}

int64_t cider_get_small_m_threshold(void) { return g_small_m_threshold.load(); }

cider_status_t cider_quantize_act(const void* x, cider_dtype_t xdt, int64_t M, int64_t K, int64_t ldx, int8_t* q,
                                  int64_t ldq, float* scale_x, void* stream) {
    t_last_error[0] = '\0';
    if (M < 0 || K < 1) return fail(CIDER_ERR_INVALID_ARG, "M >= 0 and K >= 1 required");
    if (K % 16) return fail(CIDER_ERR_INVALID_ARG, "K = %lld must be a multiple of 16", (long long)K);
    if (K > kMaxK) return fail(CIDER_ERR_INVALID_ARG, "K exceeds %lld", (long long)kMaxK);
    if (ldx < K || ldq < K)
        return fail(CIDER_ERR_INVALID_ARG, "row strides ldx = %lld and ldq = %lld must be >= K = %lld", (long long)ldx,
                    (long long)ldq, (long long)K);
    if (ldx % 8 || ldq % 16)
        return fail(CIDER_ERR_INVALID_ARG, "ldx must be a multiple of 8 elements and ldq of 16 bytes (16-byte rows)");
    if (xdt != CIDER_F16 && xdt != CIDER_BF16) return fail(CIDER_ERR_INVALID_ARG, "dtype %d unknown", (int)xdt);
    if (M == 0) return CIDER_OK;
    if (M > INT32_MAX) return fail(CIDER_ERR_INVALID_ARG, "M must be < 2^31");
    if (!x || !q || !scale_x) return fail(CIDER_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scale_x) & 3u))
        return fail(CIDER_ERR_INVALID_ARG, "x and q must be 16-byte aligned, scale_x 4-byte aligned");
    const Range rx = rng(x, static_cast<size_t>((M - 1) * ldx + K) * 2);
    const Range rq = rng(q, static_cast<size_t>((M - 1) * ldq + K));
    if (overlap(rx, rq) || overlap(rx, rng(scale_x, M * 4)) || overlap(rq, rng(scale_x, M * 4)))
        return fail(CIDER_ERR_INVALID_ARG, "x, q and scale_x must not overlap");
    DeviceInfo* d = nullptr;
    cider_status_t s = device_info(&d);
    if (s != CIDER_OK) return s;
    cudaError_t e = launch_quantize_act(x, xdt, M, static_cast<int>(K), ldx, q, ldq, scale_x, d->num_sms,
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CIDER_OK : cuda_fail(e, "quantize launch");
}

cider_status_t cider_w8a8_linear_pc(const void* x, cider_dtype_t xdt, int64_t M, int64_t K, const int8_t* w,
                                    const float* scale_w, int64_t N, void* y, cider_dtype_t ydt,
                                    void* workspace, size_t workspace_bytes, void* stream) {
    return linear(kModePC, x, xdt, M, K, w, scale_w, N, 0, y, ydt, workspace, workspace_bytes, stream);
}

cider_status_t cider_w8a16_mv_pc(const void* x, cider_dtype_t xdt, int64_t M, int64_t K, const int8_t* w,
                                 const float* scale_w, int64_t N, void* y, cider_dtype_t ydt, void* stream) {
    t_last_error[0] = '\0';
    cider_status_t s = check_common(x, M, K, w, scale_w, N, y, xdt, ydt);
    if (s != CIDER_OK) return s;
    if (M == 0) return CIDER_OK;
    if (M > kMaxMvM) return fail(CIDER_ERR_INVALID_ARG, "M = %lld exceeds %d (decode shapes only)", (long long)M, kMaxMvM);
    const int64_t xbytes = M * ((K / 16 + 31) / 32) * 2048;  // fp32 activations, whole 512-wide passes
    if (xbytes > kMaxSmallXBytes)
        return fail(CIDER_ERR_INVALID_ARG, "%lld bytes of staged activations exceed %d", (long long)xbytes,
                    kMaxSmallXBytes);
    if (K > kSmallMaxK) return fail(CIDER_ERR_INVALID_ARG, "K = %lld exceeds %lld", (long long)K, (long long)kSmallMaxK);
    const Range ry = rng(y, static_cast<size_t>(M) * N * 2);
    if (overlap(ry, rng(x, static_cast<size_t>(M) * K * 2)) || overlap(ry, rng(w, static_cast<size_t>(N) * K)) ||
        overlap(ry, rng(scale_w, N * 4)))
        return fail(CIDER_ERR_INVALID_ARG, "y overlaps an input");
    DeviceInfo* d = nullptr;
    if ((s = device_info(&d)) != CIDER_OK) return s;
    cudaError_t e = launch_mv_w8a16(x, xdt, static_cast<int>(M), static_cast<int>(K), w, scale_w, static_cast<int>(N),
                                    0, y, ydt, d->num_sms, d->status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CIDER_OK : cuda_fail(e, "W8A16 decode kernel launch");
}

cider_status_t cider_w8a16_mv_pg(const void* x, cider_dtype_t xdt, int64_t M, int64_t K, const int8_t* w,
                                 const float* scale_w, int64_t N, int64_t gs, void* y, cider_dtype_t ydt,
                                 void* stream) {
    t_last_error[0] = '\0';
    cider_status_t s = check_common(x, M, K, w, scale_w, N, y, xdt, ydt);
    if (s != CIDER_OK) return s;
    if ((s = check_gs(K, gs, false)) != CIDER_OK) return s;
    if (M == 0) return CIDER_OK;
    if (M > kMaxMvM) return fail(CIDER_ERR_INVALID_ARG, "M = %lld exceeds %d (decode shapes only)", (long long)M, kMaxMvM);
    const int64_t xbytes = M * ((K / 16 + 31) / 32) * 2048;  // fp32 activations, whole 512-wide passes
    if (xbytes > kMaxSmallXBytes)
        return fail(CIDER_ERR_INVALID_ARG, "%lld bytes of staged activations exceed %d (shared memory)",
                    (long long)xbytes, kMaxSmallXBytes);
    if (K > kSmallMaxK) return fail(CIDER_ERR_INVALID_ARG, "K = %lld exceeds %lld", (long long)K, (long long)kSmallMaxK);
    const Range ry = rng(y, static_cast<size_t>(M) * N * 2);
    if (overlap(ry, rng(x, static_cast<size_t>(M) * K * 2)) || overlap(ry, rng(w, static_cast<size_t>(N) * K)) ||
        overlap(ry, rng(scale_w, static_cast<size_t>(K / gs) * N * 4)))
        return fail(CIDER_ERR_INVALID_ARG, "y overlaps an input");
    DeviceInfo* d = nullptr;
    if ((s = device_info(&d)) != CIDER_OK) return s;
    cudaError_t e = launch_mv_w8a16(x, xdt, static_cast<int>(M), static_cast<int>(K), w, scale_w, static_cast<int>(N),
                                    static_cast<int>(gs), y, ydt, d->num_sms, d->status,
                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CIDER_OK : cuda_fail(e, "W8A16 per-group decode kernel launch");
}

cider_status_t cider_w8a8_linear_pg(const void* x, cider_dtype_t xdt, int64_t M, int64_t K, const int8_t* w,
                                    const float* scale_w, int64_t N, int64_t gs, void* y, cider_dtype_t ydt,
                                    void* workspace, size_t workspace_bytes, void* stream) {
    return linear(kModePG, x, xdt, M, K, w, scale_w, N, gs, y, ydt, workspace, workspace_bytes, stream);
}

cider_status_t cider_w4a8_linear_pg(const void* x, cider_dtype_t xdt, int64_t M, int64_t K,
                                    const uint8_t* w_packed, const float* scale_w, int64_t N, int64_t gs,
                                    void* y, cider_dtype_t ydt, void* workspace, size_t workspace_bytes,
                                    void* stream) {
    return linear(kModeW4, x, xdt, M, K, w_packed, scale_w, N, gs, y, ydt, workspace, workspace_bytes, stream);
}

cider_status_t cider_w4a8_linear_pc(const void* x, cider_dtype_t xdt, int64_t M, int64_t K, const uint8_t* w_packed,
                                    const float* scale_w, int64_t N, void* y, cider_dtype_t ydt, void* workspace,
                                    size_t workspace_bytes, void* stream) {
    return linear(kModeW4PC, x, xdt, M, K, w_packed, scale_w, N, 0, y, ydt, workspace, workspace_bytes, stream);
}

cider_status_t cider_w8a8_gemm_pc_q(const int8_t* q, const float* scale_x, int64_t M, int64_t K, const int8_t* w,
                                    const float* scale_w, int64_t N, void* y, cider_dtype_t ydt, void* stream) {
    return gemm_q(kModePC, q, scale_x, M, K, w, scale_w, N, 0, y, ydt, stream);
}

cider_status_t cider_w8a8_gemm_pg_q(const int8_t* q, const float* scale_x, int64_t M, int64_t K, const int8_t* w,
                                    const float* scale_w, int64_t N, int64_t gs, void* y, cider_dtype_t ydt,
                                    void* stream) {
    return gemm_q(kModePG, q, scale_x, M, K, w, scale_w, N, gs, y, ydt, stream);
}

cider_status_t cider_w4a8_gemm_pg_q(const int8_t* q, const float* scale_x, int64_t M, int64_t K,
                                    const uint8_t* w_packed, const float* scale_w, int64_t N, int64_t gs,
                                    void* y, cider_dtype_t ydt, void* stream) {
    return gemm_q(kModeW4, q, scale_x, M, K, w_packed, scale_w, N, gs, y, ydt, stream);
}

cider_status_t cider_w4a8_gemm_pc_q(const int8_t* q, const float* scale_x, int64_t M, int64_t K, const uint8_t* w_packed,
                                    const float* scale_w, int64_t N, void* y, cider_dtype_t ydt, void* stream) {
    return gemm_q(kModeW4PC, q, scale_x, M, K, w_packed, scale_w, N, 0, y, ydt, stream);
}

cider_status_t cider_silu_mul_quantize(const void* gate, const void* up, cider_dtype_t dt, int64_t M, int64_t F,
                                       int8_t* q, float* scale_x, void* a_out, void* stream) {
    t_last_error[0] = '\0';
    if (M < 0 || F < 1) return fail(CIDER_ERR_INVALID_ARG, "M >= 0 and F >= 1 required");
    if (F % 16 || F > 32768) return fail(CIDER_ERR_INVALID_ARG, "F = %lld must be a multiple of 16 and <= 32768", (long long)F);
    if (dt != CIDER_F16 && dt != CIDER_BF16) return fail(CIDER_ERR_INVALID_ARG, "dtype %d unknown", (int)dt);
    if (M == 0) return CIDER_OK;
    if (M > INT32_MAX) return fail(CIDER_ERR_INVALID_ARG, "M must be < 2^31");
    if (!gate || !up || !q || !scale_x) return fail(CIDER_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(gate) || !aligned16(up) || !aligned16(q) || (a_out && !aligned16(a_out)) ||
        (reinterpret_cast<uintptr_t>(scale_x) & 3u))
        return fail(CIDER_ERR_INVALID_ARG, "misaligned pointer");
    DeviceInfo* d = nullptr;
    cider_status_t s = device_info(&d);
    if (s != CIDER_OK) return s;
    cudaError_t e = launch_silu_mul_quantize(gate, up, dt, M, static_cast<int>(F), q, scale_x, a_out,
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CIDER_OK : cuda_fail(e, "silu-mul-quantize launch");
}

static cider_status_t quantize_weight(int mode, const float* W, int64_t N, int64_t K, int64_t gs, void* out,
                                      float* sw, void* stream) {
    t_last_error[0] = '\0';
    if (N < 1 || K < 1) return fail(CIDER_ERR_INVALID_ARG, "N, K >= 1 required");
    if (N > INT32_MAX || K > kMaxK) return fail(CIDER_ERR_INVALID_ARG, "size out of range");
    if (mode == 1 || mode == 2) {
        cider_status_t s = check_gs(K, gs, mode == 2);
        if (s != CIDER_OK) return s;
    }
    if (mode == 3 && K % 2) return fail(CIDER_ERR_INVALID_ARG, "INT4 packing needs an even K (K = %lld)", (long long)K);
    if (!W || !out || !sw) return fail(CIDER_ERR_INVALID_ARG, "NULL pointer");
    DeviceInfo* d = nullptr;
    cider_status_t s = device_info(&d);
    if (s != CIDER_OK) return s;
    cudaError_t e = launch_quantize_weight(mode, W, N, static_cast<int>(K), static_cast<int>(gs), out, sw,
                                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CIDER_OK : cuda_fail(e, "weight quantize launch");
}

// Percentile-clipped scales.  The position of the percentile within a slab of
// len values is p/100 * (len - 1) in double, split into the order statistic
// k0 = floor and the fraction t (rounded once to float); the kernels
// interpolate in fp32.
static cider_status_t quantize_weight_clip(const float* W, int64_t N, int64_t K, int64_t gs, double p,
                                           int8_t* out, float* sw, void* stream) {
    t_last_error[0] = '\0';
    if (!(p >= 0.0 && p <= 100.0))
        return fail(CIDER_ERR_INVALID_ARG, "clip_percentile = %g must lie in [0, 100]", p);
    if (N < 1 || K < 1) return fail(CIDER_ERR_INVALID_ARG, "N, K >= 1 required");
    if (N > INT32_MAX || K > kMaxK) return fail(CIDER_ERR_INVALID_ARG, "size out of range");
    if (gs != 0) {
        cider_status_t s = check_gs(K, gs, false);
        if (s != CIDER_OK) return s;
    }
    if (!W || !out || !sw) return fail(CIDER_ERR_INVALID_ARG, "NULL pointer");
    DeviceInfo* d = nullptr;
    cider_status_t s = device_info(&d);
    if (s != CIDER_OK) return s;
    const int64_t len = gs != 0 ? gs : K;
    const double pos = p / 100.0 * static_cast<double>(len - 1);
    int64_t k0 = static_cast<int64_t>(std::floor(pos));
    k0 = std::min<int64_t>(std::max<int64_t>(k0, 0), len - 1);
    const float t = static_cast<float>(pos - static_cast<double>(k0));
    cudaError_t e = launch_quantize_weight_clip(W, N, static_cast<int>(K), static_cast<int>(gs), static_cast<int>(k0),
                                                t, out, sw, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CIDER_OK : cuda_fail(e, "clipped weight quantize launch");
}

cider_status_t cider_quantize_weight_pc_clip(const float* W, int64_t N, int64_t K, double clip_percentile, int8_t* w,
                                             float* scale_w, void* stream) {
    return quantize_weight_clip(W, N, K, 0, clip_percentile, w, scale_w, stream);
}

cider_status_t cider_quantize_weight_pg_clip(const float* W, int64_t N, int64_t K, int64_t gs, double clip_percentile,
                                             int8_t* w, float* scale_w, void* stream) {
    return quantize_weight_clip(W, N, K, gs, clip_percentile, w, scale_w, stream);
}

cider_status_t cider_quantize_weight_pc(const float* W, int64_t N, int64_t K, int8_t* w, float* scale_w,
                                        void* stream) {
    return quantize_weight(0, W, N, K, 0, w, scale_w, stream);
}

cider_status_t cider_quantize_weight_pg(const float* W, int64_t N, int64_t K, int64_t gs, int8_t* w,
                                        float* scale_w, void* stream) {
    return quantize_weight(1, W, N, K, gs, w, scale_w, stream);
}

cider_status_t cider_pack_weight_int4_pg(const float* W, int64_t N, int64_t K, int64_t gs, uint8_t* w_packed,
                                         float* scale_w, void* stream) {
    return quantize_weight(2, W, N, K, gs, w_packed, scale_w, stream);
}

cider_status_t cider_pack_weight_int4_pc(const float* W, int64_t N, int64_t K, uint8_t* w_packed, float* scale_w,
                                         void* stream) {
    return quantize_weight(3, W, N, K, 0, w_packed, scale_w, stream);
}

// ---- decode attention ---------------------------------------------------------
static cider_status_t sdpa_check(int64_t H_q, int64_t H_kv, int64_t N, int64_t D) {
    if (D != kSdpaD) return fail(CIDER_ERR_INVALID_ARG, "D = %lld: the decode-attention kernels take D = 128", (long long)D);
    if (H_q < 1 || H_kv < 1 || H_q % H_kv)
        return fail(CIDER_ERR_INVALID_ARG, "H_q = %lld must be a positive multiple of H_kv = %lld", (long long)H_q, (long long)H_kv);
    if (H_q > 65535) return fail(CIDER_ERR_INVALID_ARG, "H_q = %lld exceeds 65535", (long long)H_q);
    // the kernels index keys with 32-bit ints (chunk ends up to N + chunk)
    if (N < 1 || N > (int64_t(1) << 30)) return fail(CIDER_ERR_INVALID_ARG, "N = %lld must lie in [1, 2^30]", (long long)N);
    return CIDER_OK;
}

size_t cider_sdpa_decode_workspace_bytes(int64_t H_q, int64_t H_kv, int64_t N, int64_t D) {
    if (sdpa_check(H_q, H_kv, N, D) != CIDER_OK) return 0;
    DeviceInfo* d = nullptr;
    if (device_info(&d) != CIDER_OK) return 0;
    return sdpa_part_bytes(H_q, sdpa_plan(H_q, H_kv, N, d->num_sms));
}

cider_status_t cider_test_sdpa_plan(int64_t H_q, int64_t H_kv, int64_t N, int64_t num_sms, int32_t* out4) {
    t_last_error[0] = '\0';
    cider_status_t s = sdpa_check(H_q, H_kv, N, kSdpaD);
    if (s != CIDER_OK) return s;
    if (num_sms < 1 || num_sms > 4096 || !out4) return fail(CIDER_ERR_INVALID_ARG, "num_sms in [1, 4096] and out4 required");
    const SdpaPlan p = sdpa_plan(H_q, H_kv, N, static_cast<int>(num_sms));
    out4[0] = p.th;
    out4[1] = p.tiles;
    out4[2] = p.chunk;
    out4[3] = p.chunks;
    return CIDER_OK;
}

cider_status_t cider_sdpa_decode(const void* q, const void* k, const void* v, cider_dtype_t dt, int64_t H_q,
                                 int64_t H_kv, int64_t N, int64_t D, void* out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    t_last_error[0] = '\0';
    cider_status_t s = sdpa_check(H_q, H_kv, N, D);
    if (s != CIDER_OK) return s;
    if (dt != CIDER_F16 && dt != CIDER_BF16) return fail(CIDER_ERR_INVALID_ARG, "dtype %d unknown", (int)dt);
    if (!q || !k || !v || !out || !workspace) return fail(CIDER_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace))
        return fail(CIDER_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    DeviceInfo* d = nullptr;
    if ((s = device_info(&d)) != CIDER_OK) return s;
    const SdpaPlan plan = sdpa_plan(H_q, H_kv, N, d->num_sms);
    const size_t need = sdpa_part_bytes(H_q, plan);
    if (workspace_bytes < need)
        return fail(CIDER_ERR_INVALID_ARG, "workspace of %zu bytes needed (got %zu)", need, workspace_bytes);
    const size_t kv = static_cast<size_t>(H_kv) * N * D * 2;
    const Range ro = rng(out, static_cast<size_t>(H_q) * D * 2);
    if (overlap(ro, rng(q, static_cast<size_t>(H_q) * D * 2)) || overlap(ro, rng(k, kv)) || overlap(ro, rng(v, kv)) ||
        overlap(ro, rng(workspace, need)))
        return fail(CIDER_ERR_INVALID_ARG, "out overlaps an input or the workspace");
    cudaError_t e = launch_sdpa_decode(q, k, v, dt == CIDER_BF16 ? 1 : 0, static_cast<int>(H_q), static_cast<int>(H_kv),
                                       static_cast<int>(N), plan, static_cast<float*>(workspace), out, d->status,
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CIDER_OK : cuda_fail(e, "decode-attention launch");
}

cider_status_t cider_test_gemm_i32(const int8_t* q, const int8_t* w, int64_t M, int64_t N, int64_t K,
                                   int32_t* acc, void* stream) {
    t_last_error[0] = '\0';
    alignas(16) static const float dummy[4] = {1, 1, 1, 1};  // scales are never read by the INT32 epilogue
    cider_status_t s = check_common(q, M, K, w, dummy, N, acc, CIDER_F16, CIDER_F16);
    if (s != CIDER_OK) return s;
    if (M == 0) return CIDER_OK;
    DeviceInfo* d = nullptr;
    if ((s = device_info(&d)) != CIDER_OK) return s;
    return run_gemm(kModeI32, q, nullptr, M, K, w, nullptr, N, 0, acc, 0, d, static_cast<cudaStream_t>(stream));
}

cider_status_t cider_test_gemm_i32_grouped(const int8_t* q, const int8_t* w, int64_t M, int64_t N, int64_t K,
                                           int64_t gs, int32_t* acc_g, void* stream) {
    t_last_error[0] = '\0';
    alignas(16) static const float dummy[4] = {1, 1, 1, 1};
    cider_status_t s = check_common(q, M, K, w, dummy, N, acc_g, CIDER_F16, CIDER_F16);
    if (s != CIDER_OK) return s;
    if ((s = check_gs(K, gs, false)) != CIDER_OK) return s;
    if (M == 0) return CIDER_OK;
    DeviceInfo* d = nullptr;
    if ((s = device_info(&d)) != CIDER_OK) return s;
    const int forced = g_split_override.load();
    const SplitPlan sp{0, forced > 1 ? forced : 1, 0, 0};
    return run_gemm(kModeI32G, q, nullptr, M, K, w, nullptr, N, gs, acc_g, 0, d, static_cast<cudaStream_t>(stream),
                    sp, nullptr);
}

cider_status_t cider_test_set_sdpa_kernel(int kernel) {
    if (set_sdpa_kernel(kernel) != cudaSuccess) return fail(CIDER_ERR_INVALID_ARG, "kernel %d outside [0, 3]", kernel);
    return CIDER_OK;
}

cider_status_t cider_test_set_small_m_kernel(int kernel) {
    if (set_small_m_kernel(kernel) != cudaSuccess)
        return fail(CIDER_ERR_INVALID_ARG, "kernel %d outside [0, 4]", kernel);
    return CIDER_OK;
}

cider_status_t cider_test_set_fused_quantize(int mode) {
    if (mode < 0 || mode > 2) return fail(CIDER_ERR_INVALID_ARG, "mode %d outside [0, 2]", mode);
    g_fuse_override.store(mode);
    return CIDER_OK;
}

cider_status_t cider_test_set_gemm_variant(int variant) {
    if (variant < kGemmAuto || variant > kGemmPair192)
        return fail(CIDER_ERR_INVALID_ARG, "variant %d outside [0, 5]", variant);
    g_gemm_variant.store(variant);
    return CIDER_OK;
}

cider_status_t cider_test_bounded_wait(int64_t limit_ns, void* stream) {
    t_last_error[0] = '\0';
    if (limit_ns < 1 || limit_ns > 100000000)
        return fail(CIDER_ERR_INVALID_ARG, "limit_ns = %lld outside [1, 1e8]", (long long)limit_ns);
    DeviceInfo* d = nullptr;
    cider_status_t s = device_info(&d);
    if (s != CIDER_OK) return s;
    cudaError_t e = launch_wait_selftest(d->status, static_cast<unsigned long long>(limit_ns),
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CIDER_OK : cuda_fail(e, "wait self-test launch");
}

cider_status_t cider_test_unpack_int4(const uint8_t* w_packed, int64_t N, int64_t K, int8_t* w, void* stream) {
    t_last_error[0] = '\0';
    if (N < 1 || K < 1 || K % 32) return fail(CIDER_ERR_INVALID_ARG, "N >= 1, K >= 1, K %% 32 == 0 required");
    if (!w_packed || !w || !aligned16(w_packed) || !aligned16(w)) return fail(CIDER_ERR_INVALID_ARG, "bad pointer");
    DeviceInfo* d = nullptr;
    cider_status_t s = device_info(&d);
    if (s != CIDER_OK) return s;
    cudaError_t e = launch_unpack_int4(w_packed, N, static_cast<int>(K), w, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CIDER_OK : cuda_fail(e, "unpack launch");
}

}  // extern "C"
