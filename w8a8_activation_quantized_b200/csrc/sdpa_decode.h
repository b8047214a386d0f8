// sdpa_decode.h -- launchers of the decode-attention kernels (sdpa_decode.cu).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace cider {

constexpr int kSdpaD = 128;  // head dimension of the kernels
// One chunk's partial result: o [D], then its max and its sum, padded to a
// multiple of four floats so that every row starts 16-byte aligned.
constexpr int kSdpaPartStride = kSdpaD + 4;

// How a decode-attention call is cut: TH query heads per CTA (a head tile of
// one KV group), C chunks of `chunk` keys along the sequence.
// tc = 1: the tensor-core kernel of sdpa_tc.cu (one CTA per KV head and
// chunk, th = the group's query heads).
struct SdpaPlan {
    int th, tiles, chunk, chunks;
    int tc = 0;
};
SdpaPlan sdpa_plan(int64_t H_q, int64_t H_kv, int64_t N, int num_sms);
// fp32 partial results [H_q][chunks][kSdpaPartStride] (o, then max and sum)
size_t sdpa_part_bytes(int64_t H_q, const SdpaPlan& p);
cudaError_t launch_sdpa_decode(const void* q, const void* k, const void* v, int dt, int H_q, int H_kv, int N,
                               const SdpaPlan& plan, float* part, void* out, unsigned* status, cudaStream_t st);
// The chunk merge: out[h] = sum_c o_c 2^(m_c - M) / sum_c l_c 2^(m_c - M).
cudaError_t launch_sdpa_merge(const float* part, int chunks, void* out, int H_q, int dt, cudaStream_t st);

// sdpa_tc.cu: whether the tensor-core kernel takes the shape (2 <= H_q / H_kv
// <= 16), its plan, its launch (split kernel, then the merge), and the test
// override (0 automatic, 1 CUDA cores only, 2 tensor cores, 3 tensor cores
// with the V descriptor's offset fields swapped).
bool sdpa_tc_applies(int64_t H_q, int64_t H_kv, int64_t N);
SdpaPlan sdpa_tc_plan(int64_t H_q, int64_t H_kv, int64_t N, int num_sms);
cudaError_t launch_sdpa_tc(const void* q, const void* k, const void* v, int dt, int H_q, int H_kv, int N,
                           const SdpaPlan& plan, float* part, void* out, unsigned* status, cudaStream_t st);
cudaError_t set_sdpa_kernel(int k);

}  // namespace cider
