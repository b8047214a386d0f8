// sdpa_decode.h -- launchers of the decode-attention kernels (sdpa_decode.cu).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace cider {

constexpr int kSdpaD = 128;  // head dimension of the kernels

// How a decode-attention call is cut: TH query heads per CTA (a head tile of
// one KV group), C chunks of `chunk` keys along the sequence.
struct SdpaPlan {
    int th, tiles, chunk, chunks;
};
SdpaPlan sdpa_plan(int64_t H_q, int64_t H_kv, int64_t N, int num_sms);
// fp32 partial results [H_q][chunks][D + 2] (o, then max and sum)
size_t sdpa_part_bytes(int64_t H_q, const SdpaPlan& p);
cudaError_t launch_sdpa_decode(const void* q, const void* k, const void* v, int dt, int H_q, int H_kv, int N,
                               const SdpaPlan& plan, float* part, void* out, cudaStream_t st);

}  // namespace cider
