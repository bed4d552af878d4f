// Host-side launchers of the expert-parallel kernels (csrc/ep.cu), used by the
// C-ABI layer (api.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace e4b {

cudaError_t launch_ep_dest(const int32_t* ids, int64_t n, int32_t E, int32_t epr, int32_t* dest, cudaStream_t st,
                           int sms);
cudaError_t launch_ep_pack(const uint16_t* x, int64_t H, const int32_t* ids, const float* gates, int32_t top_k,
                           const int32_t* perm, const int64_t* offsets, int32_t G, int64_t R_max, int32_t epr,
                           uint16_t* xs, int32_t* local_ids, float* local_gates, cudaStream_t st, int sms);
cudaError_t launch_ep_combine(const uint16_t* ys, int64_t H, const int32_t* inv, int64_t T, int32_t top_k,
                              uint16_t* y, cudaStream_t st, int sms);

}  // namespace e4b
