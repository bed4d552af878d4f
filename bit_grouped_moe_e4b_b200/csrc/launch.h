// Internal host-side launchers shared by the C-ABI layer (api.cu).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "e4b.h"

namespace e4b {

cudaError_t launch_quantize_nf4(const float* w, int64_t nblocks, uint8_t* codes, float* absmax,
                                cudaStream_t st, int sms);
cudaError_t launch_quantize_mxfp4(const float* w, int64_t nblocks, uint8_t* blocks, uint8_t* scales,
                                  cudaStream_t st, int sms);
cudaError_t launch_dequantize(int fmt, const uint8_t* codes, const void* scales, int64_t nweights,
                              uint16_t* out, cudaStream_t st, int sms);
void host_nf4_levels(float* out);

size_t route_smem_bytes(int32_t E);
cudaError_t launch_route(const int32_t* ids, int32_t R, int32_t E, int32_t* counts, int64_t* offsets,
                         int32_t* perm, int32_t* inv, int32_t* active, int32_t* status,
                         cudaStream_t st, int32_t* clear = nullptr, int32_t nclear = 0);
// xs[p] = x[perm[p] / top_k] for p < offsets[E] (H % 8 == 0, 16-byte aligned).
cudaError_t launch_gather_rows(const uint16_t* x, int64_t H, const int32_t* perm, int32_t top_k,
                               const int64_t* offsets, int32_t E, int64_t R_max, uint16_t* xs,
                               cudaStream_t st, int sms);
// Smallest workspace e4b_moe_forward accepts (without the staging copy of the
// routed rows that e4b_moe_workspace_size includes).
size_t moe_workspace_min_bytes(int64_t E, int64_t H, int64_t I, int64_t T, int64_t top_k);

// GemmProblem::epilogue for the input gradient through the weights
// (e4b_grouped_dgrad): out [R, K] bf16, row p = a_p . W_e, a [R, N].
constexpr int kEpiDgrad = 3;

// Description of one grouped projection as the kernels see it.
struct GemmProblem {
  int fmt;          // e4b_format
  int epilogue;     // e4b_epilogue
  int E;
  int top_k;
  int64_t N, K;     // weight rows (both halves for SWIGLU), inner dim
  int64_t R_max;    // bound on offsets[E]
  const uint8_t* codes;
  const void* scales;
  const uint16_t* a;
  int64_t lda;
  const int32_t* row_slot;  // may be null: row p reads a[p]; else a[row_slot[p] / top_k]
  const int32_t* out_slot;  // COMBINE: slot of row p (p when null)
  const int64_t* offsets;   // [E+1]
  const float* gates;       // COMBINE
  void* out;
  int64_t ldo;
  float* zero_buf;          // optional buffer the kernel clears first (fp32 accumulator)
  int64_t zero_count;       // floats in zero_buf
  int32_t* status;          // device status word or null
  uint32_t flags;
  // expert variant (include/e4b.h); bias: fp32 [E, N] per weight row or null
  int layout, act;
  float alpha, limit;
  const float* bias;
};

cudaError_t launch_gemv(const GemmProblem& p, cudaStream_t st, int sms);

// The whole small-M layer in one persistent launch (csrc/smallm.cu).
struct SmallMLayer {
  int fmt, E, H, I, top_k;
  int64_t T;
  const uint8_t* gu_codes;
  const void* gu_scales;
  const uint8_t* dn_codes;
  const void* dn_scales;
  const uint16_t* x;
  const int32_t* perm;
  const int64_t* offsets;
  const float* gates;
  uint16_t* h;
  float* acc;
  uint16_t* y;
  int32_t* sync;   // smallm_sync_ints(E, H) ints, zero on entry
  int32_t* status;
  uint32_t flags;
  int layout, act;  // expert variant (include/e4b.h)
  float alpha, limit;
  const float* gu_bias;  // fp32 [E, 2I] or null
  const float* dn_bias;  // fp32 [E, H] or null
};
size_t smallm_sync_ints(int E, int H);
cudaError_t launch_smallm_layer(const SmallMLayer& L, cudaStream_t st, int sms);
cudaError_t launch_tc_gemm(const GemmProblem& p, cudaStream_t st, int sms);
cudaError_t launch_finalize(const float* acc, int64_t n, uint16_t* y, cudaStream_t st, int sms);

}  // namespace e4b
