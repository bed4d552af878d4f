// e4b_moe_forward_noalloc: the layer forward for callers that cannot
// allocate device memory. Its scratch (routing arrays, the bf16
// intermediate, the fp32 combine accumulator, the status word) lives in one
// file-scope device array instead of a caller workspace; the kernels are the
// same ones e4b_moe_forward launches.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace {

// Scratch of the allocation-free entry point. Every GPU that loads the
// library holds it until the process exits.
constexpr size_t kNoallocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once
// per device (the array's name in host code is only a host-side stand-in).
// The cached address belongs to the device's current context: a
// cudaDeviceReset (or any teardown of the primary context) invalidates it, so
// the process must not call this entry point again on that device afterwards.
e4b_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return E4B_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return E4B_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return E4B_OK;
}

}  // namespace

extern "C" e4b_status e4b_moe_forward_noalloc(const e4b_moe_weights* w, const uint16_t* x,
                                              int64_t T, int32_t top_k, const int32_t* ids,
                                              const float* gates, uint16_t* y, uint32_t flags,
                                              void* stream) {
  if (!w || T < 0 || top_k <= 0) return E4B_ERR_INVALID_ARG;
  size_t full = 0;
  e4b_status st = e4b_moe_workspace_size(w, T, top_k, &full);
  if (st != E4B_OK) return st;
  // int4-b32 stacks need only the status words and h [top_k, I], whatever T.
  // For NF4 / MXFP4 the staging copy of the routed rows is optional: without
  // room for it the large-M path gathers the rows inside its kernel.
  const size_t need = w->fmt == E4B_FMT_INT4B32 ? full : e4b::moe_workspace_min_bytes(w, T, top_k, flags);
  if (need > kNoallocScratchBytes) return E4B_ERR_EXCEEDS_STATIC_SCRATCH;
  if (T == 0) return e4b_moe_forward(w, x, T, top_k, ids, gates, y, nullptr, 0, flags, stream);
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != E4B_OK) return st;
  // The routing kernel clears the status word and the gate_up kernel clears
  // the fp32 accumulator, so nothing from an earlier call leaks into this one.
  return e4b_moe_forward(w, x, T, top_k, ids, gates, y, scratch, kNoallocScratchBytes, flags, stream);
}
