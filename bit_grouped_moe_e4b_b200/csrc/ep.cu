// Expert parallelism around the layer (one process per GPU; rank r holds the
// experts [r * epr, (r + 1) * epr)): the destination rank of every routed
// slot, the send buffer of the routed rows in destination order (each row
// with its local expert id and gate), and the combine of the rows that come
// back. The routed rows cross NVLink in an all-to-all between these kernels,
// made by the caller; the experts run in e4b_moe_forward with one slot a row.
#include "common.cuh"
#include "ep.h"

namespace e4b {
namespace {

constexpr int kEpThreads = 256;

// dest[i] = ids[i] / epr for ids in [0, E); -1 (a slot the routing pass drops) else.
__global__ void __launch_bounds__(kEpThreads) ep_dest_kernel(const int32_t* __restrict__ ids, int64_t n, int32_t E,
                                                             int32_t epr, int32_t* __restrict__ dest) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int32_t e = ids[i];
    dest[i] = (e >= 0 && e < E) ? e / epr : -1;
  }
}

// One warp per position p < offsets[G] of the destination order:
// xs[p] = x[perm[p] / top_k] (16-byte copies), local_ids[p] = ids[slot] % epr,
// local_gates[p] = gates[slot].
__global__ void __launch_bounds__(kEpThreads) ep_pack_kernel(const uint16_t* __restrict__ x, int64_t H,
                                                             const int32_t* __restrict__ ids,
                                                             const float* __restrict__ gates, int32_t top_k,
                                                             const int32_t* __restrict__ perm,
                                                             const int64_t* __restrict__ offsets, int32_t G,
                                                             int64_t R_max, int32_t epr, uint16_t* __restrict__ xs,
                                                             int32_t* __restrict__ local_ids,
                                                             float* __restrict__ local_gates) {
  const int64_t R = min(offsets[G], R_max);
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t p = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); p < R; p += warps) {
    const int32_t slot = perm[p];
    const uint4* src = reinterpret_cast<const uint4*>(x + int64_t(slot / top_k) * H);
    uint4* dst = reinterpret_cast<uint4*>(xs + p * H);
    for (int64_t v = lane; v < H / 8; v += 32) dst[v] = src[v];
    if (lane == 0) {
      local_ids[p] = ids[slot] % epr;
      local_gates[p] = gates[slot];
    }
  }
}

// y[t] = bf16(sum_j ys[inv_perm[t * top_k + j]]) in fp32, slots with
// inv_perm -1 (dropped) left out; one CTA per token, 8 values a thread-step.
__global__ void __launch_bounds__(kEpThreads) ep_combine_kernel(const uint16_t* __restrict__ ys, int64_t H,
                                                                const int32_t* __restrict__ inv, int64_t T,
                                                                int32_t top_k, uint16_t* __restrict__ y) {
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    for (int64_t v = threadIdx.x; v < H / 8; v += blockDim.x) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int j = 0; j < top_k; ++j) {
        const int32_t p = inv[t * top_k + j];
        if (p < 0) continue;
        const uint4 r = reinterpret_cast<const uint4*>(ys + int64_t(p) * H)[v];
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] += __uint_as_float(w[i] << 16);
          acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(y + t * H)[v] = o;
    }
  }
}

int grid_for(int64_t work, int per_block, int sms) {
  const int64_t want = (work + per_block - 1) / per_block;
  const int64_t cap = int64_t(sms) * 8;
  return int(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_ep_dest(const int32_t* ids, int64_t n, int32_t E, int32_t epr, int32_t* dest, cudaStream_t st,
                           int sms) {
  if (n <= 0) return cudaSuccess;
  ep_dest_kernel<<<grid_for(n, kEpThreads, sms), kEpThreads, 0, st>>>(ids, n, E, epr, dest);
  return cudaGetLastError();
}

cudaError_t launch_ep_pack(const uint16_t* x, int64_t H, const int32_t* ids, const float* gates, int32_t top_k,
                           const int32_t* perm, const int64_t* offsets, int32_t G, int64_t R_max, int32_t epr,
                           uint16_t* xs, int32_t* local_ids, float* local_gates, cudaStream_t st, int sms) {
  if (R_max <= 0) return cudaSuccess;
  ep_pack_kernel<<<grid_for(R_max, kEpThreads / 32, sms), kEpThreads, 0, st>>>(
      x, H, ids, gates, top_k, perm, offsets, G, R_max, epr, xs, local_ids, local_gates);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const uint16_t* ys, int64_t H, const int32_t* inv, int64_t T, int32_t top_k,
                              uint16_t* y, cudaStream_t st, int sms) {
  if (T <= 0) return cudaSuccess;
  ep_combine_kernel<<<grid_for(T, 1, sms), kEpThreads, 0, st>>>(ys, H, inv, T, top_k, y);
  return cudaGetLastError();
}

}  // namespace e4b
