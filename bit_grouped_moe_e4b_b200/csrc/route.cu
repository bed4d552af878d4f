// Routing pass: per-expert histogram, prefix scan, and a stable scatter of the
// T*top_k routing slots into expert-contiguous order, in one CTA.
//
// "grouped-nf4-gemm" README, intro: one launch covers all active experts of a
// projection, which needs the routed rows grouped by expert; the decode glue
// lists a router epilogue in front of the grouped GEMM.
//
// The 32 warps of the CTA own consecutive ranges of slots and walk them in
// 32-slot pieces. __match_any_sync groups the lanes of a piece that share an
// expert, so ranks inside a piece come from a popcount and the order of slots
// within an expert is the slot order (stable), as the layer's combine and the
// oracle both assume.
#include "common.cuh"
#include "launch.h"

namespace e4b {

constexpr int kRouteThreads = 1024;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kBatch = 8;  // 32-slot pieces whose ids are loaded together
constexpr int32_t kRouteMultiMin = 16384;  // slots from which the layer routes over many CTAs

__global__ void __launch_bounds__(kRouteThreads, 1)
route_kernel(const int32_t* __restrict__ ids, int32_t R, int32_t E, int32_t* __restrict__ counts,
             int64_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
             int32_t* __restrict__ active, int32_t* __restrict__ status, int32_t* __restrict__ clear,
             int32_t nclear) {
  extern __shared__ int32_t smem[];
  int32_t* wcnt = smem;                        // [kRouteWarps][E] counts, then bases
  int32_t* scan = smem + kRouteWarps * E;      // [kRouteThreads] scan scratch
  __shared__ int32_t s_bad;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  // launched as a programmatic dependent: the work before it may still read
  // what this kernel writes; the layer kernel after it may start launching
  // (it waits for this kernel before reading the routing)
  grid_dependency_wait();
  grid_launch_dependents();
  for (int i = tid; i < kRouteWarps * E; i += kRouteThreads) wcnt[i] = 0;
  // counters the following layer kernels expect at zero
  for (int i = tid; i < nclear; i += kRouteThreads) clear[i] = 0;
  if (tid == 0) {
    s_bad = 0;
    // The status word describes the most recent call: route runs first.
    if (status)
      for (int i = 0; i < 8; ++i) status[i] = 0;  // error code, dropped slots, wait diagnostics
  }
  __syncthreads();

  const int32_t chunk = (R + kRouteWarps - 1) / kRouteWarps;
  const int32_t beg = min(R, warp * chunk);
  const int32_t end = min(R, beg + chunk);
  int32_t* my = wcnt + warp * E;

  // pass 1: per-warp histogram (the ids of kBatch pieces are loaded together
  // so that their latencies overlap)
  for (int32_t b0 = beg; b0 < end; b0 += 32 * kBatch) {
    int32_t ev[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int32_t s = b0 + 32 * u + lane;
      ev[u] = s < end ? __ldg(ids + s) : 0;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int32_t s = b0 + 32 * u + lane;
      if (b0 + 32 * u >= end) break;  // uniform
      const bool in = s < end;
      int32_t e = ev[u];
      const bool ok = in && e >= 0 && e < E;
      if (in && !ok) atomicAdd(&s_bad, 1);
      if (!ok) e = -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      const int leader = __ffs(peers) - 1;
      if (ok && lane == leader) my[e] += __popc(peers);
    }
  }
  __syncthreads();

  // per expert: totals and per-warp exclusive bases
  int32_t total = 0;
  if (tid < E) {
    for (int w = 0; w < kRouteWarps; ++w) {
      const int32_t c = wcnt[w * E + tid];
      wcnt[w * E + tid] = total;
      total += c;
    }
  }
  // block-wide exclusive scan of totals over experts (E <= 1024)
  scan[tid] = (tid < E) ? total : 0;
  __syncthreads();
  for (int d = 1; d < kRouteThreads; d <<= 1) {
    const int32_t v = tid >= d ? scan[tid - d] : 0;
    __syncthreads();
    scan[tid] += v;
    __syncthreads();
  }
  const int32_t incl = scan[tid];
  const int32_t excl = incl - ((tid < E) ? total : 0);
  if (tid < E) {
    counts[tid] = total;
    offsets[tid] = excl;
    for (int w = 0; w < kRouteWarps; ++w) wcnt[w * E + tid] += excl;
  }
  if (tid == E - 1) offsets[E] = incl;
  __syncthreads();

  // active-expert list for the small-M kernels: active[0] = count, then ids
  if (active) {
    scan[tid] = (tid < E && total > 0) ? 1 : 0;
    __syncthreads();
    for (int d = 1; d < kRouteThreads; d <<= 1) {
      const int32_t v = tid >= d ? scan[tid - d] : 0;
      __syncthreads();
      scan[tid] += v;
      __syncthreads();
    }
    if (tid < E && total > 0) active[scan[tid]] = tid;  // 1-based slot
    if (tid == kRouteThreads - 1) active[0] = scan[tid];
  }

  // pass 2: stable scatter, pieces in slot order
  for (int32_t b0 = beg; b0 < end; b0 += 32 * kBatch) {
    int32_t ev[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int32_t s = b0 + 32 * u + lane;
      ev[u] = s < end ? __ldg(ids + s) : 0;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int32_t s = b0 + 32 * u + lane;
      if (b0 + 32 * u >= end) break;  // uniform
      const bool in = s < end;
      int32_t e = ev[u];
      const bool ok = in && e >= 0 && e < E;
      if (!ok) e = -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      const int leader = __ffs(peers) - 1;
      int32_t pos = -1;
      if (ok) {
        pos = my[e] + __popc(peers & ((1u << lane) - 1u));
        perm[pos] = s;
      }
      if (in) inv[s] = pos;
      __syncwarp();
      if (ok && lane == leader) my[e] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  if (tid == 0 && s_bad) {
    record_status(status, E4B_ERR_BAD_EXPERT_ID);
    atomicAdd(status + 1, s_bad);
  }
}

size_t route_smem_bytes(int32_t E) { return size_t(kRouteWarps) * E * 4 + kRouteThreads * 4; }

// The same routing over many CTAs, for large T*k (one CTA spends ~1400 clocks
// per 32-slot piece, ~90 us at 65536 slots). CTA b owns the slots of chunk b
// (kRouteChunk of them):
//   route_count_kernel    per-chunk expert histograms -> cnt[b][e] (and the
//                         chunk's count of bad ids -> cnt[G*E + b]);
//   route_scatter_kernel  every CTA sums the histograms (totals, offsets and,
//                         for its chunk, the slots of earlier chunks per
//                         expert), CTA 0 writes counts/offsets, and each CTA
//                         scatters its chunk as the one-CTA kernel does, so
//                         perm and inv are the same, bit for bit.
constexpr int kRouteChunk = 2048;

__global__ void __launch_bounds__(kRouteThreads, 1)
route_count_kernel(const int32_t* __restrict__ ids, int32_t R, int32_t E, int32_t* __restrict__ cnt,
                   int32_t* __restrict__ status, int32_t* __restrict__ clear, int32_t nclear) {
  extern __shared__ int32_t smem[];
  int32_t* hist = smem;  // [E]
  __shared__ int32_t s_bad;
  const int tid = threadIdx.x;
  grid_dependency_wait();
  grid_launch_dependents();
  for (int i = tid; i < E; i += kRouteThreads) hist[i] = 0;
  if (tid == 0) s_bad = 0;
  if (blockIdx.x == 0) {
    for (int i = tid; i < nclear; i += kRouteThreads) clear[i] = 0;
    if (status && tid < 8) status[tid] = 0;  // the status words describe the most recent call
  }
  __syncthreads();
  const int32_t beg = int32_t(blockIdx.x) * kRouteChunk;
  const int32_t end = min(R, beg + kRouteChunk);
  for (int32_t s = beg + tid; s < end; s += kRouteThreads) {
    const int32_t e = __ldg(ids + s);
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    else atomicAdd(&s_bad, 1);
  }
  __syncthreads();
  for (int i = tid; i < E; i += kRouteThreads) cnt[int64_t(blockIdx.x) * E + i] = hist[i];
  if (tid == 0) cnt[int64_t(gridDim.x) * E + blockIdx.x] = s_bad;
}

__global__ void __launch_bounds__(kRouteThreads, 1)
route_scatter_kernel(const int32_t* __restrict__ ids, int32_t R, int32_t E, const int32_t* __restrict__ cnt,
                     int32_t* __restrict__ counts, int64_t* __restrict__ offsets, int32_t* __restrict__ perm,
                     int32_t* __restrict__ inv, int32_t* __restrict__ status) {
  extern __shared__ int32_t smem[];
  int32_t* wcnt = smem;                        // [kRouteWarps][E] counts, then bases
  int32_t* scan = smem + kRouteWarps * E;      // [kRouteThreads]
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int G = int(gridDim.x);
  const int b = int(blockIdx.x);
  grid_dependency_wait();
  grid_launch_dependents();
  for (int i = tid; i < kRouteWarps * E; i += kRouteThreads) wcnt[i] = 0;

  // per expert: the total, and the slots of the chunks before this one
  int32_t total = 0, before = 0;
  if (tid < E) {
    for (int c = 0; c < G; ++c) {
      const int32_t v = __ldg(cnt + int64_t(c) * E + tid);
      if (c < b) before += v;
      total += v;
    }
  }
  scan[tid] = (tid < E) ? total : 0;
  __syncthreads();
  for (int d = 1; d < kRouteThreads; d <<= 1) {
    const int32_t v = tid >= d ? scan[tid - d] : 0;
    __syncthreads();
    scan[tid] += v;
    __syncthreads();
  }
  const int32_t incl = scan[tid];
  const int32_t excl = incl - ((tid < E) ? total : 0);
  if (b == 0) {
    if (tid < E) {
      counts[tid] = total;
      offsets[tid] = excl;
    }
    if (tid == E - 1) offsets[E] = incl;
    if (tid == 0 && status) {
      int32_t bad = 0;
      for (int c = 0; c < G; ++c) bad += __ldg(cnt + int64_t(G) * E + c);
      if (bad) {
        record_status(status, E4B_ERR_BAD_EXPERT_ID);
        atomicAdd(status + 1, bad);
      }
    }
  }

  // this chunk, split over the warps as in the one-CTA kernel
  const int32_t cbeg = b * kRouteChunk;
  const int32_t cend = min(R, cbeg + kRouteChunk);
  const int32_t chunk = (cend - cbeg + kRouteWarps - 1) / kRouteWarps;
  const int32_t beg = min(cend, cbeg + warp * chunk);
  const int32_t end = min(cend, beg + chunk);
  int32_t* my = wcnt + warp * E;
  for (int32_t s0 = beg; s0 < end; s0 += 32) {
    const int32_t s = s0 + lane;
    const bool in = s < end;
    int32_t e = in ? __ldg(ids + s) : -1;
    const bool ok = in && e >= 0 && e < E;
    if (!ok) e = -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    if (ok && lane == leader) my[e] += __popc(peers);
  }
  __syncthreads();
  if (tid < E) {
    int32_t run = excl + before;
    for (int w = 0; w < kRouteWarps; ++w) {
      const int32_t c = wcnt[w * E + tid];
      wcnt[w * E + tid] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int32_t s0 = beg; s0 < end; s0 += 32) {
    const int32_t s = s0 + lane;
    const bool in = s < end;
    int32_t e = in ? __ldg(ids + s) : -1;
    const bool ok = in && e >= 0 && e < E;
    if (!ok) e = -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    int32_t pos = -1;
    if (ok) {
      pos = my[e] + __popc(peers & ((1u << lane) - 1u));
      perm[pos] = s;
    }
    if (in) inv[s] = pos;
    __syncwarp();
    if (ok && lane == leader) my[e] += __popc(peers);
    __syncwarp();
  }
}

size_t route_scratch_bytes(int32_t R, int32_t E) {
  if (R < kRouteMultiMin) return 0;  // one CTA
  const int64_t G = (int64_t(R) + kRouteChunk - 1) / kRouteChunk;
  return size_t(G) * size_t(E + 1) * 4;
}

cudaError_t launch_route(const int32_t* ids, int32_t R, int32_t E, int32_t* counts, int64_t* offsets,
                         int32_t* perm, int32_t* inv, int32_t* active, int32_t* status,
                         cudaStream_t st, int32_t* clear, int32_t nclear, int32_t* scratch,
                         size_t scratch_bytes, int* launches) {
  static int configured = -1;  // the attributes are per device context
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured != dev) {
    cudaError_t err = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(route_smem_bytes(1024)));
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(route_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(route_smem_bytes(1024)));
    if (err != cudaSuccess) return err;
    configured = dev;
  }
  // many CTAs for large batches when the caller lends scratch space (and
  // needs no active-expert list, which only the one-CTA kernel builds)
  const size_t need = route_scratch_bytes(R, E);
  const bool multi = scratch && !active && need > 0 && scratch_bytes >= need;
  if (launches) *launches = multi ? 2 : 1;
  if (multi) {
    const int G = int((int64_t(R) + kRouteChunk - 1) / kRouteChunk);
    cudaError_t err = launch_dependent(route_count_kernel, dim3(G), dim3(kRouteThreads), size_t(E) * 4, st, ids, R,
                                       E, scratch, status, clear, nclear);
    if (err != cudaSuccess) return err;
    return launch_dependent(route_scatter_kernel, dim3(G), dim3(kRouteThreads), route_smem_bytes(E), st, ids, R, E,
                            const_cast<const int32_t*>(scratch), counts, offsets, perm, inv, status);
  }
  return launch_dependent(route_kernel, dim3(1), dim3(kRouteThreads), route_smem_bytes(E), st, ids, R, E, counts,
                          offsets, perm, inv, active, status, clear, nclear);
}

// The routed activation rows in expert order, xs[p] = x[perm[p] / top_k] for
// p < offsets[E], so that the large-M projection reads its B operand as
// contiguous row tiles. One warp per row, 16-byte copies, each lane holding up
// to kGatherBatch copies in flight before it stores them (a row of H = 2048
// bf16 values is one batch); the next row's slot is loaded while this row is
// copied. Rows of dropped slots (p >= offsets[E]) are not written.
constexpr int kGatherThreads = 256;
constexpr int kGatherBatch = 8;

__global__ void __launch_bounds__(kGatherThreads)
gather_rows_kernel(const uint16_t* __restrict__ x, int64_t H, const int32_t* __restrict__ perm,
                   int32_t top_k, const int64_t* __restrict__ offsets, int32_t E,
                   uint16_t* __restrict__ xs) {
  const int64_t R = offsets[E];
  const int64_t chunks = H / 8;
  const int warps = kGatherThreads / 32;
  const int lane = threadIdx.x & 31;
  const int64_t stride = int64_t(gridDim.x) * warps;
  int64_t p = int64_t(blockIdx.x) * warps + (threadIdx.x >> 5);
  int32_t slot = p < R ? __ldg(perm + p) : 0;
  for (; p < R; p += stride) {
    const int32_t next = p + stride < R ? __ldg(perm + p + stride) : 0;
    const uint4* src = reinterpret_cast<const uint4*>(x + int64_t(slot / top_k) * H);
    uint4* dst = reinterpret_cast<uint4*>(xs + p * H);
    for (int64_t c0 = lane; c0 < chunks; c0 += 32 * kGatherBatch) {
      uint4 v[kGatherBatch];
#pragma unroll
      for (int u = 0; u < kGatherBatch; ++u) {
        const int64_t c = c0 + 32 * u;
        if (c < chunks) v[u] = __ldg(src + c);
      }
#pragma unroll
      for (int u = 0; u < kGatherBatch; ++u) {
        const int64_t c = c0 + 32 * u;
        if (c < chunks) dst[c] = v[u];
      }
    }
    slot = next;
  }
}

cudaError_t launch_gather_rows(const uint16_t* x, int64_t H, const int32_t* perm, int32_t top_k,
                               const int64_t* offsets, int32_t E, int64_t R_max, uint16_t* xs,
                               cudaStream_t st, int sms) {
  const int64_t warps = kGatherThreads / 32;
  int64_t grid = (R_max + warps - 1) / warps;
  if (grid > int64_t(sms) * 8) grid = int64_t(sms) * 8;
  if (grid < 1) grid = 1;
  gather_rows_kernel<<<int(grid), kGatherThreads, 0, st>>>(x, H, perm, top_k, offsets, E, xs);
  return cudaGetLastError();
}

}  // namespace e4b
