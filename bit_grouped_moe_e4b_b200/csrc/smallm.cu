// Small-M MoE layer in one persistent launch: both projections, the SwiGLU,
// the weighted combine and the bf16 output.
//
// "grouped-nf4-gemm" README, intro: the grouped GEMM over all active experts
// on packed weights with table decode, fp32 accumulation and a bf16 epilogue;
// bitsandbytes PR #1984, Design: gated SiLU between the projections and the
// weighted sum over the chosen experts.
//
// With few routed rows per expert every packed byte is read once, and the
// cost is the integer work of decoding (B200 issues the byte-permute /
// logic / shift ops at half the fp32 rate), so the kernel is organised to
// spend nothing else on the integer pipe and to keep every SM busy to the end:
//  * warps take work items from one atomic counter: first gate_up items
//    (one expert, 16 gate rows + the same 16 up rows, all of K), then down
//    items (one expert, 16 output rows, one K slice). A down item waits,
//    bounded, until every gate_up item of its expert has stored h;
//  * a lane owns 32 contiguous packed bytes (64 weights) of two rows per
//    256-wide K chunk, copied ahead into a private shared-memory slot with
//    cp.async; it decodes them through the block's 16-entry bf16 table straight
//    into the A fragment of mma.sync m16n8k16 (bf16 in, fp32 accumulate), with
//    the K order permuted so that fragment columns are the lane's own weights;
//  * down items add gate * output into an fp32 accumulator; the last item to
//    finish a 16-row slice of the output converts that slice to bf16.
#include "common.cuh"
#include "launch.h"

namespace e4b {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 256;              // K per step of a warp
constexpr int kSlotBytesPerLane = 128;   // 2 rows x (2 matrices) x 32 B
constexpr int kSlots = 2;
constexpr int kMaxNT = 2;                // token chunks of 8 per pass (16 rows)
constexpr int kGroup = 8 * kMaxNT;
constexpr uint32_t kPolls = 1u << 24;

// sync words (int32) at the start of the layer's sync area:
//   work item counter, zeroing-chunk counter, zeroed-chunk count, then
//   done_A[E] (gate_up items finished per active expert) and arrive[H/16]
//   (down items finished per 16-row output slice). Cleared by the routing
//   kernel before every layer call.
enum : int { kWork = 0, kZeroWork = 1, kZeroDone = 2, kDoneA = 3 };
constexpr int64_t kZeroChunk = 16384;  // floats per zeroing chunk

E4B_DEV void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                      uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

E4B_DEV void cp16(uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
E4B_DEV void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
E4B_DEV void cp_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
E4B_DEV void cp_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

E4B_DEV uint4 lds128(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

E4B_DEV uint4 ld_cg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

E4B_DEV int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *p >= target; false if it gave up. limit == 0 (the
// test flag) gives up at once, so the error path can be exercised.
E4B_DEV bool wait_geq(const int* p, int target, uint32_t limit) {
  if (limit == 0) return false;
  uint32_t polls = 0;
  while (ld_acquire(p) < target) {
    if (++polls > limit) return false;
    __nanosleep(128);
  }
  return true;
}

struct Params {
  int E, H, I, top_k;
  int64_t T;
  const uint8_t* gu_codes;
  const uint8_t* gu_scales;
  const uint8_t* dn_codes;
  const uint8_t* dn_scales;
  const uint16_t* x;
  const int32_t* perm;
  const int64_t* offsets;
  const float* gates;
  uint16_t* h;       // [R, I] bf16, expert-ordered rows
  float* acc;        // [T, H] fp32
  uint16_t* y;       // [T, H] bf16
  int32_t* sync;     // work, zero_done, done_A[E], arrive[H/16]
  int32_t* status;
  int ksplit;        // K slice of a down item (multiple of 256)
  uint32_t flags;
};

// Scale words of one row for the chunk: NF4 = the absmax of the lane's
// 64-weight block (bits of a float); MXFP4 = its two e8m0 bytes.
template <int FMT>
E4B_DEV uint32_t load_scale(const uint8_t* srow, int kl, int K) {
  if (kl >= K) return 0u;
  if constexpr (FMT == E4B_FMT_NF4) {
    return __float_as_uint(__ldg(reinterpret_cast<const float*>(srow) + (kl >> 6)));
  } else {
    const uint32_t b0 = __ldg(srow + (kl >> 5));
    const uint32_t b1 = (kl + 32 < K) ? uint32_t(__ldg(srow + (kl >> 5) + 1)) : 0u;
    return b0 | (b1 << 8);
  }
}

// One warp-item over the K range [k0, k1) of one weight matrix (row
// pointers crow/srow for rows g and g+8 of the 16-row tile) and NT chunks of
// 8 token rows (brow: activation row of this lane's token in each chunk, or
// null). Accumulates into acc[j][4].
template <int FMT, int NT, bool COHERENT_B>
E4B_DEV void run_item(const uint8_t* const (&crow)[2], const uint8_t* const (&srow)[2],
                      const uint16_t* const (&brow)[kMaxNT], int k0, int k1, int K, uint32_t slot_base,
                      float (&acc)[kMaxNT][4]) {
  const int lane = threadIdx.x & 31;
  const int c = lane & 3;
  const int kend = min(K, k1);
  const int nchunks = (k1 - k0 + kChunk - 1) / kChunk;

  auto issue = [&](int ci, int slot) {
    const int kl = k0 + ci * kChunk + c * 64;
    const int left = kend - kl;  // weights this lane may copy
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int piece = 0; piece < 2; ++piece) {
        const uint32_t dst = slot_base + uint32_t(slot * kSlotBytesPerLane * 32) +
                             uint32_t((h * 2 + piece) * 512 + lane * 16);
        const bool ok = left >= 32 * (piece + 1);
        cp16(dst, ok ? (const void*)(crow[h] + (kl >> 1) + piece * 16) : (const void*)crow[h],
             ok ? 16u : 0u);
      }
    cp_commit();
  };
  auto load_b = [&](int koff, uint4 (&b)[NT]) {
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      b[j] = make_uint4(0, 0, 0, 0);
      if (brow[j] && koff < kend) {
        if constexpr (COHERENT_B) b[j] = ld_cg_v4(brow[j] + koff);
        else b[j] = __ldg(reinterpret_cast<const uint4*>(brow[j] + koff));
      }
    }
  };

  // two accumulator sets (the two MMA sub-steps of a word) shorten the
  // dependency chains through the tensor pipe
  float acc2[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc2[j][q] = 0.f;

  issue(0, 0);
  uint32_t sc_next0 = load_scale<FMT>(srow[0], k0 + c * 64, kend);
  uint32_t sc_next1 = load_scale<FMT>(srow[1], k0 + c * 64, kend);
  uint4 bcur[NT];
  load_b(k0 + c * 64, bcur);

  for (int ci = 0; ci < nchunks; ++ci) {
    const int slot = ci & 1;
    const int kl = k0 + ci * kChunk + c * 64;
    const uint32_t sc0 = sc_next0, sc1 = sc_next1;
    if (ci + 1 < nchunks) {
      issue(ci + 1, slot ^ 1);
      sc_next0 = load_scale<FMT>(srow[0], kl + kChunk, kend);
      sc_next1 = load_scale<FMT>(srow[1], kl + kChunk, kend);
      cp_wait1();
    } else {
      cp_wait0();
    }
    const uint32_t sbase = slot_base + uint32_t(slot * kSlotBytesPerLane * 32) + uint32_t(lane * 16);
    Lut L0, L1;
    if constexpr (FMT == E4B_FMT_NF4) {  // one 64-weight block per row and lane
      lut_nf4(L0, __uint_as_float(sc0));
      lut_nf4(L1, __uint_as_float(sc1));
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint4 w0 = lds128(sbase + uint32_t((0 * 2 + half) * 512));
      const uint4 w1 = lds128(sbase + uint32_t((1 * 2 + half) * 512));
      if constexpr (FMT == E4B_FMT_MXFP4) {  // one 32-weight block per half
        lut_mxfp4(L0, (sc0 >> (8 * half)) & 0xFFu);
        lut_mxfp4(L1, (sc1 >> (8 * half)) & 0xFFu);
      }
      const uint32_t r0w[4] = {w0.x, w0.y, w0.z, w0.w};
      const uint32_t r1w[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        // prefetch the next word's activations (next chunk's first word at the end)
        uint4 bnext[NT];
        const int knext = (half == 1 && wi == 3) ? kl + kChunk : kl + half * 32 + wi * 8 + 8;
        const bool more = !(half == 1 && wi == 3) || (ci + 1 < nchunks);
        if (more) load_b(knext, bnext);
        uint32_t o0[4], o1[4];
        lut_decode8<FMT>(L0, r0w[wi], o0);
        lut_decode8<FMT>(L1, r1w[wi], o1);
        // sub-step 0: weights 0..3 of the word, sub-step 1: weights 4..7;
        // fragment registers {row g | row g+8} x {cols 2c,2c+1 | 2c+8,2c+9}
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          mma16816(acc[j], o0[0], o1[0], o0[1], o1[1], bcur[j].x, bcur[j].y);
          mma16816(acc2[j], o0[2], o1[2], o0[3], o1[3], bcur[j].z, bcur[j].w);
        }
        if (more) {
#pragma unroll
          for (int j = 0; j < NT; ++j) bcur[j] = bnext[j];
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[j][q] += acc2[j][q];
}

// run_item with the token-chunk count as a compile-time constant
template <int FMT, bool COHERENT_B>
E4B_DEV void run_item_nt(int nt, const uint8_t* const (&crow)[2], const uint8_t* const (&srow)[2],
                         const uint16_t* const (&brow)[kMaxNT], int k0, int k1, int K, uint32_t slot_base,
                         float (&acc)[kMaxNT][4]) {
  if (nt == 1) run_item<FMT, 1, COHERENT_B>(crow, srow, brow, k0, k1, K, slot_base, acc);
  else run_item<FMT, 2, COHERENT_B>(crow, srow, brow, k0, k1, K, slot_base, acc);
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, 2) smallm_layer_kernel(Params p) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int32_t s_act[1024];
  __shared__ int32_t s_n;
  __shared__ int32_t s_wscr[kWarps + 1];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int g = lane >> 2;
  const int c = lane & 3;
  const int H = p.H, I = p.I;
  const uint32_t limit = (p.flags & E4B_FLAG_TEST_TIMEOUT) ? 0u : kPolls;

  // Clear the fp32 accumulator in chunks handed out by a counter, so that
  // waiting on the zeroed count only depends on CTAs that are running.
  const int64_t nacc = p.T * int64_t(H);
  const int nzero = int((nacc + kZeroChunk - 1) / kZeroChunk);
  __shared__ int s_zc;
  while (true) {
    if (threadIdx.x == 0) s_zc = atomicAdd(p.sync + kZeroWork, 1);
    __syncthreads();
    const int zc = s_zc;
    __syncthreads();
    if (zc >= nzero) break;
    const int64_t b0 = int64_t(zc) * kZeroChunk;
    const int64_t b1 = min(nacc, b0 + kZeroChunk);
    for (int64_t i = b0 + threadIdx.x; i < b1; i += kThreads) p.acc[i] = 0.f;
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      atomicAdd(p.sync + kZeroDone, 1);
    }
  }
  block_active_experts(p.offsets, p.E, s_act, &s_n, s_wscr);  // ends with __syncthreads
  const int nact = s_n;
  if (nact == 0) {  // no routed slot at all: the output is zero
    for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < nacc; i += int64_t(gridDim.x) * kThreads)
      p.y[i] = 0;
    return;
  }
  const int MTA = I / 16;                  // gate_up items per expert
  const int MTB = H / 16;                  // down row tiles
  const int NKS = (I + p.ksplit - 1) / p.ksplit;
  const int nA = nact * MTA;
  const int nB = nact * MTB * NKS;
  int32_t* done_A = p.sync + kDoneA;
  int32_t* arrive = p.sync + kDoneA + p.E;
  const uint32_t slot_base = uint32_t(__cvta_generic_to_shared(smem)) + uint32_t(wid * kSlots * kSlotBytesPerLane * 32);

  while (true) {
    int item = 0;
    if (lane == 0) item = atomicAdd(p.sync + kWork, 1);
    item = __shfl_sync(0xffffffffu, item, 0);
    if (item >= nA + nB) break;

    if (item < nA) {
      // ------------------------------------------------ gate_up + SwiGLU
      const int ai = item / MTA;
      const int mt = item % MTA;
      const int e = s_act[ai];
      const int64_t p0 = p.offsets[e], p1 = p.offsets[e + 1];
      const uint8_t* crow[2];
      const uint8_t* srow[2];
      const int64_t sstride = FMT == E4B_FMT_NF4 ? (H / 64) * 4 : (H / 32);
      for (int64_t tg = p0; tg < p1; tg += kGroup) {
        const int nt = int((min(p1 - tg, int64_t(kGroup)) + 7) / 8);
        const uint16_t* brow[kMaxNT];
#pragma unroll
        for (int j = 0; j < kMaxNT; ++j) {
          const int64_t pr = tg + 8 * j + g;
          brow[j] = (j < nt && pr < p1) ? p.x + int64_t(p.perm[pr] / p.top_k) * H : nullptr;
        }
        float accg[kMaxNT][4], accu[kMaxNT][4];
#pragma unroll
        for (int j = 0; j < kMaxNT; ++j)
#pragma unroll
          for (int q = 0; q < 4; ++q) accg[j][q] = accu[j][q] = 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int64_t row = int64_t(e) * 2 * I + mt * 16 + g + 8 * hh;
          crow[hh] = p.gu_codes + row * (H / 2);
          srow[hh] = p.gu_scales + row * sstride;
        }
        run_item_nt<FMT, false>(nt, crow, srow, brow, 0, H, H, slot_base, accg);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int64_t row = int64_t(e) * 2 * I + I + mt * 16 + g + 8 * hh;
          crow[hh] = p.gu_codes + row * (H / 2);
          srow[hh] = p.gu_scales + row * sstride;
        }
        run_item_nt<FMT, false>(nt, crow, srow, brow, 0, H, H, slot_base, accu);
        // h[p][n] = bf16(silu(g) * u); fragment (row g / g+8, tokens 2c, 2c+1)
#pragma unroll
        for (int j = 0; j < kMaxNT; ++j) {
          if (j >= nt) continue;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int64_t pr = tg + 8 * j + 2 * c + (q & 1);
            if (pr < p1) {
              const int n = mt * 16 + g + ((q & 2) ? 8 : 0);
              p.h[pr * I + n] = to_bf16_bits(silu_mul(accg[j][q], accu[j][q]));
            }
          }
        }
      }
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicAdd(done_A + ai, 1);
    } else {
      // ------------------------------------------------ down + combine
      const int b = item - nA;
      const int ai = b / (MTB * NKS);
      const int rem = b % (MTB * NKS);
      const int ks = rem / MTB;
      const int mt = rem % MTB;
      const int e = s_act[ai];
      bool ok = true;
      if (lane == 0) {
        ok = wait_geq(done_A + ai, MTA, limit) && wait_geq(p.sync + kZeroDone, nzero, limit);
        if (!ok) record_status(p.status, E4B_ERR_DEVICE_TIMEOUT);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      __syncwarp();
      if (ok) {
        const int64_t p0 = p.offsets[e], p1 = p.offsets[e + 1];
        const int k0 = ks * p.ksplit;
        const int k1 = min(I, k0 + p.ksplit);
        const uint8_t* crow[2];
        const uint8_t* srow[2];
        const int64_t sstride = FMT == E4B_FMT_NF4 ? (I / 64) * 4 : (I / 32);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int64_t row = int64_t(e) * H + mt * 16 + g + 8 * hh;
          crow[hh] = p.dn_codes + row * (I / 2);
          srow[hh] = p.dn_scales + row * sstride;
        }
        for (int64_t tg = p0; tg < p1; tg += kGroup) {
          const int nt = int((min(p1 - tg, int64_t(kGroup)) + 7) / 8);
          const uint16_t* brow[kMaxNT];
#pragma unroll
          for (int j = 0; j < kMaxNT; ++j) {
            const int64_t pr = tg + 8 * j + g;
            brow[j] = (j < nt && pr < p1) ? p.h + pr * I : nullptr;
          }
          float acc[kMaxNT][4];
#pragma unroll
          for (int j = 0; j < kMaxNT; ++j)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;
          run_item_nt<FMT, true>(nt, crow, srow, brow, k0, k1, I, slot_base, acc);
#pragma unroll
          for (int j = 0; j < kMaxNT; ++j) {
            if (j >= nt) continue;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int64_t pr = tg + 8 * j + 2 * c + (q & 1);
              if (pr < p1) {
                const int slot = p.perm[pr];
                const int n = mt * 16 + g + ((q & 2) ? 8 : 0);
                atomicAdd(p.acc + int64_t(slot / p.top_k) * H + n, p.gates[slot] * acc[j][q]);
              }
            }
          }
        }
      }
      // the last item of this 16-row output slice converts it to bf16
      __threadfence();
      __syncwarp();
      int last = 0;
      if (lane == 0) last = (atomicAdd(arrive + mt, 1) == nact * NKS - 1) ? 1 : 0;
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence();
        for (int64_t i = lane; i < p.T * 4; i += 32) {
          const int64_t t = i >> 2;
          const int part = int(i & 3);
          const float* src = p.acc + t * H + mt * 16 + part * 4;
          float4 v;
          asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
                       : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                       : "l"(src));
          *reinterpret_cast<uint2*>(p.y + t * H + mt * 16 + part * 4) =
              make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
        }
      }
    }
  }
}

}  // namespace

size_t smallm_sync_ints(int E, int H) { return size_t(kDoneA) + E + H / 16; }

cudaError_t launch_smallm_layer(const SmallMLayer& L, cudaStream_t st, int sms) {
  Params p;
  p.E = L.E;
  p.H = L.H;
  p.I = L.I;
  p.top_k = L.top_k;
  p.T = L.T;
  p.gu_codes = L.gu_codes;
  p.gu_scales = static_cast<const uint8_t*>(L.gu_scales);
  p.dn_codes = L.dn_codes;
  p.dn_scales = static_cast<const uint8_t*>(L.dn_scales);
  p.x = L.x;
  p.perm = L.perm;
  p.offsets = L.offsets;
  p.gates = L.gates;
  p.h = L.h;
  p.acc = L.acc;
  p.y = L.y;
  p.sync = L.sync;
  p.status = L.status;
  p.ksplit = 2048;
  p.flags = L.flags;
  const size_t smem = size_t(kWarps) * kSlots * kSlotBytesPerLane * 32;
  static int configured = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured != dev) {
    cudaError_t e1 = cudaFuncSetAttribute(smallm_layer_kernel<E4B_FMT_NF4>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    cudaError_t e2 = cudaFuncSetAttribute(smallm_layer_kernel<E4B_FMT_MXFP4>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e1 != cudaSuccess) return e1;
    if (e2 != cudaSuccess) return e2;
    configured = dev;
  }
  // persistent: every CTA resident at once (2 per SM)
  const int grid = sms * 2;
  if (L.fmt == E4B_FMT_NF4)
    smallm_layer_kernel<E4B_FMT_NF4><<<grid, kThreads, smem, st>>>(p);
  else
    smallm_layer_kernel<E4B_FMT_MXFP4><<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace e4b
