// Small-M MoE layer in one persistent launch: both projections, the SwiGLU,
// the weighted combine and the bf16 output.
//
// "grouped-nf4-gemm" README, intro: the grouped GEMM over all active experts
// on packed weights with table decode, fp32 accumulation and a bf16 epilogue;
// bitsandbytes PR #1984, Design: gated SiLU between the projections and the
// weighted sum over the chosen experts.
//
// With few routed rows per expert every packed byte is read once and the
// layer streams the packed weights from HBM. What limits such a stream is how
// many bytes each SM keeps in flight, so the kernel is a pipeline with one
// persistent CTA per SM:
//  * a producer warp takes work items from one atomic counter and fetches, for
//    each 256-wide K chunk of an item, the packed codes of the item's 256
//    weight rows (two TMA tiles, 128B-swizzled), the chunk of each routed
//    activation row (four-row TMA gathers from x, or TMA tiles of h) and the
//    block scales into a shared-memory stage (four stages of 44 KB);
//  * sixteen consumer warps take 16 weight rows each from a stage, decode the
//    codes through a 256-entry byte table (conflict-free shared loads) into
//    the A fragments of mma.sync m16n8k16 (bf16 in, fp32 accumulate), with the
//    activations of the stage as B, and release the stage;
//  * gate_up items (one expert, 128 gate rows and the matching 128 up rows,
//    all of K) end in the SwiGLU and store bf16 h; down items (one expert,
//    256 output rows, a 2048-wide K slice) wait, bounded, until every gate_up
//    item of their expert has stored h, and store their fp32 partial sums,
//    one per K slice and routed row, with no atomics;
//  * a second, small kernel (launched as a programmatic dependent) sums each
//    token's slots and K slices in a fixed order, weights them by the gates
//    and writes bf16 y, so the result does not depend on the order in which
//    the passes ran.
// Every wait is bounded; a wait that gives up records E4B_ERR_DEVICE_TIMEOUT
// and all warps stop.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"
#include "tmap.h"

namespace e4b {
namespace {

using namespace sm100;

constexpr int kConsumers = 16;                   // consumer warps
constexpr int kThreads = (kConsumers + 1) * 32;  // + the producer warp
constexpr int kChunk = 256;                      // K per stage
constexpr int kRows = 256;                       // weight rows per stage (16 per consumer)
constexpr int kMaxTok = 16;                      // routed rows per pass (two chunks of 8)
// Byte-to-weight-pair table, 256 entries of 128 bytes each, replicated so
// that the lanes' lookups never conflict. NF4: two fp32 levels per entry, one
// copy per half-warp lane (entry v of lane l at v * 128 + 8 * (l % 16)).
// MXFP4: two bf16 values per entry, one copy per lane (v * 128 + 4 * l).
constexpr int kLutBytes = 256 * 128;
// MXFP4 scale table: 2^(s-127) as fp32 for every byte s, 8 copies side by
// side ([s][g], g = the lane's fragment row modulo 8) so the 8 rows a warp
// reads at once sit in 8 different banks.
constexpr int kScaleTabBytes = 256 * 8 * 4;
constexpr uint64_t kStageWaitNs = 100000000;  // 100 ms for a stage; 16x that for h of an expert
constexpr uint64_t kDrainNs = 1000000000;     // the copies still landing at exit
constexpr int kKSplit = 2048;                    // K slice of a down item

// sync words (int32) at the start of the layer's sync area: the work item
// counter, then done_A[E] (finished gate_up passes per active expert, one
// count per consumer warp). Cleared by the routing kernel before every layer
// call.
enum : int { kWork = 0, kDoneA = 1 };

E4B_DEV void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                      uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 4-byte copy; the first src_bytes bytes come from src, the rest are zero.
E4B_DEV void cp4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// Arrives on the mbarrier once every cp.async this thread issued so far has
// landed (the barrier's expected count includes this arrival).
E4B_DEV void cp_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
E4B_DEV void cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

E4B_DEV uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded waits of this kernel: they give up after `ns` nanoseconds (at once
// when ns == 0, the test flag) or when *abort becomes nonzero.
E4B_DEV bool wait_phase(uint64_t* bar, uint32_t parity, uint64_t ns, const volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (ns == 0 || (abort && *abort) || now_ns() - t0 > ns) return false;
    __nanosleep(32);
  }
}

// Records the first wait that gave up: status[2] = site, [3] = CTA, [4] = stage.
E4B_DEV void record_wait_site(int32_t* status, int site, int64_t stage) {
  if (status && atomicCAS(status + 2, 0, site) == 0) {
    status[3] = int32_t(blockIdx.x);
    status[4] = int32_t(stage);
  }
}

E4B_DEV int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *p >= target (same rules as wait_phase).
E4B_DEV bool wait_geq(const int* p, int target, uint64_t ns, const volatile int* abort) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t t0 = now_ns();
  while (ld_acquire(p) < target) {
    if (ns == 0 || *abort || now_ns() - t0 > ns) return false;
    __nanosleep(128);
  }
  return true;
}

E4B_DEV uint32_t lds32(uint32_t addr) {
  uint32_t r;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
  return r;
}
E4B_DEV uint4 lds128(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}

// TMA descriptors of the operands (see launch_smallm_layer).
struct Maps {
  CUtensorMap gu_codes;   // [E*2I rows, H/2 bytes], box 128 x 128, 128B swizzle
  CUtensorMap dn_codes;   // [E*H rows, I/2 bytes], box 128 x 128, 128B swizzle
  CUtensorMap x;          // [T rows, H] bf16, box 32 x 1 (four-row gathers)
  CUtensorMap h;          // [T*top_k rows, I] bf16, box 32 x 4
  // NF4 absmax rows [E*N rows, K/64*4 bytes], box 16 x 128 (when *_scales_tma)
  CUtensorMap gu_scales;
  CUtensorMap dn_scales;
};

struct Params {
  int E, H, I, top_k;
  int gu_scales_tma, dn_scales_tma;  // NF4: fetch the absmax rows by TMA (else cp.async)
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
  float* part;       // [NKS, R, H] fp32: down partial sums per K slice and routed row
  int32_t* sync;     // see the sync words above
  int32_t* status;
  uint32_t flags;
  int layout, act;       // expert variant: gate_up row layout, activation
  float alpha, limit;    // clamped GLU constants
  const float* gu_bias;  // [E, 2I] or null
  const float* dn_bias;  // [E, H] or null
};

// What a stage holds (written by the producer before it releases the stage).
struct StageInfo {
  int kind;    // 0 gate_up, 1 down, -1 no more work
  int ai;      // index of the expert among the active ones
  int e;       // expert
  int mt;      // row block: 128 gate/up outputs (gate_up) or 256 outputs (down)
  int kc;      // first weight of the chunk along K
  int last;    // last chunk of the pass: the consumers finish the pass
  int p0;      // first routed row of the pass
  int ntok;    // routed rows in the pass (1..16)
};

// How a block's scale is applied (template parameter SA).
//  * SA = true, "level" decode: the table holds bf16 operands and the block's
//    scale multiplies the block's fp32 MMA result. MXFP4 always: e2m1 values
//    and 2^(s-127) are exact, so this is the decoded weight exactly. NF4 by
//    default: the operand is bf16(level) and the weight bf16(level) * absmax
//    (one 4-byte table entry per code byte).
//  * SA = false, "product" decode (NF4 with E4B_FLAG_NF4_PRODUCT_DECODE): each
//    weight is bf16(fp32(level * absmax)) before the MMA, the operand the
//    tcgen05 path decodes (an 8-byte entry of two fp32 levels per code byte,
//    twice the shared-memory traffic of the lookups).

// Fills the byte table (whole CTA; ends with a barrier). The earlier weight of
// a byte is the high nibble for NF4 and the low nibble for MXFP4; it goes
// first in the entry. The 16 values of a nibble are staged in shared memory
// first: indexing the constant level arrays with a per-thread value would
// rebuild them in local memory at every call.
template <int FMT, bool SA>
E4B_DEV void build_lut(uint8_t* lut, float* s_val) {
  if (threadIdx.x < 16) {
    const int n = threadIdx.x;
    s_val[n] = FMT == E4B_FMT_NF4 ? nf4_level(n) : ((n & 8) ? -e2m1_magnitude(n & 7) : e2m1_magnitude(n & 7));
  }
  __syncthreads();
  if constexpr (!SA) {
    for (int i = threadIdx.x; i < 256 * 16; i += blockDim.x)
      reinterpret_cast<float2*>(lut)[i] = make_float2(s_val[i >> 8], s_val[(i >> 4) & 15]);
  } else {
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
      const int v = i >> 5, lo = v & 15, hi = v >> 4;
      const float first = FMT == E4B_FMT_NF4 ? s_val[hi] : s_val[lo];
      const float second = FMT == E4B_FMT_NF4 ? s_val[lo] : s_val[hi];
      reinterpret_cast<uint32_t*>(lut)[i] = pack_bf16x2(first, second);
    }
  }
  __syncthreads();
}

// 8 codes (one 32-bit word, weights in byte order) -> 4 bf16x2 weight pairs,
// one byte extract and one conflict-free shared load per pair.
// NF4 pair: both fp32 levels of the entry at `addr` times the absmax (one
// packed f32x2 multiply, round-to-nearest per element), rounded to bf16x2.
E4B_DEV uint32_t scaled_pair(uint32_t addr, uint64_t absmax2) {
  uint32_t r;
  asm("{\n\t.reg .b64 l, p;\n\t.reg .f32 a, b;\n\t"
      "ld.shared.b64 l, [%1];\n\t"
      "mul.rn.f32x2 p, l, %2;\n\t"
      "mov.b64 {a, b}, p;\n\t"
      "cvt.rn.bf16x2.f32 %0, b, a;\n\t}"
      : "=r"(r)
      : "r"(addr), "l"(absmax2));
  return r;
}

template <bool SA>
E4B_DEV void lut_lookup8(uint32_t lut_lane, uint32_t w, uint64_t absmax2, uint32_t* o) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t a = lut_lane + (prmt(w, 0u, 0x4440u | uint32_t(j)) << 7);
    if constexpr (!SA) o[j] = scaled_pair(a, absmax2);
    else o[j] = lds32(a);
  }
}

// Scale of block b of a row in a stage. NF4: the absmax staged at `slot`.
// MXFP4: 2^(s-127) for byte b of `mx` (the row's 8 scale bytes of the
// chunk), looked up in this lane's column `tab_lane` of the scale table
// (byte 0 = 2^-127, byte 255 = NaN).
template <int FMT>
E4B_DEV float stage_scale(uint32_t slot, int b, uint64_t mx, uint32_t tab_lane) {
  if constexpr (FMT == E4B_FMT_NF4) {
    return __uint_as_float(lds32(slot + uint32_t(4 * b)));
  } else {
    const uint32_t w = b < 4 ? uint32_t(mx) : uint32_t(mx >> 32);
    const int sh = 8 * (b & 3);  // the byte's offset in w; the table row is 32 bytes
    const uint32_t off = sh >= 5 ? (w >> (sh - 5)) & 0x1FE0u : (w << 5) & 0x1FE0u;
    return __uint_as_float(lds32(tab_lane + off));
  }
}

// MXFP4: the 3 aligned words of the scale array (total bytes `n`) that hold
// bytes [o, o + 8), read through L1; words past the end read as zero bytes.
E4B_DEV void mx_words(const uint8_t* scales, int64_t n, int64_t o, uint32_t (&w)[3]) {
  const int64_t a = o & ~int64_t(3);
  if (a + 12 <= n) {  // every row but the array's last few: three plain loads
#pragma unroll
    for (int j = 0; j < 3; ++j) w[j] = __ldg(reinterpret_cast<const uint32_t*>(scales + a + 4 * j));
    return;
  }
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int64_t q = a + 4 * j;
    if (q + 4 <= n) {
      w[j] = __ldg(reinterpret_cast<const uint32_t*>(scales + q));
    } else {
      w[j] = 0;
      for (int64_t t = q; t < n && t < q + 4; ++t) w[j] |= uint32_t(__ldg(scales + t)) << (8 * (t - q));
    }
  }
}

// The 8 bytes [o, o + 8) out of mx_words' result.
E4B_DEV uint64_t mx_bytes(const uint32_t (&w)[3], int64_t o) {
  const uint32_t sh = uint32_t(o & 3) * 8;
  const uint64_t lo = (uint64_t(w[1]) << 32) | w[0];
  return sh ? (lo >> sh) | (uint64_t(w[2]) << (64 - sh)) : lo;
}

// Stage layout (1024-byte aligned, as the 128B swizzle needs):
//   codes   256 rows x 128 bytes, 16-byte chunk q of row r at chunk q ^ (r % 8)
//   x       8 slabs of 32 K values: 16 routed rows x 64 bytes each
//   scales  256 rows x 16 bytes
constexpr int kCodeOff = 0;
constexpr int kXOff = kRows * 128;
constexpr int kSOff = kXOff + 8 * kMaxTok * 64;
// Scale bytes per row (NF4: the chunk's 4 absmax words; MXFP4: the 3 aligned
// words that hold its 8 scale bytes), stage size, stage count.
template <int FMT>
struct Geo {
  static constexpr int kSlot = 16;
  static constexpr int kStageBytes = kSOff + kRows * kSlot;
  static constexpr int kStages = 4;
  // MXFP4: + the e8m0 scale table after the barriers and stage info
  static constexpr int kTabBytes = FMT == E4B_FMT_MXFP4 ? kScaleTabBytes : 0;
  static constexpr int kSmemBytes = 1024 + kLutBytes + kStages * kStageBytes + 256 + kTabBytes;
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned");
  static_assert(kSmemBytes + 8192 <= 232448, "shared memory budget");
};

// Work items: gate_up items ai * MTA + mt (mt: a block of 128 gate rows and
// the matching 128 up rows), then down items nA + (ai * NKS + ks) * MTB + mt
// (mt: a block of 256 output rows, ks: a 2048-wide K slice). Each item runs
// one pass per group of up to 16 routed rows of its expert.
struct Work {
  int MTA, MTB, NKS, nA, nB;
};

// Producer warp: fills the stages, chunk by chunk, item after item, then
// posts one stage with kind -1. Returns early, with the abort flag set, if a
// bounded wait gives up.
template <int FMT>
E4B_DEV void produce(const Maps& maps, const Params& p, const Work& W, const int32_t* s_act, uint8_t* stages,
                     uint64_t* full, uint64_t* empty, StageInfo* info, volatile int* s_abort,
                     uint64_t limit) {
  constexpr int kStages = Geo<FMT>::kStages;
  constexpr int kSlot = Geo<FMT>::kSlot;
  const int lane = threadIdx.x & 31;
  const int H = p.H, I = p.I;
  int64_t i = 0;  // stages posted
  bool aborted = false;
  auto give_up = [&]() {
    if (lane == 0) {
      *s_abort = 1;
      record_status(p.status, E4B_ERR_DEVICE_TIMEOUT);
    }
    aborted = true;
  };
  // waits (bounded) until stage s of post i is free and announces `tx` bytes
  // of TMA copies to it; false if it gave up
  auto acquire_stage = [&](int s, uint32_t tx) -> bool {
    int ok = 1;
    if (lane == 0) {
      ok = wait_phase(&empty[s], (uint32_t(i / kStages) & 1u) ^ 1u, limit, s_abort);
      if (!ok) record_wait_site(p.status, 1, i);
      if (ok && tx) mbar_expect_tx(&full[s], tx);
    }
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
  };

  while (!aborted) {
    int item = 0;
    if (lane == 0) item = atomicAdd(p.sync + kWork, 1);
    item = __shfl_sync(0xffffffffu, item, 0);
    if (item >= W.nA + W.nB) break;
    const bool down = item >= W.nA;
    int ai, mt, ks = 0;
    if (!down) {
      ai = item / W.MTA;
      mt = item % W.MTA;
    } else {
      const int b = item - W.nA;
      ai = b / (W.MTB * W.NKS);
      const int r = b % (W.MTB * W.NKS);
      ks = r / W.MTB;
      mt = r % W.MTB;
    }
    const int e = s_act[ai];
    const int64_t p0 = p.offsets[e], p1 = p.offsets[e + 1];
    const int ngroups = int((p1 - p0 + kMaxTok - 1) / kMaxTok);
    if (down) {
      // h of this expert complete (every gate_up pass of it, one count per
      // consumer warp)
      int ok = 1;
      if (lane == 0) {
        ok = wait_geq(p.sync + kDoneA + ai, W.MTA * ngroups * kConsumers, 16 * limit, s_abort);
        if (!ok) record_wait_site(p.status, 2, i);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        give_up();
        break;
      }
      ld_acquire(p.sync + kDoneA + ai);  // every lane reads h after the acquire
      // h was written through the generic proxy; the TMA reads it through the async one
      asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    // interleaved gate_up: the item's 128 outputs own the 256 consecutive
    // rows 256 mt .. (gate 2n, up 2n + 1)
    const bool il = !down && p.layout == E4B_GATE_UP_INTERLEAVED;
    const int K = down ? I : H;
    const int k0 = down ? ks * kKSplit : 0;
    const int k1 = down ? min(I, k0 + kKSplit) : H;
    const uint8_t* scales = down ? p.dn_scales : p.gu_scales;
    const int64_t sstride = FMT == E4B_FMT_NF4 ? (K / 64) * 4 : K / 32;  // scale bytes per row
    // global weight row of stage row r, or -1 past the matrix
    auto wrow = [&](int r) -> int64_t {
      if (down) {
        const int n = mt * 256 + r;
        return n < H ? int64_t(e) * H + n : -1;
      }
      if (il) {
        const int q = mt * 256 + r;
        return q < 2 * I ? int64_t(e) * 2 * I + q : -1;
      }
      const int n = mt * 128 + (r & 127);
      return n < I ? int64_t(e) * 2 * I + int64_t(r >> 7) * I + n : -1;
    };

    const CUtensorMap* cmap = down ? &maps.dn_codes : &maps.gu_codes;
    const bool scales_tma = down ? p.dn_scales_tma : p.gu_scales_tma;
    const CUtensorMap* smap = down ? &maps.dn_scales : &maps.gu_scales;
    // first global weight row of the stage's two 128-row halves
    const int64_t row0 = down ? int64_t(e) * H + int64_t(mt) * 256
                         : int64_t(e) * 2 * I + int64_t(mt) * (il ? 256 : 128);
    const int64_t row1 = (down || il) ? row0 + 128 : row0 + I;
    const uint32_t tx_fixed = uint32_t(kRows * 128 + (FMT == E4B_FMT_NF4 && scales_tma ? kRows * 16 : 0));

    for (int64_t tg = p0; tg < p1 && !aborted; tg += kMaxTok) {
      const int ntok = int(min(p1 - tg, int64_t(kMaxTok)));
      // activations arrive in groups of 4 routed rows: only the groups that
      // hold routed rows of the pass are fetched (the consumers read rows < ntok)
      const int ngrp = (ntok + 3) / 4;
      const uint32_t tx = tx_fixed + uint32_t(8 * ngrp * 4 * 64);
      // gate_up: the x row of each of the pass's routed rows (rows past the
      // pass repeat its first row; their products are never stored)
      int32_t xrow = 0;
      if (!down) xrow = p.perm[tg + (lane < ntok ? lane : 0)] / p.top_k;
      int32_t gr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) gr[u] = __shfl_sync(0xffffffffu, xrow, 4 * (lane & 3) + u);
      for (int kc = k0; kc < k1; kc += kChunk, ++i) {
        const int s = int(i % kStages);
        if (!acquire_stage(s, tx)) {
          give_up();
          break;
        }
        uint8_t* st = stages + s * Geo<FMT>::kStageBytes;
        if (lane == 0) {
          tma_load_2d(st + kCodeOff, cmap, &full[s], kc / 2, int32_t(row0));
          tma_load_2d(st + kCodeOff + 128 * 128, cmap, &full[s], kc / 2, int32_t(row1));
          if (FMT == E4B_FMT_NF4 && scales_tma) {
            tma_load_2d(st + kSOff, smap, &full[s], (kc / 64) * 4, int32_t(row0));
            tma_load_2d(st + kSOff + 128 * 16, smap, &full[s], (kc / 64) * 4, int32_t(row1));
          }
        }
        {
          // lane l fetches routed rows 4(l%4)..+3 of 32-wide slab l/4: a
          // 4-row tile of h (rows tg.. are contiguous) or a four-row gather of x
          const int slab = lane >> 2, grp = lane & 3;
          uint8_t* dst = st + kXOff + slab * kMaxTok * 64 + grp * 4 * 64;
          if (grp < ngrp) {
            if (down) tma_load_2d(dst, &maps.h, &full[s], kc + 32 * slab, int32_t(tg) + 4 * grp);
            else tma_gather4_2d(dst, &maps.x, &full[s], kc + 32 * slab, gr[0], gr[1], gr[2], gr[3]);
          }
        }
        if (FMT == E4B_FMT_NF4 && !scales_tma) {
          // absmax by cp.async: the chunk's 4 words of each row
          const uint32_t sbase = smem_u32(st + kSOff);
          for (int m = 0; m < kRows / 8; ++m) {
            const int q = lane + 32 * m, r = q >> 2, w = q & 3;
            const int64_t grow = wrow(r);
            const uint32_t dst = sbase + uint32_t(r * kSlot + 4 * w);
            const bool v = grow >= 0 && kc + 64 * w < k1;
            cp4(dst, v ? (const void*)(scales + grow * sstride + (kc / 64 + w) * 4) : (const void*)scales,
                v ? 4u : 0u);
          }
        }
        if (lane == 0) {
          StageInfo& f = info[s];
          f.kind = down ? 1 : 0;
          f.ai = ai;
          f.e = e;
          f.mt = mt;
          f.kc = kc;
          f.last = kc + kChunk >= k1;
          f.p0 = int(tg);
          f.ntok = ntok;
        }
        cp_arrive_noinc(&full[s]);
        if (lane == 0) mbar_arrive(&full[s]);
      }
    }
  }
  // the end-of-work stage
  if (!aborted) {
    const int s = int(i % kStages);
    if (acquire_stage(s, 0u)) {
      if (lane == 0) info[s].kind = -1;
      cp_arrive_noinc(&full[s]);
      if (lane == 0) mbar_arrive(&full[s]);
      ++i;  // a post like any other: the drain below must not alias its slot
    } else {
      give_up();
    }
  }
  cp_wait_all();  // no cp.async may land after the CTA has exited
  // ... nor a TMA copy: wait (bounded) for the stages posted last
  if (lane == 0)
    for (int64_t q = i > kStages ? i - kStages : 0; q < i; ++q)
      if (!wait_phase(&full[q % kStages], uint32_t(q / kStages) & 1u, kDrainNs, nullptr))
        record_wait_site(p.status, 5, q);
}

// One stage for one consumer warp: one 16-row tile (MMA rows g from stage
// row rA + g, rows g + 8 from stage row rB + g) times NT chunks of 8 routed
// rows, accumulated into acc.
// K order: the stage's 256 K values are 8 chunks of 32 (16 code bytes); in
// every chunk, lane c of a quad takes the 8 consecutive weights 8c..8c+7
// (code word c), so every mma k16 step stays inside one 32-wide chunk and
// hence inside one scale block of each row.
template <int FMT, int NT, bool SA>
E4B_DEV void consume_stage(uint32_t st, const StageInfo& f, int kend, int rA, int rB, uint64_t mxA,
                           uint64_t mxB, uint32_t lut_lane, uint32_t tab_lane, float (&acc)[2][4]) {
  static_assert(SA || FMT == E4B_FMT_NF4, "MXFP4 scales always apply after the block's MMA");
  constexpr int kSlot = Geo<FMT>::kSlot;
  constexpr int BLK = FMT == E4B_FMT_NF4 ? 64 : 32;  // weights per scale block
  constexpr int NB = kChunk / BLK;                     // blocks per stage
  constexpr int CPB = BLK / 32;                        // 32-wide chunks per block
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int c = lane & 3;
  const uint32_t cA = st + uint32_t(kCodeOff + (rA + g) * 128 + 4 * c);  // both rows are g modulo 8
  const uint32_t cB = st + uint32_t(kCodeOff + (rB + g) * 128 + 4 * c);
  uint32_t x_lane[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) x_lane[j] = uint32_t(min(8 * j + g, f.ntok - 1) * 64 + 16 * c);
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    // blocks past K: codes and activations are zero, scale 0. The scale slot
    // of every block exists, so it is read either way and then selected.
    const bool live = f.kc + BLK * b < kend;
    float sA = stage_scale<FMT>(st + uint32_t(kSOff + (rA + g) * kSlot), b, mxA, tab_lane);
    float sB = stage_scale<FMT>(st + uint32_t(kSOff + (rB + g) * kSlot), b, mxB, tab_lane);
    sA = live ? sA : 0.f;
    sB = live ? sB : 0.f;
    const uint64_t sA2 = (uint64_t(__float_as_uint(sA)) << 32) | __float_as_uint(sA);
    const uint64_t sB2 = (uint64_t(__float_as_uint(sB)) << 32) | __float_as_uint(sB);
    float P[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) P[j][q] = 0.f;
#pragma unroll
    for (int it = 0; it < CPB; ++it) {
      const int ch = CPB * b + it;  // 32-wide chunk of the stage
      // activations: 8 values of this lane's token in each chunk of 8 routed
      // rows. Lanes past the pass's routed rows read the last routed row
      // instead (no branch; the same addresses as other lanes): those values
      // reach only MMA columns that no epilogue stores.
      uint4 xv[NT];
#pragma unroll
      for (int j = 0; j < NT; ++j) xv[j] = lds128(st + uint32_t(kXOff + ch * kMaxTok * 64) + x_lane[j]);
      const uint32_t sw = uint32_t((ch ^ g) << 4);  // the 128B swizzle of chunk ch in row g (mod 8)
      uint32_t dA[4], dB[4];
      lut_lookup8<SA>(lut_lane, lds32(cA + sw), sA2, dA);
      lut_lookup8<SA>(lut_lane, lds32(cB + sw), sB2, dB);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        float(&D)[4] = SA ? P[j] : acc[j];
        // fragment registers {row g | row g+8} x {pair 0,2 | pair 1,3}
        mma16816(D, dA[0], dB[0], dA[1], dB[1], xv[j].x, xv[j].y);
        mma16816(D, dA[2], dB[2], dA[3], dB[3], xv[j].z, xv[j].w);
      }
    }
    if constexpr (SA) {
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        acc[j][0] = fmaf(sA, P[j][0], acc[j][0]);
        acc[j][1] = fmaf(sA, P[j][1], acc[j][1]);
        acc[j][2] = fmaf(sB, P[j][2], acc[j][2]);
        acc[j][3] = fmaf(sB, P[j][3], acc[j][3]);
      }
    }
  }
}

// Consumer warps: take the stages in order until the kind -1 stage, finishing
// each pass with its epilogue. Warp w takes, per stage, gate rows 8w..8w+7
// (MMA rows g) and the matching up rows 128+8w.. (MMA rows g+8) for gate_up
// with the two halves, so gate and up of an output sit in the same lane;
// stage rows 16w..16w+15 for down and for interleaved gate_up, where the gate
// and up rows of an output are neighbours, four lanes apart in the fragment.
template <int FMT, bool SA>
E4B_DEV void consume(const Params& p, uint8_t* stages, uint64_t* full, uint64_t* empty,
                     const StageInfo* info, volatile int* s_abort, uint32_t lut_lane, uint32_t tab_lane,
                     uint64_t limit) {
  constexpr int kStages = Geo<FMT>::kStages;
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;  // 0 .. kConsumers-1
  const int g = lane >> 2;
  const int c = lane & 3;
  const int H = p.H, I = p.I;
  int32_t* done_A = p.sync + kDoneA;
  float acc[2][4];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;
  uint32_t pfA[3] = {0, 0, 0}, pfB[3] = {0, 0, 0};  // MXFP4: prefetched scale words
  int64_t pf_o = -1;                                // ... of the chunk at row-A offset pf_o

  for (int64_t i = 0;; ++i) {
    const int s = int(i % kStages);
    if (!wait_phase(&full[s], uint32_t(i / kStages) & 1u, limit, s_abort)) {
      if (!*s_abort) {
        record_wait_site(p.status, 4, i);
        *s_abort = 1;
        record_status(p.status, E4B_ERR_DEVICE_TIMEOUT);
      }
      break;
    }
    const StageInfo f = info[s];
    if (f.kind < 0) break;
    const bool down = f.kind == 1;
    const int kend = down ? min(I, (f.kc / kKSplit + 1) * kKSplit) : H;
    const uint32_t st = smem_u32(stages + s * Geo<FMT>::kStageBytes);
    const bool il = !down && p.layout == E4B_GATE_UP_INTERLEAVED;
    const int rA = (down || il) ? 16 * w : 8 * w;
    const int rB = (down || il) ? 16 * w + 8 : 128 + 8 * w;
    // MXFP4: each lane reads its two rows' scale bytes of the chunk itself
    // (L1: consecutive chunks of a row share lines), the next chunk's
    // prefetched while the pass continues
    uint64_t mxA = 0, mxB = 0;
    if constexpr (FMT == E4B_FMT_MXFP4) {
      const int64_t k32 = (down ? I : H) / 32;
      const uint8_t* scales = down ? p.dn_scales : p.gu_scales;
      const int64_t n = int64_t(p.E) * (down ? H : 2 * I) * k32;
      auto grow = [&](int r) -> int64_t {
        if (down) return int64_t(f.e) * H + int64_t(f.mt) * 256 + r;
        if (il) return int64_t(f.e) * 2 * I + int64_t(f.mt) * 256 + r;
        return int64_t(f.e) * 2 * I + int64_t(r >> 7) * I + int64_t(f.mt) * 128 + (r & 127);
      };
      const int64_t oA = grow(rA + g) * k32 + f.kc / 32, oB = grow(rB + g) * k32 + f.kc / 32;
      uint32_t wA[3], wB[3];
      if (oA == pf_o) {
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          wA[j] = pfA[j];
          wB[j] = pfB[j];
        }
      } else {
        mx_words(scales, n, oA, wA);
        mx_words(scales, n, oB, wB);
      }
      mxA = mx_bytes(wA, oA);
      mxB = mx_bytes(wB, oB);
      pf_o = -1;
      if (!f.last) {
        pf_o = oA + 8;
        mx_words(scales, n, oA + 8, pfA);
        mx_words(scales, n, oB + 8, pfB);
      }
    }
    if (f.ntok > 8) consume_stage<FMT, 2, SA>(st, f, kend, rA, rB, mxA, mxB, lut_lane, tab_lane, acc);
    else consume_stage<FMT, 1, SA>(st, f, kend, rA, rB, mxA, mxB, lut_lane, tab_lane, acc);
    mbar_arrive(&empty[s]);  // this lane's reads of the stage are done
    if (!f.last) continue;

    // ---------------------------------------------------- end of a pass
    const int nt = f.ntok > 8 ? 2 : 1;
    if (!down) {
      // h[p][n] = bf16(act(gate + bias, up + bias)), tokens 2c, 2c+1. Halves:
      // gate in fragment rows g (d0, d1), up in rows g + 8 (d2, d3).
      // Interleaved: rows g and g + 8 are stage rows 16w + g and 16w + 8 + g;
      // an even g holds the gate of output 8w + g/2 in d0, d1 and gets its up
      // from lane g + 1, an odd g holds the up of output 8w + 4 + (g-1)/2 in
      // d2, d3 and gets its gate from lane g - 1.
      const bool odd = g & 1;
      const int n = f.mt * 128 + 8 * w + (!il ? g : odd ? 4 + (g >> 1) : (g >> 1));
      const float* gb = p.gu_bias ? p.gu_bias + int64_t(f.e) * 2 * I : nullptr;
      const float bg = gb && n < I ? gb[gate_up_row(p.layout, I, 0, n)] : 0.f;
      const float bu = gb && n < I ? gb[gate_up_row(p.layout, I, 1, n)] : 0.f;
      for (int j = 0; j < nt; ++j) {
        float gv[2] = {acc[j][0], acc[j][1]}, uv[2] = {acc[j][2], acc[j][3]};
        if (il) {
          const float r0 = __shfl_xor_sync(0xffffffffu, odd ? acc[j][0] : acc[j][2], 4);
          const float r1 = __shfl_xor_sync(0xffffffffu, odd ? acc[j][1] : acc[j][3], 4);
          if (odd) {
            gv[0] = r0;
            gv[1] = r1;
          } else {
            uv[0] = r0;
            uv[1] = r1;
          }
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int tok = 8 * j + 2 * c + q;
          if (tok < f.ntok && n < I)
            p.h[int64_t(f.p0 + tok) * I + n] =
                to_bf16_bits(glu_act(p.act, gv[q] + bg, uv[q] + bu, p.alpha, p.limit));
        }
      }
      __threadfence();
      // h is read next by TMA (the async proxy) in other CTAs
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __syncwarp();
      if (lane == 0) atomicAdd(done_A + f.ai, 1);
    } else {
      // the partial sum of this K slice for every routed row of the pass; the
      // down bias joins the first K slice only
      const int ks = f.kc / kKSplit;
      const int64_t R = p.T * p.top_k;
      const float* db = p.dn_bias && ks == 0 ? p.dn_bias + int64_t(f.e) * H : nullptr;
      float* part = p.part + int64_t(ks) * R * H;
      for (int j = 0; j < nt; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int tok = 8 * j + 2 * c + (q & 1);
          const int n = f.mt * 256 + 16 * w + g + ((q & 2) ? 8 : 0);
          if (tok >= f.ntok || n >= H) continue;
          part[int64_t(f.p0 + tok) * H + n] = acc[j][q] + (db ? db[n] : 0.f);
        }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;
  }
}

template <int FMT, bool SA>
__global__ void __launch_bounds__(kThreads, 1)
smallm_layer_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ int32_t s_act[1024];
  __shared__ int32_t s_n;
  __shared__ int32_t s_wscr[kThreads / 32 + 1];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int H = p.H, I = p.I;
  const uint64_t limit = (p.flags & E4B_FLAG_TEST_TIMEOUT) ? 0u : kStageWaitNs;
  uint8_t* stages = smem + kLutBytes;
  constexpr int kStages = Geo<FMT>::kStages;
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + kStages * Geo<FMT>::kStageBytes);
  uint64_t* empty = full + kStages;
  StageInfo* info = reinterpret_cast<StageInfo*>(empty + kStages);
  volatile int* s_abort = reinterpret_cast<volatile int*>(info + kStages);
  static_assert(2 * kStages * sizeof(uint64_t) + kStages * sizeof(StageInfo) + sizeof(int) <= 256,
                "barriers, stage info and the abort flag fit their 256 bytes");
  float* scale_tab = reinterpret_cast<float*>(stages + kStages * Geo<FMT>::kStageBytes + 256);

  // The byte table (and, for MXFP4, the scale table), made visible by the
  // barrier that ends build_lut.
  __shared__ float s_val[16];
  if constexpr (FMT == E4B_FMT_MXFP4)
    for (int i = threadIdx.x; i < kScaleTabBytes / 4; i += blockDim.x)
      scale_tab[i] = e8m0_to_f32(uint32_t(i >> 3));
  build_lut<FMT, SA>(smem, s_val);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 33);                  // 32 producer lanes' copies + the stage info
      mbar_init(&empty[s], kConsumers * 32);    // every consumer lane
    }
    *s_abort = 0;
    mbar_init_fence();
  }
  // launched as a programmatic dependent of the routing pass: the table and
  // barriers above are set up while it runs; everything below reads its
  // output or the counters it clears
  grid_dependency_wait();

  block_active_experts(p.offsets, p.E, s_act, &s_n, s_wscr);  // ends with __syncthreads
  const int nact = s_n;
  if (nact == 0) {  // no routed slot: nothing to compute (the combine writes zeros)
    grid_launch_dependents();
    return;
  }
  Work W;
  W.MTA = (I + 127) / 128;
  W.MTB = (H + 255) / 256;
  W.NKS = (I + kKSplit - 1) / kKSplit;
  W.nA = nact * W.MTA;
  W.nB = nact * W.MTB * W.NKS;
  if (wid == kConsumers) {
    produce<FMT>(maps, p, W, s_act, stages, full, empty, info, s_abort, limit);
    // no more work items for this CTA: the combine kernel may start launching
    // (it waits for this whole grid before reading the partial sums)
    grid_launch_dependents();
  } else {
    const uint32_t lut_lane = smem_u32(smem) + uint32_t(!SA ? 8 * (lane & 15) : 4 * lane);
    // MXFP4: this lane's column of the scale table
    const uint32_t tab_lane = smem_u32(scale_tab) + uint32_t(4 * ((lane >> 2) & 7));
    consume<FMT, SA>(p, stages, full, empty, info, s_abort, lut_lane, tab_lane, limit);
  }
}

}  // namespace

size_t smallm_sync_ints(int E, int H) {
  (void)H;
  return size_t(kDoneA) + E;
}

// y[t, n] = bf16( sum_j gates[s] * sum_ks part[ks][inv[s]][n] ), s = t*k + j,
// in that order (fp32); slots whose inv is -1 add nothing. One thread per 4
// consecutive outputs of a token.
__global__ void __launch_bounds__(256) smallm_combine_kernel(const float* __restrict__ part,
                                                              const int32_t* __restrict__ inv,
                                                              const float* __restrict__ gates, int64_t T,
                                                              int32_t k, int64_t H4, int32_t nks, int64_t R,
                                                              uint16_t* __restrict__ y) {
  grid_dependency_wait();  // the layer kernel's partial sums
  const int64_t total = T * H4;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = i / H4;
    const int64_t c = i - t * H4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int64_t s = t * k + j;
      const int32_t p = __ldg(inv + s);
      if (p < 0) continue;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int ks = 0; ks < nks; ++ks) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(part + (int64_t(ks) * R + p) * (H4 * 4)) + c);
        o.x += v.x;
        o.y += v.y;
        o.z += v.z;
        o.w += v.w;
      }
      const float gw = __ldg(gates + s);
      acc.x += gw * o.x;
      acc.y += gw * o.y;
      acc.z += gw * o.z;
      acc.w += gw * o.w;
    }
    reinterpret_cast<uint2*>(y)[i] = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
  }
}

int smallm_k_slices(int I) { return (I + kKSplit - 1) / kKSplit; }

cudaError_t launch_smallm_combine(const SmallMLayer& L, cudaStream_t st, int sms) {
  const int64_t total = L.T * (L.H / 4);
  int64_t grid = (total + 255) / 256;
  if (grid > int64_t(sms) * 8) grid = int64_t(sms) * 8;
  if (grid < 1) grid = 1;
  return launch_dependent(smallm_combine_kernel, dim3(unsigned(grid)), dim3(256), 0, st,
                          static_cast<const float*>(L.part), static_cast<const int32_t*>(L.inv), L.gates, L.T,
                          int32_t(L.top_k), int64_t(L.H / 4), int32_t(smallm_k_slices(L.I)),
                          int64_t(L.T * L.top_k), L.y);
}

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
  p.part = L.part;
  p.sync = L.sync;
  p.status = L.status;
  p.flags = L.flags;
  p.layout = L.layout;
  p.act = L.act;
  p.alpha = L.alpha;
  p.limit = L.limit;
  p.gu_bias = L.gu_bias;
  p.dn_bias = L.dn_bias;
  const int64_t E = L.E, H = L.H, I = L.I;
  Maps m;
  bool ok = encode_2d(&m.gu_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.gu_codes, uint64_t(H / 2), uint64_t(E * 2 * I),
                      uint64_t(H / 2), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_2d(&m.dn_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.dn_codes, uint64_t(I / 2), uint64_t(E * H),
                      uint64_t(I / 2), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_2d(&m.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.x, uint64_t(H), uint64_t(L.T), uint64_t(H) * 2, 32, 1,
                      CU_TENSOR_MAP_SWIZZLE_NONE) &&
            encode_2d(&m.h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.h, uint64_t(I), uint64_t(L.T * L.top_k),
                      uint64_t(I) * 2, 32, 4, CU_TENSOR_MAP_SWIZZLE_NONE);
  // Scales by TMA where the layout allows: NF4 absmax rows when their byte
  // stride is a multiple of 16; MXFP4 scale bytes when their total is.
  m.gu_scales = m.gu_codes;
  m.dn_scales = m.dn_codes;
  if (L.fmt == E4B_FMT_NF4) {
    p.gu_scales_tma = H % 256 == 0;
    p.dn_scales_tma = I % 256 == 0;
    if (ok && p.gu_scales_tma)
      ok = encode_2d(&m.gu_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.gu_scales, uint64_t(H / 64 * 4),
                     uint64_t(E * 2 * I), uint64_t(H / 64 * 4), 16, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && p.dn_scales_tma)
      ok = encode_2d(&m.dn_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.dn_scales, uint64_t(I / 64 * 4),
                     uint64_t(E * H), uint64_t(I / 64 * 4), 16, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    // MXFP4 scale bytes: 8 per row and chunk at any alignment, fetched by
    // cp.async (one bulk copy per row measured slower)
    p.gu_scales_tma = 0;
    p.dn_scales_tma = 0;
  }
  if (!ok) return cudaErrorInvalidValue;
  static int configured = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured != dev) {
    cudaError_t e[3] = {
        cudaFuncSetAttribute(smallm_layer_kernel<E4B_FMT_NF4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Geo<E4B_FMT_NF4>::kSmemBytes),
        cudaFuncSetAttribute(smallm_layer_kernel<E4B_FMT_NF4, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Geo<E4B_FMT_NF4>::kSmemBytes),
        cudaFuncSetAttribute(smallm_layer_kernel<E4B_FMT_MXFP4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Geo<E4B_FMT_MXFP4>::kSmemBytes)};
    for (cudaError_t x : e)
      if (x != cudaSuccess) return x;
    configured = dev;
  }
  // persistent: one CTA per SM, all resident at once
  if (L.fmt == E4B_FMT_NF4) {
    if (L.flags & E4B_FLAG_NF4_PRODUCT_DECODE)
      return launch_dependent(smallm_layer_kernel<E4B_FMT_NF4, false>, dim3(sms), dim3(kThreads),
                              Geo<E4B_FMT_NF4>::kSmemBytes, st, m, p);
    return launch_dependent(smallm_layer_kernel<E4B_FMT_NF4, true>, dim3(sms), dim3(kThreads),
                            Geo<E4B_FMT_NF4>::kSmemBytes, st, m, p);
  }
  return launch_dependent(smallm_layer_kernel<E4B_FMT_MXFP4, true>, dim3(sms), dim3(kThreads),
                          Geo<E4B_FMT_MXFP4>::kSmemBytes, st, m, p);
}

}  // namespace e4b
