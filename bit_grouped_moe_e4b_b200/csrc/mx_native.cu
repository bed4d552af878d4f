// MXFP4 on Blackwell's block-scaled tensor cores: the large-M layer path that
// multiplies the e2m1 codes and their e8m0 scales directly.
//
// "grouped-nf4-gemm" README, intro: MXFP4 as OCP e2m1 + e8m0; one launch over
// all active experts per projection, fp32 accumulation, bf16 epilogue.
// tcgen05.mma kind::mxf8f6f4 takes A = e2m1 weights and B = e4m3 activations,
// each with one e8m0 scale per 32 elements of K, so the weights reach the
// tensor cores without any decode. Three kernels:
//
//  * mx_prepare_kernel (once per weight stack): the packed codes are copied to
//    rows padded to a multiple of 128 in K (the tensor map of 4-bit elements
//    that TMA unpacks into the MMA's shared-memory format needs that), gate and
//    up rows de-interleaved into two matrices of 128-row blocks, and the scale
//    bytes rearranged into the MMA's scale-factor chunks: 512 bytes per 128
//    rows x 128 K, row r = 32 m1 + m0 and k-block b at byte 16 m0 + 4 m1 + b.
//
//  * mx_act_quant_kernel (per layer call, twice): bf16 activation rows -> e4m3
//    elements with one e8m0 scale per 32, into rows padded per expert to a
//    multiple of 112, one scale-factor chunk per 112 rows (x rows gathered
//    through the routing permutation; h rows already in that order). Two readings (flags):
//      - one term: the OCP MXFP8 rule, shared exponent floor(log2 amax) - 8,
//        e4m3 round to nearest even, saturating at 448;
//      - two terms (default): x = x1 + x2 with x1 = e4m3(x / 2^X1),
//        X1 = floor(log2 amax) - 7 (no saturation), and x2 the same rule on the
//        residual x - x1. A bf16 value has 8 significant bits and each e4m3
//        term carries 4, so the sum reproduces every bf16 input exactly except
//        for elements below ~2^-13 of their block's largest magnitude, and the
//        layer keeps the bf16-activation result at twice the MMA count.
//
//  * mx_gemm_kernel: one persistent CTA per SM, warp-specialised:
//      warp 0      TMA producer: per 128-wide K chunk, the A tile(s) (128
//                  weight rows, e2m1 unpacked by TMA to one byte per element,
//                  128B-swizzled), the B tile(s) (112 routed rows of each term),
//                  and the scale-factor chunks by bulk copies;
//      warp 1      TMEM owner and single-thread MMA issuer: the chunk's scale
//                  factors go to TMEM with tcgen05.cp (one TMEM slot per ring
//                  stage), then 4 MMAs of K = 32 per matrix and term;
//      warps 2-5   epilogue from TMEM (two accumulator buffers, so it
//                  overlaps the next tile's MMAs): the gated activation into bf16 h
//                  (gate_up), or the gate-weighted fp32 row of every routed row
//                  (down), summed per token afterwards in a fixed order.
//    Every wait is bounded; a wait that gives up records E4B_ERR_DEVICE_TIMEOUT,
//    stops all roles, drains what was issued, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace e4b {
namespace {

using namespace sm100;

constexpr int MBM = 128;  // weight rows per tile (MMA M)
// routed rows per tile (MMA N) and the unit of the per-expert row padding:
// 112 leaves TMEM room for two accumulator buffers of gate and up (448
// columns) plus the scale-factor slots, so every epilogue overlaps the next
// tile's MMAs
constexpr int MBN = kMxRowBlock;
constexpr int MBK = 128;  // K per stage
constexpr int kMxMaxE = 256;
constexpr int kMxThreads = 192;
constexpr uint32_t kTile = MBM * MBK;         // 16 KB: a 128 x 128 A tile at one byte per element
constexpr uint32_t kBTile = MBN * MBK;        // 14 KB: a B tile (e4m3)
constexpr uint32_t kATx = MBM * MBK / 2;      // TMA counts the packed 4-bit bytes of an A tile
constexpr uint32_t kChunk = 512;              // scale-factor chunk: up to 128 rows x 4 k-blocks
static_assert(MBN % 16 == 0 && MBN <= 128 && kBTile % 1024 == 0, "routed-row tile");

// s_poff[e] = sum over e' < e of the expert's rows rounded up to MBN, for
// e = 0..E (one warp).
E4B_DEV void warp_padded_offsets(const int64_t* offsets, int E, int32_t* s_poff, int lane) {
  int run = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    int v = 0;
    if (e < E) v = int((offsets[e + 1] - offsets[e] + kMxRowBlock - 1) / kMxRowBlock) * kMxRowBlock;
    int incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += o;
    }
    if (e < E) s_poff[e] = run + incl - v;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) s_poff[E] = run;
}

// The expert whose padded rows hold padded row pp: the largest e < E with
// s_poff[e] <= pp (experts without rows share their successor's offset).
E4B_DEV int expert_of_padded_row(const int32_t* s_poff, int E, int64_t pp) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_poff[mid] <= pp) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------- weight preparation
__global__ void mx_prepare_kernel(const uint8_t* __restrict__ blocks, const uint8_t* __restrict__ scales,
                                  int E, int64_t Nm, int nmat, int64_t K, int layout, int64_t Np, int64_t Kp,
                                  uint8_t* __restrict__ out_codes, uint8_t* __restrict__ out_sf) {
  const int64_t nbk = Kp / 32;      // 32-weight blocks per padded row
  const int64_t nb_src = K / 32;
  const int64_t total = int64_t(E) * nmat * Np * nbk;
  const int64_t src_rows = int64_t(nmat) * Nm;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t b = i % nbk;
    const int64_t rest = i / nbk;
    const int64_t np = rest % Np;
    const int64_t em = rest / Np;  // e * nmat + m
    const int m = int(em % nmat);
    const int64_t e = em / nmat;
    const bool valid = np < Nm && b < nb_src;
    uint4 v = make_uint4(0, 0, 0, 0);
    uint8_t sb = 0;
    if (valid) {
      const int64_t row = nmat == 2 ? gate_up_row(layout, Nm, m, np) : np;
      const int64_t src = (e * src_rows + row) * nb_src + b;
      v = __ldg(reinterpret_cast<const uint4*>(blocks) + src);
      sb = __ldg(scales + src);
    }
    reinterpret_cast<uint4*>(out_codes)[(em * Np + np) * nbk + b] = v;
    const int64_t chunk = (em * (Np / 128) + np / 128) * (Kp / 128) + b / 4;
    const int r = int(np % 128);
    out_sf[chunk * kChunk + (r % 32) * 16 + (r / 32) * 4 + (b % 4)] = sb;
  }
}

// ------------------------------------------------- activation quantisation
E4B_DEV int floor_log2_pos(float a) {
  const uint32_t bits = __float_as_uint(a);
  const int ex = int(bits >> 23);
  return ex > 0 ? ex - 127 : (31 - __clz(int(bits))) - 149;
}

// 2^n as fp32 for n in [-127, 127] (2^-127 is a subnormal).
E4B_DEV float exp2i(int n) { return n >= -126 ? __uint_as_float(uint32_t(n + 127) << 23) : __uint_as_float(0x00400000u); }

// One 32-value block held by 4 consecutive lanes (8 values each, lane & 3 =
// position in the block): NT e4m3 terms with their e8m0 bytes. shift: 8 for
// the OCP rule, 7 for the two-term split. Every lane of the warp must call.
template <int NT>
E4B_DEV void quant_block8(float (&v)[8], int shift, uint2 (&out)[NT], uint32_t (&sb)[NT]) {
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    int X = -127;
    uint32_t byte = 0;
    if (a > 0.f) {
      X = floor_log2_pos(a) - shift;
      X = X < -127 ? -127 : (X > 127 ? 127 : X);
      byte = uint32_t(X + 127);
    }
    const float inv = exp2i(-X);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = a > 0.f ? e4m3x2_from_f32(v[2 * i] * inv, v[2 * i + 1] * inv) : 0u;
    out[t] = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
    sb[t] = byte;
    if (t + 1 < NT) {
      // the residual for the next term (exact: both terms are few-bit values)
      const float sc = exp2i(X);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 d = f32x2_from_e4m3x2(w[i]);
        v[2 * i] -= d.x * sc;
        v[2 * i + 1] -= d.y * sc;
      }
    }
  }
}

enum : int { kActGather = 0, kActPadded = 1, kActPlain = 2 };

struct ActQuant {
  const uint16_t* src;   // bf16 rows
  int64_t ld_src;        // elements between source rows
  const int32_t* perm;   // gather: padded row -> slot -> source row slot / top_k
  int32_t top_k;
  const int64_t* offsets;
  int32_t E;
  int64_t K, Kp;         // row length and padded row length (elements)
  int64_t rows;          // plain: rows; otherwise the padded row bound Rp_max
  uint8_t* elems;        // [NT][rows][Kp] e4m3 (plain: [rows][K])
  uint8_t* sf;           // [NT][rows/MBN][Kp/128][512] (plain: [rows][K/32])
  int shift;
};

template <int NT, int MODE>
__global__ void __launch_bounds__(256) mx_act_quant_kernel(ActQuant q) {
  __shared__ int32_t s_poff[kMxMaxE + 1];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int64_t used = q.rows;
  if constexpr (MODE != kActPlain) {
    if (warp == 0) warp_padded_offsets(q.offsets, q.E, s_poff, lane);
    __syncthreads();
    used = s_poff[q.E];
  }
  const int64_t steps = (q.Kp + 255) / 256;
  const int64_t kbp = q.Kp / 128;
  for (int64_t pp = int64_t(blockIdx.x) * 8 + warp; pp < used; pp += int64_t(gridDim.x) * 8) {
    bool valid = true;
    int64_t row = pp;
    if constexpr (MODE != kActPlain) {
      const int e = expert_of_padded_row(s_poff, q.E, pp);
      const int64_t local = pp - s_poff[e];
      valid = local < q.offsets[e + 1] - q.offsets[e];
      if (MODE == kActGather && valid) row = q.perm[q.offsets[e] + local] / q.top_k;
    }
    const uint16_t* src = q.src + row * q.ld_src;
    for (int64_t st = 0; st < steps; ++st) {
      const int64_t k0 = st * 256 + lane * 8;
      const bool in_row = k0 < q.Kp;  // uniform per 4-lane block (Kp % 32 == 0)
      float v[8];
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (valid && k0 < q.K) raw = __ldg(reinterpret_cast<const uint4*>(src + k0));
      const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16_bits_to_f32(rw[i] & 0xFFFFu);
        v[2 * i + 1] = bf16_bits_to_f32(rw[i] >> 16);
      }
      uint2 out[NT];
      uint32_t sb[NT];
      quant_block8<NT>(v, q.shift, out, sb);
      if (!in_row) continue;
      const int64_t blk = k0 / 32;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if constexpr (MODE == kActPlain) {
          *reinterpret_cast<uint2*>(q.elems + pp * q.K + k0) = out[t];
          if ((lane & 3) == 0) q.sf[pp * (q.K / 32) + blk] = uint8_t(sb[t]);
        } else {
          *reinterpret_cast<uint2*>(q.elems + (int64_t(t) * q.rows + pp) * q.Kp + k0) = out[t];
          if ((lane & 3) == 0) {
            const int64_t chunk = (int64_t(t) * (q.rows / MBN) + pp / MBN) * kbp + blk / 4;
            const int r = int(pp % MBN);
            q.sf[chunk * kChunk + (r % 32) * 16 + (r / 32) * 4 + (blk % 4)] = uint8_t(sb[t]);
          }
        }
      }
    }
  }
}

// ------------------------------------------------------------ the GEMM
template <int NMAT, int NT>
struct MxCfg {
  // the tiles, then one 512-byte scale-factor chunk per tile, rounded up to
  // 1 KB so that the next stage's tiles stay 1024-byte aligned
  static constexpr uint32_t kSfBytes = ((NMAT + NT) * kChunk + 1023) / 1024 * 1024;
  static constexpr uint32_t kStage = NMAT * kTile + NT * kBTile + kSfBytes;
  static constexpr int S = NMAT + NT == 4 ? 3 : (NMAT + NT == 3 ? 4 : 6);
  static constexpr int NACC = 2;
  static constexpr uint32_t kBars = S * kStage;
  static constexpr int kNumBars = 2 * S + 4;
  static constexpr uint32_t kScal = kBars + kNumBars * 8;  // tmem base, abort, n active
  static constexpr uint32_t kAct = kScal + 16;
  static constexpr uint32_t kPre = kAct + kMxMaxE * 4;
  static constexpr uint32_t kPoff = kPre + (kMxMaxE + 1) * 4;
  static constexpr uint32_t kGate = (kPoff + (kMxMaxE + 1) * 4 + 15) / 16 * 16;
  static constexpr uint32_t kRow = kGate + 4 * MBN * 4;
  static constexpr uint32_t kEnd = kRow + 4 * MBN * 4;
  static constexpr uint32_t kSmemBytes = kEnd + 1024;
  static constexpr uint32_t kSfCol = NMAT * MBN * NACC;  // scale-factor slots after the accumulators
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert((NMAT + NT) * kChunk <= kSfBytes && kStage % 1024 == 0, "stage layout");
  static_assert(kSfCol + S * (NMAT + NT) * 4 <= kTmemCols, "TMEM budget");
  static_assert(kSfCol % 4 == 0, "scale-factor slots");
};

struct MxGemm {
  int epilogue;  // E4B_EPI_SWIGLU or kEpiGatedRows
  int E, top_k;
  int64_t Nm, Np;          // weight rows per matrix, padded to 128
  int64_t K, Kp;
  int64_t Rp_max;
  const uint8_t* codes;    // prepared [E][nmat][Np][Kp/2]
  const uint8_t* sfa;      // prepared [E][nmat][Np/128][Kp/128][512]
  const uint8_t* act;      // [nt][Rp_max][Kp] e4m3
  const uint8_t* sfb;      // [nt][Rp_max/MBN][Kp/128][512]
  const int64_t* offsets;  // [E+1]
  const int32_t* perm;     // [R] slot of each routed row
  const float* gates;      // [T*top_k]
  void* out;               // SWIGLU: bf16 [Rp_max, ldo] (padded rows); gated: fp32 [R, ldo]
  int64_t ldo;
  int layout, act_fn;
  float alpha, limit;
  const float* bias;       // fp32 [E, nmat*Nm] in the source stack's row order, or null
  int32_t* status;
  uint32_t flags;
};

struct MxTile {
  int e;
  int64_t mt, nt, rows;  // weight-row block, routed-row block, valid routed rows (<= 128)
  int64_t pp0, p0;       // first padded row, first routed row
};

template <int EPI, int NT>
__global__ void __launch_bounds__(kMxThreads, 1)
mx_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
               MxGemm p) {
  constexpr int NMAT = EPI == E4B_EPI_SWIGLU ? 2 : 1;
  using C = MxCfg<NMAT, NT>;
  constexpr int S = C::S;
  constexpr int NACC = C::NACC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBars);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kScal);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kScal + 4);
  int32_t* s_n = reinterpret_cast<int32_t*>(smem + C::kScal + 8);
  int32_t* s_act = reinterpret_cast<int32_t*>(smem + C::kAct);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + C::kPre);
  int32_t* s_poff = reinterpret_cast<int32_t*>(smem + C::kPoff);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int64_t MT = p.Np / MBM;
  const int KB = int(p.Kp / MBK);
  const uint32_t limit = (p.flags & E4B_FLAG_TEST_TIMEOUT) ? 0u : kWaitPolls;

  // active experts, their padded row offsets and tile prefix sums
  {
    int32_t* s_warp = reinterpret_cast<int32_t*>(smem);  // scratch in stage 0, reused below
    block_active_experts(p.offsets, p.E, s_act, s_n, s_warp);
    if (warp == 0) {
      warp_padded_offsets(p.offsets, p.E, s_poff, lane);
      const int nact = *s_n;
      int run = 0;
      for (int base = 0; base < nact; base += 32) {
        const int a = base + lane;
        int v = 0;
        if (a < nact) {
          const int e = s_act[a];
          v = int((p.offsets[e + 1] - p.offsets[e] + MBN - 1) / MBN * MT);
        }
        int incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int o = __shfl_up_sync(0xffffffffu, incl, d);
          if (lane >= d) incl += o;
        }
        if (a < nact) s_pre[a] = run + incl - v;
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) s_pre[nact] = run;
    }
    __syncthreads();
  }
  const int nact = *s_n;
  const int total = s_pre[nact];
  if (int(blockIdx.x) >= total) return;  // no tile for this CTA (uniform)

  auto tile = [&](int t) -> MxTile {
    int lo = 0, hi = nact - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= t) lo = mid;
      else hi = mid - 1;
    }
    MxTile r;
    r.e = s_act[lo];
    const int64_t cnt = p.offsets[r.e + 1] - p.offsets[r.e];
    const int64_t ntn = (cnt + MBN - 1) / MBN;
    const int64_t local = t - s_pre[lo];
    r.mt = local / ntn;
    r.nt = local % ntn;
    r.rows = cnt - r.nt * MBN < MBN ? cnt - r.nt * MBN : MBN;
    r.pp0 = s_poff[r.e] + r.nt * MBN;
    r.p0 = p.offsets[r.e] + r.nt * MBN;
    return r;
  };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    *s_abort = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  auto give_up = [&]() {
    *s_abort = 1;
    record_status(p.status, E4B_ERR_DEVICE_TIMEOUT);
  };
  const int my_tiles = (total - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x);
  auto stage = [&](int s) { return smem + uint32_t(s) * C::kStage; };
  auto a_tile = [&](int s, int m) { return stage(s) + uint32_t(m) * kTile; };
  auto b_tile = [&](int s, int t) { return stage(s) + uint32_t(NMAT) * kTile + uint32_t(t) * kBTile; };
  auto sf_chunk = [&](int s, int i) {
    return stage(s) + uint32_t(NMAT) * kTile + uint32_t(NT) * kBTile + uint32_t(i) * kChunk;
  };

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      int64_t i = 0;
      bool aborted = false;
      const int64_t kbp = p.Kp / MBK;
      for (int j = 0; j < my_tiles && !aborted; ++j) {
        const MxTile T = tile(int(blockIdx.x) + j * int(gridDim.x));
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int s = int(i % S);
          if (!mbar_wait_bounded(&empty[s], (uint32_t(i / S) & 1u) ^ 1u, limit, s_abort)) {
            give_up();
            aborted = true;
            break;
          }
          mbar_arrive_expect_tx(&full[s], NMAT * kATx + NT * kBTile + (NMAT + NT) * kChunk);
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            tma_load_2d(a_tile(s, m), &tmap_a, &full[s], kb * MBK,
                        int32_t((int64_t(T.e) * NMAT + m) * p.Np + T.mt * MBM));
            const int64_t ca = ((int64_t(T.e) * NMAT + m) * MT + T.mt) * kbp + kb;
            bulk_load(sf_chunk(s, m), p.sfa + ca * kChunk, kChunk, &full[s]);
          }
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            tma_load_3d(b_tile(s, t), &tmap_b, &full[s], kb * MBK, int32_t(T.pp0), t);
            const int64_t cb = (int64_t(t) * (p.Rp_max / MBN) + T.pp0 / MBN) * kbp + kb;
            bulk_load(sf_chunk(s, NMAT + t), p.sfb + cb * kChunk, kChunk, &full[s]);
          }
        }
      }
      for (int64_t q = i > S ? i - S : 0; q < i; ++q)
        mbar_wait_bounded(&full[q % S], uint32_t(q / S) & 1u, kWaitPolls, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc0 = idesc_mx(MBM, MBN, 5u /* e2m1 */, 0u /* e4m3 */);
      int64_t i = 0;
      uint64_t* last_bar = nullptr;
      uint32_t last_ph = 0;
      bool aborted = false;
      for (int j = 0; j < my_tiles && !aborted; ++j) {
        const int ab = j % NACC;
        if (!mbar_wait_bounded(&acc_empty[ab], (uint32_t(j / NACC) & 1u) ^ 1u, limit, s_abort)) {
          give_up();
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + uint32_t(ab * NMAT * MBN);
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int s = int(i % S);
          if (!mbar_wait_bounded(&full[s], uint32_t(i / S) & 1u, limit, s_abort)) {
            give_up();
            aborted = true;
            break;
          }
          tc_fence_after();
          // this stage's scale factors into its own TMEM slot
          const uint32_t sfcol = tmem + C::kSfCol + uint32_t(s * (NMAT + NT) * 4);
#pragma unroll
          for (int c = 0; c < NMAT + NT; ++c)
            tmem_cp_32x128b_warpx4(sfcol + uint32_t(4 * c), chunk512_desc(smem_u32(sf_chunk(s, c))));
#pragma unroll
          for (int kk = 0; kk < MBK / 32; ++kk) {
            const uint32_t idesc = idesc_mx_ids(idesc0, uint32_t(kk), uint32_t(kk));
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
              const uint64_t adesc = sw128_kmajor_desc(smem_u32(a_tile(s, m)) + kk * 32);
#pragma unroll
              for (int t = 0; t < NT; ++t) {
                const uint64_t bdesc = sw128_kmajor_desc(smem_u32(b_tile(s, t)) + kk * 32);
                mma_mxf8f6f4_ss(dcol + uint32_t(m * MBN), adesc, bdesc, idesc, sfcol + uint32_t(4 * m),
                                sfcol + uint32_t(4 * (NMAT + t)), (kb | kk | t) ? 1u : 0u);
              }
            }
          }
          mma_commit(&empty[s]);
          last_bar = &empty[s];
          last_ph = uint32_t(i / S) & 1u;
        }
        if (aborted) break;
        mma_commit(&acc_full[ab]);
      }
      if (*s_abort && last_bar) mbar_wait_bounded(last_bar, last_ph, kWaitPolls, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // the TMEM lane quarter this warp may read
    const int r = q * 32 + lane;
    constexpr bool GATED = EPI == kEpiGatedRows;
    float* s_g = reinterpret_cast<float*>(smem + C::kGate) + q * MBN;
    int32_t* s_p = reinterpret_cast<int32_t*>(smem + C::kRow) + q * MBN;
    for (int j = 0; j < my_tiles; ++j) {
      const int ab = j % NACC;
      const MxTile T = tile(int(blockIdx.x) + j * int(gridDim.x));
      if constexpr (GATED) {
        // each routed row's gate weight and position, staged by this warp for
        // itself while the tile's MMAs run
        __syncwarp();
#pragma unroll
        for (int u = 0; u < (MBN + 31) / 32; ++u) {
          const int ii = lane + 32 * u;
          if (ii >= MBN) break;
          const bool ok = ii < T.rows;
          const int32_t slot = ok ? p.perm[T.p0 + ii] : 0;
          s_p[ii] = ok ? int32_t(T.p0 + ii) : -1;
          s_g[ii] = ok ? p.gates[slot] : 0.f;
        }
        __syncwarp();
      }
      if (!mbar_wait_bounded(&acc_full[ab], uint32_t(j / NACC) & 1u, limit, s_abort)) {
        give_up();
        break;
      }
      tc_fence_after();
      const int64_t n = T.mt * MBM + r;
      const bool nvalid = n < p.Nm;
      float b0 = 0.f, b1 = 0.f;
      if (p.bias && nvalid) {
        const float* b = p.bias + int64_t(T.e) * NMAT * p.Nm;
        b0 = b[NMAT == 2 ? gate_up_row(p.layout, p.Nm, 0, n) : n];
        if constexpr (NMAT == 2) b1 = b[gate_up_row(p.layout, p.Nm, 1, n)];
      }
      const uint32_t lane_base = tmem + (uint32_t(q * 32) << 16) + uint32_t(ab * NMAT * MBN);
      for (int cc = 0; cc < MBN / 16; ++cc) {
        if (cc * 16 >= T.rows) break;  // uniform: the rest of the tile is padding
        uint32_t g[16];
        uint32_t u[16];
        tmem_ld_32x32b_x16(lane_base + uint32_t(cc * 16), g);
        if constexpr (NMAT == 2) tmem_ld_32x32b_x16(lane_base + uint32_t(MBN + cc * 16), u);
        tmem_ld_wait();
        if (!nvalid) continue;
        if (cc * 16 + 16 <= T.rows) {
          // all 16 rows valid: no per-row check, pointer stepping (the gated
          // rows' gates as four 16-byte shared loads; row ii is T.p0 + ii)
          if constexpr (GATED) {
            float gw[16];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const float4 q4 = reinterpret_cast<const float4*>(s_g + cc * 16)[v];
              gw[4 * v] = q4.x;
              gw[4 * v + 1] = q4.y;
              gw[4 * v + 2] = q4.z;
              gw[4 * v + 3] = q4.w;
            }
            float* o = static_cast<float*>(p.out) + (T.p0 + cc * 16) * p.ldo + n;
#pragma unroll
            for (int t = 0; t < 16; ++t) o[t * p.ldo] = gw[t] * (__uint_as_float(g[t]) + b0);
          } else {
            uint16_t* o = static_cast<uint16_t*>(p.out) + (T.pp0 + cc * 16) * p.ldo + n;
#pragma unroll
            for (int t = 0; t < 16; ++t)
              o[t * p.ldo] = to_bf16_bits(
                  glu_act(p.act_fn, __uint_as_float(g[t]) + b0, __uint_as_float(u[t]) + b1, p.alpha, p.limit));
          }
          continue;
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int ii = cc * 16 + t;
          if (ii >= T.rows) break;
          const float gv = __uint_as_float(g[t]) + b0;
          if constexpr (GATED) {
            static_cast<float*>(p.out)[int64_t(s_p[ii]) * p.ldo + n] = s_g[ii] * gv;
          } else {
            const float hv = glu_act(p.act_fn, gv, __uint_as_float(u[t]) + b1, p.alpha, p.limit);
            static_cast<uint16_t*>(p.out)[(T.pp0 + ii) * p.ldo + n] = to_bf16_bits(hv);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn mx_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

template <int EPI, int NT>
cudaError_t launch_mx_t(const MxGemm& p, cudaStream_t st, int sms) {
  constexpr int NMAT = EPI == E4B_EPI_SWIGLU ? 2 : 1;
  using C = MxCfg<NMAT, NT>;
  EncodeTiledFn enc = mx_encode_fn();
  if (!enc) return cudaErrorInitializationError;
  CUtensorMap ta, tb;
  {
    // prepared codes [E * nmat * Np rows, Kp 4-bit elements]; TMA unpacks each
    // 16 elements into a 16-byte unit (8 bytes of codes, 8 unused)
    const cuuint64_t gdim[2] = {cuuint64_t(p.Kp), cuuint64_t(int64_t(p.E) * NMAT * p.Np)};
    const cuuint64_t gstride[1] = {cuuint64_t(p.Kp / 2)};
    const cuuint32_t box[2] = {MBK, MBM};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&ta, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<uint8_t*>(p.codes), gdim, gstride, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // activation terms [NT][Rp_max rows][Kp bytes]
    const cuuint64_t gdim[3] = {cuuint64_t(p.Kp), cuuint64_t(p.Rp_max), cuuint64_t(NT)};
    const cuuint64_t gstride[2] = {cuuint64_t(p.Kp), cuuint64_t(p.Kp) * cuuint64_t(p.Rp_max)};
    const cuuint32_t box[3] = {MBK, MBN, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(p.act), gdim, gstride, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  auto kern = mx_gemm_kernel<EPI, NT>;
  static int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    const cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::kSmemBytes));
    if (err != cudaSuccess) return err;
    configured_dev = dev;
  }
  const int64_t max_tiles = (p.Np / MBM) * (p.Rp_max / MBN);
  int grid = int(max_tiles < sms ? max_tiles : sms);
  if (grid < 1) grid = 1;
  kern<<<grid, kMxThreads, C::kSmemBytes, st>>>(ta, tb, p);
  return cudaGetLastError();
}

}  // namespace

int64_t mx_padded_rows_max(int64_t R, int64_t E) {
  const int64_t active = R < E ? R : E;
  return (R + kMxRowBlock - 1) / kMxRowBlock * kMxRowBlock + int64_t(kMxRowBlock) * active;
}

cudaError_t launch_mx_prepare(const uint8_t* blocks, const uint8_t* scales, int E, int64_t Nm, int nmat,
                              int64_t K, int layout, uint8_t* out_codes, uint8_t* out_sf, cudaStream_t st,
                              int sms) {
  const int64_t Np = (Nm + 127) / 128 * 128;
  const int64_t Kp = (K + 127) / 128 * 128;
  const int64_t total = int64_t(E) * nmat * Np * (Kp / 32);
  int64_t grid = (total + 255) / 256;
  if (grid > int64_t(sms) * 32) grid = int64_t(sms) * 32;
  if (grid < 1) grid = 1;
  mx_prepare_kernel<<<int(grid), 256, 0, st>>>(blocks, scales, E, Nm, nmat, K, layout, Np, Kp, out_codes, out_sf);
  return cudaGetLastError();
}

cudaError_t launch_mx_act_quant(const MxActArgs& a, cudaStream_t st, int sms) {
  ActQuant q{};
  q.src = a.src;
  q.ld_src = a.ld_src;
  q.perm = a.perm;
  q.top_k = a.top_k;
  q.offsets = a.offsets;
  q.E = a.E;
  q.K = a.K;
  q.Kp = a.plain ? a.K : (a.K + 127) / 128 * 128;
  q.rows = a.rows;
  q.elems = a.elems;
  q.sf = a.sf;
  q.shift = a.nterms == 2 ? 7 : 8;
  int64_t grid = (a.rows + 7) / 8;
  if (grid > int64_t(sms) * 16) grid = int64_t(sms) * 16;
  if (grid < 1) grid = 1;
  if (a.plain) {
    mx_act_quant_kernel<1, kActPlain><<<int(grid), 256, 0, st>>>(q);
  } else if (a.nterms == 2) {
    if (a.perm) mx_act_quant_kernel<2, kActGather><<<int(grid), 256, 0, st>>>(q);
    else mx_act_quant_kernel<2, kActPadded><<<int(grid), 256, 0, st>>>(q);
  } else {
    if (a.perm) mx_act_quant_kernel<1, kActGather><<<int(grid), 256, 0, st>>>(q);
    else mx_act_quant_kernel<1, kActPadded><<<int(grid), 256, 0, st>>>(q);
  }
  return cudaGetLastError();
}

cudaError_t launch_mx_gemm(const MxGemmArgs& a, cudaStream_t st, int sms) {
  if (a.E > kMxMaxE) return cudaErrorInvalidValue;
  MxGemm p{};
  p.epilogue = a.gated_rows ? kEpiGatedRows : E4B_EPI_SWIGLU;
  p.E = a.E;
  p.top_k = a.top_k;
  p.Nm = a.Nm;
  p.Np = (a.Nm + 127) / 128 * 128;
  p.K = a.K;
  p.Kp = (a.K + 127) / 128 * 128;
  p.Rp_max = a.Rp_max;
  p.codes = a.codes;
  p.sfa = a.sfa;
  p.act = a.act;
  p.sfb = a.sfb;
  p.offsets = a.offsets;
  p.perm = a.perm;
  p.gates = a.gates;
  p.out = a.out;
  p.ldo = a.ldo;
  p.layout = a.layout;
  p.act_fn = a.act_fn;
  p.alpha = a.alpha;
  p.limit = a.limit;
  p.bias = a.bias;
  p.status = a.status;
  p.flags = a.flags;
  if (a.gated_rows) {
    return a.nterms == 2 ? launch_mx_t<kEpiGatedRows, 2>(p, st, sms) : launch_mx_t<kEpiGatedRows, 1>(p, st, sms);
  }
  return a.nterms == 2 ? launch_mx_t<E4B_EPI_SWIGLU, 2>(p, st, sms) : launch_mx_t<E4B_EPI_SWIGLU, 1>(p, st, sms);
}

}  // namespace e4b
