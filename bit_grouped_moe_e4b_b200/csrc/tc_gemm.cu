// Large-M grouped projection on the 5th-generation tensor cores.
//
// "grouped-nf4-gemm" README, intro: one launch covers all active experts;
// weights stay packed in HBM and are decoded through a table on the fly; fp32
// accumulation; bf16 epilogue. bitsandbytes PR #1984, Design: gated SiLU
// (SwiGLU) between the projections; the top-k weighted sum after the second.
//
// sm_100a design, one persistent CTA per SM, warp-specialised, with three
// independent shared-memory rings so that no producer waits on a consumer
// further down the chain than its own ring:
//   codes ring  (warp 0, TMA)  packed codes of the tile's weight rows,
//               [128 rows x 32 B] per matrix and 64-wide K block; a slot is
//               released by the decoders as soon as they hold the codes in
//               registers, so code fetches run far ahead of the MMAs;
//   B ring      (warp 2, TMA)  the routed activation rows, 128B-swizzled
//               K-major: rows gathered four at a time (tile::gather4) from
//               a[row_slot[p] / top_k], or one 256-row tile when the rows are
//               contiguous; released by the MMA;
//   A ring      (warps 4-11)   decoders: each thread takes one weight row of a
//               job, builds its block's 16-entry bf16 table and writes 64
//               decoded weights (128B-swizzled K-major); released by the MMA.
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer
//               (M = 128 weight rows, N = 256 routed rows, K = 16 per MMA).
//   warps 12-15 epilogue: tcgen05.ld of the fp32 accumulators, then the
//               biases and the gated activation (gate and up accumulate in two
//               TMEM column ranges of the same lanes, so it is thread-local),
//               the gate-weighted combine (atomics, e4b_grouped_gemm), or the
//               layer's gate-weighted rows (one fp32 row per routed row,
//               summed per token afterwards in a fixed order).
// Interleaved gate/up rows (gate 2n, up 2n+1) reach the same tiles through a
// 3-D view of the codes, [E*I rows, 2, K/2 bytes]: one box fetches 128 gate
// (or up) rows at a two-row stride.
//               A single-matrix projection has two accumulators in TMEM, so
//               the epilogue of one tile overlaps the MMAs of the next.
// Tiles: per active expert, (weight-row block of 128) x (routed-row block of
// 256), routed-row blocks fastest so CTAs running together share A in L2.
// Every wait is bounded; a wait that gives up records E4B_ERR_DEVICE_TIMEOUT,
// stops all roles, drains the copies and MMAs already issued, frees TMEM and
// returns.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace e4b {
namespace {

using namespace sm100;

constexpr int BM = 128;   // weight rows per matrix per tile (MMA M)
constexpr int BN = 256;   // routed rows per tile (MMA N)
constexpr int BK = 64;    // K per job: one 128-byte swizzle row of bf16
constexpr int kThreads = 512;
constexpr int kMaxE = 256;
constexpr int kDecoderThreads = 256;
constexpr int kEpiThreads = 128;
constexpr uint32_t kATileBytes = BM * BK * 2;   // 16 KB
constexpr uint32_t kBTileBytes = BN * BK * 2;   // 32 KB
constexpr uint32_t kCTileBytes = BM * BK / 2;   // 4 KB packed codes
constexpr int kScalePrefetch = 4;               // jobs of absmax / scale loads in flight

template <int NMAT>
struct Cfg {
  static constexpr int CS = NMAT == 2 ? 6 : 10;    // codes stages
  static constexpr int AS = NMAT == 2 ? 2 : 4;     // decoded-A stages
  static constexpr int BS = 3;                     // activation stages
  static constexpr int NACC = NMAT == 2 ? 1 : 2;   // accumulators in TMEM
  static constexpr int kDecPerJob = NMAT == 2 ? kDecoderThreads : kDecoderThreads / 2;
  static constexpr uint32_t kA = 0;
  static constexpr uint32_t kB = kA + AS * NMAT * kATileBytes;
  static constexpr uint32_t kC = kB + BS * kBTileBytes;
  static constexpr uint32_t kMisc = kC + CS * NMAT * kCTileBytes;
  // misc: barriers, scalars, the expert tables
  static constexpr int kNumBars = 2 * (CS + AS + BS + 2);
  static constexpr uint32_t kBars = kMisc;
  static constexpr uint32_t kScal = kBars + kNumBars * 8;       // 16 B
  static constexpr uint32_t kAct = kScal + 16;                  // kMaxE x 4
  static constexpr uint32_t kPre = kAct + kMaxE * 4;            // (kMaxE + 1) x 4
  // per epilogue warp: the gate weight and token of each of a tile's BN rows
  static constexpr uint32_t kGate = (kPre + (kMaxE + 1) * 4 + 15) / 16 * 16;
  static constexpr uint32_t kTok = kGate + 4 * BN * 4;
  static constexpr uint32_t kEnd = kTok + 4 * BN * 4;
  static constexpr uint32_t kSmemBytes = kEnd + 1024;           // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // With one matrix the decoders split into two groups that take alternate
  // jobs. A parity wait must never run two phases ahead of its barrier, so
  // every slot of a ring the groups wait on must belong to one group only:
  // an even number of slots.
  static_assert(NMAT == 2 || (CS % 2 == 0 && AS % 2 == 0), "decoder groups own alternate slots");
  static_assert(NMAT * BN * (NMAT == 2 ? 1 : NACC) <= 512, "TMEM budget");
};

struct Tile {
  int e;
  int64_t mt, p0, p1;
};

// The static tile decomposition shared by every role of the CTA.
struct Sched {
  const int32_t* act;
  const int32_t* pre;
  int nact;
  int total;
  const int64_t* offsets;

  __device__ Tile tile(int t) const {
    int lo = 0, hi = nact - 1;  // largest a with pre[a] <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= t) lo = mid;
      else hi = mid - 1;
    }
    const int e = act[lo];
    const int64_t b = offsets[e];
    const int64_t end = offsets[e + 1];
    const int64_t ntn = (end - b + BN - 1) / BN;
    const int64_t local = t - pre[lo];
    Tile r;
    r.e = e;
    r.mt = local / ntn;
    r.p0 = b + (local % ntn) * BN;
    r.p1 = end;
    return r;
  }
};

template <int FMT, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmap_codes,
               const __grid_constant__ CUtensorMap tmap_act, GemmProblem p) {
  constexpr bool DG = EPI == kEpiDgrad;
  constexpr int NMAT = (EPI == E4B_EPI_SWIGLU) ? 2 : 1;
  using C = Cfg<NMAT>;
  constexpr int CS = C::CS;
  constexpr int AS = C::AS;
  constexpr int BS = C::BS;
  constexpr int NACC = C::NACC;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBars);
  uint64_t* c_full = bars;
  uint64_t* c_empty = c_full + CS;
  uint64_t* a_full = c_empty + CS;
  uint64_t* a_empty = a_full + AS;
  uint64_t* b_full = a_empty + AS;
  uint64_t* b_empty = b_full + BS;
  uint64_t* acc_full = b_empty + BS;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kScal);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kScal + 4);
  int32_t* s_n = reinterpret_cast<int32_t*>(smem + C::kScal + 8);
  int32_t* s_act = reinterpret_cast<int32_t*>(smem + C::kAct);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + C::kPre);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int64_t N = p.N;
  const int64_t K = p.K;
  const int64_t rows_per_mat = NMAT == 2 ? N / 2 : N;
  // dgrad: the MMA's M runs over the weight's columns, its reduction over the
  // weight's rows
  const int64_t Mdim = DG ? K : rows_per_mat;
  const int64_t Kred = DG ? N : K;
  const int64_t MT = (Mdim + BM - 1) / BM;
  const int KB = int((Kred + BK - 1) / BK);
  const bool il = NMAT == 2 && p.layout == E4B_GATE_UP_INTERLEAVED;
  const uint32_t limit = (p.flags & E4B_FLAG_TEST_TIMEOUT) ? 0u : kWaitPolls;

  // Clear the caller's fp32 accumulator (the layer's combine buffer) first.
  if (p.zero_buf) {
    for (int64_t i = int64_t(blockIdx.x) * kThreads + tid; i < p.zero_count;
         i += int64_t(gridDim.x) * kThreads)
      p.zero_buf[i] = 0.f;
  }

  // Active experts and their tile prefix sums.
  {
    int32_t* s_warp = reinterpret_cast<int32_t*>(smem + C::kA);  // scratch, reused below
    block_active_experts(p.offsets, p.E, s_act, s_n, s_warp);
    if (warp == 0) {
      const int nact = *s_n;
      int run = 0;
      for (int base = 0; base < nact; base += 32) {
        const int a = base + lane;
        int v = 0;
        if (a < nact) {
          const int e = s_act[a];
          const int64_t rows = p.offsets[e + 1] - p.offsets[e];
          v = int(((rows + BN - 1) / BN) * MT);
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
  Sched sc{s_act, s_pre, *s_n, s_pre[*s_n], p.offsets};
  if (int(blockIdx.x) >= sc.total) return;  // no tile for this CTA (uniform)

  if (tid == 0) {
    for (int s = 0; s < CS; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_empty[s], C::kDecPerJob);
    }
    for (int s = 0; s < AS; ++s) {
      mbar_init(&a_full[s], C::kDecPerJob);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < BS; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiThreads);
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

  const int my_tiles = (sc.total - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x);
  const int64_t njobs = int64_t(my_tiles) * KB;  // (tile, k-block) jobs this CTA walks

  if (warp == 0) {
    // --------------------------------------------------- codes ring (TMA)
    if (lane == 0) {
      int64_t i = 0;
      bool aborted = false;
      for (int j = 0; j < my_tiles && !aborted; ++j) {
        const Tile T = sc.tile(int(blockIdx.x) + j * int(gridDim.x));
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int s = int(i % CS);
          if (!mbar_wait_bounded(&c_empty[s], (uint32_t(i / CS) & 1u) ^ 1u, limit, s_abort)) {
            give_up();
            aborted = true;
            break;
          }
          mbar_arrive_expect_tx(&c_full[s], NMAT * kCTileBytes);
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            uint8_t* dst = smem + C::kC + (s * NMAT + m) * kCTileBytes;
            if (DG) {
              // 64 weight rows x 128 weight columns (64 bytes)
              tma_load_2d(dst, &tmap_codes, &c_full[s], int32_t(T.mt * (BM / 2)),
                          int32_t(int64_t(T.e) * N + int64_t(kb) * BK));
            } else if (il) {
              tma_load_3d(dst, &tmap_codes, &c_full[s], kb * (BK / 2), m,
                          int32_t(int64_t(T.e) * rows_per_mat + T.mt * BM));
            } else {
              const int64_t row = int64_t(T.e) * N + m * rows_per_mat + T.mt * BM;
              tma_load_2d(dst, &tmap_codes, &c_full[s], kb * (BK / 2), int32_t(row));
            }
          }
        }
      }
      // Drain: every load issued must land before the CTA can exit.
      for (int64_t q = i > CS ? i - CS : 0; q < i; ++q)
        mbar_wait_bounded(&c_full[q % CS], uint32_t(q / CS) & 1u, kWaitPolls, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      // dgrad: A is MN-major (bit 15, "transpose A")
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN) | (DG ? (1u << 15) : 0u);
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
        const uint32_t dcol = tmem + uint32_t(NMAT == 2 ? 0 : ab * BN);
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int as = int(i % AS);
          const int bs = int(i % BS);
          if (!mbar_wait_bounded(&a_full[as], uint32_t(i / AS) & 1u, limit, s_abort) ||
              !mbar_wait_bounded(&b_full[bs], uint32_t(i / BS) & 1u, limit, s_abort)) {
            give_up();
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint32_t bbase = smem_u32(smem + C::kB + bs * kBTileBytes);
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const uint32_t abase = smem_u32(smem + C::kA + (as * NMAT + m) * kATileBytes);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t adesc = DG ? sw128_mnmajor_desc(abase + kk * 2048, 8192, 1024)
                                        : sw128_kmajor_desc(abase + kk * 32);
              mma_bf16_ss(dcol + uint32_t(m * BN), adesc, sw128_kmajor_desc(bbase + kk * 32), idesc,
                          (kb | kk) ? 1u : 0u);
            }
          }
          mma_commit(&a_empty[as]);
          mma_commit(&b_empty[bs]);
          last_bar = &b_empty[bs];
          last_ph = uint32_t(i / BS) & 1u;
        }
        if (aborted) break;
        mma_commit(&acc_full[ab]);
      }
      // Drain: the MMAs issued so far must finish before TMEM is freed.
      if (*s_abort && last_bar) mbar_wait_bounded(last_bar, last_ph, kWaitPolls, nullptr);
    }
  } else if (warp == 2) {
    // ------------------------------------ activation rows, B ring (TMA)
    // Gathered rows: lane l issues the four-row gathers l and l + 32 of each
    // job (rows 4l..4l+3 and 128+4l..128+4l+3 of the tile), so the 64 copies
    // of a job leave in two warp-wide instructions.
    const bool gather = p.row_slot != nullptr;
    int64_t i = 0;
    bool aborted = false;
    for (int j = 0; j < my_tiles && !aborted; ++j) {
      const Tile T = sc.tile(int(blockIdx.x) + j * int(gridDim.x));
      int32_t gr[8];
      if (gather) {
        // rows past the expert's end repeat its first row (products discarded)
        const int32_t first = p.row_slot[T.p0] / p.top_k;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int64_t pr = T.p0 + 4 * lane + (q >> 2) * 128 + (q & 3);
          gr[q] = pr < T.p1 ? p.row_slot[pr] / p.top_k : first;
        }
      }
      for (int kb = 0; kb < KB; ++kb, ++i) {
        const int s = int(i % BS);
        int ok = 1;
        if (lane == 0) {
          ok = mbar_wait_bounded(&b_empty[s], (uint32_t(i / BS) & 1u) ^ 1u, limit, s_abort);
          if (ok) mbar_arrive_expect_tx(&b_full[s], kBTileBytes);
          else give_up();
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          aborted = true;
          break;
        }
        uint8_t* dst = smem + C::kB + s * kBTileBytes;
        if (gather) {
          tma_gather4_2d(dst + lane * 512, &tmap_act, &b_full[s], kb * BK, gr[0], gr[1], gr[2], gr[3]);
          tma_gather4_2d(dst + (lane + 32) * 512, &tmap_act, &b_full[s], kb * BK, gr[4], gr[5], gr[6],
                         gr[7]);
        } else if (lane == 0) {
          tma_load_2d(dst, &tmap_act, &b_full[s], kb * BK, int32_t(T.p0));
        }
      }
    }
    if (lane == 0) {
      for (int64_t q = i > BS ? i - BS : 0; q < i; ++q)
        mbar_wait_bounded(&b_full[q % BS], uint32_t(q / BS) & 1u, kWaitPolls, nullptr);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------ decoders (A operand)
    const int d = tid - 128;                  // 0..255
    const int m = NMAT == 2 ? (d >> 7) : 0;   // matrix (gate / up)
    const int r = d & 127;                    // row within the tile
    // dgrad: weight row dr of the job's 64, columns 64 db .. 64 db + 63 of the tile
    const int dr = r & 63, db = r >> 6;
    const int grp = NMAT == 2 ? 0 : (d >> 7); // NMAT == 1: two groups take alternate jobs
    constexpr int step = NMAT == 2 ? 1 : 2;
    const uint8_t* scales = static_cast<const uint8_t*>(p.scales);
    const int64_t sstride = FMT == E4B_FMT_NF4 ? (K / 64) * 4 : (K / 32);

    // Absmax (NF4, as fp32 bits) or the two scale bytes (MXFP4) of this
    // thread's row at job q.
    int cached_j = -1;
    const uint8_t* srow = nullptr;
    auto scale_at = [&](int64_t q) -> uint32_t {
      if (q >= njobs) return 0u;
      const int j = int(q / KB);
      const int kb = int(q % KB);
      if constexpr (DG) {
        // the absmax (or the two scale bytes) of weight row kb*64 + dr at
        // columns 128 mt + 64 db ..; zero past the expert's rows or columns
        // (those products meet zero-filled dy columns or unstored outputs)
        if (j != cached_j) {
          cached_j = j;
          const Tile T = sc.tile(int(blockIdx.x) + j * int(gridDim.x));
          const int64_t col0 = T.mt * BM + 64 * db;
          srow = col0 < K ? scales + int64_t(T.e) * N * sstride + (FMT == E4B_FMT_NF4 ? (col0 / 64) * 4 : col0 / 32)
                          : nullptr;
        }
        const int64_t wr = int64_t(kb) * BK + dr;
        if (!srow || wr >= N) return 0u;
        if constexpr (FMT == E4B_FMT_NF4) {
          return __float_as_uint(__ldg(reinterpret_cast<const float*>(srow + wr * sstride)));
        } else {
          const uint8_t* sb = srow + wr * sstride;
          return uint32_t(__ldg(sb)) | (uint32_t(__ldg(sb + 1)) << 8);
        }
      }
      if (j != cached_j) {
        cached_j = j;
        const Tile T = sc.tile(int(blockIdx.x) + j * int(gridDim.x));
        const int64_t n = T.mt * BM + r;
        const int64_t row = NMAT == 2 ? gate_up_row(p.layout, rows_per_mat, m, n) : n;
        srow = n < rows_per_mat ? scales + (int64_t(T.e) * N + row) * sstride : nullptr;
      }
      if (!srow) return 0u;
      if constexpr (FMT == E4B_FMT_NF4) {
        return __float_as_uint(__ldg(reinterpret_cast<const float*>(srow) + kb));
      } else {
        const int64_t b0 = int64_t(kb) * 2;
        const uint32_t lo = b0 < K / 32 ? uint32_t(__ldg(srow + b0)) : 0u;
        const uint32_t hi = b0 + 1 < K / 32 ? uint32_t(__ldg(srow + b0 + 1)) : 0u;
        return lo | (hi << 8);
      }
    };
    uint32_t ring[kScalePrefetch];
#pragma unroll
    for (int u = 0; u < kScalePrefetch; ++u) ring[u] = scale_at(grp + int64_t(u) * step);

    bool aborted = false;
    for (int64_t i0 = grp; i0 < njobs && !aborted; i0 += int64_t(kScalePrefetch) * step) {
#pragma unroll
      for (int u = 0; u < kScalePrefetch; ++u) {
        const int64_t i = i0 + int64_t(u) * step;
        if (i >= njobs) break;
        const uint32_t cur = ring[u];
        ring[u] = scale_at(i + int64_t(kScalePrefetch) * step);
        const int cs = int(i % CS);
        if (!mbar_wait_bounded(&c_full[cs], uint32_t(i / CS) & 1u, limit, s_abort)) {
          give_up();
          aborted = true;
          break;
        }
        const uint4* crow = reinterpret_cast<const uint4*>(
            smem + C::kC + (cs * NMAT + m) * kCTileBytes + (DG ? dr * 64 + db * 32 : r * 32));
        const uint4 c0 = crow[0];
        const uint4 c1 = crow[1];
        // The slot's next fill is a TMA write (async proxy); without this
        // fence it can overtake the generic-proxy reads just issued.
        fence_proxy_async_smem();
        mbar_arrive(&c_empty[cs]);
        const int as = int(i % AS);
        if (!mbar_wait_bounded(&a_empty[as], (uint32_t(i / AS) & 1u) ^ 1u, limit, s_abort)) {
          give_up();
          aborted = true;
          break;
        }
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        // K-major: the 128-byte row r of the tile. dgrad, MN-major: the
        // 128-byte row of K index dr (8-row atoms of 1024 bytes) in the atom
        // column db (8 KB apart); the same 128B swizzle by row within the atom.
        const int sw = DG ? (dr & 7) : (r & 7);
        uint8_t* arow = smem + C::kA + (as * NMAT + m) * kATileBytes +
                        (DG ? db * 8192 + (dr >> 3) * 1024 + (dr & 7) * 128 : r * 128);
        Lut L;
        lut_build<FMT>(L, __uint_as_float(cur), cur & 0xFFu);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (FMT == E4B_FMT_MXFP4 && c == 4) lut_build<FMT>(L, 0.f, (cur >> 8) & 0xFFu);
          uint32_t o[4];
          lut_decode8<FMT>(L, words[c], o);
          *reinterpret_cast<uint4*>(arow + ((c ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&a_full[as]);
      }
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int rloc = q * 32 + lane;
    constexpr bool GATED = EPI == E4B_EPI_COMBINE || EPI == kEpiGatedRows;
    float* s_g = reinterpret_cast<float*>(smem + C::kGate) + q * BN;
    int32_t* s_t = reinterpret_cast<int32_t*>(smem + C::kTok) + q * BN;
    for (int j = 0; j < my_tiles; ++j) {
      const int ab = j % NACC;
      const Tile T = sc.tile(int(blockIdx.x) + j * int(gridDim.x));
      if constexpr (GATED) {
        // Every row's gate weight and token, staged by this warp for itself
        // while the tile's MMAs run: the loop below reads them from shared
        // memory instead of two dependent global loads per row.
        __syncwarp();
        int32_t sl[BN / 32];
#pragma unroll
        for (int u = 0; u < BN / 32; ++u) {
          const int64_t pr = T.p0 + lane + 32 * u;
          sl[u] = pr < T.p1 ? (p.out_slot ? p.out_slot[pr] : int32_t(pr)) : -1;
        }
#pragma unroll
        for (int u = 0; u < BN / 32; ++u) {
          s_g[lane + 32 * u] = sl[u] >= 0 ? p.gates[sl[u]] : 0.f;
          s_t[lane + 32 * u] = sl[u] >= 0 ? sl[u] / p.top_k : 0;
        }
        __syncwarp();
      }
      if (!mbar_wait_bounded(&acc_full[ab], uint32_t(j / NACC) & 1u, limit, s_abort)) {
        give_up();
        break;
      }
      tc_fence_after();
      const int64_t n = T.mt * BM + rloc;
      const bool nvalid = n < Mdim;
      // bias of this thread's row(s): gate and up, or the single output row
      float b0 = 0.f, b1 = 0.f;
      if (p.bias && nvalid) {
        const float* b = p.bias + int64_t(T.e) * N;
        b0 = b[NMAT == 2 ? gate_up_row(p.layout, rows_per_mat, 0, n) : n];
        if constexpr (NMAT == 2) b1 = b[gate_up_row(p.layout, rows_per_mat, 1, n)];
      }
      const uint32_t lane_base =
          tmem + (uint32_t(q * 32) << 16) + uint32_t(NMAT == 2 ? 0 : ab * BN);
      for (int cc = 0; cc < BN / 16; ++cc) {
        const int64_t pbase = T.p0 + cc * 16;
        if (pbase >= T.p1) break;  // uniform: the rest of the tile is past the expert's rows
        uint32_t g[16];
        uint32_t u[16];
        tmem_ld_32x32b_x16(lane_base + uint32_t(cc * 16), g);
        if constexpr (NMAT == 2) tmem_ld_32x32b_x16(lane_base + uint32_t(BN + cc * 16), u);
        tmem_ld_wait();
        if (!nvalid) continue;
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int64_t pr = pbase + t;
          if (pr >= T.p1) break;
          const float gv = __uint_as_float(g[t]) + b0;
          if constexpr (EPI == E4B_EPI_SWIGLU) {
            const float hv = glu_act(p.act, gv, __uint_as_float(u[t]) + b1, p.alpha, p.limit);
            static_cast<uint16_t*>(p.out)[pr * p.ldo + n] = to_bf16_bits(hv);
          } else if constexpr (EPI == E4B_EPI_STORE || DG) {
            static_cast<uint16_t*>(p.out)[pr * p.ldo + n] = to_bf16_bits(gv);
          } else if constexpr (EPI == kEpiGatedRows) {
            static_cast<float*>(p.out)[pr * p.ldo + n] = s_g[cc * 16 + t] * gv;
          } else {
            const int64_t tok = s_t[cc * 16 + t];
            atomicAdd(static_cast<float*>(p.out) + tok * p.ldo + n, s_g[cc * 16 + t] * gv);
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

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

template <int FMT, int EPI>
cudaError_t launch_t(const GemmProblem& p, cudaStream_t st, int sms) {
  constexpr int NMAT = (EPI == E4B_EPI_SWIGLU) ? 2 : 1;
  using C = Cfg<NMAT>;
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cudaErrorInitializationError;
  constexpr bool DG = EPI == kEpiDgrad;
  // Packed codes viewed as a 2-D byte tensor [E*N rows, K/2 bytes] (dgrad:
  // boxes of 64 rows x 128 weight columns), or for interleaved gate/up rows as
  // [E*I, 2, K/2] (boxes of 128 gate or up rows).
  CUtensorMap tmap_codes;
  if (DG) {
    const cuuint64_t gdim[2] = {cuuint64_t(p.K / 2), cuuint64_t(int64_t(p.E) * p.N)};
    const cuuint64_t gstride[1] = {cuuint64_t(p.K / 2)};
    const cuuint32_t box[2] = {BM / 2, BK};
    const cuuint32_t estride[2] = {1, 1};
    CUresult cr = enc(&tmap_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p.codes),
                      gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  } else if (NMAT == 2 && p.layout == E4B_GATE_UP_INTERLEAVED) {
    const cuuint64_t gdim[3] = {cuuint64_t(p.K / 2), 2, cuuint64_t(int64_t(p.E) * (p.N / 2))};
    const cuuint64_t gstride[2] = {cuuint64_t(p.K / 2), cuuint64_t(p.K)};
    const cuuint32_t box[3] = {BK / 2, 1, BM};
    const cuuint32_t estride[3] = {1, 1, 1};
    CUresult cr = enc(&tmap_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(p.codes),
                      gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  } else {
    const cuuint64_t gdim[2] = {cuuint64_t(p.K / 2), cuuint64_t(int64_t(p.E) * p.N)};
    const cuuint64_t gstride[1] = {cuuint64_t(p.K / 2)};
    const cuuint32_t box[2] = {BK / 2, BM};
    const cuuint32_t estride[2] = {1, 1};
    CUresult cr = enc(&tmap_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p.codes),
                      gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  // Activations [rows, K] bf16 with row stride lda, landing 128B-swizzled:
  // single rows for the four-row gather, 256-row tiles for contiguous rows.
  // dgrad: dy [rows, N], the reduction running over the weight's rows.
  CUtensorMap tmap_act;
  {
    const bool gather = p.row_slot != nullptr;
    const int64_t rows = gather ? (p.R_max + p.top_k - 1) / p.top_k : p.R_max;
    const cuuint64_t gdim[2] = {cuuint64_t(DG ? p.N : p.K), cuuint64_t(rows)};
    const cuuint64_t gstride[1] = {cuuint64_t(p.lda) * 2};
    const cuuint32_t box[2] = {BK, gather ? 1u : cuuint32_t(BN)};
    const cuuint32_t estride[2] = {1, 1};
    CUresult cr = enc(&tmap_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(p.a),
                      gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }

  auto kern = tc_gemm_kernel<FMT, EPI>;
  static int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(C::kSmemBytes));
    if (err != cudaSuccess) return err;
    configured_dev = dev;
  }
  const int64_t rows_per_mat = NMAT == 2 ? p.N / 2 : p.N;
  const int64_t MT = ((DG ? p.K : rows_per_mat) + BM - 1) / BM;
  const int64_t max_tiles = MT * ((p.R_max + BN - 1) / BN + p.E);
  int grid = int(max_tiles < sms ? max_tiles : sms);
  if (grid < 1) grid = 1;
  kern<<<grid, kThreads, C::kSmemBytes, st>>>(tmap_codes, tmap_act, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_gemm(const GemmProblem& p, cudaStream_t st, int sms) {
  if (p.E > kMaxE) return cudaErrorInvalidValue;
  if (tc_pair_supported(p)) return launch_tc_pair(p, st, sms);
  if (p.epilogue == kEpiDgrad) {
    if (p.row_slot) return cudaErrorInvalidValue;  // dy rows are expert-ordered
    return p.fmt == E4B_FMT_NF4 ? launch_t<E4B_FMT_NF4, kEpiDgrad>(p, st, sms)
                                : launch_t<E4B_FMT_MXFP4, kEpiDgrad>(p, st, sms);
  }
  if (p.epilogue == kEpiGatedRows)
    return p.fmt == E4B_FMT_NF4 ? launch_t<E4B_FMT_NF4, kEpiGatedRows>(p, st, sms)
                                : launch_t<E4B_FMT_MXFP4, kEpiGatedRows>(p, st, sms);
  if (p.fmt == E4B_FMT_NF4) {
    if (p.epilogue == E4B_EPI_SWIGLU) return launch_t<E4B_FMT_NF4, E4B_EPI_SWIGLU>(p, st, sms);
    if (p.epilogue == E4B_EPI_COMBINE) return launch_t<E4B_FMT_NF4, E4B_EPI_COMBINE>(p, st, sms);
    return launch_t<E4B_FMT_NF4, E4B_EPI_STORE>(p, st, sms);
  }
  if (p.epilogue == E4B_EPI_SWIGLU) return launch_t<E4B_FMT_MXFP4, E4B_EPI_SWIGLU>(p, st, sms);
  if (p.epilogue == E4B_EPI_COMBINE) return launch_t<E4B_FMT_MXFP4, E4B_EPI_COMBINE>(p, st, sms);
  return launch_t<E4B_FMT_MXFP4, E4B_EPI_STORE>(p, st, sms);
}

}  // namespace e4b
