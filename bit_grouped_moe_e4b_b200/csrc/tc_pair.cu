// Large-M grouped projection on SM pairs (tcgen05.mma.cta_group::2).
//
// "grouped-nf4-gemm" README, intro: one launch covers all active experts;
// weights stay packed in HBM and are decoded through a table on the fly; fp32
// accumulation; bf16 epilogue. bitsandbytes PR #1984, Design: gated SiLU
// (SwiGLU) between the projections; the top-k weighted sum after the second.
//
// Why pairs. A one-SM tcgen05.mma of M=128, N=256, K=16 reads 12 KB of
// shared memory in the 128 clocks it runs, ~96 of the ~128 bytes per clock an
// SM's shared memory serves; the TMA fills of the activation tiles and the
// decoders' stores of the weight tiles then exceed the budget, and the kernel
// is bound by shared-memory bandwidth, not by the tensor pipe (measured on
// the one-SM kernel: ~790 busy MMA clocks per 64-wide K job where the MMAs
// alone need 512). Two CTAs on two SMs issue one M=256 MMA: each holds its
// own 128 weight rows and HALF of the 256 activation rows, and each half is
// read once for both SMs (~64 bytes per clock per SM). The activation fill
// per SM halves too. For gate_up the pair's 256 weight rows are the gate AND
// up rows of 128 features, so one accumulator is 256 TMEM columns and two fit:
// the epilogue of one tile overlaps the MMAs of the next.
//
// Roles of each CTA (512 threads; the even CTA of the pair is the leader):
//   warp 0       packed codes of this CTA's 128 weight rows -> codes ring (TMA)
//   warp 1       TMEM (both CTAs allocate as a pair); the leader's lane 0
//                issues the pair MMAs and their commits (multicast to both)
//   warp 2       this CTA's 128 activation rows -> the stage's B tile (TMA,
//                128B swizzle), completing on this CTA's b_full barrier
//   warp 3       forwards each landed B tile to the leader's full barrier
//                (one arrival; remote for the odd CTA)
//   warps 4-11   decoders: two groups of 128 threads take alternate jobs; a
//                thread decodes one weight row of the job (64 weights, its
//                block's 16-entry table) into the stage's A tile; one arrival
//                per warp on the leader's full barrier (remote for the odd CTA)
//   warps 12-15  epilogue: tcgen05.ld of this CTA's 128 accumulator lanes
//                over the tile's 256 routed rows, then the projection's
//                epilogue; one arrival per warp on the leader's acc_empty
// Rings: codes (local), and the operand stages (an A and a B tile in each
// CTA): one full barrier per stage in the leader counts both CTAs' decoder
// warps and both CTAs' landed activation tiles, so the MMA thread waits on ONE
// barrier per job (each mbarrier wait costs ~100+ clocks next to the MMAs'
// shared-memory traffic, and the MMA thread cannot run ahead of the tensor
// pipe to hide it); one empty barrier per stage in each CTA, arrived on by
// the leader's commit. Every wait is bounded; a wait that
// gives up records E4B_ERR_DEVICE_TIMEOUT and stops this CTA's roles (the
// other CTA's waits then give up too). Both CTAs meet at a cluster barrier
// before TMEM is freed and before either exits, so no remote arrival or MMA
// read ever targets a CTA that has left.
//
// The input gradient (kEpiDgrad, e4b_grouped_dgrad) runs here too: the MMA's
// M then runs over the weight's columns (each CTA 128 of them, its A tile
// MN-major as in the one-SM kernel) and its reduction over the weight's rows.
//
// gate_up rows in a CTA (SWIGLU): the pair covers features F .. F+127, the
// CTA of rank r features F + 64r .. F + 64r + 63. Lane quarter q (lanes
// 32q .. 32q+31) holds features 16q .. 16q+15 of the CTA: gate rows in its
// first 16 lanes, the same features' up rows in the last 16. The epilogue
// pairs lane l with lane l ^ 16 by a shuffle; each lane computes half of the
// 16 routed rows of a column chunk.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace e4b {
namespace {

using namespace sm100;

constexpr int PM = 128;   // weight rows per CTA (the pair's MMA has M = 256)
constexpr int PN = 256;   // routed rows per tile (MMA N); each CTA stages 128
constexpr int PK = 64;    // K per job
constexpr int kPThreads = 512;
constexpr int kPMaxE = 256;
constexpr int kPDec = 128;       // decoder threads per job (one group)
constexpr int kPEpi = 128;
constexpr uint32_t kPATile = PM * PK * 2;         // 16 KB decoded weights
constexpr uint32_t kPBTile = (PN / 2) * PK * 2;   // 16 KB of this CTA's activation rows
constexpr uint32_t kPCTile = PM * PK / 2;         // 4 KB packed codes
constexpr int kPScalePrefetch = 4;
// wait sites recorded in the status words when a wait gives up
enum { kSiteCodesEmpty = 101, kSiteAccEmpty, kSiteFull, kSiteBEmpty, kSiteCodesFull, kSiteAEmpty, kSiteAccFull, kSiteBFull };

struct PCfg {
  // codes stages: the packed codes are the HBM stream, and 16 stages of 4 KB
  // (~8 jobs per decoder group) hide its latency (4 stages cost gate_up 55%);
  // operand stages: an A and a B tile each (4 or 6 measured alike)
  static constexpr int CS = 16;
  static constexpr int S = 4;
  static constexpr uint32_t kA = 0;
  static constexpr uint32_t kB = kA + S * kPATile;
  static constexpr uint32_t kC = kB + S * kPBTile;
  static constexpr uint32_t kMisc = kC + CS * kPCTile;
  // c_full, c_empty, full, empty, b_full, acc_full, acc_empty
  static constexpr int kNumBars = 2 * CS + 3 * S + 4;
  static constexpr uint32_t kBars = kMisc;
  static constexpr uint32_t kScal = kBars + kNumBars * 8;
  static constexpr uint32_t kAct = kScal + 16;
  static constexpr uint32_t kPre = kAct + kPMaxE * 4;
  static constexpr uint32_t kGate = (kPre + (kPMaxE + 1) * 4 + 15) / 16 * 16;
  static constexpr uint32_t kTok = kGate + 4 * PN * 4;
  static constexpr uint32_t kProg = kTok + 4 * PN * 4;          // 8 progress words
  static constexpr uint32_t kEnd = kProg + 32;
  static constexpr uint32_t kSmemBytes = kEnd + 1024;
  static constexpr uint32_t kTmemCols = 512;   // two accumulators of 256 columns
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // the two decoder groups take alternate jobs: a slot must belong to one group
  static_assert(CS % 2 == 0 && S % 2 == 0, "decoder groups own alternate slots");
};

struct PTile {
  int e;
  int64_t mt, p0, p1;
};

// The static tile list of the pair: per active expert, (block of 256 weight
// rows, or 128 gate/up features) x (block of 256 routed rows), routed-row
// blocks fastest.
struct PSched {
  const int32_t* act;
  const int32_t* pre;
  int nact;
  int total;
  const int64_t* offsets;

  __device__ PTile tile(int t) const {
    int lo = 0, hi = nact - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= t) lo = mid;
      else hi = mid - 1;
    }
    const int e = act[lo];
    const int64_t b = offsets[e];
    const int64_t end = offsets[e + 1];
    const int64_t ntn = (end - b + PN - 1) / PN;
    const int64_t local = t - pre[lo];
    PTile r;
    r.e = e;
    r.mt = local / ntn;
    r.p0 = b + (local % ntn) * PN;
    r.p1 = end;
    return r;
  }
};

template <int FMT, int EPI>
__global__ void __launch_bounds__(kPThreads, 1)
tc_pair_kernel(const __grid_constant__ CUtensorMap tmap_codes,
               const __grid_constant__ CUtensorMap tmap_act, GemmProblem p) {
  constexpr int NMAT = (EPI == E4B_EPI_SWIGLU) ? 2 : 1;
  constexpr bool DG = EPI == kEpiDgrad;
  using C = PCfg;
  constexpr int CS = C::CS;
  constexpr int S = C::S;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBars);
  uint64_t* c_full = bars;
  uint64_t* c_empty = c_full + CS;
  uint64_t* full = c_empty + CS;      // leader's: both CTAs' decoders and B bytes
  uint64_t* empty = full + S;         // each CTA's, arrived on by the leader's commit
  uint64_t* b_full = empty + S;       // each CTA's own B copy
  uint64_t* acc_full = b_full + S;
  uint64_t* acc_empty = acc_full + 2; // leader's counts both CTAs' epilogues
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kScal);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kScal + 4);
  int32_t* s_n = reinterpret_cast<int32_t*>(smem + C::kScal + 8);
  int32_t* s_act = reinterpret_cast<int32_t*>(smem + C::kAct);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + C::kPre);
  // progress words, read by a wait that gives up: [0..3] tiles each epilogue
  // warp has released, [4] jobs decoded by the first decoder warp, [5] jobs
  // whose B tile this CTA has requested, [6] tiles the MMA has committed
  volatile int32_t* s_prog = reinterpret_cast<volatile int32_t*>(smem + C::kProg);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = int(blockIdx.x >> 1);
  const int npairs = int(gridDim.x >> 1);
  const int64_t N = p.N;
  const int64_t K = p.K;
  const int64_t rows_per_mat = NMAT == 2 ? N / 2 : N;
  // dgrad: the MMA's M runs over the weight's columns, its reduction over the
  // weight's rows
  const int64_t Mdim = DG ? K : rows_per_mat;
  const int64_t Kred = DG ? N : K;
  constexpr int64_t TM = NMAT == 2 ? 128 : 256;   // M rows (features) per pair tile
  const int64_t MT = (Mdim + TM - 1) / TM;
  const int KB = int((Kred + PK - 1) / PK);
  const bool il = NMAT == 2 && p.layout == E4B_GATE_UP_INTERLEAVED;
  const uint32_t limit = (p.flags & E4B_FLAG_TEST_TIMEOUT) ? 0u : kWaitPolls;

  if (p.zero_buf) {
    for (int64_t i = int64_t(blockIdx.x) * kPThreads + tid; i < p.zero_count;
         i += int64_t(gridDim.x) * kPThreads)
      p.zero_buf[i] = 0.f;
  }

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
          v = int(((rows + PN - 1) / PN) * MT);
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
  PSched sc{s_act, s_pre, *s_n, s_pre[*s_n], p.offsets};
  if (pair >= sc.total) return;  // no tile for this pair (uniform over both CTAs)

  if (tid == 0) {
    for (int s = 0; s < CS; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_empty[s], kPDec);
    }
    for (int s = 0; s < S; ++s) {
      // one arrival per decoder warp of both CTAs, plus one per CTA for its
      // landed B tile
      mbar_init(&full[s], 2 * (kPDec / 32) + 2);
      mbar_init(&empty[s], 1);
      mbar_init(&b_full[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * (kPEpi / 32));  // one per epilogue warp of both CTAs
    }
    *s_abort = 0;
    for (int w = 0; w < 8; ++w) s_prog[w] = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc_pair(s_tmem, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  // A wait that gave up: the error code, and (first one only) status[2] =
  // the site, [3] = the CTA, [4] = the job (or tile) index it waited for.
  auto give_up_at = [&](int site, int64_t job) {
    // recorded before the abort flag is raised, so the first wait that gave
    // up is the one recorded (the flag makes the CTA's other waits give up)
    record_status(p.status, E4B_ERR_DEVICE_TIMEOUT);
    if (p.status && atomicCAS(p.status + 2, 0, site) == 0) {
      p.status[3] = int32_t(blockIdx.x);
      p.status[4] = int32_t(job);
      // [5]: this CTA's epilogue warps' released tiles (a byte each), [6] the
      // other CTA's, [7] this CTA's decoded / requested jobs and MMA tiles
      uint32_t mine = 0, other = 0;
      const uint32_t peer_prog = cluster_addr(const_cast<int32_t*>(s_prog), rank ^ 1u);
      for (int w = 0; w < 4; ++w) {
        uint32_t v;
        asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(peer_prog + 4u * w));
        mine |= (uint32_t(s_prog[w]) & 0xFFu) << (8 * w);
        other |= (v & 0xFFu) << (8 * w);
      }
      p.status[5] = int32_t(mine);
      p.status[6] = int32_t(other);
      p.status[7] = int32_t((uint32_t(s_prog[4]) & 0xFFFu) | ((uint32_t(s_prog[5]) & 0xFFFu) << 12) |
                            ((uint32_t(s_prog[6]) & 0xFFu) << 24));
    }
    *s_abort = 1;
  };

  const int my_tiles = (sc.total - pair + npairs - 1) / npairs;
  const int64_t njobs = int64_t(my_tiles) * KB;

  if (warp == 0) {
    // ------------------------------------------------ codes ring (TMA, local)
    if (lane == 0) {
      int64_t i = 0;
      bool aborted = false;
      for (int j = 0; j < my_tiles && !aborted; ++j) {
        const PTile T = sc.tile(pair + j * npairs);
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int s = int(i % CS);
          if (!mbar_wait_bounded(&c_empty[s], (uint32_t(i / CS) & 1u) ^ 1u, limit, s_abort)) {
            give_up_at(kSiteCodesEmpty, i);
            aborted = true;
            break;
          }
          mbar_arrive_expect_tx(&c_full[s], kPCTile);
          uint8_t* dst = smem + C::kC + s * kPCTile;
          if constexpr (DG) {
            // 64 weight rows x this CTA's 128 weight columns (64 bytes)
            tma_load_2d(dst, &tmap_codes, &c_full[s], int32_t((T.mt * TM + int64_t(rank) * 128) / 2),
                        int32_t(int64_t(T.e) * N + int64_t(kb) * PK));
          } else if constexpr (NMAT == 1) {
            tma_load_2d(dst, &tmap_codes, &c_full[s], kb * (PK / 2),
                        int32_t(int64_t(T.e) * N + T.mt * TM + int64_t(rank) * 128));
          } else {
            const int64_t f0 = T.mt * TM + int64_t(rank) * 64;   // this CTA's first feature
            if (il) {
              tma_load_3d(dst, &tmap_codes, &c_full[s], kb * (PK / 2), 0, int32_t(int64_t(T.e) * rows_per_mat + f0));
              tma_load_3d(dst + kPCTile / 2, &tmap_codes, &c_full[s], kb * (PK / 2), 1,
                          int32_t(int64_t(T.e) * rows_per_mat + f0));
            } else {
              tma_load_2d(dst, &tmap_codes, &c_full[s], kb * (PK / 2), int32_t(int64_t(T.e) * N + f0));
              tma_load_2d(dst + kPCTile / 2, &tmap_codes, &c_full[s], kb * (PK / 2),
                          int32_t(int64_t(T.e) * N + rows_per_mat + f0));
            }
          }
        }
      }
      for (int64_t q = i > CS ? i - CS : 0; q < i; ++q)
        mbar_wait_bounded(&c_full[q % CS], uint32_t(q / CS) & 1u, kWaitPolls, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- pair MMA (leader)
    if (lane == 0 && leader) {
      // dgrad: A is MN-major (bit 15, "transpose A")
      constexpr uint32_t idesc = idesc_bf16_f32(2 * PM, PN) | (DG ? (1u << 15) : 0u);
      int64_t i = 0;
      bool aborted = false;
      uint64_t* last_bar = nullptr;
      uint32_t last_ph = 0;
      for (int j = 0; j < my_tiles && !aborted; ++j) {
        const int ab = j & 1;
        if (!mbar_wait_cluster_bounded(&acc_empty[ab], (uint32_t(j >> 1) & 1u) ^ 1u, limit, s_abort)) {
          give_up_at(kSiteAccEmpty, j);
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + uint32_t(ab * PN);
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int st = int(i % S);
          const uint32_t ph = uint32_t(i / S) & 1u;
          if (!mbar_wait_cluster_bounded(&full[st], ph, limit, s_abort)) {
            give_up_at(kSiteFull, i);
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint32_t abase = smem_u32(smem + C::kA + st * kPATile);
          const uint32_t bbase = smem_u32(smem + C::kB + st * kPBTile);
#pragma unroll
          for (int kk = 0; kk < PK / 16; ++kk) {
            const uint64_t adesc = DG ? sw128_mnmajor_desc(abase + kk * 2048, 8192, 1024)
                                      : sw128_kmajor_desc(abase + kk * 32);
            mma_bf16_pair(dcol, adesc, sw128_kmajor_desc(bbase + kk * 32), idesc, (kb | kk) ? 1u : 0u);
          }
          mma_commit_pair(&empty[st]);
          last_bar = &empty[st];
          last_ph = ph;
        }
        if (aborted) break;
        mma_commit_pair(&acc_full[ab]);
        s_prog[6] = j + 1;
      }
      // Drain after an abort: the pair MMAs issued so far must finish before
      // TMEM is freed and before the other CTA (whose shared memory they
      // read) may leave. Without an abort the epilogues have waited for them.
      if (*s_abort && last_bar) mbar_wait_cluster_bounded(last_bar, last_ph, kWaitPolls, nullptr);
    }
  } else if (warp == 2) {
    // -------------------------------- this CTA's activation rows, B tiles (TMA)
    if (lane == 0) {
      int64_t i = 0;
      bool aborted = false;
      for (int j = 0; j < my_tiles && !aborted; ++j) {
        const PTile T = sc.tile(pair + j * npairs);
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int st = int(i % S);
          if (!mbar_wait_cluster_bounded(&empty[st], (uint32_t(i / S) & 1u) ^ 1u, limit, s_abort)) {
            give_up_at(kSiteBEmpty, i);
            aborted = true;
            break;
          }
          mbar_arrive_expect_tx(&b_full[st], kPBTile);
          tma_load_2d(smem + C::kB + st * kPBTile, &tmap_act, &b_full[st], kb * PK,
                      int32_t(T.p0 + int64_t(rank) * (PN / 2)));
          s_prog[5] = int32_t(i + 1);
        }
      }
      for (int64_t q = i > S ? i - S : 0; q < i; ++q)
        mbar_wait_bounded(&b_full[q % S], uint32_t(q / S) & 1u, kWaitPolls, nullptr);
    }
  } else if (warp == 3) {
    // ------------------------- each landed B tile: one arrival on the leader
    if (lane == 0) {
      for (int64_t i = 0; i < njobs; ++i) {
        const int st = int(i % S);
        if (!mbar_wait_bounded(&b_full[st], uint32_t(i / S) & 1u, limit, s_abort)) {
          give_up_at(kSiteBFull, i);
          break;
        }
        mbar_arrive_cluster(cluster_addr(&full[st], 0));
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // -------------------------------------------------- decoders (A operand)
    const int d = tid - 128;            // 0..255
    const int grp = d >> 7;             // groups take alternate jobs
    const int m = d & 127;              // row of this CTA's A tile
    // gate_up: lane quarter q = m / 32 holds features 16q..16q+15 of the CTA,
    // gate rows in its first 16 lanes and up rows in the last 16
    const int mat = NMAT == 2 ? ((m >> 4) & 1) : 0;
    const int floc = NMAT == 2 ? ((m >> 5) * 16 + (m & 15)) : m;      // feature within the CTA's 64
    const int crow = NMAT == 2 ? (mat * 64 + floc) : m;                // row of the codes stage
    // dgrad: weight row dr of the job's 64, columns 64 db .. 64 db + 63 of the CTA's 128
    const int dr = m & 63, db = m >> 6;
    const uint8_t* scales = static_cast<const uint8_t*>(p.scales);
    const int64_t sstride = FMT == E4B_FMT_NF4 ? (K / 64) * 4 : (K / 32);

    int cached_j = -1;
    const uint8_t* srow = nullptr;
    auto scale_at = [&](int64_t q) -> uint32_t {
      if (q >= njobs) return 0u;
      const int j = int(q / KB);
      const int kb = int(q % KB);
      if constexpr (DG) {
        // the absmax (or the two scale bytes) of weight row kb*64 + dr at the
        // columns 64 db.. of this CTA; zero past the weight's rows or columns
        if (j != cached_j) {
          cached_j = j;
          const PTile T = sc.tile(pair + j * npairs);
          const int64_t col0 = T.mt * TM + int64_t(rank) * 128 + 64 * db;
          srow = col0 < K ? scales + int64_t(T.e) * N * sstride + (FMT == E4B_FMT_NF4 ? (col0 / 64) * 4 : col0 / 32)
                          : nullptr;
        }
        const int64_t wr = int64_t(kb) * PK + dr;
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
        const PTile T = sc.tile(pair + j * npairs);
        int64_t n, row;
        if constexpr (NMAT == 2) {
          n = T.mt * TM + int64_t(rank) * 64 + floc;
          row = gate_up_row(p.layout, rows_per_mat, mat, n);
        } else {
          n = T.mt * TM + int64_t(rank) * 128 + m;
          row = n;
        }
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
    uint32_t ring[kPScalePrefetch];
#pragma unroll
    for (int u = 0; u < kPScalePrefetch; ++u) ring[u] = scale_at(grp + int64_t(u) * 2);

    bool aborted = false;
    for (int64_t i0 = grp; i0 < njobs && !aborted; i0 += int64_t(kPScalePrefetch) * 2) {
#pragma unroll
      for (int u = 0; u < kPScalePrefetch; ++u) {
        const int64_t i = i0 + int64_t(u) * 2;
        if (i >= njobs) break;
        const uint32_t cur = ring[u];
        ring[u] = scale_at(i + int64_t(kPScalePrefetch) * 2);
        const int cs = int(i % CS);
        // every wait of a multi-lane role gives up for the whole warp at once:
        // its lanes then never split between a warp-wide step and the exit
        if (__any_sync(0xffffffffu, !mbar_wait_bounded(&c_full[cs], uint32_t(i / CS) & 1u, limit, s_abort))) {
          give_up_at(kSiteCodesFull, i);
          aborted = true;
          break;
        }
        const uint4* cp =
            reinterpret_cast<const uint4*>(smem + C::kC + cs * kPCTile + (DG ? dr * 64 + db * 32 : crow * 32));
        const uint4 c0 = cp[0];
        const uint4 c1 = cp[1];
        // the slot's next fill is a TMA write (async proxy)
        fence_proxy_async_smem();
        mbar_arrive(&c_empty[cs]);
        const int st = int(i % S);
        if (__any_sync(0xffffffffu,
                       !mbar_wait_cluster_bounded(&empty[st], (uint32_t(i / S) & 1u) ^ 1u, limit, s_abort))) {
          give_up_at(kSiteAEmpty, i);
          aborted = true;
          break;
        }
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        // K-major: the 128-byte row m of the tile. dgrad, MN-major: the
        // 128-byte row of K index dr (8-row atoms of 1024 bytes) in the atom
        // column db (8 KB apart); the same 128B swizzle by row within the atom.
        const int sw = DG ? (dr & 7) : (m & 7);
        uint8_t* arow = smem + C::kA + st * kPATile +
                        (DG ? db * 8192 + (dr >> 3) * 1024 + (dr & 7) * 128 : m * 128);
        Lut L;
        lut_build<FMT>(L, __uint_as_float(cur), cur & 0xFFu);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (FMT == E4B_FMT_MXFP4 && c == 4) lut_build<FMT>(L, 0.f, (cur >> 8) & 0xFFu);
          uint32_t o[4];
          lut_decode8<FMT>(L, words[c], o);
          *reinterpret_cast<uint4*>(arow + ((c ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        // the pair MMA reads this tile through the async proxy, possibly from
        // the other SM: every thread fences its own stores, then one arrival
        // per warp
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cluster_addr(&full[st], 0));
        if (warp == 4 && lane == 0) s_prog[4] = int32_t(i + 1);
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int q = warp & 3;
    constexpr bool GATED = EPI == E4B_EPI_COMBINE || EPI == kEpiGatedRows;
    float* s_g = reinterpret_cast<float*>(smem + C::kGate) + q * PN;
    int32_t* s_t = reinterpret_cast<int32_t*>(smem + C::kTok) + q * PN;
    for (int j = 0; j < my_tiles; ++j) {
      const int ab = j & 1;
      const PTile T = sc.tile(pair + j * npairs);
      if constexpr (GATED) {
        __syncwarp();
        int32_t sl[PN / 32];
#pragma unroll
        for (int u = 0; u < PN / 32; ++u) {
          const int64_t pr = T.p0 + lane + 32 * u;
          sl[u] = pr < T.p1 ? (p.out_slot ? p.out_slot[pr] : int32_t(pr)) : -1;
        }
#pragma unroll
        for (int u = 0; u < PN / 32; ++u) {
          s_g[lane + 32 * u] = sl[u] >= 0 ? p.gates[sl[u]] : 0.f;
          s_t[lane + 32 * u] = sl[u] >= 0 ? sl[u] / p.top_k : 0;
        }
        __syncwarp();
      }
      if (__any_sync(0xffffffffu, !mbar_wait_cluster_bounded(&acc_full[ab], uint32_t(j >> 1) & 1u, limit, s_abort))) {
        give_up_at(kSiteAccFull, j);
        break;
      }
      tc_fence_after();
      const uint32_t lane_base = tmem + (uint32_t(q * 32) << 16) + uint32_t(ab * PN);
      if constexpr (NMAT == 2) {
        // lane l: feature f of gate (l < 16) or up (l >= 16); its partner l ^ 16
        const bool isup = lane >= 16;
        const int64_t f = T.mt * TM + int64_t(rank) * 64 + q * 16 + (lane & 15);
        const bool fvalid = f < rows_per_mat;
        float bmine = 0.f;
        if (p.bias && fvalid)
          bmine = p.bias[int64_t(T.e) * N + gate_up_row(p.layout, rows_per_mat, isup ? 1 : 0, f)];
        const float bother = __shfl_xor_sync(0xffffffffu, bmine, 16);
        const float bg = isup ? bother : bmine;
        const float bu = isup ? bmine : bother;
        uint16_t* out = static_cast<uint16_t*>(p.out);
        for (int cc = 0; cc < PN / 16; ++cc) {
          const int64_t pbase = T.p0 + cc * 16;
          if (pbase >= T.p1) break;  // uniform
          uint32_t v[16];
          tmem_ld_32x32b_x16(lane_base + uint32_t(cc * 16), v);
          tmem_ld_wait();
          // lanes < 16 keep rows 0-7 of the chunk (gate here, up from the
          // partner); lanes >= 16 rows 8-15 (gate from the partner, up here)
          float g[8], u[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const uint32_t send = isup ? v[t] : v[8 + t];
            const float recv = __uint_as_float(__shfl_xor_sync(0xffffffffu, send, 16));
            g[t] = isup ? recv : __uint_as_float(v[t]);
            u[t] = isup ? __uint_as_float(v[8 + t]) : recv;
          }
          if (!fvalid) continue;
          const int64_t r0 = pbase + (isup ? 8 : 0);
          uint16_t* o = out + r0 * p.ldo + f;
          if (r0 + 8 <= T.p1) {
            // all 8 rows valid (every chunk but an expert's last): no per-row check
#pragma unroll
            for (int t = 0; t < 8; ++t)
              o[t * p.ldo] = to_bf16_bits(glu_act(p.act, g[t] + bg, u[t] + bu, p.alpha, p.limit));
          } else {
#pragma unroll
            for (int t = 0; t < 8; ++t)
              if (r0 + t < T.p1)
                o[t * p.ldo] = to_bf16_bits(glu_act(p.act, g[t] + bg, u[t] + bu, p.alpha, p.limit));
          }
        }
      } else {
        const int64_t n = T.mt * TM + int64_t(rank) * 128 + q * 32 + lane;
        const bool nvalid = n < Mdim;
        const float b0 = (!DG && p.bias && nvalid) ? p.bias[int64_t(T.e) * N + n] : 0.f;
        for (int cc = 0; cc < PN / 16; ++cc) {
          const int64_t pbase = T.p0 + cc * 16;
          if (pbase >= T.p1) break;  // uniform
          uint32_t g[16];
          tmem_ld_32x32b_x16(lane_base + uint32_t(cc * 16), g);
          tmem_ld_wait();
          if (!nvalid) continue;
          if constexpr (EPI == kEpiGatedRows) {
            if (pbase + 16 <= T.p1) {
              // all 16 rows valid: the gates as four 16-byte shared loads (the
              // same address for every lane), no per-row check
              float gw[16];
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const float4 q4 = reinterpret_cast<const float4*>(s_g + cc * 16)[v];
                gw[4 * v] = q4.x;
                gw[4 * v + 1] = q4.y;
                gw[4 * v + 2] = q4.z;
                gw[4 * v + 3] = q4.w;
              }
              float* o = static_cast<float*>(p.out) + pbase * p.ldo + n;
#pragma unroll
              for (int t = 0; t < 16; ++t) o[t * p.ldo] = gw[t] * (__uint_as_float(g[t]) + b0);
              continue;
            }
          }
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int64_t pr = pbase + t;
            if (pr >= T.p1) break;
            const float gv = __uint_as_float(g[t]) + b0;
            if constexpr (EPI == E4B_EPI_STORE || DG) {
              static_cast<uint16_t*>(p.out)[pr * p.ldo + n] = to_bf16_bits(gv);
            } else if constexpr (EPI == kEpiGatedRows) {
              static_cast<float*>(p.out)[pr * p.ldo + n] = s_g[cc * 16 + t] * gv;
            } else {
              const int64_t tok = s_t[cc * 16 + t];
              atomicAdd(static_cast<float*>(p.out) + tok * p.ldo + n, s_g[cc * 16 + t] * gv);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_cluster(cluster_addr(&acc_empty[ab], 0));
        s_prog[q] = j + 1;
      }
    }
  }

  // Both CTAs meet here: every remote arrival and every pair MMA that reads
  // either CTA's shared memory is done before TMEM is freed or a CTA leaves.
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, C::kTmemCols);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn pair_encode_fn() {
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
cudaError_t launch_pair_t(const GemmProblem& p, cudaStream_t st, int sms) {
  constexpr int NMAT = (EPI == E4B_EPI_SWIGLU) ? 2 : 1;
  constexpr bool DG = EPI == kEpiDgrad;
  using C = PCfg;
  EncodeTiledFn enc = pair_encode_fn();
  if (!enc) return cudaErrorInitializationError;
  // Packed codes [E*N rows, K/2 bytes]: boxes of this CTA's 128 weight rows,
  // or of 64 gate and 64 up rows (interleaved rows: the 3-D view [E*I, 2, K/2]).
  CUtensorMap tmap_codes;
  CUresult cr;
  if (DG) {
    // boxes of 64 weight rows x 128 weight columns (64 bytes)
    const cuuint64_t gdim[2] = {cuuint64_t(p.K / 2), cuuint64_t(int64_t(p.E) * p.N)};
    const cuuint64_t gstride[1] = {cuuint64_t(p.K / 2)};
    const cuuint32_t box[2] = {PM / 2, PK};
    const cuuint32_t estride[2] = {1, 1};
    cr = enc(&tmap_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p.codes), gdim, gstride, box,
             estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else if (NMAT == 2 && p.layout == E4B_GATE_UP_INTERLEAVED) {
    const cuuint64_t gdim[3] = {cuuint64_t(p.K / 2), 2, cuuint64_t(int64_t(p.E) * (p.N / 2))};
    const cuuint64_t gstride[2] = {cuuint64_t(p.K / 2), cuuint64_t(p.K)};
    const cuuint32_t box[3] = {PK / 2, 1, 64};
    const cuuint32_t estride[3] = {1, 1, 1};
    cr = enc(&tmap_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(p.codes), gdim, gstride, box,
             estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t gdim[2] = {cuuint64_t(p.K / 2), cuuint64_t(int64_t(p.E) * p.N)};
    const cuuint64_t gstride[1] = {cuuint64_t(p.K / 2)};
    const cuuint32_t box[2] = {PK / 2, NMAT == 2 ? 64u : 128u};
    const cuuint32_t estride[2] = {1, 1};
    cr = enc(&tmap_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p.codes), gdim, gstride, box,
             estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  // Activations [R_max, K] bf16 (row stride lda; dgrad: dy [R_max, N]),
  // 128-row boxes, 128B swizzle.
  CUtensorMap tmap_act;
  {
    const cuuint64_t gdim[2] = {cuuint64_t(DG ? p.N : p.K), cuuint64_t(p.R_max)};
    const cuuint64_t gstride[1] = {cuuint64_t(p.lda) * 2};
    const cuuint32_t box[2] = {PK, PN / 2};
    const cuuint32_t estride[2] = {1, 1};
    cr = enc(&tmap_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(p.a), gdim, gstride, box,
             estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }

  auto kern = tc_pair_kernel<FMT, EPI>;
  static int configured_dev = -1;
  static int max_pairs = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (configured_dev != dev) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::kSmemBytes));
    if (err != cudaSuccess) return err;
    // pairs that can be resident at once (one CTA per SM, both CTAs of a pair
    // in one GPC): the persistent grid never exceeds it
    cfg.gridDim = dim3(2 * (sms / 2));
    int n = 0;
    err = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (err != cudaSuccess) return err;
    if (n < 1) return cudaErrorInvalidConfiguration;
    max_pairs = n;
    configured_dev = dev;
  }
  const int64_t rows_per_mat = NMAT == 2 ? p.N / 2 : p.N;
  const int64_t TM = NMAT == 2 ? 128 : 256;
  const int64_t MT = ((DG ? p.K : rows_per_mat) + TM - 1) / TM;
  const int64_t max_tiles = MT * ((p.R_max + PN - 1) / PN + p.E);
  int np = int(max_tiles < max_pairs ? max_tiles : max_pairs);
  if (np < 1) np = 1;
  cfg.gridDim = dim3(2 * np);
  return cudaLaunchKernelEx(&cfg, kern, tmap_codes, tmap_act, p);
}

}  // namespace

bool tc_pair_supported(const GemmProblem& p) {
  // contiguous activation rows (the gathered form stays on the one-SM kernel)
  return p.row_slot == nullptr && p.E <= kPMaxE && (p.flags & E4B_FLAG_TC_SINGLE_SM) == 0;
}

cudaError_t launch_tc_pair(const GemmProblem& p, cudaStream_t st, int sms) {
  if (!tc_pair_supported(p)) return cudaErrorInvalidValue;
  if (p.epilogue == kEpiDgrad)
    return p.fmt == E4B_FMT_NF4 ? launch_pair_t<E4B_FMT_NF4, kEpiDgrad>(p, st, sms)
                                : launch_pair_t<E4B_FMT_MXFP4, kEpiDgrad>(p, st, sms);
  if (p.epilogue == kEpiGatedRows)
    return p.fmt == E4B_FMT_NF4 ? launch_pair_t<E4B_FMT_NF4, kEpiGatedRows>(p, st, sms)
                                : launch_pair_t<E4B_FMT_MXFP4, kEpiGatedRows>(p, st, sms);
  if (p.fmt == E4B_FMT_NF4) {
    if (p.epilogue == E4B_EPI_SWIGLU) return launch_pair_t<E4B_FMT_NF4, E4B_EPI_SWIGLU>(p, st, sms);
    if (p.epilogue == E4B_EPI_COMBINE) return launch_pair_t<E4B_FMT_NF4, E4B_EPI_COMBINE>(p, st, sms);
    return launch_pair_t<E4B_FMT_NF4, E4B_EPI_STORE>(p, st, sms);
  }
  if (p.epilogue == E4B_EPI_SWIGLU) return launch_pair_t<E4B_FMT_MXFP4, E4B_EPI_SWIGLU>(p, st, sms);
  if (p.epilogue == E4B_EPI_COMBINE) return launch_pair_t<E4B_FMT_MXFP4, E4B_EPI_COMBINE>(p, st, sms);
  return launch_pair_t<E4B_FMT_MXFP4, E4B_EPI_STORE>(p, st, sms);
}

}  // namespace e4b
