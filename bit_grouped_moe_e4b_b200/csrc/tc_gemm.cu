// Large-M grouped projection on the 5th-generation tensor cores.
//
// "grouped-nf4-gemm" README, intro: one launch covers all active experts;
// weights stay packed in HBM and are decoded through a table on the fly; fp32
// accumulation; bf16 epilogue. bitsandbytes PR #1984, Design: gated SiLU
// (SwiGLU) between the projections; the top-k weighted sum after the second.
//
// sm_100a design, one persistent CTA per SM, warp-specialised:
//   warp 0      TMA: packed codes of the tile's weight rows, [128 rows x 32 B]
//               per matrix and 64-wide K block, into a staging ring.
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer
//               (M = 128 weight rows, N = 256 routed rows, K = 16 per MMA).
//   warps 2-3   cp.async gather of the routed activation rows (row p of an
//               expert reads a[row_slot[p] / top_k]) into the B ring, written
//               in the 128B-swizzled K-major layout; missing rows zero-filled.
//   warps 4-11  decoders: each thread owns one weight row of a stage, builds
//               its block's 16-entry bf16 table and writes 64 decoded weights
//               as the A operand (128B-swizzled K-major) for the MMA.
//   warps 12-15 epilogue: tcgen05.ld of the fp32 accumulators, then SwiGLU
//               (gate and up accumulate in two TMEM column ranges of the same
//               lanes, so it is thread-local) or the gate-weighted combine.
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
constexpr int BK = 64;    // K per stage: one 128-byte swizzle row of bf16
constexpr int kThreads = 512;
constexpr int kMaxE = 256;
constexpr int kLoaderThreads = 64;
constexpr int kDecoderThreads = 256;
constexpr int kEpiThreads = 128;
constexpr uint32_t kATileBytes = BM * BK * 2;   // 16 KB
constexpr uint32_t kBTileBytes = BN * BK * 2;   // 32 KB
constexpr uint32_t kCTileBytes = BM * BK / 2;   // 4 KB packed codes

template <int NMAT>
struct Cfg {
  static constexpr int NS = NMAT == 2 ? 3 : 4;
  static constexpr uint32_t kA = 0;
  static constexpr uint32_t kB = kA + NS * NMAT * kATileBytes;
  static constexpr uint32_t kC = kB + NS * kBTileBytes;
  static constexpr uint32_t kMisc = kC + NS * NMAT * kCTileBytes;
  // misc: barriers, then scalars, then the expert tables
  static constexpr uint32_t kBars = kMisc;                      // (4*NS + 2) x 8 B
  static constexpr uint32_t kScal = kBars + (4 * NS + 2) * 8;   // 16 B
  static constexpr uint32_t kAct = kScal + 16;                  // kMaxE x 4
  static constexpr uint32_t kPre = kAct + kMaxE * 4;            // (kMaxE + 1) x 4
  static constexpr uint32_t kEnd = kPre + (kMaxE + 1) * 4;
  static constexpr uint32_t kSmemBytes = kEnd + 1024;           // + alignment slack
  static constexpr uint32_t kTmemCols = NMAT * BN;              // 256 or 512
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
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmap_codes, GemmProblem p) {
  constexpr int NMAT = (EPI == E4B_EPI_SWIGLU) ? 2 : 1;
  using C = Cfg<NMAT>;
  constexpr int NS = C::NS;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBars);
  uint64_t* tma_full = bars;
  uint64_t* a_full = bars + NS;
  uint64_t* b_full = bars + 2 * NS;
  uint64_t* empty = bars + 3 * NS;
  uint64_t* acc_full = bars + 4 * NS;
  uint64_t* acc_empty = bars + 4 * NS + 1;
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
  const int64_t MT = (rows_per_mat + BM - 1) / BM;
  const int KB = int((K + BK - 1) / BK);
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
    for (int s = 0; s < NS; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&a_full[s], NMAT == 2 ? kDecoderThreads : kDecoderThreads / 2);
      mbar_init(&b_full[s], kLoaderThreads);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiThreads);
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
  const int64_t njobs = int64_t(my_tiles) * KB;  // k-blocks this CTA walks

  if (warp == 0) {
    // ---------------------------------------------------------- TMA codes
    if (lane == 0) {
      int64_t i = 0;
      for (int j = 0; j < my_tiles && !*s_abort; ++j) {
        const Tile T = sc.tile(int(blockIdx.x) + j * int(gridDim.x));
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int s = int(i % NS);
          const uint32_t ph = uint32_t(i / NS) & 1u;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, s_abort)) {
            give_up();
            break;
          }
          mbar_arrive_expect_tx(&tma_full[s], NMAT * kCTileBytes);
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const int64_t row = int64_t(T.e) * N + m * rows_per_mat + T.mt * BM;
            tma_load_2d(smem + C::kC + (s * NMAT + m) * kCTileBytes, &tmap_codes, &tma_full[s],
                        kb * (BK / 2), int32_t(row));
          }
        }
      }
      // Drain: every load issued must land before the CTA can exit.
      const int64_t first = i > NS ? i - NS : 0;
      for (int64_t q = first; q < i; ++q)
        mbar_wait_bounded(&tma_full[q % NS], uint32_t(q / NS) & 1u, kWaitPolls, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      int64_t i = 0;
      uint64_t* last_bar = nullptr;
      uint32_t last_ph = 0;
      for (int j = 0; j < my_tiles && !*s_abort; ++j) {
        if (!mbar_wait_bounded(acc_empty, (uint32_t(j) & 1u) ^ 1u, limit, s_abort)) {
          give_up();
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int s = int(i % NS);
          const uint32_t ph = uint32_t(i / NS) & 1u;
          if (!mbar_wait_bounded(&a_full[s], ph, limit, s_abort) ||
              !mbar_wait_bounded(&b_full[s], ph, limit, s_abort)) {
            give_up();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t bbase = smem_u32(smem + C::kB + s * kBTileBytes);
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const uint32_t abase = smem_u32(smem + C::kA + (s * NMAT + m) * kATileBytes);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              mma_bf16_ss(tmem + uint32_t(m * BN), sw128_kmajor_desc(abase + kk * 32),
                          sw128_kmajor_desc(bbase + kk * 32), idesc, (kb | kk) ? 1u : 0u);
            }
          }
          mma_commit(&empty[s]);
          last_bar = &empty[s];
          last_ph = ph;
        }
        if (!ok) break;
        mma_commit(acc_full);
        last_bar = acc_full;
        last_ph = uint32_t(j) & 1u;
      }
      // Drain: the MMAs issued so far must finish before TMEM is freed.
      if (*s_abort && last_bar) mbar_wait_bounded(last_bar, last_ph, kWaitPolls, nullptr);
    }
  } else if (warp < 4) {
    // ------------------------------------------- activation rows (B operand)
    const int lt = tid - 64;  // 0..63
    const uint16_t* src[4];
    int64_t i = 0;
    int64_t signaled = 0;
    constexpr int LAG = NS - 1;
    bool aborted = false;
    for (int j = 0; j < my_tiles && !aborted; ++j) {
      const Tile T = sc.tile(int(blockIdx.x) + j * int(gridDim.x));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t pr = T.p0 + lt + 64 * q;
        src[q] = nullptr;
        if (pr < T.p1) {
          const int64_t ar = p.row_slot ? int64_t(p.row_slot[pr] / p.top_k) : pr;
          src[q] = p.a + ar * p.lda;
        }
      }
      for (int kb = 0; kb < KB; ++kb, ++i) {
        const int s = int(i % NS);
        const uint32_t ph = uint32_t(i / NS) & 1u;
        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, s_abort)) {
          give_up();
          aborted = true;
          break;
        }
        uint8_t* bt = smem + C::kB + s * kBTileBytes;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = lt + 64 * q;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int64_t k = int64_t(kb) * BK + c * 8;
            const bool v = src[q] != nullptr && k < K;
            cp_async_16(bt + r * 128 + ((c ^ (r & 7)) << 4), v ? (const void*)(src[q] + k) : (const void*)p.a,
                        v ? 16u : 0u);
          }
        }
        cp_async_commit();
        if (i - signaled >= LAG) {
          cp_async_wait<LAG>();
          fence_proxy_async_smem();
          mbar_arrive(&b_full[signaled % NS]);
          ++signaled;
        }
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    if (!aborted) {
      for (; signaled < i; ++signaled) mbar_arrive(&b_full[signaled % NS]);
    }
  } else if (warp < 12) {
    // ------------------------------------------------ decoders (A operand)
    const int d = tid - 128;                  // 0..255
    const int m = NMAT == 2 ? (d >> 7) : 0;   // matrix (gate / up)
    const int r = d & 127;                    // row within the tile
    const int grp = NMAT == 2 ? 0 : (d >> 7); // NMAT == 1: two groups take alternate k-blocks
    const int step = NMAT == 2 ? 1 : 2;
    const uint8_t* scales = static_cast<const uint8_t*>(p.scales);
    const int64_t sstride = FMT == E4B_FMT_NF4 ? (K / 64) * 4 : (K / 32);

    // Scale of this thread's row at job i (k-block i % KB of its tile).
    int cached_j = -1;
    const uint8_t* srow = nullptr;
    auto scale_at = [&](int64_t i, int& cj, const uint8_t*& sr) -> uint32_t {
      if (i >= njobs) return 0u;
      const int j = int(i / KB);
      const int kb = int(i % KB);
      if (j != cj) {
        cj = j;
        const Tile T = sc.tile(int(blockIdx.x) + j * int(gridDim.x));
        const int64_t n = T.mt * BM + r;
        sr = n < rows_per_mat ? scales + (int64_t(T.e) * N + m * rows_per_mat + n) * sstride : nullptr;
      }
      if (!sr) return 0u;
      if constexpr (FMT == E4B_FMT_NF4) {
        return __float_as_uint(__ldg(reinterpret_cast<const float*>(sr) + kb));
      } else {
        const int64_t b0 = int64_t(kb) * 2;
        const uint32_t lo = b0 < K / 32 ? uint32_t(__ldg(sr + b0)) : 0u;
        const uint32_t hi = b0 + 1 < K / 32 ? uint32_t(__ldg(sr + b0 + 1)) : 0u;
        return lo | (hi << 8);
      }
    };
    int cj2 = -1;
    const uint8_t* sr2 = nullptr;
    int64_t i = grp;
    uint32_t sc1 = scale_at(i, cached_j, srow);
    uint32_t sc2 = scale_at(i + step, cj2, sr2);
    for (; i < njobs; i += step) {
      const uint32_t cur = sc1;
      sc1 = sc2;
      sc2 = scale_at(i + 2 * step, cj2, sr2);
      const int s = int(i % NS);
      const uint32_t ph = uint32_t(i / NS) & 1u;
      if (!mbar_wait_bounded(&tma_full[s], ph, limit, s_abort)) {
        give_up();
        break;
      }
      const uint4* crow = reinterpret_cast<const uint4*>(smem + C::kC + (s * NMAT + m) * kCTileBytes + r * 32);
      const uint4 c0 = crow[0];
      const uint4 c1 = crow[1];
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      uint8_t* arow = smem + C::kA + (s * NMAT + m) * kATileBytes + r * 128;
      Lut L;
      lut_build<FMT>(L, __uint_as_float(cur), cur & 0xFFu);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (FMT == E4B_FMT_MXFP4 && c == 4) lut_build<FMT>(L, 0.f, (cur >> 8) & 0xFFu);
        uint32_t o[4];
        lut_decode8<FMT>(L, words[c], o);
        *reinterpret_cast<uint4*>(arow + ((c ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&a_full[s]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int rloc = q * 32 + lane;
    for (int j = 0; j < my_tiles; ++j) {
      if (!mbar_wait_bounded(acc_full, uint32_t(j) & 1u, limit, s_abort)) {
        give_up();
        break;
      }
      tc_fence_after();
      const Tile T = sc.tile(int(blockIdx.x) + j * int(gridDim.x));
      const int64_t n = T.mt * BM + rloc;
      const bool nvalid = n < rows_per_mat;
      const uint32_t lane_base = tmem + (uint32_t(q * 32) << 16);
      for (int cc = 0; cc < BN / 16; ++cc) {
        uint32_t g[16];
        uint32_t u[16];
        tmem_ld_32x32b_x16(lane_base + uint32_t(cc * 16), g);
        if constexpr (NMAT == 2) tmem_ld_32x32b_x16(lane_base + uint32_t(BN + cc * 16), u);
        tmem_ld_wait();
        const int64_t pbase = T.p0 + cc * 16;
        if (!nvalid || pbase >= T.p1) continue;
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int64_t pr = pbase + t;
          if (pr >= T.p1) break;
          const float gv = __uint_as_float(g[t]);
          if constexpr (EPI == E4B_EPI_SWIGLU) {
            const float hv = silu_mul(gv, __uint_as_float(u[t]));
            static_cast<uint16_t*>(p.out)[pr * p.ldo + n] = to_bf16_bits(hv);
          } else if constexpr (EPI == E4B_EPI_STORE) {
            static_cast<uint16_t*>(p.out)[pr * p.ldo + n] = to_bf16_bits(gv);
          } else {
            const int32_t slot = p.out_slot ? p.out_slot[pr] : int32_t(pr);
            const int64_t tok = slot / p.top_k;
            atomicAdd(static_cast<float*>(p.out) + tok * p.ldo + n, p.gates[slot] * gv);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
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
  // Packed codes viewed as a 2-D byte tensor [E*N rows, K/2 bytes].
  CUtensorMap tmap;
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cudaErrorInitializationError;
  const cuuint64_t gdim[2] = {cuuint64_t(p.K / 2), cuuint64_t(int64_t(p.E) * p.N)};
  const cuuint64_t gstride[1] = {cuuint64_t(p.K / 2)};
  const cuuint32_t box[2] = {BK / 2, BM};
  const cuuint32_t estride[2] = {1, 1};
  CUresult cr = enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p.codes), gdim,
                    gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;

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
  const int64_t MT = (rows_per_mat + BM - 1) / BM;
  const int64_t max_tiles = MT * ((p.R_max + BN - 1) / BN + p.E);
  int grid = int(max_tiles < sms ? max_tiles : sms);
  if (grid < 1) grid = 1;
  kern<<<grid, kThreads, C::kSmemBytes, st>>>(tmap, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_gemm(const GemmProblem& p, cudaStream_t st, int sms) {
  if (p.E > kMaxE) return cudaErrorInvalidValue;
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
