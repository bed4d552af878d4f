// Small-M grouped projection: few routed rows per expert, so every packed
// weight byte is read once and the layer is bound by HBM and by the decode.
//
// "grouped-nf4-gemm" README, intro: one launch over all active experts, LUT
// decode in registers, blockwise scale, fp32 accumulation, bf16 epilogue;
// the decode glue's swiglu and combine are fused into the two epilogues.
//
// Design (sm_100a): a warp owns 16 weight rows of one expert (32 for the
// SwiGLU gate/up pair) and streams them along K in chunks of 256 weights; each
// lane loads 32 contiguous packed bytes per row (one NF4 block, two MXFP4
// blocks) with 16-byte non-allocating loads, builds that block's 16-entry
// bf16 table, and decodes straight into the A fragment of an
// m16n8k16 bf16 MMA with fp32 accumulators. The K index is permuted inside
// each chunk so that a lane's fragment columns are its own consecutive
// weights; the activation fragment follows the same permutation (4
// consecutive bf16 per lane and step). Decoded weights never touch shared
// memory: staging them there would cost more shared bandwidth than the
// tensor work saves at these row counts.
#include "common.cuh"
#include "launch.h"

namespace e4b {

constexpr int kGemvWarps = 8;
constexpr int kMaxExpertsSmem = 1024;

E4B_DEV void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Per-lane state for one weight row (16-row tile row g or g+8) within a chunk.
struct RowChunk {
  uint32_t w[8];  // 64 packed codes
  float absmax;   // NF4 block scale
  uint32_t mx;    // MXFP4: two scale bytes (block 0 low byte, block 1 next)
};

template <int FMT>
E4B_DEV void load_row_chunk(RowChunk& rc, const uint8_t* crow, const uint8_t* srow, int64_t kl,
                            int64_t K) {
  const int64_t left = K - kl;
  if (left >= 64) {
    const uint4 q0 = ldg_nc_v4(crow + kl / 2);
    const uint4 q1 = ldg_nc_v4(crow + kl / 2 + 16);
    rc.w[0] = q0.x; rc.w[1] = q0.y; rc.w[2] = q0.z; rc.w[3] = q0.w;
    rc.w[4] = q1.x; rc.w[5] = q1.y; rc.w[6] = q1.z; rc.w[7] = q1.w;
  } else if (left >= 32) {
    const uint4 q0 = ldg_nc_v4(crow + kl / 2);
    rc.w[0] = q0.x; rc.w[1] = q0.y; rc.w[2] = q0.z; rc.w[3] = q0.w;
    rc.w[4] = rc.w[5] = rc.w[6] = rc.w[7] = 0;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) rc.w[i] = 0;
  }
  if constexpr (FMT == E4B_FMT_NF4) {
    rc.absmax = left > 0 ? __ldg(reinterpret_cast<const float*>(srow) + kl / 64) : 0.f;
    rc.mx = 0;
  } else {
    const uint32_t s0 = left > 0 ? __ldg(srow + kl / 32) : 0u;
    const uint32_t s1 = left > 32 ? __ldg(srow + kl / 32 + 1) : 0u;
    rc.mx = s0 | (s1 << 8);
    rc.absmax = 0.f;
  }
}

template <int FMT, int EPI>
__global__ void __launch_bounds__(kGemvWarps * 32, 2)
gemv_kernel(GemmProblem p) {
  __shared__ int32_t s_act[kMaxExpertsSmem];
  __shared__ int32_t s_nact;
  __shared__ int32_t s_warp[kGemvWarps + 1];
  constexpr int NM = (EPI == E4B_EPI_SWIGLU) ? 2 : 1;  // matrices per item (gate, up)

  // Clear the caller's fp32 accumulator (the layer's combine buffer) first.
  if (p.zero_buf) {
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < p.zero_count;
         i += int64_t(gridDim.x) * blockDim.x)
      p.zero_buf[i] = 0.f;
  }
  block_active_experts(p.offsets, p.E, s_act, &s_nact, s_warp);

  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int c = lane & 3;
  const int64_t N = p.N;
  const int64_t K = p.K;
  const int64_t rows_per_mat = (EPI == E4B_EPI_SWIGLU) ? N / 2 : N;
  const int64_t MT = rows_per_mat / 16;
  const int64_t nitems = int64_t(s_nact) * MT;
  const int64_t warp0 = int64_t(blockIdx.x) * kGemvWarps + (threadIdx.x >> 5);
  const int64_t nwarps = int64_t(gridDim.x) * kGemvWarps;
  const int64_t cbytes = K / 2;
  const int64_t sstride = (FMT == E4B_FMT_NF4) ? (K / 64) * 4 : (K / 32);  // scale row bytes
  const uint8_t* scales = static_cast<const uint8_t*>(p.scales);

  for (int64_t item = warp0; item < nitems; item += nwarps) {
    const int e = s_act[item / MT];
    const int64_t mt = item % MT;
    const int64_t p0 = p.offsets[e];
    const int64_t p1 = p.offsets[e + 1];
    const uint8_t* crow[NM][2];
    const uint8_t* srow[NM][2];
#pragma unroll
    for (int m = 0; m < NM; ++m)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t n = mt * 16 + g + 8 * h;
        const int64_t row =
            int64_t(e) * N + (NM == 2 ? gate_up_row(p.layout, rows_per_mat, m, n) : n);
        crow[m][h] = p.codes + row * cbytes;
        srow[m][h] = scales + row * sstride;
      }

    for (int64_t tg0 = p0; tg0 < p1; tg0 += 32) {
      const int nt = int((min(p1 - tg0, int64_t(32)) + 7) / 8);
      const uint16_t* xrow[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t pr = tg0 + 8 * j + g;
        xrow[j] = nullptr;
        if (j < nt && pr < p1) {
          const int64_t ar = p.row_slot ? int64_t(p.row_slot[pr] / p.top_k) : pr;
          xrow[j] = p.a + ar * p.lda;
        }
      }
      float acc[NM][4][4];
#pragma unroll
      for (int m = 0; m < NM; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[m][j][i] = 0.f;

      for (int64_t kc = 0; kc < K; kc += 256) {
        const int64_t kl = kc + c * 64;
        RowChunk rc[NM][2];
#pragma unroll
        for (int m = 0; m < NM; ++m)
#pragma unroll
          for (int h = 0; h < 2; ++h) load_row_chunk<FMT>(rc[m][h], crow[m][h], srow[m][h], kl, K);
        const bool kvalid = kl < K;
        Lut L[NM][2];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          // one NF4 block (64 weights) per row and lane: its table serves both
          // halves; MXFP4 has a block (and table) per half
          if (FMT == E4B_FMT_MXFP4 || half == 0) {
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
              for (int h = 0; h < 2; ++h)
                lut_build<FMT>(L[m][h], rc[m][h].absmax, (rc[m][h].mx >> (8 * half)) & 0xFFu);
          }
#pragma unroll
          for (int ss = 0; ss < 8; ++ss) {
            const int s = half * 8 + ss;  // MMA k-step within the chunk
            uint32_t A[NM][4];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
              const uint32_t v0 = (s & 1) ? (rc[m][0].w[s >> 1] >> 16) : rc[m][0].w[s >> 1];
              const uint32_t v1 = (s & 1) ? (rc[m][1].w[s >> 1] >> 16) : rc[m][1].w[s >> 1];
              lut_decode4<FMT>(L[m][0], v0, A[m][0], A[m][2]);
              lut_decode4<FMT>(L[m][1], v1, A[m][1], A[m][3]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if (j < nt) {
                uint32_t b0 = 0, b1 = 0;
                if (xrow[j] && kvalid && (kl + 4 * s) < K) {
                  const uint2 bv = __ldg(reinterpret_cast<const uint2*>(xrow[j] + kl + 4 * s));
                  b0 = bv.x;
                  b1 = bv.y;
                }
#pragma unroll
                for (int m = 0; m < NM; ++m) mma_bf16_16816(acc[m][j], A[m], b0, b1);
              }
            }
          }
        }
      }

      // Epilogue. Fragment: acc[.][j][0..1] -> row g, tokens 2c, 2c+1 of
      // chunk j; acc[.][j][2..3] -> row g+8, same tokens.
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (j >= nt) continue;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t pr = tg0 + 8 * j + 2 * c + (i & 1);
          if (pr >= p1) continue;
          const int64_t n = mt * 16 + g + ((i & 2) ? 8 : 0);
          if constexpr (EPI == E4B_EPI_SWIGLU) {
            float gv = acc[0][j][i], uv = acc[NM - 1][j][i];
            if (p.bias) {
              const float* b = p.bias + int64_t(e) * N;
              gv += b[gate_up_row(p.layout, rows_per_mat, 0, n)];
              uv += b[gate_up_row(p.layout, rows_per_mat, 1, n)];
            }
            const float hv = glu_act(p.act, gv, uv, p.alpha, p.limit);
            static_cast<uint16_t*>(p.out)[pr * p.ldo + n] = to_bf16_bits(hv);
          } else {
            const float v = acc[0][j][i] + (p.bias ? p.bias[int64_t(e) * N + n] : 0.f);
            if constexpr (EPI == E4B_EPI_STORE) {
              static_cast<uint16_t*>(p.out)[pr * p.ldo + n] = to_bf16_bits(v);
            } else {
              const int32_t slot = p.out_slot ? p.out_slot[pr] : int32_t(pr);
              const int64_t t = slot / p.top_k;
              atomicAdd(static_cast<float*>(p.out) + t * p.ldo + n, p.gates[slot] * v);
            }
          }
        }
      }
    }
  }
}

template <int FMT, int EPI>
static cudaError_t launch_gemv_t(const GemmProblem& p, cudaStream_t st, int sms) {
  const int64_t rows_per_mat = (EPI == E4B_EPI_SWIGLU) ? p.N / 2 : p.N;
  const int64_t items = int64_t(p.E) * (rows_per_mat / 16);
  int64_t grid = (items + kGemvWarps - 1) / kGemvWarps;
  const int64_t cap = int64_t(sms) * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  gemv_kernel<FMT, EPI><<<int(grid), kGemvWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemv(const GemmProblem& p, cudaStream_t st, int sms) {
  if (p.fmt == E4B_FMT_NF4) {
    if (p.epilogue == E4B_EPI_SWIGLU) return launch_gemv_t<E4B_FMT_NF4, E4B_EPI_SWIGLU>(p, st, sms);
    if (p.epilogue == E4B_EPI_COMBINE) return launch_gemv_t<E4B_FMT_NF4, E4B_EPI_COMBINE>(p, st, sms);
    return launch_gemv_t<E4B_FMT_NF4, E4B_EPI_STORE>(p, st, sms);
  }
  if (p.epilogue == E4B_EPI_SWIGLU) return launch_gemv_t<E4B_FMT_MXFP4, E4B_EPI_SWIGLU>(p, st, sms);
  if (p.epilogue == E4B_EPI_COMBINE) return launch_gemv_t<E4B_FMT_MXFP4, E4B_EPI_COMBINE>(p, st, sms);
  return launch_gemv_t<E4B_FMT_MXFP4, E4B_EPI_STORE>(p, st, sms);
}

// y = bf16(acc), 4 values per thread.
__global__ void finalize_kernel(const float* __restrict__ acc, int64_t n4, uint16_t* __restrict__ y) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(acc)[i];
    reinterpret_cast<uint2*>(y)[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

// One thread per 4 consecutive outputs of a token: the token's k rows are
// read in slot order and summed in fp32, so the result does not depend on the
// order in which the rows were produced.
__global__ void combine_rows_kernel(const float* __restrict__ rows, const int32_t* __restrict__ inv,
                                    int64_t T, int32_t k, int64_t H4, uint16_t* __restrict__ y) {
  const int64_t total = T * H4;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = i / H4;
    const int64_t c = i - t * H4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int32_t p = __ldg(inv + t * k + j);
      if (p < 0) continue;
      const float4 v = __ldg(reinterpret_cast<const float4*>(rows + int64_t(p) * (H4 * 4)) + c);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    reinterpret_cast<uint2*>(y)[i] = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
  }
}

cudaError_t launch_combine_rows(const float* rows, const int32_t* inv, int64_t T, int32_t k, int64_t H,
                                uint16_t* y, cudaStream_t st, int sms) {
  const int64_t total = T * (H / 4);
  int64_t grid = (total + 255) / 256;
  if (grid > int64_t(sms) * 16) grid = int64_t(sms) * 16;
  if (grid < 1) grid = 1;
  combine_rows_kernel<<<int(grid), 256, 0, st>>>(rows, inv, T, k, H / 4, y);
  return cudaGetLastError();
}

cudaError_t launch_finalize(const float* acc, int64_t n, uint16_t* y, cudaStream_t st, int sms) {
  const int64_t n4 = n / 4;  // callers guarantee n % 4 == 0
  int64_t grid = (n4 + 255) / 256;
  if (grid > int64_t(sms) * 8) grid = int64_t(sms) * 8;
  if (grid < 1) grid = 1;
  finalize_kernel<<<int(grid), 256, 0, st>>>(acc, n4, y);
  return cudaGetLastError();
}

}  // namespace e4b
