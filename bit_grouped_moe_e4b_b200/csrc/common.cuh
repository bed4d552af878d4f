// Shared device helpers for the e4b kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "e4b.h"

#define E4B_DEV __device__ __forceinline__

namespace e4b {

// Workspace status word layout (first 256 bytes of every workspace):
//   [0] int32 first error code recorded by any kernel (0 = none)
//   [1] int32 count of dropped slots (bad expert ids)
constexpr int kStatusBytes = 256;

// Wait bounds: a spin on an mbarrier gives up after this many polls
// (each poll backs off with nanosleep once it has spun for a while).
// ~2^26 polls of >= 32 ns each is well over a second.
constexpr uint32_t kWaitPolls = 1u << 26;

E4B_DEV void record_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// Programmatic dependent launch: wait until the grid this one depends on has
// completed and its memory is visible (returns at once when there is none);
// allow the grid that depends on this one to start launching.
E4B_DEV void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
E4B_DEV void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launches `kernel` as a programmatic dependent of the work before it on the
// stream: it may start before that work completes and must call
// grid_dependency_wait() before touching memory that work writes or reads.
template <typename Kernel, typename... Args>
inline cudaError_t launch_dependent(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                    Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ------------------------------------------------------------------ bf16
E4B_DEV uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  // d.hi = cvt(a), d.lo = cvt(b)
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

E4B_DEV uint16_t to_bf16_bits(float v) {
  return static_cast<uint16_t>(pack_bf16x2(v, 0.f) & 0xFFFFu);
}

E4B_DEV float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

E4B_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// ------------------------------------------------------------- NF4 levels
// The 16 NormalFloat-4 levels as published with QLoRA (Dettmers et al. 2023,
// Appendix E), the codebook of the bitsandbytes gemm_4bit layout.
__host__ __device__ constexpr float nf4_level(int i) {
  constexpr float kLevels[16] = {
      -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
      -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
      0.07958029955625534f, 0.16093020141124725f, 0.24611230611801147f, 0.33791524171829224f,
      0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, 1.0f};
  return kLevels[i];
}

// e2m1 magnitudes (OCP MX v1.0 FP4 E2M1), index = 3-bit magnitude code.
__host__ __device__ constexpr float e2m1_magnitude(int i) {
  constexpr float kMag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  return kMag[i];
}

// ------------------------------------------------------------- 16-entry LUT
// A per-block decode table of 16 bf16 values held as byte planes:
//   lo[q] = low bytes of entries 4q..4q+3, hi[q] = high bytes.
// A 4-bit code selects its entry with two levels of byte permutes: the low
// three bits pick within entries 0..7 (planes 0,1) and 8..15 (planes 2,3),
// the top bit picks between the two.
struct Lut {
  uint32_t lo[4];
  uint32_t hi[4];
};

// Build from 8 packed pairs p[j] = bf16x2(T[2j], T[2j+1]) (T[2j] in the low half).
E4B_DEV void lut_from_pairs(Lut& L, const uint32_t (&p)[8]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    L.lo[q] = prmt(p[2 * q], p[2 * q + 1], 0x6420);
    L.hi[q] = prmt(p[2 * q], p[2 * q + 1], 0x7531);
  }
}

// NF4: T[i] = bf16_rne(fp32(level_i * absmax)).
E4B_DEV void lut_nf4(Lut& L, float absmax) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    p[j] = pack_bf16x2(__fmul_rn(nf4_level(2 * j), absmax), __fmul_rn(nf4_level(2 * j + 1), absmax));
  lut_from_pairs(L, p);
}

// e8m0 byte -> fp32 2^(s-127); byte 0 is the subnormal 2^-127, byte 255 NaN.
E4B_DEV float e8m0_to_f32(uint32_t s) {
  if (s == 0) return __uint_as_float(0x00400000u);
  if (s == 255) return __uint_as_float(0x7FC00000u);
  return __uint_as_float(s << 23);
}

// MXFP4: T[i] = sign(i) * e2m1(i & 7) * 2^(s-127), exact in fp32 and bf16.
// Entries 8..15 are entries 0..7 with the sign bit set (code 8 is -0).
E4B_DEV void lut_mxfp4(Lut& L, uint32_t scale_byte) {
  const float sc = e8m0_to_f32(scale_byte);
  uint32_t p[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    p[j] = pack_bf16x2(__fmul_rn(e2m1_magnitude(2 * j), sc), __fmul_rn(e2m1_magnitude(2 * j + 1), sc));
  L.lo[0] = prmt(p[0], p[1], 0x6420);
  L.hi[0] = prmt(p[0], p[1], 0x7531);
  L.lo[1] = prmt(p[2], p[3], 0x6420);
  L.hi[1] = prmt(p[2], p[3], 0x7531);
  L.lo[2] = L.lo[0];
  L.lo[3] = L.lo[1];
  L.hi[2] = L.hi[0] | 0x80808080u;
  L.hi[3] = L.hi[1] | 0x80808080u;
}

template <int FMT>
E4B_DEV void lut_build(Lut& L, float nf4_absmax, uint32_t mx_scale) {
  if constexpr (FMT == E4B_FMT_NF4) lut_nf4(L, nf4_absmax);
  else lut_mxfp4(L, mx_scale);
}

// Decode one 32-bit word of 8 codes into 4 bf16x2 registers in weight order.
// NF4 bytes hold the earlier weight in the high nibble, MXFP4 in the low one.
template <int FMT>
E4B_DEV void lut_decode8(const Lut& L, uint32_t w, uint32_t (&out)[4]) {
  const uint32_t idx = w & 0x77777777u;
  const uint32_t sel = ((w >> 1) & 0x44444444u) | 0x32103210u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t i = h ? (idx >> 16) : idx;
    const uint32_t s = h ? (sel >> 16) : sel;
    const uint32_t la = prmt(L.lo[0], L.lo[1], i);
    const uint32_t lb = prmt(L.lo[2], L.lo[3], i);
    const uint32_t ha = prmt(L.hi[0], L.hi[1], i);
    const uint32_t hb = prmt(L.hi[2], L.hi[3], i);
    const uint32_t l = prmt(la, lb, s);
    const uint32_t hh = prmt(ha, hb, s);
    if constexpr (FMT == E4B_FMT_NF4) {
      out[2 * h] = prmt(l, hh, 0x4051);
      out[2 * h + 1] = prmt(l, hh, 0x6273);
    } else {
      out[2 * h] = prmt(l, hh, 0x5140);
      out[2 * h + 1] = prmt(l, hh, 0x7362);
    }
  }
}

// Decode the 4 codes in the low 16 bits of v (two weight pairs).
template <int FMT>
E4B_DEV void lut_decode4(const Lut& L, uint32_t v, uint32_t& out01, uint32_t& out23) {
  const uint32_t i = v & 0x7777u;
  const uint32_t s = ((v >> 1) & 0x4444u) | 0x3210u;
  const uint32_t la = prmt(L.lo[0], L.lo[1], i);
  const uint32_t lb = prmt(L.lo[2], L.lo[3], i);
  const uint32_t ha = prmt(L.hi[0], L.hi[1], i);
  const uint32_t hb = prmt(L.hi[2], L.hi[3], i);
  const uint32_t l = prmt(la, lb, s);
  const uint32_t hh = prmt(ha, hb, s);
  if constexpr (FMT == E4B_FMT_NF4) {
    out01 = prmt(l, hh, 0x4051);
    out23 = prmt(l, hh, 0x6273);
  } else {
    out01 = prmt(l, hh, 0x5140);
    out23 = prmt(l, hh, 0x7362);
  }
}

// ----------------------------------------------------------- global loads
E4B_DEV uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// silu(g) * u in fp32 with the hardware exp2 approximation and an approximate
// reciprocal (__expf, __fdividef): relative error ~2^-20, so the bf16 h the
// layer keeps is the correctly rounded value or one ulp off in rare elements.
// The epilogues evaluate it once per gate/up pair; with IEEE expf and division
// it took issue slots the tcgen05 path's decoder warps (on the same SM
// sub-partitions) need. g -> -inf: __expf = inf and __fdividef(g, inf) = -0.
E4B_DEV float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// The gate_up activation of the expert variant (include/e4b.h): SwiGLU, or
// the clamped GLU (u' + 1) * g' * sigmoid(alpha * g') with g' = min(g, limit)
// and u' = clamp(u, -limit, limit). Comparisons keep NaN inputs NaN.
E4B_DEV float glu_act(int act, float g, float u, float alpha, float limit) {
  if (act == E4B_ACT_CLAMPED_GLU) {
    g = g > limit ? limit : g;
    u = u > limit ? limit : (u < -limit ? -limit : u);
    return __fdividef((u + 1.0f) * g, 1.0f + __expf(-alpha * g));
  }
  return silu_mul(g, u);
}

// gate_up row of output n's gate (m = 0) or up (m = 1) row: the two halves,
// or interleaved (gate 2n, up 2n+1).
E4B_DEV int64_t gate_up_row(int layout, int64_t I, int m, int64_t n) {
  return layout == E4B_GATE_UP_INTERLEAVED ? 2 * n + m : int64_t(m) * I + n;
}

// Compacts the experts with at least one routed row (offsets[e+1] > offsets[e])
// into s_act[0..*s_n), in expert order. Whole block; ends with __syncthreads.
// s_warp needs blockDim.x/32 + 1 ints.
E4B_DEV void block_active_experts(const int64_t* offsets, int E, int32_t* s_act, int32_t* s_n,
                                  int32_t* s_warp) {
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int wid = tid >> 5;
  const int nw = blockDim.x >> 5;
  if (tid == 0) *s_n = 0;
  __syncthreads();
  for (int base = 0; base < E; base += blockDim.x) {
    const int e = base + tid;
    const bool on = e < E && offsets[e + 1] > offsets[e];
    const uint32_t bal = __ballot_sync(0xffffffffu, on);
    if (lane == 0) s_warp[wid] = __popc(bal);
    __syncthreads();
    if (tid == 0) {
      int run = *s_n;
      for (int w = 0; w < nw; ++w) {
        const int c = s_warp[w];
        s_warp[w] = run;
        run += c;
      }
      s_warp[nw] = run;
    }
    __syncthreads();
    if (on) s_act[s_warp[wid] + __popc(bal & ((1u << lane) - 1u))] = e;
    __syncthreads();
    if (tid == 0) *s_n = s_warp[nw];
    __syncthreads();
  }
}

}  // namespace e4b
