// Blockwise 4-bit quantisation (NF4, MXFP4) and the table decode used by the
// GEMM kernels, exposed for bit-exact checks.
//
// NF4: "grouped-nf4-gemm" README, CPU block 1 (quantize_pack_nf4 /
// dequant_ref); bitsandbytes PR #1984, Summary (per-expert absmax).
// MXFP4: README intro and CPU block 2 (OCP e2m1 + e8m0).
#include "common.cuh"
#include "launch.h"

namespace e4b {

// Largest fp32 not above the midpoint of two adjacent NF4 levels. A value s
// is nearer the upper level exactly when s > this threshold (ties, s equal
// to the exact midpoint, stay with the lower level).
E4B_DEV float nf4_threshold(int i) {
  return __fadd_rd(nf4_level(i), nf4_level(i + 1)) * 0.5f;
}

// One warp handles 4 blocks of 64 weights: 8 lanes per block, 8 weights per lane.
__global__ void quantize_nf4_kernel(const float* __restrict__ w, int64_t nblocks,
                                    uint8_t* __restrict__ codes, float* __restrict__ absmax) {
  float thr[15];
#pragma unroll
  for (int i = 0; i < 15; ++i) thr[i] = nf4_threshold(i);
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t g = warp; g * 4 < nblocks; g += nwarps) {
    const int64_t b = g * 4 + (lane >> 3);
    const bool valid = b < nblocks;
    const int64_t base = b * 64 + (lane & 7) * 8;
    float v[8];
    if (valid) {
      const float4 p0 = *reinterpret_cast<const float4*>(w + base);
      const float4 p1 = *reinterpret_cast<const float4*>(w + base + 4);
      v[0] = p0.x; v[1] = p0.y; v[2] = p0.z; v[3] = p0.w;
      v[4] = p1.x; v[5] = p1.y; v[6] = p1.z; v[7] = p1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t c = 7;
      if (a > 0.f) {
        const float s = __fdiv_rn(v[i], a);
        c = 0;
#pragma unroll
        for (int t = 0; t < 15; ++t) c += (s > thr[t]) ? 1u : 0u;
      }
      // byte i/2: earlier weight in the high nibble
      const int byte = i >> 1;
      const int shift = byte * 8 + ((i & 1) ? 0 : 4);
      word |= c << shift;
    }
    if (valid) {
      *reinterpret_cast<uint32_t*>(codes + base / 2) = word;
      if ((lane & 7) == 0) absmax[b] = a;
    }
  }
}

// 2^p for p in [-127, 127] as an exact fp32 (2^-127 is subnormal).
E4B_DEV float exp2_exact(int p) {
  return p >= -126 ? __uint_as_float(uint32_t(p + 127) << 23) : __uint_as_float(0x00400000u);
}

// Nearest e2m1 magnitude code of |q|, ties to the even code, saturating at 6.
E4B_DEV uint32_t e2m1_round(float m) {
  return (m > 0.25f) + (m >= 0.75f) + (m > 1.25f) + (m >= 1.75f) + (m > 2.5f) + (m >= 3.5f) +
         (m > 5.0f);
}

// One warp handles 8 blocks of 32 weights: 4 lanes per block, 8 weights per lane.
__global__ void quantize_mxfp4_kernel(const float* __restrict__ w, int64_t nblocks,
                                      uint8_t* __restrict__ blocks, uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t g = warp; g * 8 < nblocks; g += nwarps) {
    const int64_t b = g * 8 + (lane >> 2);
    const bool valid = b < nblocks;
    const int64_t base = b * 32 + (lane & 3) * 8;
    float v[8];
    if (valid) {
      const float4 p0 = *reinterpret_cast<const float4*>(w + base);
      const float4 p1 = *reinterpret_cast<const float4*>(w + base + 4);
      v[0] = p0.x; v[1] = p0.y; v[2] = p0.z; v[3] = p0.w;
      v[4] = p1.x; v[5] = p1.y; v[6] = p1.z; v[7] = p1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    uint32_t word = 0;
    uint32_t sbyte = 0;
    if (a > 0.f) {
      int e = ilogbf(a) - 2;
      e = max(-127, min(127, e));
      sbyte = uint32_t(e + 127);
      const float inv = exp2_exact(-e);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float q = __fmul_rn(v[i], inv);  // exact: a power-of-two scaling of a normal result
        const uint32_t c = e2m1_round(fabsf(q)) | ((__float_as_uint(v[i]) >> 31) << 3);
        word |= c << (i * 4);  // earlier weight in the low nibble
      }
    }
    if (valid) {
      *reinterpret_cast<uint32_t*>(blocks + base / 2) = word;
      if ((lane & 3) == 0) scales[b] = uint8_t(sbyte);
    }
  }
}

// Each thread decodes one 32-bit word (8 weights) through the block's table.
template <int FMT>
__global__ void dequantize_kernel(const uint8_t* __restrict__ codes, const void* __restrict__ scales,
                                  int64_t nwords, uint16_t* __restrict__ out) {
  constexpr int kWordsPerBlock = FMT == E4B_FMT_NF4 ? 8 : 4;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t blk = i / kWordsPerBlock;
    Lut L;
    if constexpr (FMT == E4B_FMT_NF4) lut_nf4(L, static_cast<const float*>(scales)[blk]);
    else lut_mxfp4(L, static_cast<const uint8_t*>(scales)[blk]);
    const uint32_t wd = reinterpret_cast<const uint32_t*>(codes)[i];
    uint32_t o[4];
    lut_decode8<FMT>(L, wd, o);
    reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

static int grid_for(int64_t work, int per_block, int sms) {
  int64_t g = (work + per_block - 1) / per_block;
  const int64_t cap = int64_t(sms) * 8;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return int(g);
}

cudaError_t launch_quantize_nf4(const float* w, int64_t nblocks, uint8_t* codes, float* absmax,
                                cudaStream_t st, int sms) {
  const int threads = 256;  // 8 warps x 4 blocks
  quantize_nf4_kernel<<<grid_for(nblocks, 32, sms), threads, 0, st>>>(w, nblocks, codes, absmax);
  return cudaGetLastError();
}

cudaError_t launch_quantize_mxfp4(const float* w, int64_t nblocks, uint8_t* blocks, uint8_t* scales,
                                  cudaStream_t st, int sms) {
  const int threads = 256;  // 8 warps x 8 blocks
  quantize_mxfp4_kernel<<<grid_for(nblocks, 64, sms), threads, 0, st>>>(w, nblocks, blocks, scales);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(int fmt, const uint8_t* codes, const void* scales, int64_t nweights,
                              uint16_t* out, cudaStream_t st, int sms) {
  const int64_t nwords = nweights / 8;
  const int threads = 256;
  if (fmt == E4B_FMT_NF4)
    dequantize_kernel<E4B_FMT_NF4><<<grid_for(nwords, threads, sms), threads, 0, st>>>(codes, scales, nwords, out);
  else
    dequantize_kernel<E4B_FMT_MXFP4><<<grid_for(nwords, threads, sms), threads, 0, st>>>(codes, scales, nwords, out);
  return cudaGetLastError();
}

void host_nf4_levels(float* out) {
  for (int i = 0; i < 16; ++i) out[i] = nf4_level(i);
}

}  // namespace e4b
