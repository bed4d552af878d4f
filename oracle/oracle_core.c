/*
 * oracle_core.c -- plain C restatement of the oracle's heavy loops (test
 * infrastructure only; compiled without fast-math or FMA contraction).
 *
 * The same definitions as oracle/formats.py and oracle/moe.py, written as
 * straight loops so full-size layers can be checked in seconds:
 *   NF4 ("grouped-nf4-gemm" README, CPU block 1; bitsandbytes PR #1984):
 *     absmax per 64-weight block, s = fp32(w / absmax), nearest level with
 *     ties to the lower index (decided exactly: 2s > c[i] + c[i+1] in double),
 *     zero block -> level 7; packed with the earlier weight in the high nibble;
 *     decoded value bf16_rne(fp32(c[code] * absmax)) ("product"), or
 *     bf16_rne(c[code]) * absmax as the exact double product ("level").
 *   MXFP4 (README intro, CPU block 2; OCP MX v1.0): e = floor(log2 amax) - 2
 *     clamped to [-127, 127], elements rounded to e2m1 with ties to even,
 *     sign bit copied, earlier weight in the low nibble.
 *   fp64 matrix-vector products for the per-expert matmuls.
 * The codebook is passed in by the caller (the Python oracle builds it).
 * No table or helper here is shared with the CUDA library.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float bf16_rne_f32(float v) {
  uint32_t u;
  memcpy(&u, &v, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) { /* inf / nan */
    if (u & 0x007FFFFFu) u = 0x7FC00000u;
    memcpy(&v, &u, 4);
    return v;
  }
  const uint32_t lsb = (u >> 16) & 1u;
  u = (u + 0x7FFFu + lsb) & 0xFFFF0000u;
  memcpy(&v, &u, 4);
  return v;
}

void e4bref_nf4_quantize(const float* w, int64_t rows, int64_t K, const float* cb, uint8_t* codes,
                         float* absmax) {
  double sums[15];
  for (int i = 0; i < 15; ++i) sums[i] = (double)cb[i] + (double)cb[i + 1];
  const int64_t nb = K / 64;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const float* blk = w + r * K + b * 64;
      float a = 0.0f;
      for (int i = 0; i < 64; ++i) {
        const float v = fabsf(blk[i]);
        if (v > a) a = v;
      }
      absmax[r * nb + b] = a;
      uint8_t cs[64];
      for (int i = 0; i < 64; ++i) {
        if (a == 0.0f) {
          cs[i] = 7;
          continue;
        }
        const volatile float s = blk[i] / a;
        const double two_s = 2.0 * (double)s;
        int c = 0;
        for (int t = 0; t < 15; ++t)
          if (two_s > sums[t]) ++c;
        cs[i] = (uint8_t)c;
      }
      uint8_t* out = codes + r * (K / 2) + b * 32;
      for (int j = 0; j < 32; ++j) out[j] = (uint8_t)((cs[2 * j] << 4) | cs[2 * j + 1]);
    }
  }
}

void e4bref_nf4_decode(const uint8_t* codes, const float* absmax, int64_t rows, int64_t K,
                       const float* cb, float* out) {
  const int64_t nb = K / 64;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      const uint8_t byte = codes[r * (K / 2) + k / 2];
      const int c = (k & 1) ? (byte & 15) : (byte >> 4);
      const volatile float prod = cb[c] * absmax[r * nb + k / 64];
      out[r * K + k] = bf16_rne_f32(prod);
    }
  }
}

void e4bref_nf4_decode_level(const uint8_t* codes, const float* absmax, int64_t rows, int64_t K,
                             const float* cb, double* out) {
  const int64_t nb = K / 64;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      const uint8_t byte = codes[r * (K / 2) + k / 2];
      const int c = (k & 1) ? (byte & 15) : (byte >> 4);
      out[r * K + k] = (double)bf16_rne_f32(cb[c]) * (double)absmax[r * nb + k / 64];
    }
  }
}

static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static int e2m1_nearest(double m) {
  int lo = 0;
  for (int i = 0; i < 8; ++i)
    if (kE2M1[i] <= m) lo = i;
  if (lo == 7) return 7;
  const double dl = m - kE2M1[lo], dh = kE2M1[lo + 1] - m;
  if (dh < dl) return lo + 1;
  if (dh == dl && (lo & 1)) return lo + 1;
  return lo;
}

void e4bref_mxfp4_quantize(const float* w, int64_t rows, int64_t K, uint8_t* blocks,
                           uint8_t* scales) {
  const int64_t nb = K / 32;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const float* blk = w + r * K + b * 32;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) {
        const double v = fabs((double)blk[i]);
        if (v > amax) amax = v;
      }
      uint8_t* out = blocks + r * (K / 2) + b * 16;
      if (amax == 0.0) {
        scales[r * nb + b] = 0;
        memset(out, 0, 16);
        continue;
      }
      int ex;
      frexp(amax, &ex); /* amax = m 2^ex, m in [0.5, 1) */
      int e = (ex - 1) - 2;
      if (e < -127) e = -127;
      if (e > 127) e = 127;
      scales[r * nb + b] = (uint8_t)(e + 127);
      uint8_t cs[32];
      for (int i = 0; i < 32; ++i) {
        const double q = ldexp((double)blk[i], -e);
        const int mag = e2m1_nearest(fabs(q));
        const int sgn = signbit(blk[i]) ? 8 : 0;
        cs[i] = (uint8_t)(sgn | mag);
      }
      for (int j = 0; j < 16; ++j) out[j] = (uint8_t)(cs[2 * j] | (cs[2 * j + 1] << 4));
    }
  }
}

void e4bref_mxfp4_decode(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int64_t K,
                         float* out) {
  const int64_t nb = K / 32;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      const uint8_t byte = blocks[r * (K / 2) + k / 2];
      const int c = (k & 1) ? (byte >> 4) : (byte & 15);
      const int s = scales[r * nb + k / 32];
      double v = kE2M1[c & 7];
      if (c & 8) v = -v;
      out[r * K + k] = (s == 255) ? NAN : (float)ldexp(v, s - 127);
    }
  }
}

/* y[i, r] = sum_k W[r, k] * x[i, k] in fp64, for n vectors x. */
void e4bref_matvec_f64w(const double* W, int64_t rows, int64_t K, const double* x, int64_t n,
                        double* y) {
  for (int64_t i = 0; i < n; ++i) {
    const double* xi = x + i * K;
    for (int64_t r = 0; r < rows; ++r) {
      const double* wr = W + r * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += wr[k] * xi[k];
      y[i * rows + r] = acc;
    }
  }
}

void e4bref_matvec_f64(const float* W, int64_t rows, int64_t K, const double* x, int64_t n,
                       double* y) {
  for (int64_t i = 0; i < n; ++i) {
    const double* xi = x + i * K;
    for (int64_t r = 0; r < rows; ++r) {
      const float* wr = W + r * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += (double)wr[k] * xi[k];
      y[i * rows + r] = acc;
    }
  }
}
