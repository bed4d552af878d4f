// int4-b32: signed 4-bit weights (two's complement, two per byte, the earlier
// weight in the low nibble) with one fp16 scale per 32 weights along K. The
// batch-1 decode GEMV over a token's routed experts with exact integer block
// sums, its quantiser, and the repack of symmetric GPTQ tensors onto the same
// bytes ("How do I run a single-token INT4 decode GEMV over routed MoE experts,
// and pack calibrated (GPTQ) weights for it?", grouped-nf4-gemm solutions
// page; the measured row "int4-b32 decode GEMV, dense M=1" in the
// grouped-nf4-gemm README).
//
// GEMV design (HBM-bound: 0.5625 bytes per weight, read once):
//   * one CTA of 8 warps per SM; it quantises the token (or each routed
//     slot's row) to int8 in shared memory, one fp32 product per value,
//     laid out so a 16-byte load pairs with the nibbles of one 4-byte code
//     word: per 32-weight block two 16-byte planes (word i holds the bytes of
//     the even or odd positions of weights 8i..8i+7), plus -8 * (block sum)
//     as int16;
//   * an item is four weight rows (two outputs) over a chunk of up to 128
//     blocks; every warp owns a contiguous run of items and keeps kStages of
//     them in flight in its own shared-memory stages, filled by bulk copies
//     that the whole warp starts (lane 0 writes the item's descriptor and
//     posts the bytes; lanes 0-3 copy one row position each, two
//     neighbouring rows of one expert in one copy when the chunk is the
//     whole row; the scales ride along when 16-byte aligned);
//   * a code word w gives (w ^ 0x88888888) & 0x0F0F0F0F = q + 8 of the even
//     positions and (w ^ 0x88888888) & 0xF0F0F0F0 = 16 (q + 8) of the odd
//     ones as unsigned bytes, so two LOP3 and two unsigned x signed dp4a per
//     word, with the chains seeded by the block's -8 * sum(xq), give exactly
//     16 * sum(q * xq) = 16 D (|16 D| < 2^20);
//   * the 16 block dot products of an item run without branches; the four
//     row sums leave the warp in one butterfly and are added to the round's
//     fp32 accumulators in shared memory, which the epilogue (store / SwiGLU
//     / gate-weighted combine over the routed slots) turns into bf16;
//   * the kernel is a programmatic dependent of the work before it on the
//     stream: it waits (griddepcontrol.wait) before it reads the ids and
//     gates (with E4B_FLAG_IDS_READY only before it reads x, so its set-up
//     overlaps that work), quantises x before its first weight copies, and
//     lets the next kernel launch once its copies are all issued.
#include <cuda_fp16.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace e4b {
namespace {

using namespace sm100;

constexpr int kI4Block = 32;
constexpr int kGemvThreads = 256;  // 8 warps, one CTA per SM
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kStages = 3;         // per-warp stages in flight
constexpr int kRows = 4;           // weight rows per item (two outputs)
constexpr int kChunkBlocks = 128;  // blocks of one row per item (2 KiB of codes)
constexpr int kLaneBlocks = kChunkBlocks / 32;
constexpr int kStageBytes = kRows * kChunkBlocks * (16 + 2);  // codes, then the rows' fp16 scales
constexpr int kRoundOutputs = 256;  // outputs whose fp32 sums sit in shared memory at once
constexpr int kQuantGroups = 8;     // groups of 8 activations a thread keeps in registers
constexpr int kMaxSlots = 64;       // routed experts of one token
// head of shared memory: sx[64] @0, ids[64] @256, gates[64] @512, reduction
// scratch[8] @768, abort flag @832, barriers [8][kStages] @1024, item
// descriptors [8][kStages] @2048
constexpr int kBarOff = 1024;
constexpr int kDescOff = 2048;
constexpr int kHeadBytes = 4096;

// Bytes of one quantised activation row in shared memory: the two planes
// (K bytes) and an int16 -8 * sum(xq) per block, rounded up to 16 so every
// row starts 16-byte aligned.
__host__ __device__ constexpr int64_t xrow_bytes(int64_t K) { return (K + K / 16 + 15) / 16 * 16; }

E4B_DEV float half_bits_to_f32(uint32_t h) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

E4B_DEV int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// 16 * (sum over one block of q * xq): w holds the block's 32 nibbles, xa and
// xb its activation planes, s8 = -8 * sum(xq) over the block.
E4B_DEV int block_dot16(const uint4 w, const uint4 xa, const uint4 xb, int s8) {
  const uint32_t f = 0x88888888u, lo = 0x0F0F0F0Fu, hi = 0xF0F0F0F0u;
  int dl = s8, dh = 0;
  dl = dp4a_us((w.x ^ f) & lo, xa.x, dl);
  dh = dp4a_us((w.x ^ f) & hi, xa.y, dh);
  dl = dp4a_us((w.y ^ f) & lo, xa.z, dl);
  dh = dp4a_us((w.y ^ f) & hi, xa.w, dh);
  dl = dp4a_us((w.z ^ f) & lo, xb.x, dl);
  dh = dp4a_us((w.z ^ f) & hi, xb.y, dh);
  dl = dp4a_us((w.w ^ f) & lo, xb.z, dl);
  dh = dp4a_us((w.w ^ f) & hi, xb.w, dh);
  return dl * 16 + dh;
}

E4B_DEV uint4 lds_v4(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

E4B_DEV uint32_t ldg_nc_u16(const uint16_t* p) {
  unsigned short r;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}

E4B_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// clamp(rint(fl(v * r)), -127, 127), ties to even, with r = fl(127 / amax):
// one fp32 product decides each int8 (r = 0 for a token treated as zero).
E4B_DEV int quant_x(float v, float r) {
  const int n = __float2int_rn(__fmul_rn(v, r));
  return min(max(n, -127), 127);
}

E4B_DEV uint32_t pack4(int a, int b, int c, int d) {
  return uint32_t(a & 0xFF) | (uint32_t(b & 0xFF) << 8) | (uint32_t(c & 0xFF) << 16) | (uint32_t(d & 0xFF) << 24);
}

// Stores the 8 quantised values of group g (weights 8i..8i+7 of block g / 4,
// i = g % 4) into the row's planes.
E4B_DEV void store_group(uint8_t* row, int64_t K, int64_t g, const int (&q)[8]) {
  const int64_t b = g >> 2;
  const int i = int(g & 3);
  uint8_t* dst = row + (i >> 1) * (K / 2) + b * 16 + (i & 1) * 8;
  *reinterpret_cast<uint2*>(dst) = make_uint2(pack4(q[0], q[2], q[4], q[6]), pack4(q[1], q[3], q[5], q[7]));
}

E4B_DEV float group_absmax(const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32(w[i] & 0xFFFFu)), fabsf(bf16_bits_to_f32(w[i] >> 16))));
  return m;
}

E4B_DEV int quant_group(const uint4 v, float r, int (&q)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    q[2 * i] = quant_x(__uint_as_float(w[i] << 16), r);
    q[2 * i + 1] = quant_x(__uint_as_float(w[i] & 0xFFFF0000u), r);
    sum += q[2 * i] + q[2 * i + 1];
  }
  return sum;
}

// Quantises one group of 8 activations of row `row` (values v) and stores
// them; returns their sum (0 for a group past the row).
E4B_DEV int quant_store(uint8_t* row, int64_t K, int64_t g, bool valid, const uint4 v, float r) {
  int q[8], sum = 0;
  if (valid) {
    sum = quant_group(v, r, q);
    store_group(row, K, g, q);
  }
  return sum;
}

// Block sums: the 4 groups of a block sit in 4 neighbouring lanes.
E4B_DEV void store_block_sum(uint8_t* row, int64_t K, int64_t g, bool valid, int sum) {
  sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
  sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
  if (valid && (g & 3) == 0) reinterpret_cast<int16_t*>(row + K)[g >> 2] = int16_t(-8 * sum);
}

// Quantises the nx activation rows into xs (row r at r * xrow_bytes(K): plane
// A, plane B, then the int16 -8 * sum(xq) of every block) and their scales
// into s_sx. Rows go two at a time; when a row has at most kQuantGroups groups
// of 8 values a thread, every load of both rows is issued at once and the
// values stay in registers between the max and the quantisation; longer rows
// are read twice. Whole block; ends with __syncthreads.
E4B_DEV void quantize_rows(const Int4Gemv& p, uint8_t* xs, float* s_sx, float* s_red) {
  const int tid = threadIdx.x, nthreads = blockDim.x, nwarps = nthreads >> 5;
  const int64_t K = p.K, G = K / 8;  // groups of 8 values; 4 groups a block
  const bool cached = G <= int64_t(kQuantGroups) * nthreads;
  const int passes = int((G + nthreads - 1) / nthreads);
  for (int r0 = 0; r0 < p.nx; r0 += 2) {
    const bool two = r0 + 1 < p.nx;
    const uint16_t* xa = p.x + r0 * p.ld_x;
    const uint16_t* xb = two ? xa + p.ld_x : xa;
    uint4 va[kQuantGroups], vb[kQuantGroups];
    float ma = 0.f, mb = 0.f;
    if (cached) {
#pragma unroll
      for (int i = 0; i < kQuantGroups; ++i) {
        const int64_t g = tid + int64_t(i) * nthreads;
        const bool ok = g < G;
        va[i] = ok ? *reinterpret_cast<const uint4*>(xa + 8 * g) : make_uint4(0, 0, 0, 0);
        vb[i] = (ok && two) ? *reinterpret_cast<const uint4*>(xb + 8 * g) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < kQuantGroups; ++i) {
        ma = fmaxf(ma, group_absmax(va[i]));
        mb = fmaxf(mb, group_absmax(vb[i]));
      }
    } else {
      for (int64_t g = tid; g < G; g += nthreads) {
        ma = fmaxf(ma, group_absmax(*reinterpret_cast<const uint4*>(xa + 8 * g)));
        if (two) mb = fmaxf(mb, group_absmax(*reinterpret_cast<const uint4*>(xb + 8 * g)));
      }
    }
    ma = warp_max(ma);
    mb = warp_max(mb);
    if ((tid & 31) == 0) s_red[2 * (tid >> 5)] = ma, s_red[2 * (tid >> 5) + 1] = mb;
    __syncthreads();
    float amax_a = 0.f, amax_b = 0.f;
    for (int w = 0; w < nwarps; ++w) amax_a = fmaxf(amax_a, s_red[2 * w]), amax_b = fmaxf(amax_b, s_red[2 * w + 1]);
    // r = fl(127 / amax); a token whose r is not finite is treated as zero
    float ra = __fdiv_rn(127.f, amax_a), rb = __fdiv_rn(127.f, amax_b);
    const bool za = !(amax_a > 0.f) || isinf(ra), zb = !(amax_b > 0.f) || isinf(rb);
    const float sxa = za ? 0.f : __fdiv_rn(amax_a, 127.f), sxb = zb ? 0.f : __fdiv_rn(amax_b, 127.f);
    ra = za ? 0.f : ra;
    rb = zb ? 0.f : rb;
    if (tid == 0) {
      s_sx[r0] = sxa;
      if (two) s_sx[r0 + 1] = sxb;
    }
    uint8_t* rowa = xs + r0 * xrow_bytes(K);
    uint8_t* rowb = rowa + xrow_bytes(K);
    // every thread runs the same passes: the block sums reduce over 4 lanes
    // with full-warp shuffles
    if (cached) {
#pragma unroll
      for (int i = 0; i < kQuantGroups; ++i) {
        if (i < passes) {
          const int64_t g = tid + int64_t(i) * nthreads;
          const bool ok = g < G;
          store_block_sum(rowa, K, g, ok, quant_store(rowa, K, g, ok, va[i], ra));
          if (two) store_block_sum(rowb, K, g, ok, quant_store(rowb, K, g, ok, vb[i], rb));
        }
      }
    } else {
      for (int i = 0; i < passes; ++i) {
        const int64_t g = tid + int64_t(i) * nthreads;
        const bool ok = g < G;
        const uint4 v0 = ok ? *reinterpret_cast<const uint4*>(xa + 8 * g) : make_uint4(0, 0, 0, 0);
        store_block_sum(rowa, K, g, ok, quant_store(rowa, K, g, ok, v0, ra));
        if (two) {
          const uint4 v1 = ok ? *reinterpret_cast<const uint4*>(xb + 8 * g) : make_uint4(0, 0, 0, 0);
          store_block_sum(rowb, K, g, ok, quant_store(rowb, K, g, ok, v1, rb));
        }
      }
    }
    __syncthreads();  // s_red is reused by the next row pair
  }
}

// ------------------------------------------------------------ the GEMV
// Outputs: a row pair of one slot (STORE), the gate/up pair of one h value
// (SWIGLU), one row of y over all slots (COMBINE). An item is two consecutive
// outputs of a CTA's round, one slot pair (COMBINE: np = ceil(n_slots / 2)
// pairs; else np = 1) and one chunk of 128 blocks. Its four rows:
//   STORE   (j, n), (j, n+1) | (j', n'), (j', n'+1)    of output pair o, o+1
//   SWIGLU  gate i, up i     | gate i', up i'
//   COMBINE (a, n), (b, n)   | (a, n+1), (b, n+1)       slots a = 2pp, b = a+1
struct __align__(16) ItemDesc {
  const uint16_t* s[kRows];  // scales of the chunk of each row (null: no row)
  uint32_t x0, x1;           // activation rows (byte offsets into xs)
  uint32_t pad;
  uint32_t nb;               // blocks in the chunk
  uint32_t acc;              // accumulator of the item's first output (2 floats an output)
  uint32_t flags;            // bits 0-3: row r present; bit 4: the item has its second output
  uint32_t ja, jb;           // COMBINE: slots a and b (jb == n_slots: none)
};
static_assert(sizeof(ItemDesc) == 64, "descriptor slot is 64 bytes");

// Stage position of row r: rows that are neighbours in memory (same expert,
// consecutive weight rows) sit in neighbouring positions, so that when a
// chunk is a whole row they arrive in one copy. STORE: rows n, n+1, n', n'+1;
// SWIGLU: gate i, gate i', up i, up i'; COMBINE: (a, n), (a, n+1), (b, n), (b, n+1).
template <int EPI>
__host__ __device__ constexpr int row_pos(int r) {
  return EPI == E4B_EPI_STORE ? r : (r == 1 ? 2 : r == 2 ? 1 : r);
}

struct Cursor {
  uint32_t c, pp, ol;  // chunk, slot pair, first output of the item within the round
  uint32_t j, n;       // slot and row of that output (COMBINE: n = row)
};

template <int EPI>
E4B_DEV void out_next(uint32_t& j, uint32_t& n, const Int4Gemv& p) {
  if constexpr (EPI == E4B_EPI_STORE) {
    n += 2;
    if (n >= uint32_t(p.N)) n = 0, ++j;
  } else if constexpr (EPI == E4B_EPI_SWIGLU) {
    if (++n == uint32_t(p.N / 2)) n = 0, ++j;
  } else {
    ++n;
  }
}

template <int EPI>
E4B_DEV void cursor_init(Cursor& k, uint32_t it, const Int4Gemv& p, const Int4Plan& q, uint32_t r0) {
  const uint32_t tl = it / q.nch;
  k.c = it - tl * q.nch;
  const uint32_t pair = tl / q.np;
  k.pp = tl - pair * q.np;
  k.ol = 2 * pair;
  const uint32_t o = r0 + k.ol;
  if constexpr (EPI == E4B_EPI_STORE) {
    const uint32_t tpr = uint32_t((p.N + 1) / 2);
    k.j = o / tpr;
    k.n = 2 * (o - k.j * tpr);
  } else if constexpr (EPI == E4B_EPI_SWIGLU) {
    const uint32_t I = uint32_t(p.N / 2);
    k.j = o / I;
    k.n = o - k.j * I;
  } else {
    k.j = 0;
    k.n = o;
  }
}

template <int EPI>
E4B_DEV void cursor_next(Cursor& k, const Int4Gemv& p, const Int4Plan& q) {
  if (++k.c < q.nch) return;
  k.c = 0;
  if (++k.pp < q.np) return;
  k.pp = 0;
  k.ol += 2;
  out_next<EPI>(k.j, k.n, p);
  out_next<EPI>(k.j, k.n, p);
}

E4B_DEV int64_t pick4(int i, int64_t v0, int64_t v1, int64_t v2, int64_t v3) {
  return i == 0 ? v0 : i == 1 ? v1 : i == 2 ? v2 : v3;
}

// The whole warp starts item k into a stage: lane 0 writes the descriptor and
// posts the expected bytes on the stage's barrier; lanes 0-3 then take one
// stage position each and copy its row chunk (two neighbouring rows in one
// copy when the chunk is the whole row and the rows are consecutive rows of
// one expert), and prefetch the row's scales into L2. `nout` = outputs of
// the round. Ends with every lane past a __syncwarp.
template <int EPI>
E4B_DEV void issue_item(const Cursor& k, uint32_t nout, const Int4Gemv& p, const Int4Plan& q,
                        const int32_t* s_ids, ItemDesc* d, uint8_t* stage, uint64_t* bar, int lane) {
  const int64_t N = p.N, NB = p.K / kI4Block, halfK = p.K / 2;
  const int64_t coff = int64_t(k.c) * kChunkBlocks;
  const uint32_t nb = uint32_t(min(int64_t(kChunkBlocks), NB - coff));
  const bool two = k.ol + 1 < nout;
  uint32_t j2 = k.j, n2 = k.n;
  out_next<EPI>(j2, n2, p);
  // expert (-1: none) and weight row of logical rows 0..3
  int e0, e1, e2, e3;
  int64_t w0, w1, w2, w3;
  uint32_t xj0, xj1, ja = 0, jb = 0;
  if constexpr (EPI == E4B_EPI_STORE) {
    const int ea = s_ids[k.j], eb = two ? s_ids[j2] : -1;
    e0 = ea, w0 = k.n;
    e1 = k.n + 1 < uint32_t(N) ? ea : -1, w1 = k.n + 1;
    e2 = eb, w2 = n2;
    e3 = (two && n2 + 1 < uint32_t(N)) ? eb : -1, w3 = n2 + 1;
    xj0 = k.j, xj1 = two ? j2 : k.j;
  } else if constexpr (EPI == E4B_EPI_SWIGLU) {
    const int64_t I = N / 2;
    const int ea = s_ids[k.j], eb = two ? s_ids[j2] : -1;
    e0 = ea, w0 = k.n;
    e1 = ea, w1 = k.n + I;
    e2 = eb, w2 = n2;
    e3 = eb, w3 = n2 + I;
    xj0 = k.j, xj1 = two ? j2 : k.j;
  } else {
    ja = 2 * k.pp, jb = ja + 1;
    const int ea = s_ids[ja], eb = jb < uint32_t(p.n_slots) ? s_ids[jb] : -1;
    e0 = ea, w0 = k.n;
    e1 = eb, w1 = k.n;
    e2 = two ? ea : -1, w2 = k.n + 1;
    e3 = two ? eb : -1, w3 = k.n + 1;
    xj0 = ja, xj1 = jb < uint32_t(p.n_slots) ? jb : ja;
  }
  const uint32_t flags = (two ? 16u : 0u) | (e0 >= 0 ? 1u : 0u) | (e1 >= 0 ? 2u : 0u) | (e2 >= 0 ? 4u : 0u) |
                         (e3 >= 0 ? 8u : 0u);
  if (lane == 0) {
    const uint32_t xrb = uint32_t(xrow_bytes(p.K));
    d->s[0] = e0 >= 0 ? p.scales + (int64_t(e0) * N + w0) * NB + coff : nullptr;
    d->s[1] = e1 >= 0 ? p.scales + (int64_t(e1) * N + w1) * NB + coff : nullptr;
    d->s[2] = e2 >= 0 ? p.scales + (int64_t(e2) * N + w2) * NB + coff : nullptr;
    d->s[3] = e3 >= 0 ? p.scales + (int64_t(e3) * N + w3) * NB + coff : nullptr;
    d->x0 = (p.nx == 1 ? 0 : xj0) * xrb;
    d->x1 = (p.nx == 1 ? 0 : xj1) * xrb;
    d->nb = nb;
    d->acc = 2 * k.ol;
    d->flags = flags;
    d->ja = ja;
    d->jb = jb;
    mbar_arrive_expect_tx(bar, uint32_t(__popc(flags & 15u)) * nb * (q.sbulk ? 18u : 16u));
  }
  __syncwarp();  // the expected bytes are posted before any copy lands
  if (lane < kRows) {
    // logical row at this position and at the next one
    const int r = row_pos<EPI>(lane);  // the position map is its own inverse
    const int rn = row_pos<EPI>((lane + 1) & 3);
    const int64_t e = pick4(r, e0, e1, e2, e3), w = pick4(r, w0, w1, w2, w3);
    const int64_t en = pick4(rn, e0, e1, e2, e3), wn = pick4(rn, w0, w1, w2, w3);
    const int rp = row_pos<EPI>((lane + 3) & 3);  // the previous position's row
    const int64_t ep = pick4(rp, e0, e1, e2, e3), wp = pick4(rp, w0, w1, w2, w3);
    // positions pair up as (0, 1) and (2, 3)
    const bool whole = q.nch == 1;
    const bool joins_next = whole && (lane & 1) == 0 && e >= 0 && en == e && wn == w + 1;
    const bool joined = whole && (lane & 1) == 1 && e >= 0 && ep == e && w == wp + 1;
    if (e >= 0 && !joined) {
      const int64_t er = e * N + w;
      const uint32_t rows = joins_next ? 2u : 1u;
      bulk_load(stage + lane * nb * 16, p.codes + er * halfK + coff * 16, rows * nb * 16, bar);
      const uint16_t* sc = p.scales + er * NB + coff;
      if (q.sbulk) {
        // scales ride with the codes (every row's chunk of them is 16-byte aligned)
        bulk_load(stage + kRows * nb * 16 + lane * nb * 2, sc, rows * nb * 2, bar);
      } else {
        prefetch_l2(sc);
        if (nb > 64) prefetch_l2(sc + 64);
        if (joins_next) {
          prefetch_l2(sc + NB);
          if (nb > 64) prefetch_l2(sc + NB + 64);
        }
      }
    }
  }
  __syncwarp();
}

// The lane's scales of an item: row r, lane block u (0 where the row is
// absent or the block is past the chunk).
E4B_DEV void load_scales(const ItemDesc& d, int lane, uint32_t (&h)[kRows][kLaneBlocks]) {
#pragma unroll
  for (int r = 0; r < kRows; ++r)
#pragma unroll
    for (int u = 0; u < kLaneBlocks; ++u) {
      const uint32_t lb = lane + 32 * u;
      h[r][u] = (((d.flags >> r) & 1u) && lb < d.nb) ? ldg_nc_u16(d.s[r] + lb) : 0u;
    }
}

template <int EPI>
__global__ void __launch_bounds__(kGemvThreads, 1) int4_gemv_kernel(const Int4Gemv p, const Int4Plan q) {
  extern __shared__ __align__(128) uint8_t smem[];
  float* s_sx = reinterpret_cast<float*>(smem);             // [64]
  int32_t* s_ids = reinterpret_cast<int32_t*>(smem + 256);  // [64], -1 = dropped slot
  float* s_gate = reinterpret_cast<float*>(smem + 512);     // [64]
  float* s_red = reinterpret_cast<float*>(smem + 768);      // [8 warps][2 rows]
  int32_t* s_abort = reinterpret_cast<int32_t*>(smem + 832);
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem + kBarOff);   // [8][kStages]
  ItemDesc* s_desc = reinterpret_cast<ItemDesc*>(smem + kDescOff);  // [8][kStages]
  uint8_t* xs = smem + kHeadBytes;
  float* s_acc = reinterpret_cast<float*>(smem + q.acc_off);
  uint8_t* ring = smem + q.ring_off;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool streams = warp < q.warps;
  uint8_t* my_ring = ring + size_t(warp) * kStages * kStageBytes;
  uint64_t* my_bar = s_bar + warp * kStages;
  ItemDesc* my_desc = s_desc + warp * kStages;
  const int64_t halfK = p.K / 2;

  // programmatic dependent launch: x, and unless the caller says otherwise
  // the ids and gates, may come from the kernel before this one in the
  // stream, and y may still be read by it
  const bool ids_ready = (p.flags & E4B_FLAG_IDS_READY) != 0;
  if (!ids_ready) grid_dependency_wait();
  if (tid < p.n_slots) {
    const int e = p.ids[tid];
    const bool bad = e < 0 || e >= p.E;
    if (bad && blockIdx.x == 0) record_status(p.status, E4B_ERR_BAD_EXPERT_ID);
    s_ids[tid] = bad ? -1 : e;
    s_gate[tid] = EPI == E4B_EPI_COMBINE ? p.gates[tid] : 0.f;
  }
  if (tid == 0) *s_abort = 0;
  if (streams && lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(my_bar + s, 1);
    mbar_init_fence();
  }
  __syncthreads();  // ids, gates, barriers

  const uint32_t O = uint32_t(q.outputs);
  const uint32_t o0 = uint32_t(uint64_t(blockIdx.x) * O / gridDim.x);
  const uint32_t o1 = uint32_t(uint64_t(blockIdx.x + 1) * O / gridDim.x);
  uint32_t parity = 0;  // bit s: parity of the next wait on stage s
  bool first = true;
  for (uint32_t r0 = o0; r0 < o1; r0 += kRoundOutputs) {
    const uint32_t nout = min(o1 - r0, uint32_t(kRoundOutputs));
    const uint32_t items = (nout + 1) / 2 * q.np * q.nch;
    const uint32_t i0 = streams ? uint32_t(uint64_t(warp) * items / q.warps) : 0;
    const uint32_t i1 = streams ? uint32_t(uint64_t(warp + 1) * items / q.warps) : 0;
    for (uint32_t i = tid; i < 2 * nout; i += blockDim.x) s_acc[i] = 0.f;
    // the activation rows are quantised before the first weight copies
    // start: copies issued earlier hold up the quantisation's loads behind
    // them (one token through the decode layer: quantisation 6-7 -> 4-5 us a
    // launch, the two-launch step 74.8 -> 70.7 us, timed on one B200)
    Cursor ki{}, kc{};
    if (i0 < i1) {
      cursor_init<EPI>(ki, i0, p, q, r0);
      kc = ki;
    }
    uint32_t issued = i0, waited = i0;
    if (first) {
      if (ids_ready) grid_dependency_wait();
      quantize_rows(p, xs, s_sx, s_red);  // ends with __syncthreads (s_acc cleared too)
      first = false;
    } else {
      __syncthreads();  // s_acc cleared
    }
    if (issued < i1) {
      issue_item<EPI>(ki, nout, p, q, s_ids, my_desc, my_ring, my_bar, lane);
      cursor_next<EPI>(ki, p, q);
      ++issued;
    }
    uint32_t hn[kRows][kLaneBlocks];  // scales of the next item (when they are not copied)
    if (!q.sbulk && i0 < i1) load_scales(my_desc[0], lane, hn);
    bool ok = true;
    for (uint32_t it = i0; it < i1; ++it) {
      // keep kStages items in flight: the stages of items before `it` are free
      while (issued < i1 && issued < it + kStages) {
        const int sn = int((issued - i0) % kStages);
        issue_item<EPI>(ki, nout, p, q, s_ids, my_desc + sn, my_ring + sn * kStageBytes, my_bar + sn, lane);
        cursor_next<EPI>(ki, p, q);
        ++issued;
      }
      const int s = int((it - i0) % kStages);
      // the descriptor was written before at least one __syncwarp
      const ItemDesc d = my_desc[s];
      // the inner loop has no branches, so the 16 block dot products of an
      // item overlap: a row that is absent, or a block past the chunk, gets
      // scale 0 (its reads stay inside this CTA's stage and activation rows).
      // The scales of the next item are loaded now (L2 hits after the
      // prefetch at issue time) and used one item later.
      uint32_t h[kRows][kLaneBlocks];
#pragma unroll
      for (int r = 0; r < kRows; ++r)
#pragma unroll
        for (int u = 0; u < kLaneBlocks; ++u) h[r][u] = hn[r][u];
      if (!q.sbulk && it + 1 < i1) load_scales(my_desc[(s + 1) % kStages], lane, hn);
      // polls == 0 (E4B_FLAG_TEST_TIMEOUT): give up at the first wait
      if (q.polls == 0 || !mbar_wait_bounded(my_bar + s, (parity >> s) & 1u, q.polls, s_abort)) {
        ok = false;
        break;
      }
      parity ^= 1u << s;
      ++waited;
      const uint8_t* st = my_ring + s * kStageBytes;
      if (q.sbulk) {
        const uint16_t* ss = reinterpret_cast<const uint16_t*>(st + kRows * d.nb * 16);
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
          for (int u = 0; u < kLaneBlocks; ++u) {
            const uint32_t lb = lane + 32 * u;
            const uint32_t v = ss[row_pos<EPI>(r) * d.nb + lb];
            h[r][u] = (((d.flags >> r) & 1u) && lb < d.nb) ? v : 0u;
          }
      }
      const uint8_t* x0 = xs + d.x0 + kc.c * kChunkBlocks * 16;
      const uint8_t* x1 = xs + d.x1 + kc.c * kChunkBlocks * 16;
      const int16_t* b0 = reinterpret_cast<const int16_t*>(xs + d.x0 + p.K) + kc.c * kChunkBlocks;
      const int16_t* b1 = reinterpret_cast<const int16_t*>(xs + d.x1 + p.K) + kc.c * kChunkBlocks;
      float a[kRows] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int u = 0; u < kLaneBlocks; ++u) {
        const uint32_t lb = lane + 32 * u;
        const uint4 xa0 = lds_v4(x0 + lb * 16), xb0 = lds_v4(x0 + halfK + lb * 16);
        const uint4 xa1 = lds_v4(x1 + lb * 16), xb1 = lds_v4(x1 + halfK + lb * 16);
        const int s0 = b0[lb], s1 = b1[lb];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          // the activation row of row r is fixed by the epilogue: rows 2, 3
          // (STORE / SWIGLU) or 1, 3 (COMBINE) read x1
          constexpr uint32_t kSel = EPI == E4B_EPI_COMBINE ? 0xAu : 0xCu;
          const uint4 w = lds_v4(st + (row_pos<EPI>(r) * d.nb + lb) * 16);
          const int v = ((kSel >> r) & 1u) ? block_dot16(w, xa1, xb1, s1) : block_dot16(w, xa0, xb0, s0);
          a[r] = fmaf(half_bits_to_f32(h[r][u]), float(v), a[r]);
        }
      }
      // four row sums leave the warp in one butterfly: after it, lane 8 m
      // (m = 0..3) holds the sum of value m
      if constexpr (EPI == E4B_EPI_COMBINE) {
        // y[n] += g_a sx_a / 16 * row (a, n) + g_b sx_b / 16 * row (b, n)
        const float ma = s_gate[d.ja] * s_sx[p.nx == 1 ? 0 : d.ja] * 0.0625f;
        const float mb = d.jb < uint32_t(p.n_slots) ? s_gate[d.jb] * s_sx[p.nx == 1 ? 0 : d.jb] * 0.0625f : 0.f;
        const float va = a[0] * ma + a[1] * mb, vb = a[2] * ma + a[3] * mb;
        const bool up = lane >= 16;
        float v = (up ? vb : va) + __shfl_xor_sync(0xFFFFFFFFu, up ? va : vb, 16);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        if (lane == 0) atomicAdd(s_acc + d.acc, v);
        if (lane == 16 && (d.flags & 16u)) atomicAdd(s_acc + d.acc + 2, v);
      } else {
        const bool up = lane >= 16;
        const float k0 = (up ? a[2] : a[0]) + __shfl_xor_sync(0xFFFFFFFFu, up ? a[0] : a[2], 16);
        const float k1 = (up ? a[3] : a[1]) + __shfl_xor_sync(0xFFFFFFFFu, up ? a[1] : a[3], 16);
        const bool odd = lane & 8;
        float v = (odd ? k1 : k0) + __shfl_xor_sync(0xFFFFFFFFu, odd ? k0 : k1, 8);
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        const int m = lane >> 3;  // value index held by lanes 8m..8m+7
        if ((lane & 7) == 0 && ((d.flags >> m) & 1u)) atomicAdd(s_acc + d.acc + m, v);
      }
      __syncwarp();  // every lane has read the stage and its descriptor before its refill
      cursor_next<EPI>(kc, p, q);
    }
    if (!ok) {
      // a wait gave up: record it, stop every warp, and let the copies this
      // warp started land before the CTA can exit
      if (lane == 0) {
        record_status(p.status, E4B_ERR_DEVICE_TIMEOUT);
        atomicExch(s_abort, 1);
      }
      for (uint32_t x = waited; x < issued; ++x) {  // issued, not yet waited on
        const int s = int((x - i0) % kStages);
        mbar_wait_bounded(my_bar + s, (parity >> s) & 1u, kWaitPolls, nullptr);
        parity ^= 1u << s;
      }
    }
    // every copy of this CTA has been issued: the next grid may start
    // launching (its CTAs take SMs as this grid's CTAs leave)
    if (r0 + kRoundOutputs >= o1) grid_launch_dependents();
    __syncthreads();  // all sums of the round are in s_acc
    const bool aborted = *reinterpret_cast<volatile int32_t*>(s_abort) != 0;
    for (uint32_t ol = tid; ol < nout && !aborted; ol += blockDim.x) {
      const uint32_t o = r0 + ol;
      const float g = s_acc[2 * ol], u = s_acc[2 * ol + 1];
      if constexpr (EPI == E4B_EPI_STORE) {
        const uint32_t tpr = uint32_t((p.N + 1) / 2);
        const uint32_t j = o / tpr, n = 2 * (o - j * tpr);
        const float f = s_sx[p.nx == 1 ? 0 : j] * 0.0625f;
        p.y[int64_t(j) * p.ld_y + n] = to_bf16_bits(g * f);
        if (n + 1 < uint32_t(p.N)) p.y[int64_t(j) * p.ld_y + n + 1] = to_bf16_bits(u * f);
      } else if constexpr (EPI == E4B_EPI_SWIGLU) {
        const uint32_t I = uint32_t(p.N / 2);
        const uint32_t j = o / I, i = o - j * I;
        const float f = s_sx[p.nx == 1 ? 0 : j] * 0.0625f;
        p.y[int64_t(j) * p.ld_y + i] = s_ids[j] >= 0 ? to_bf16_bits(silu_mul(g * f, u * f)) : uint16_t(0);
      } else {
        p.y[o] = to_bf16_bits(g);
      }
    }
    __syncthreads();  // s_acc is cleared by the next round
    if (aborted) break;
  }
}

// One thread per 32-weight block: s = fp16(fp32(absmax / 7)),
// q = clamp(rint(fp32(w / s)), -8, 7) (0 where s is 0), nibbles packed with
// the earlier weight low.
__global__ void __launch_bounds__(256) quantize_int4_kernel(const float* __restrict__ w, int64_t nblocks,
                                                            uint8_t* __restrict__ codes,
                                                            uint16_t* __restrict__ scales) {
  for (int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; b < nblocks;
       b += int64_t(gridDim.x) * blockDim.x) {
    const float4* src = reinterpret_cast<const float4*>(w + b * kI4Block);
    float v[kI4Block];
#pragma unroll
    for (int i = 0; i < kI4Block / 4; ++i) {
      const float4 f = src[i];
      v[4 * i] = f.x;
      v[4 * i + 1] = f.y;
      v[4 * i + 2] = f.z;
      v[4 * i + 3] = f.w;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < kI4Block; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const __half s16 = __float2half_rn(__fdiv_rn(amax, 7.f));
    const float s = __half2float(s16);
    uint32_t word[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < kI4Block; ++i) {
      int q = 0;
      if (s > 0.f) q = int(fminf(fmaxf(rintf(__fdiv_rn(v[i], s)), -8.f), 7.f));
      word[i >> 3] |= uint32_t(q & 15) << (4 * (i & 7));
    }
    *reinterpret_cast<uint4*>(codes + b * 16) = make_uint4(word[0], word[1], word[2], word[3]);
    scales[b] = __half_as_ushort(s16);
  }
}

// out[z][c][r] = in[z][r][c] ^ mask through a 32 x 32 shared tile (block 32 x 8).
template <typename T>
__global__ void __launch_bounds__(256) transpose_xor_kernel(const T* __restrict__ in, T* __restrict__ out,
                                                            int64_t rows, int64_t cols, T mask) {
  __shared__ T tile[32][33];
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int64_t r0 = int64_t(blockIdx.y) * 32, c0 = int64_t(blockIdx.x) * 32;
  const T* src = in + int64_t(blockIdx.z) * rows * cols;
  T* dst = out + int64_t(blockIdx.z) * rows * cols;
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int64_t r = r0 + ty + i, c = c0 + tx;
    if (r < rows && c < cols) tile[ty + i][tx] = src[r * cols + c];
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int64_t c = c0 + ty + i, r = r0 + tx;
    if (r < rows && c < cols) dst[c * rows + r] = T(tile[tx][ty + i] ^ mask);
  }
}


}  // namespace

static size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared memory of the GEMV: head, the nx quantised activation rows, the
// round's accumulators, and kStages stages of every streaming warp.
static size_t acc_offset(int nx, int64_t K) {
  return round_up(size_t(kHeadBytes) + size_t(nx) * size_t(xrow_bytes(K)), 128);
}
static size_t ring_offset(int nx, int64_t K) {
  return round_up(acc_offset(nx, K) + size_t(kRoundOutputs) * 2 * sizeof(float), 128);
}

size_t int4_gemv_smem_bytes(int nx, int64_t K, int warps) {
  return ring_offset(nx, K) + size_t(warps) * kStages * kStageBytes;
}

int int4_gemv_max_slots() { return kMaxSlots; }

int int4_gemv_warps(int nx, int64_t K) {
  int dev = 0, smem_max = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (smem_max <= 0) smem_max = 227 * 1024;
  int w = kGemvWarps;
  while (w > 0 && int4_gemv_smem_bytes(nx, K, w) > size_t(smem_max)) --w;
  return w;
}

cudaError_t launch_int4_gemv(const Int4Gemv& p, cudaStream_t st, int sms) {
  Int4Plan q{};
  q.warps = int4_gemv_warps(p.nx, p.K);
  if (q.warps <= 0) return cudaErrorInvalidValue;
  const int64_t NB = p.K / kI4Block;
  q.nch = uint32_t((NB + kChunkBlocks - 1) / kChunkBlocks);
  q.np = p.epilogue == E4B_EPI_COMBINE ? uint32_t((p.n_slots + 1) / 2) : 1u;
  q.outputs = p.epilogue == E4B_EPI_STORE    ? int64_t(p.n_slots) * ((p.N + 1) / 2)
              : p.epilogue == E4B_EPI_SWIGLU ? int64_t(p.n_slots) * (p.N / 2)
                                             : p.N;
  q.polls = (p.flags & E4B_FLAG_TEST_TIMEOUT) ? 0u : kWaitPolls;
  q.sbulk = (NB % 8 == 0 && (reinterpret_cast<uintptr_t>(p.scales) & 15u) == 0) ? 1u : 0u;
  q.acc_off = uint32_t(acc_offset(p.nx, p.K));
  q.ring_off = uint32_t(ring_offset(p.nx, p.K));
  const size_t smem = int4_gemv_smem_bytes(p.nx, p.K, q.warps);
  // one CTA per SM; at least two outputs a CTA
  const int64_t want = (q.outputs + 1) / 2;
  const int grid = int(want < int64_t(sms) ? want : int64_t(sms));
  if (grid <= 0) return cudaSuccess;
  auto launch = [&](auto kernel) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: the kernel waits on its predecessor in
    // the stream itself (griddepcontrol.wait) before it reads x or writes y
    return launch_dependent(kernel, dim3(grid), dim3(kGemvThreads), smem, st, p, q);
  };
  switch (p.epilogue) {
    case E4B_EPI_STORE: return launch(int4_gemv_kernel<E4B_EPI_STORE>);
    case E4B_EPI_SWIGLU: return launch(int4_gemv_kernel<E4B_EPI_SWIGLU>);
    default: return launch(int4_gemv_kernel<E4B_EPI_COMBINE>);
  }
}

cudaError_t launch_quantize_int4(const float* w, int64_t nblocks, uint8_t* codes, uint16_t* scales,
                                 cudaStream_t st, int sms) {
  if (nblocks <= 0) return cudaSuccess;
  const int64_t want = (nblocks + 255) / 256;
  const int grid = int(want < int64_t(sms) * 8 ? want : int64_t(sms) * 8);
  quantize_int4_kernel<<<grid, 256, 0, st>>>(w, nblocks, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_gptq_repack(const int32_t* qweight, const uint16_t* gscales, int64_t E, int64_t N, int64_t K,
                               uint8_t* codes, uint16_t* scales, cudaStream_t st) {
  if (E <= 0 || N <= 0 || K <= 0) return cudaSuccess;
  const dim3 block(32, 8);
  // qweight [E, K/8, N] words -> codes [E, N, K/8] words; u ^ 8 == (u - 8) & 15 per nibble
  const dim3 g1(unsigned((N + 31) / 32), unsigned((K / 8 + 31) / 32), unsigned(E));
  transpose_xor_kernel<uint32_t><<<g1, block, 0, st>>>(reinterpret_cast<const uint32_t*>(qweight),
                                                       reinterpret_cast<uint32_t*>(codes), K / 8, N,
                                                       0x88888888u);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 g2(unsigned((N + 31) / 32), unsigned((K / 32 + 31) / 32), unsigned(E));
  transpose_xor_kernel<uint16_t><<<g2, block, 0, st>>>(gscales, scales, K / 32, N, uint16_t(0));
  return cudaGetLastError();
}

}  // namespace e4b
