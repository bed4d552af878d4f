// The C ABI of libe4b: argument checks, workspace layout, path choice and
// launch order. Every entry point is declared and documented in include/e4b.h.
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "ep.h"
#include "launch.h"

namespace {

using namespace e4b;

thread_local int32_t g_last_path = E4B_PATH_NONE;
thread_local int32_t g_last_launches = 0;
thread_local cudaEvent_t g_events[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
thread_local bool g_timing = false;

void mark(int i, cudaStream_t s) {
  if (g_timing) cudaEventRecord(g_events[i], s);
}

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace of the layer forward. After the routing arrays and h comes one
// fp32 region that the small-M path uses for the partial sums of its down
// passes, [K slices][T*top_k][H] (needs up to small_min), and the large-M path
// for the gate-weighted rows [T*top_k, H] (needs up to large_min); xs (the
// routed rows of x in expert order) is the large-M path's staging copy, after
// the larger of the two, used when the workspace reaches total.
struct MoeWs {
  size_t status, sync, nsync, counts, offsets, perm, inv, h, acc, small_min, rows, large_min, xs, total;
};

MoeWs moe_ws_layout(int64_t E, int64_t H, int64_t I, int64_t T, int64_t top_k) {
  MoeWs w;
  const int64_t R = T * top_k;
  size_t o = 0;
  w.status = o;  o += kStatusBytes;
  w.nsync = smallm_sync_ints(int(E), int(H));
  w.sync = o;    o = align_up(o + w.nsync * 4, 256);
  w.counts = o;  o = align_up(o + size_t(E) * 4, 256);
  w.offsets = o; o = align_up(o + size_t(E + 1) * 8, 256);
  w.perm = o;    o = align_up(o + size_t(R) * 4, 256);
  w.inv = o;     o = align_up(o + size_t(R) * 4, 256);
  w.h = o;       o = align_up(o + size_t(R) * size_t(I) * 2, 256);
  w.acc = o;
  w.rows = o;
  w.small_min = align_up(o + size_t(smallm_k_slices(int(I))) * size_t(R) * size_t(H) * 4, 256);
  w.large_min = align_up(o + size_t(R) * size_t(H) * 4, 256);
  o = w.small_min > w.large_min ? w.small_min : w.large_min;
  w.xs = o;      o = align_up(o + size_t(R) * size_t(H) * 2, 256);
  w.total = o;
  return w;
}

// Workspace regions of the block-scaled MXFP4 path, after the routing
// arrays, h and the gate-weighted rows (the staging copy's place): the two
// e4m3 terms of x and of h in padded per-expert rows, their scale chunks, and
// bf16 h in padded rows.
struct MxWs {
  int64_t Rp_max, Hp, Ip;
  size_t xq, sfx, hp, hq, sfh, total;
};

MxWs mx_ws_layout(const MoeWs& L, int64_t E, int64_t H, int64_t I, int64_t T, int64_t top_k) {
  MxWs m;
  m.Rp_max = mx_padded_rows_max(T * top_k, E);
  m.Hp = (H + 127) / 128 * 128;
  m.Ip = (I + 127) / 128 * 128;
  const size_t rp = size_t(m.Rp_max);
  size_t o = L.large_min;
  m.xq = o;  o = align_up(o + 2 * rp * size_t(m.Hp), 256);
  m.sfx = o; o = align_up(o + 2 * (rp / kMxRowBlock) * size_t(m.Hp / 128) * 512, 256);
  m.hp = o;  o = align_up(o + rp * size_t(I) * 2, 256);
  m.hq = o;  o = align_up(o + 2 * rp * size_t(m.Ip), 256);
  m.sfh = o; o = align_up(o + 2 * (rp / kMxRowBlock) * size_t(m.Ip / 128) * 512, 256);
  m.total = o;
  return m;
}

bool has_mx(const e4b_moe_weights* w) {
  return w->fmt == E4B_FMT_MXFP4 && w->gate_up_mx_codes && w->gate_up_mx_sf && w->down_mx_codes &&
         w->down_mx_sf;
}

}  // namespace

size_t e4b::moe_workspace_min_bytes(const e4b_moe_weights* w, int64_t T, int64_t top_k, uint32_t flags) {
  const MoeWs L = moe_ws_layout(w->E, w->H, w->I, T, top_k);
  if (layer_uses_small_m(T * top_k, w->E, flags)) return L.small_min;
  if (has_mx(w) && !(flags & E4B_FLAG_MX_DECODE)) return mx_ws_layout(L, w->E, w->H, w->I, T, top_k).total;
  return L.large_min;
}

namespace {

e4b_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return E4B_OK;
  return E4B_ERR_CUDA;
}

// Shape rules shared by both kernel families.
e4b_status check_projection(int fmt, int64_t N, int64_t K, bool swiglu) {
  if (fmt != E4B_FMT_NF4 && fmt != E4B_FMT_MXFP4) return E4B_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0) return E4B_ERR_INVALID_ARG;
  if (N % (swiglu ? 32 : 16)) return E4B_ERR_UNSUPPORTED;
  if (fmt == E4B_FMT_NF4 && K % E4B_NF4_BLOCK) return E4B_ERR_UNSUPPORTED;
  if (fmt == E4B_FMT_MXFP4 && K % E4B_MXFP4_BLOCK) return E4B_ERR_UNSUPPORTED;
  return E4B_OK;
}

// Expert-variant fields (include/e4b.h): known codes, a usable clamp limit
// and a 16-byte aligned bias.
e4b_status check_variant(int32_t layout, int32_t act, float limit, const float* b0,
                         const float* b1) {
  if (layout != E4B_GATE_UP_HALVES && layout != E4B_GATE_UP_INTERLEAVED) return E4B_ERR_INVALID_ARG;
  if (act != E4B_ACT_SWIGLU && act != E4B_ACT_CLAMPED_GLU) return E4B_ERR_INVALID_ARG;
  if (act == E4B_ACT_CLAMPED_GLU && !(limit >= 0.f)) return E4B_ERR_INVALID_ARG;
  if (!aligned16(b0) || !aligned16(b1)) return E4B_ERR_MISALIGNED;
  return E4B_OK;
}

// Small-M when an expert sees few rows on average; the tcgen05 kernel needs
// E <= 256 for its on-chip expert table.
bool choose_gemv(int64_t R, int64_t E, uint32_t flags) {
  if (flags & E4B_FLAG_FORCE_GEMV) return true;
  if (flags & E4B_FLAG_FORCE_TCGEN05) return false;
  if (E > 256) return true;
  return R <= 16 * E;
}

}  // namespace

bool e4b::layer_uses_small_m(int64_t R, int64_t E, uint32_t flags) { return choose_gemv(R, E, flags); }

namespace {

e4b_status run_projection(const GemmProblem& p, bool gemv, cudaStream_t st) {
  const int sms = sm_count();
  cudaError_t e = gemv ? launch_gemv(p, st, sms) : launch_tc_gemm(p, st, sms);
  return cuda_status(e);
}

}  // namespace

extern "C" {

const char* e4b_version(void) { return "e4b 0.1.0 sm_100a"; }

const char* e4b_status_string(int32_t s) {
  switch (s) {
    case E4B_OK: return "ok";
    case E4B_ERR_INVALID_ARG: return "invalid argument";
    case E4B_ERR_UNSUPPORTED: return "unsupported shape";
    case E4B_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case E4B_ERR_CUDA: return "CUDA error";
    case E4B_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case E4B_ERR_BAD_EXPERT_ID: return "expert id out of range";
    case E4B_ERR_MISALIGNED: return "misaligned pointer or stride";
    case E4B_ERR_EXCEEDS_STATIC_SCRATCH: return "needs more than the 16 MiB static scratch";
    default: return "unknown status";
  }
}

int32_t e4b_last_path(void) { return g_last_path; }

e4b_status e4b_set_timing_events(void* const* events, int32_t n) {
  if (n == 0) {
    g_timing = false;
    return E4B_OK;
  }
  if (n != 5 || !events) return E4B_ERR_INVALID_ARG;
  for (int i = 0; i < 5; ++i) {
    if (!events[i]) return E4B_ERR_INVALID_ARG;
    g_events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  g_timing = true;
  return E4B_OK;
}
int32_t e4b_last_launch_count(void) { return g_last_launches; }

e4b_status e4b_nf4_codebook(float* out_host) {
  if (!out_host) return E4B_ERR_INVALID_ARG;
  host_nf4_levels(out_host);
  return E4B_OK;
}

e4b_status e4b_quantize_nf4(const float* w, int64_t E, int64_t N, int64_t K, int32_t blocksize,
                            uint8_t* codes, float* absmax, void* stream) {
  if (!w || !codes || !absmax || E <= 0 || N <= 0 || K <= 0) return E4B_ERR_INVALID_ARG;
  if (blocksize != E4B_NF4_BLOCK || K % E4B_NF4_BLOCK) return E4B_ERR_UNSUPPORTED;
  if (!aligned16(w) || (reinterpret_cast<uintptr_t>(codes) & 3u) ||
      (reinterpret_cast<uintptr_t>(absmax) & 3u))
    return E4B_ERR_MISALIGNED;
  const int64_t nblocks = E * N * (K / E4B_NF4_BLOCK);
  return cuda_status(launch_quantize_nf4(w, nblocks, codes, absmax,
                                         static_cast<cudaStream_t>(stream), sm_count()));
}

e4b_status e4b_quantize_mxfp4(const float* w, int64_t E, int64_t N, int64_t K, uint8_t* blocks,
                              uint8_t* scales, void* stream) {
  if (!w || !blocks || !scales || E <= 0 || N <= 0 || K <= 0) return E4B_ERR_INVALID_ARG;
  if (K % E4B_MXFP4_BLOCK) return E4B_ERR_UNSUPPORTED;
  if (!aligned16(w) || (reinterpret_cast<uintptr_t>(blocks) & 3u)) return E4B_ERR_MISALIGNED;
  const int64_t nblocks = E * N * (K / E4B_MXFP4_BLOCK);
  return cuda_status(launch_quantize_mxfp4(w, nblocks, blocks, scales,
                                           static_cast<cudaStream_t>(stream), sm_count()));
}

e4b_status e4b_dequantize(int32_t fmt, const uint8_t* codes, const void* scales, int64_t E,
                          int64_t N, int64_t K, uint16_t* out, void* stream) {
  if (!codes || !scales || !out || E <= 0 || N <= 0 || K <= 0) return E4B_ERR_INVALID_ARG;
  if (fmt != E4B_FMT_NF4 && fmt != E4B_FMT_MXFP4) return E4B_ERR_INVALID_ARG;
  if (fmt == E4B_FMT_NF4 && K % E4B_NF4_BLOCK) return E4B_ERR_UNSUPPORTED;
  if (fmt == E4B_FMT_MXFP4 && K % E4B_MXFP4_BLOCK) return E4B_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(codes) & 3u) || !aligned16(out)) return E4B_ERR_MISALIGNED;
  if (fmt == E4B_FMT_NF4 && (reinterpret_cast<uintptr_t>(scales) & 3u)) return E4B_ERR_MISALIGNED;
  return cuda_status(launch_dequantize(fmt, codes, scales, E * N * K, out,
                                       static_cast<cudaStream_t>(stream), sm_count()));
}

e4b_status e4b_route_workspace_size(int64_t T, int32_t top_k, int32_t E, size_t* bytes) {
  if (!bytes || T < 0 || top_k <= 0 || E <= 0) return E4B_ERR_INVALID_ARG;
  const int64_t R = T * int64_t(top_k);
  *bytes = kStatusBytes + (E <= 1024 && R < (int64_t(1) << 31) ? route_scratch_bytes(int32_t(R), E) : 0);
  return E4B_OK;
}

e4b_status e4b_route(const int32_t* ids, int64_t T, int32_t top_k, int32_t E, int32_t* counts,
                     int64_t* offsets, int32_t* perm, int32_t* inv_perm, void* ws, size_t ws_bytes,
                     void* stream) {
  if (T < 0 || top_k <= 0 || E <= 0) return E4B_ERR_INVALID_ARG;
  if (!counts || !offsets || !ws || (T > 0 && (!ids || !perm || !inv_perm)))
    return E4B_ERR_INVALID_ARG;
  if (E > 1024 || T * int64_t(top_k) >= (int64_t(1) << 31)) return E4B_ERR_UNSUPPORTED;
  if (ws_bytes < size_t(kStatusBytes)) return E4B_ERR_WORKSPACE_TOO_SMALL;
  int launches = 1;
  // the status words, then (large batches) the many-CTA pass's scratch
  const e4b_status st = cuda_status(launch_route(
      ids, int32_t(T * top_k), E, counts, offsets, perm, inv_perm, nullptr, static_cast<int32_t*>(ws),
      static_cast<cudaStream_t>(stream), nullptr, 0,
      reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kStatusBytes), ws_bytes - kStatusBytes, &launches));
  g_last_launches = launches;
  return st;
}

e4b_status e4b_grouped_gemm(const e4b_gemm_args* a, uint32_t flags, void* stream) {
  if (!a) return E4B_ERR_INVALID_ARG;
  if (a->E <= 0 || a->top_k <= 0 || a->R_max < 0) return E4B_ERR_INVALID_ARG;
  if (a->epilogue < E4B_EPI_STORE || a->epilogue > E4B_EPI_COMBINE) return E4B_ERR_INVALID_ARG;
  e4b_status st = check_projection(a->fmt, a->N, a->K, a->epilogue == E4B_EPI_SWIGLU);
  if (st != E4B_OK) return st;
  if (!a->codes || !a->scales || !a->a || !a->offsets || !a->out) return E4B_ERR_INVALID_ARG;
  if (a->epilogue == E4B_EPI_COMBINE && !a->gates) return E4B_ERR_INVALID_ARG;
  if (!aligned16(a->codes) || !aligned16(a->a) || !aligned16(a->out) || a->lda % 8 || a->ldo % 8)
    return E4B_ERR_MISALIGNED;
  if (a->lda < a->K) return E4B_ERR_INVALID_ARG;
  st = check_variant(a->gate_up_layout, a->activation, a->glu_limit, a->bias, nullptr);
  if (st != E4B_OK) return st;
  if (a->R_max == 0) return E4B_OK;
  const bool gemv = choose_gemv(a->R_max, a->E, flags);
  if (!gemv && a->E > 256) return E4B_ERR_UNSUPPORTED;
  GemmProblem p{};
  p.fmt = a->fmt;
  p.epilogue = a->epilogue;
  p.E = a->E;
  p.top_k = a->top_k;
  p.N = a->N;
  p.K = a->K;
  p.R_max = a->R_max;
  p.codes = a->codes;
  p.scales = a->scales;
  p.a = a->a;
  p.lda = a->lda;
  p.row_slot = a->a_row_slot;
  p.out_slot = a->out_row_slot;
  p.offsets = a->offsets;
  p.gates = a->gates;
  p.out = a->out;
  p.ldo = a->ldo;
  p.flags = flags;
  p.layout = a->gate_up_layout;
  p.act = a->activation;
  p.alpha = a->glu_alpha;
  p.limit = a->glu_limit;
  p.bias = a->bias;
  g_last_path = gemv ? E4B_PATH_GEMV : E4B_PATH_TCGEN05;
  g_last_launches = 1;
  return run_projection(p, gemv, static_cast<cudaStream_t>(stream));
}

e4b_status e4b_grouped_dgrad(const e4b_dgrad_args* a, uint32_t flags, void* stream) {
  if (!a) return E4B_ERR_INVALID_ARG;
  if (a->E <= 0 || a->R_max < 0) return E4B_ERR_INVALID_ARG;
  if (a->fmt != E4B_FMT_NF4 && a->fmt != E4B_FMT_MXFP4) return E4B_ERR_INVALID_ARG;
  if (a->N <= 0 || a->K <= 0) return E4B_ERR_INVALID_ARG;
  if (a->fmt == E4B_FMT_NF4 && a->K % E4B_NF4_BLOCK) return E4B_ERR_UNSUPPORTED;
  if (a->fmt == E4B_FMT_MXFP4 && a->K % E4B_MXFP4_BLOCK) return E4B_ERR_UNSUPPORTED;
  if (a->E > 256 || (flags & E4B_FLAG_FORCE_GEMV)) return E4B_ERR_UNSUPPORTED;
  if (!a->codes || !a->scales || !a->dy || !a->offsets || !a->dx) return E4B_ERR_INVALID_ARG;
  if (!aligned16(a->codes) || !aligned16(a->dy) || !aligned16(a->dx) || a->ld_dy % 8 || a->ld_dx % 8)
    return E4B_ERR_MISALIGNED;
  if (a->ld_dy < a->N || a->ld_dx < a->K) return E4B_ERR_INVALID_ARG;
  if (a->R_max == 0) return E4B_OK;
  GemmProblem p{};
  p.fmt = a->fmt;
  p.epilogue = kEpiDgrad;
  p.E = a->E;
  p.top_k = 1;
  p.N = a->N;
  p.K = a->K;
  p.R_max = a->R_max;
  p.codes = a->codes;
  p.scales = a->scales;
  p.a = a->dy;
  p.lda = a->ld_dy;
  p.offsets = a->offsets;
  p.out = a->dx;
  p.ldo = a->ld_dx;
  p.flags = flags;
  g_last_path = E4B_PATH_TCGEN05;
  g_last_launches = 1;
  return cuda_status(launch_tc_gemm(p, static_cast<cudaStream_t>(stream), sm_count()));
}

e4b_status e4b_quantize_int4_b32(const float* w, int64_t E, int64_t N, int64_t K, uint8_t* codes,
                                 uint16_t* scales, void* stream) {
  if (E < 0 || N < 0 || K < 0) return E4B_ERR_INVALID_ARG;
  if (K % E4B_INT4_BLOCK) return E4B_ERR_UNSUPPORTED;
  const int64_t nblocks = E * N * (K / E4B_INT4_BLOCK);
  g_last_launches = 0;
  if (nblocks == 0) return E4B_OK;
  if (!w || !codes || !scales) return E4B_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 1u)) return E4B_ERR_MISALIGNED;
  g_last_launches = 1;
  return cuda_status(launch_quantize_int4(w, nblocks, codes, scales, static_cast<cudaStream_t>(stream),
                                          sm_count()));
}

e4b_status e4b_gptq_pack_int4_b32(const int32_t* qweight, const uint16_t* gptq_scales, int64_t E,
                                  int64_t N, int64_t K, uint8_t* codes, uint16_t* scales,
                                  void* stream) {
  if (E < 0 || N < 0 || K < 0) return E4B_ERR_INVALID_ARG;
  if (K % E4B_INT4_BLOCK) return E4B_ERR_UNSUPPORTED;
  if (E > 65535 || (N + 31) / 32 > 0x7FFFFFFF || K / 256 + 1 > 65535) return E4B_ERR_UNSUPPORTED;
  g_last_launches = 0;
  if (E == 0 || N == 0 || K == 0) return E4B_OK;
  if (!qweight || !gptq_scales || !codes || !scales) return E4B_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(qweight) & 3u) || (reinterpret_cast<uintptr_t>(codes) & 3u) ||
      (reinterpret_cast<uintptr_t>(gptq_scales) & 1u) || (reinterpret_cast<uintptr_t>(scales) & 1u))
    return E4B_ERR_MISALIGNED;
  g_last_launches = 2;
  return cuda_status(launch_gptq_repack(qweight, gptq_scales, E, N, K, codes, scales,
                                        static_cast<cudaStream_t>(stream)));
}

e4b_status e4b_gemv_int4_b32(const e4b_int4_gemv_args* a, uint32_t flags, void* stream) {
  if (!a || (flags & ~(E4B_FLAG_TEST_TIMEOUT | E4B_FLAG_IDS_READY))) return E4B_ERR_INVALID_ARG;
  if (a->epilogue != E4B_EPI_STORE && a->epilogue != E4B_EPI_SWIGLU && a->epilogue != E4B_EPI_COMBINE)
    return E4B_ERR_INVALID_ARG;
  if (a->E <= 0 || a->N <= 0 || a->K <= 0 || a->n_slots <= 0 || a->ld_x < 0) return E4B_ERR_INVALID_ARG;
  if (a->n_slots > int4_gemv_max_slots()) return E4B_ERR_UNSUPPORTED;
  if (a->K % E4B_INT4_BLOCK) return E4B_ERR_UNSUPPORTED;
  if (a->epilogue == E4B_EPI_SWIGLU && a->N % 2) return E4B_ERR_INVALID_ARG;
  if (!a->codes || !a->scales || !a->expert_ids || !a->x || !a->y) return E4B_ERR_INVALID_ARG;
  if (a->epilogue == E4B_EPI_COMBINE && !a->gates) return E4B_ERR_INVALID_ARG;
  if (!aligned16(a->codes) || !aligned16(a->x) || (reinterpret_cast<uintptr_t>(a->y) & 1u) ||
      (reinterpret_cast<uintptr_t>(a->scales) & 1u) || a->ld_x % 8)
    return E4B_ERR_MISALIGNED;
  if (a->ld_x != 0 && a->ld_x < a->K) return E4B_ERR_INVALID_ARG;
  if (a->epilogue == E4B_EPI_STORE && a->ld_y < a->N) return E4B_ERR_INVALID_ARG;
  if (a->epilogue == E4B_EPI_SWIGLU && a->ld_y < a->N / 2) return E4B_ERR_INVALID_ARG;
  const int nx = a->ld_x == 0 ? 1 : a->n_slots;
  if (int64_t(nx) * a->K > 200 * 1024) return E4B_ERR_UNSUPPORTED;
  // outputs and items are counted in 32 bits
  const int64_t outputs = a->epilogue == E4B_EPI_COMBINE ? a->N : int64_t(a->n_slots) * ((a->N + 1) / 2);
  if (outputs * ((a->n_slots + 1) / 2) * ((a->K / E4B_INT4_BLOCK + 127) / 128) >= (int64_t(1) << 31))
    return E4B_ERR_UNSUPPORTED;
  Int4Gemv p{};
  p.epilogue = a->epilogue;
  p.E = a->E;
  p.n_slots = a->n_slots;
  p.nx = nx;
  p.N = a->N;
  p.K = a->K;
  p.codes = a->codes;
  p.scales = a->scales;
  p.ids = a->expert_ids;
  p.gates = a->gates;
  p.x = a->x;
  p.ld_x = a->ld_x;
  p.y = a->y;
  p.ld_y = a->ld_y;
  p.status = a->status;
  p.flags = flags;
  if (int4_gemv_warps(nx, a->K) <= 0) return E4B_ERR_UNSUPPORTED;
  g_last_path = E4B_PATH_INT4_GEMV;
  g_last_launches = 1;
  return cuda_status(launch_int4_gemv(p, static_cast<cudaStream_t>(stream), sm_count()));
}

e4b_status e4b_ep_dest(const int32_t* ids, int64_t n, int32_t E, int32_t epr, int32_t* dest, void* stream) {
  if (n < 0 || E <= 0 || epr <= 0 || E % epr) return E4B_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (n == 0) return E4B_OK;
  if (!ids || !dest) return E4B_ERR_INVALID_ARG;
  g_last_launches = 1;
  return cuda_status(launch_ep_dest(ids, n, E, epr, dest, static_cast<cudaStream_t>(stream), sm_count()));
}

e4b_status e4b_ep_pack(const uint16_t* x, int64_t H, const int32_t* ids, const float* gates, int32_t top_k,
                       const int32_t* perm, const int64_t* offsets, int32_t G, int64_t R_max, int32_t epr,
                       uint16_t* xs, int32_t* local_ids, float* local_gates, void* stream) {
  if (H <= 0 || top_k <= 0 || G <= 0 || R_max < 0 || epr <= 0) return E4B_ERR_INVALID_ARG;
  if (H % 8) return E4B_ERR_UNSUPPORTED;
  g_last_launches = 0;
  if (R_max == 0) return E4B_OK;
  if (!x || !ids || !gates || !perm || !offsets || !xs || !local_ids || !local_gates) return E4B_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xs)) return E4B_ERR_MISALIGNED;
  g_last_launches = 1;
  return cuda_status(launch_ep_pack(x, H, ids, gates, top_k, perm, offsets, G, R_max, epr, xs, local_ids,
                                    local_gates, static_cast<cudaStream_t>(stream), sm_count()));
}

e4b_status e4b_ep_combine(const uint16_t* ys, int64_t H, const int32_t* inv_perm, int64_t T, int32_t top_k,
                          uint16_t* y, void* stream) {
  if (H <= 0 || T < 0 || top_k <= 0) return E4B_ERR_INVALID_ARG;
  if (H % 8) return E4B_ERR_UNSUPPORTED;
  g_last_launches = 0;
  if (T == 0) return E4B_OK;
  if (!inv_perm || !y || !ys) return E4B_ERR_INVALID_ARG;
  if (!aligned16(ys) || !aligned16(y)) return E4B_ERR_MISALIGNED;
  g_last_launches = 1;
  return cuda_status(launch_ep_combine(ys, H, inv_perm, T, top_k, y, static_cast<cudaStream_t>(stream), sm_count()));
}

// Workspace of the int4-b32 decode path: the status words, then h [top_k, I].
static size_t int4_layer_ws_bytes(int64_t I, int64_t top_k) {
  return size_t(kStatusBytes) + align_up(size_t(top_k) * size_t(I) * 2, 256);
}

e4b_status e4b_moe_workspace_size(const e4b_moe_weights* w, int64_t T, int32_t top_k,
                                  size_t* bytes) {
  if (!w || !bytes || T < 0 || top_k <= 0 || w->E <= 0 || w->H <= 0 || w->I <= 0)
    return E4B_ERR_INVALID_ARG;
  if (w->fmt == E4B_FMT_INT4B32) {
    *bytes = int4_layer_ws_bytes(w->I, top_k);
    return E4B_OK;
  }
  const MoeWs L = moe_ws_layout(w->E, w->H, w->I, T, top_k);
  *bytes = L.total;
  if (has_mx(w)) {
    const size_t mx = mx_ws_layout(L, w->E, w->H, w->I, T, top_k).total;
    if (mx > *bytes) *bytes = mx;
  }
  return E4B_OK;
}

// The layer on int4-b32 stacks: two decode GEMV launches a token.
static e4b_status moe_forward_int4(const e4b_moe_weights* w, const uint16_t* x, int64_t T, int32_t top_k,
                            const int32_t* ids, const float* gates, uint16_t* y, void* ws, size_t ws_bytes,
                            uint32_t flags, void* stream) {
  const int64_t E = w->E, H = w->H, I = w->I;
  if (H % E4B_INT4_BLOCK || I % E4B_INT4_BLOCK || top_k > int4_gemv_max_slots()) return E4B_ERR_UNSUPPORTED;
  if (w->gate_up_layout != E4B_GATE_UP_HALVES || w->activation != E4B_ACT_SWIGLU || w->gate_up_bias ||
      w->down_bias)
    return E4B_ERR_UNSUPPORTED;
  if (flags & ~E4B_FLAG_TEST_TIMEOUT) return E4B_ERR_UNSUPPORTED;
  if (int64_t(top_k) * I > 200 * 1024 || int4_gemv_warps(top_k, I) <= 0 || int4_gemv_warps(1, H) <= 0)
    return E4B_ERR_UNSUPPORTED;
  g_last_launches = 0;
  if (T == 0) return E4B_OK;
  if (!x || !ids || !gates || !y || !ws || !w->gate_up_codes || !w->gate_up_scales || !w->down_codes ||
      !w->down_scales)
    return E4B_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(ws) || !aligned16(w->gate_up_codes) ||
      !aligned16(w->down_codes) || (reinterpret_cast<uintptr_t>(w->gate_up_scales) & 1u) ||
      (reinterpret_cast<uintptr_t>(w->down_scales) & 1u))
    return E4B_ERR_MISALIGNED;
  if (ws_bytes < int4_layer_ws_bytes(I, top_k)) return E4B_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* status = static_cast<int32_t*>(ws);
  uint16_t* h = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  // the status words describe this call
  if (cudaMemsetAsync(status, 0, kStatusBytes, s) != cudaSuccess) return E4B_ERR_CUDA;
  mark(0, s);
  const int sms = sm_count();
  for (int64_t t = 0; t < T; ++t) {
    Int4Gemv gu{};
    gu.epilogue = E4B_EPI_SWIGLU;
    gu.E = int(E);
    gu.n_slots = top_k;
    gu.nx = 1;
    gu.N = 2 * I;
    gu.K = H;
    gu.codes = w->gate_up_codes;
    gu.scales = static_cast<const uint16_t*>(w->gate_up_scales);
    gu.ids = ids + t * top_k;
    gu.x = x + t * H;
    gu.ld_x = 0;
    gu.y = h;
    gu.ld_y = I;
    gu.status = status;
    gu.flags = flags;
    if (launch_int4_gemv(gu, s, sms) != cudaSuccess) return E4B_ERR_CUDA;
    Int4Gemv dn{};
    dn.epilogue = E4B_EPI_COMBINE;
    dn.E = int(E);
    dn.n_slots = top_k;
    dn.nx = top_k;
    dn.N = H;
    dn.K = I;
    dn.codes = w->down_codes;
    dn.scales = static_cast<const uint16_t*>(w->down_scales);
    dn.ids = ids + t * top_k;
    dn.gates = gates + t * top_k;
    dn.x = h;
    dn.ld_x = I;
    dn.y = y + t * H;
    dn.status = status;
    dn.flags = flags | E4B_FLAG_IDS_READY;  // the gate_up launch has read this token's ids
    if (launch_int4_gemv(dn, s, sms) != cudaSuccess) return E4B_ERR_CUDA;
  }
  mark(4, s);
  g_last_path = E4B_PATH_INT4_GEMV;
  g_last_launches = int32_t(2 * T);
  return E4B_OK;
}

// The large-M layer on the block-scaled FP4 MMA (csrc/mx_native.cu): x split
// into e4m3 terms in padded per-expert rows, gate_up with the gated
// activation into bf16 h (padded rows), h split the same way, down with the
// gate-weighted rows, then each token's rows summed in slot order.
static e4b_status moe_forward_mx(const e4b_moe_weights* w, const MoeWs& L, const uint16_t* x, int64_t T,
                                 int32_t top_k, const int32_t* perm, const int64_t* offsets, const int32_t* inv,
                                 const float* gates, uint16_t* y, uint8_t* base, size_t ws_bytes,
                                 int32_t* status, uint32_t flags, cudaStream_t s) {
  const int64_t E = w->E, H = w->H, I = w->I;
  const MxWs M = mx_ws_layout(L, E, H, I, T, top_k);
  if (ws_bytes < M.total) return E4B_ERR_WORKSPACE_TOO_SMALL;
  if (M.Rp_max >= (int64_t(1) << 31)) return E4B_ERR_UNSUPPORTED;
  const int nt = (flags & E4B_FLAG_MX_ACT_E4M3) ? 1 : 2;
  const int sms = sm_count();
  uint8_t* xq = base + M.xq;
  uint8_t* sfx = base + M.sfx;
  uint16_t* hp = reinterpret_cast<uint16_t*>(base + M.hp);
  uint8_t* hq = base + M.hq;
  uint8_t* sfh = base + M.sfh;
  float* rows = reinterpret_cast<float*>(base + L.rows);

  MxActArgs qa{};
  qa.src = x;
  qa.ld_src = H;
  qa.perm = perm;
  qa.top_k = top_k;
  qa.offsets = offsets;
  qa.E = int32_t(E);
  qa.K = H;
  qa.rows = M.Rp_max;
  qa.elems = xq;
  qa.sf = sfx;
  qa.nterms = nt;
  if (launch_mx_act_quant(qa, s, sms) != cudaSuccess) return E4B_ERR_CUDA;

  MxGemmArgs g{};
  g.gated_rows = false;
  g.nterms = nt;
  g.E = int(E);
  g.top_k = top_k;
  g.Nm = I;
  g.K = H;
  g.Rp_max = M.Rp_max;
  g.codes = w->gate_up_mx_codes;
  g.sfa = w->gate_up_mx_sf;
  g.act = xq;
  g.sfb = sfx;
  g.offsets = offsets;
  g.perm = perm;
  g.gates = gates;
  g.out = hp;
  g.ldo = I;
  g.layout = w->gate_up_layout;
  g.act_fn = w->activation;
  g.alpha = w->glu_alpha;
  g.limit = w->glu_limit;
  g.bias = w->gate_up_bias;
  g.status = status;
  g.flags = flags;
  mark(1, s);
  if (launch_mx_gemm(g, s, sms) != cudaSuccess) return E4B_ERR_CUDA;

  mark(2, s);
  MxActArgs qh = qa;
  qh.src = hp;
  qh.ld_src = I;
  qh.perm = nullptr;
  qh.K = I;
  qh.elems = hq;
  qh.sf = sfh;
  if (launch_mx_act_quant(qh, s, sms) != cudaSuccess) return E4B_ERR_CUDA;

  MxGemmArgs d = g;
  d.gated_rows = true;
  d.Nm = H;
  d.K = I;
  d.codes = w->down_mx_codes;
  d.sfa = w->down_mx_sf;
  d.act = hq;
  d.sfb = sfh;
  d.out = rows;
  d.ldo = H;
  d.bias = w->down_bias;
  if (launch_mx_gemm(d, s, sms) != cudaSuccess) return E4B_ERR_CUDA;

  mark(3, s);
  if (launch_combine_rows(rows, inv, T, top_k, H, y, s, sms) != cudaSuccess) return E4B_ERR_CUDA;
  mark(4, s);
  g_last_path = E4B_PATH_TCGEN05_MX;
  g_last_launches = 6;
  return E4B_OK;
}

e4b_status e4b_mxfp4_native_size(int32_t E, int64_t rows_per_mat, int64_t K, int32_t nmat,
                                 size_t* codes_bytes, size_t* sf_bytes) {
  if (!codes_bytes || !sf_bytes || E <= 0 || rows_per_mat <= 0 || K <= 0 || (nmat != 1 && nmat != 2))
    return E4B_ERR_INVALID_ARG;
  if (K % E4B_MXFP4_BLOCK) return E4B_ERR_UNSUPPORTED;
  const size_t Np = size_t((rows_per_mat + 127) / 128 * 128);
  const size_t Kp = size_t((K + 127) / 128 * 128);
  *codes_bytes = size_t(E) * size_t(nmat) * Np * Kp / 2;
  *sf_bytes = size_t(E) * size_t(nmat) * (Np / 128) * (Kp / 128) * 512;
  return E4B_OK;
}

e4b_status e4b_mxfp4_native_prepare(const uint8_t* blocks, const uint8_t* scales, int32_t E,
                                    int64_t rows_per_mat, int64_t K, int32_t nmat,
                                    int32_t gate_up_layout, uint8_t* codes_out, uint8_t* sf_out,
                                    void* stream) {
  size_t cb = 0, fb = 0;
  e4b_status st = e4b_mxfp4_native_size(E, rows_per_mat, K, nmat, &cb, &fb);
  if (st != E4B_OK) return st;
  if (!blocks || !scales || !codes_out || !sf_out) return E4B_ERR_INVALID_ARG;
  if (nmat == 2 && gate_up_layout != E4B_GATE_UP_HALVES && gate_up_layout != E4B_GATE_UP_INTERLEAVED)
    return E4B_ERR_INVALID_ARG;
  if (!aligned16(blocks) || (reinterpret_cast<uintptr_t>(codes_out) & 31u) || !aligned16(sf_out))
    return E4B_ERR_MISALIGNED;
  g_last_launches = 1;
  return cuda_status(launch_mx_prepare(blocks, scales, E, rows_per_mat, nmat, K,
                                       nmat == 2 ? gate_up_layout : E4B_GATE_UP_HALVES, codes_out, sf_out,
                                       static_cast<cudaStream_t>(stream), sm_count()));
}

e4b_status e4b_quantize_mxfp8(const uint16_t* x, int64_t R, int64_t K, uint8_t* elems, uint8_t* scales,
                              void* stream) {
  if (R < 0 || K <= 0) return E4B_ERR_INVALID_ARG;
  if (K % 32) return E4B_ERR_UNSUPPORTED;
  g_last_launches = 0;
  if (R == 0) return E4B_OK;
  if (!x || !elems || !scales) return E4B_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(elems) & 7u)) return E4B_ERR_MISALIGNED;
  MxActArgs a{};
  a.src = x;
  a.ld_src = K;
  a.K = K;
  a.rows = R;
  a.elems = elems;
  a.sf = scales;
  a.nterms = 1;
  a.plain = true;
  g_last_launches = 1;
  return cuda_status(launch_mx_act_quant(a, static_cast<cudaStream_t>(stream), sm_count()));
}

e4b_status e4b_moe_forward(const e4b_moe_weights* w, const uint16_t* x, int64_t T, int32_t top_k,
                           const int32_t* ids, const float* gates, uint16_t* y, void* ws,
                           size_t ws_bytes, uint32_t flags, void* stream) {
  if (!w || T < 0 || top_k <= 0) return E4B_ERR_INVALID_ARG;
  const int64_t E = w->E, H = w->H, I = w->I;
  if (E <= 0 || H <= 0 || I <= 0 || top_k > E) return E4B_ERR_INVALID_ARG;
  if (w->fmt == E4B_FMT_INT4B32)
    return moe_forward_int4(w, x, T, top_k, ids, gates, y, ws, ws_bytes, flags, stream);
  e4b_status st = check_projection(w->fmt, 2 * I, H, true);
  if (st != E4B_OK) return st;
  st = check_projection(w->fmt, H, I, false);
  if (st != E4B_OK) return st;
  if (H % 8) return E4B_ERR_UNSUPPORTED;
  if (E > 1024 || T * int64_t(top_k) >= (int64_t(1) << 31)) return E4B_ERR_UNSUPPORTED;
  st = check_variant(w->gate_up_layout, w->activation, w->glu_limit, w->gate_up_bias, w->down_bias);
  if (st != E4B_OK) return st;
  {
    const int nmx = (w->gate_up_mx_codes != nullptr) + (w->gate_up_mx_sf != nullptr) +
                    (w->down_mx_codes != nullptr) + (w->down_mx_sf != nullptr);
    if (nmx != 0 && (nmx != 4 || w->fmt != E4B_FMT_MXFP4)) return E4B_ERR_INVALID_ARG;
    if (nmx == 4 && ((reinterpret_cast<uintptr_t>(w->gate_up_mx_codes) & 31u) ||
                     (reinterpret_cast<uintptr_t>(w->down_mx_codes) & 31u) || !aligned16(w->gate_up_mx_sf) ||
                     !aligned16(w->down_mx_sf)))
      return E4B_ERR_MISALIGNED;
  }
  g_last_launches = 0;
  if (T == 0) return E4B_OK;
  if (!x || !ids || !gates || !y || !ws || !w->gate_up_codes || !w->gate_up_scales ||
      !w->down_codes || !w->down_scales)
    return E4B_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(ws) || !aligned16(w->gate_up_codes) ||
      !aligned16(w->down_codes) || !aligned16(w->gate_up_scales) || !aligned16(w->down_scales))
    return E4B_ERR_MISALIGNED;
  const MoeWs L = moe_ws_layout(E, H, I, T, top_k);
  const int64_t R = T * top_k;
  const bool gemv = choose_gemv(R, E, flags);
  if (!gemv && E > 256) return E4B_ERR_UNSUPPORTED;
  if (ws_bytes < (gemv ? L.small_min : L.large_min)) return E4B_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(base + L.status);
  int32_t* counts = reinterpret_cast<int32_t*>(base + L.counts);
  int64_t* offsets = reinterpret_cast<int64_t*>(base + L.offsets);
  int32_t* perm = reinterpret_cast<int32_t*>(base + L.perm);
  int32_t* inv = reinterpret_cast<int32_t*>(base + L.inv);
  uint16_t* h = reinterpret_cast<uint16_t*>(base + L.h);
  float* acc = reinterpret_cast<float*>(base + L.acc);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  mark(0, s);
  int32_t* sync = reinterpret_cast<int32_t*>(base + L.sync);
  // the fp32 rows / partial sums region is free until the projections: it
  // lends the many-CTA routing its scratch
  int route_launches = 1;
  cudaError_t ce = launch_route(ids, int32_t(R), int32_t(E), counts, offsets, perm, inv, nullptr,
                                status, s, sync, int32_t(L.nsync), reinterpret_cast<int32_t*>(acc),
                                (gemv ? L.small_min : L.large_min) - L.acc, &route_launches);
  if (ce != cudaSuccess) return E4B_ERR_CUDA;

  if (gemv) {
    // small-M: both projections and the SwiGLU in one launch, then the
    // fixed-order combine into bf16 y
    SmallMLayer sl{};
    sl.fmt = w->fmt;
    sl.E = int(E);
    sl.H = int(H);
    sl.I = int(I);
    sl.top_k = top_k;
    sl.T = T;
    sl.gu_codes = w->gate_up_codes;
    sl.gu_scales = w->gate_up_scales;
    sl.dn_codes = w->down_codes;
    sl.dn_scales = w->down_scales;
    sl.x = x;
    sl.perm = perm;
    sl.offsets = offsets;
    sl.gates = gates;
    sl.h = h;
    sl.part = acc;
    sl.inv = inv;
    sl.y = y;
    sl.sync = sync;
    sl.status = status;
    sl.flags = flags;
    sl.layout = w->gate_up_layout;
    sl.act = w->activation;
    sl.alpha = w->glu_alpha;
    sl.limit = w->glu_limit;
    sl.gu_bias = w->gate_up_bias;
    sl.dn_bias = w->down_bias;
    mark(1, s);
    mark(2, s);
    ce = launch_smallm_layer(sl, s, sm_count());
    if (ce != cudaSuccess) return E4B_ERR_CUDA;
    mark(3, s);
    ce = launch_smallm_combine(sl, s, sm_count());
    if (ce != cudaSuccess) return E4B_ERR_CUDA;
    mark(4, s);
    g_last_path = E4B_PATH_GEMV;
    g_last_launches = 2 + route_launches;
    return E4B_OK;
  }

  if (has_mx(w) && !(flags & E4B_FLAG_MX_DECODE)) {
    const e4b_status r =
        moe_forward_mx(w, L, x, T, top_k, perm, offsets, inv, gates, y, base, ws_bytes, status, flags, s);
    g_last_launches += route_launches - 1;
    return r;
  }

  // Large-M: stage the routed rows of x in expert order when the workspace
  // holds the copy (contiguous TMA row tiles), else gather them in the kernel.
  const bool staged = ws_bytes >= L.total;
  uint16_t* xs = staged ? reinterpret_cast<uint16_t*>(base + L.xs) : nullptr;
  if (staged) {
    ce = launch_gather_rows(x, H, perm, top_k, offsets, int32_t(E), R, xs, s, sm_count());
    if (ce != cudaSuccess) return E4B_ERR_CUDA;
  }

  GemmProblem g{};
  g.fmt = w->fmt;
  g.epilogue = E4B_EPI_SWIGLU;
  g.E = int(E);
  g.top_k = top_k;
  g.N = 2 * I;
  g.K = H;
  g.R_max = R;
  g.codes = w->gate_up_codes;
  g.scales = w->gate_up_scales;
  g.a = staged ? xs : x;
  g.lda = H;
  g.row_slot = staged ? nullptr : perm;
  g.out_slot = perm;
  g.offsets = offsets;
  g.out = h;
  g.ldo = I;
  g.status = status;
  g.flags = flags;
  g.layout = w->gate_up_layout;
  g.act = w->activation;
  g.alpha = w->glu_alpha;
  g.limit = w->glu_limit;
  g.bias = w->gate_up_bias;
  mark(1, s);
  st = run_projection(g, gemv, s);
  if (st != E4B_OK) return st;

  // down: every routed row's gate-weighted output into its own fp32 row, then
  // each token's rows summed in slot order (deterministic, no atomics)
  float* rows = reinterpret_cast<float*>(base + L.rows);
  GemmProblem d = g;
  d.epilogue = kEpiGatedRows;
  d.N = H;
  d.K = I;
  d.codes = w->down_codes;
  d.scales = w->down_scales;
  d.a = h;
  d.lda = I;
  d.row_slot = nullptr;
  d.out_slot = perm;
  d.gates = gates;
  d.out = rows;
  d.ldo = H;
  d.bias = w->down_bias;
  mark(2, s);
  st = run_projection(d, gemv, s);
  if (st != E4B_OK) return st;

  mark(3, s);
  ce = launch_combine_rows(rows, inv, T, top_k, H, y, s, sm_count());
  if (ce != cudaSuccess) return E4B_ERR_CUDA;
  mark(4, s);
  g_last_path = gemv ? E4B_PATH_GEMV : E4B_PATH_TCGEN05;
  g_last_launches = (staged ? 4 : 3) + route_launches;
  return E4B_OK;
}

e4b_status e4b_read_device_status(void* ws, int32_t* status_host, void* stream) {
  if (!ws || !status_host) return E4B_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return E4B_ERR_CUDA;
  int32_t v[2] = {0, 0};
  if (cudaMemcpy(v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return E4B_ERR_CUDA;
  if (cudaMemset(ws, 0, sizeof(v)) != cudaSuccess) return E4B_ERR_CUDA;
  *status_host = v[0];
  return E4B_OK;
}

}  // extern "C"
