// Internal host-side launchers shared by the C-ABI layer (api.cu).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "e4b.h"

namespace e4b {

cudaError_t launch_quantize_nf4(const float* w, int64_t nblocks, uint8_t* codes, float* absmax,
                                cudaStream_t st, int sms);
cudaError_t launch_quantize_mxfp4(const float* w, int64_t nblocks, uint8_t* blocks, uint8_t* scales,
                                  cudaStream_t st, int sms);
cudaError_t launch_dequantize(int fmt, const uint8_t* codes, const void* scales, int64_t nweights,
                              uint16_t* out, cudaStream_t st, int sms);
void host_nf4_levels(float* out);

size_t route_smem_bytes(int32_t E);
// Bytes of scratch the many-CTA routing of R slots over E experts needs (0:
// R is small enough for the one-CTA pass).
size_t route_scratch_bytes(int32_t R, int32_t E);
// The routing pass; with `scratch` (at least route_scratch_bytes) and a large
// R it runs over many CTAs in two launches (*launches says how many).
cudaError_t launch_route(const int32_t* ids, int32_t R, int32_t E, int32_t* counts, int64_t* offsets,
                         int32_t* perm, int32_t* inv, int32_t* active, int32_t* status,
                         cudaStream_t st, int32_t* clear = nullptr, int32_t nclear = 0,
                         int32_t* scratch = nullptr, size_t scratch_bytes = 0, int* launches = nullptr);
// xs[p] = x[perm[p] / top_k] for p < offsets[E] (H % 8 == 0, 16-byte aligned).
cudaError_t launch_gather_rows(const uint16_t* x, int64_t H, const int32_t* perm, int32_t top_k,
                               const int64_t* offsets, int32_t E, int64_t R_max, uint16_t* xs,
                               cudaStream_t st, int sms);
// Smallest workspace e4b_moe_forward accepts (without the staging copy of the
// routed rows that e4b_moe_workspace_size includes).
// The path the layer takes for these sizes and flags: true = small-M.
bool layer_uses_small_m(int64_t R, int64_t E, uint32_t flags);
// Smallest workspace e4b_moe_forward accepts for this call (NF4 / MXFP4): the
// small-M path needs the routing arrays, h and an fp32 [T, H] accumulator; the
// large-M path the routing arrays, h and the gated rows fp32 [T*top_k, H]
// (without the staging copy of the routed rows that e4b_moe_workspace_size
// includes); the block-scaled MXFP4 path also its e4m3 activation terms.
size_t moe_workspace_min_bytes(const e4b_moe_weights* w, int64_t T, int64_t top_k, uint32_t flags);

// GemmProblem::epilogue for the input gradient through the weights
// (e4b_grouped_dgrad): out [R, K] bf16, row p = a_p . W_e, a [R, N].
constexpr int kEpiDgrad = 3;
// GemmProblem::epilogue of the layer's down projection on the large-M path:
// out fp32 [R, ldo], row p = gates[s] * (a_p . W_e^T + bias), s = out_slot[p]
// (p when null); every row is written once (no accumulation), so the
// token-wise sum that follows (launch_combine_rows) runs in a fixed order.
constexpr int kEpiGatedRows = 4;

// y[t] = bf16(sum_j rows[inv[t*k + j]]) for j = 0..k-1 in that order, fp32
// sums; a slot whose inv is -1 adds nothing (rows fp32 [*, H], y bf16 [T, H],
// H % 4 == 0, both 16-byte aligned).
cudaError_t launch_combine_rows(const float* rows, const int32_t* inv, int64_t T, int32_t k, int64_t H,
                                uint16_t* y, cudaStream_t st, int sms);

// Description of one grouped projection as the kernels see it.
struct GemmProblem {
  int fmt;          // e4b_format
  int epilogue;     // e4b_epilogue
  int E;
  int top_k;
  int64_t N, K;     // weight rows (both halves for SWIGLU), inner dim
  int64_t R_max;    // bound on offsets[E]
  const uint8_t* codes;
  const void* scales;
  const uint16_t* a;
  int64_t lda;
  const int32_t* row_slot;  // may be null: row p reads a[p]; else a[row_slot[p] / top_k]
  const int32_t* out_slot;  // COMBINE: slot of row p (p when null)
  const int64_t* offsets;   // [E+1]
  const float* gates;       // COMBINE
  void* out;
  int64_t ldo;
  float* zero_buf;          // optional buffer the kernel clears first (fp32 accumulator)
  int64_t zero_count;       // floats in zero_buf
  int32_t* status;          // device status word or null
  uint32_t flags;
  // expert variant (include/e4b.h); bias: fp32 [E, N] per weight row or null
  int layout, act;
  float alpha, limit;
  const float* bias;
};

cudaError_t launch_gemv(const GemmProblem& p, cudaStream_t st, int sms);

// The whole small-M layer in one persistent launch (csrc/smallm.cu).
struct SmallMLayer {
  int fmt, E, H, I, top_k;
  int64_t T;
  const uint8_t* gu_codes;
  const void* gu_scales;
  const uint8_t* dn_codes;
  const void* dn_scales;
  const uint16_t* x;
  const int32_t* perm;
  const int64_t* offsets;
  const float* gates;
  uint16_t* h;
  float* part;     // [smallm_k_slices(I), T*top_k, H] fp32 partial sums of the down passes
  const int32_t* inv;  // [T*top_k] routed row of each slot (-1: dropped)
  uint16_t* y;
  int32_t* sync;   // smallm_sync_ints(E, H) ints, zero on entry
  int32_t* status;
  uint32_t flags;
  int layout, act;  // expert variant (include/e4b.h)
  float alpha, limit;
  const float* gu_bias;  // fp32 [E, 2I] or null
  const float* dn_bias;  // fp32 [E, H] or null
};
size_t smallm_sync_ints(int E, int H);
// K slices of the small-M down passes (the partial sums kept per slice).
int smallm_k_slices(int I);
cudaError_t launch_smallm_layer(const SmallMLayer& L, cudaStream_t st, int sms);
// The fixed-order sum of the partial sums into bf16 y (a programmatic
// dependent of launch_smallm_layer).
cudaError_t launch_smallm_combine(const SmallMLayer& L, cudaStream_t st, int sms);
cudaError_t launch_tc_gemm(const GemmProblem& p, cudaStream_t st, int sms);
// The SM-pair (cta_group::2) form of the large-M projection (csrc/tc_pair.cu):
// forward epilogues on contiguous activation rows; launch_tc_gemm takes it
// whenever tc_pair_supported says so.
bool tc_pair_supported(const GemmProblem& p);
cudaError_t launch_tc_pair(const GemmProblem& p, cudaStream_t st, int sms);
cudaError_t launch_finalize(const float* acc, int64_t n, uint16_t* y, cudaStream_t st, int sms);

// The int4-b32 decode GEMV (csrc/int4.cu): one token against n_slots routed
// experts of a stack [E, N, K] (codes [E, N, K/2], fp16 scales [E, N, K/32]).
// nx activation rows: 1 (every slot reads x) or n_slots (slot j reads row j).
struct Int4Gemv {
  int epilogue;  // E4B_EPI_STORE / E4B_EPI_SWIGLU / E4B_EPI_COMBINE
  int E, n_slots, nx;
  int64_t N, K;
  const uint8_t* codes;
  const uint16_t* scales;
  const int32_t* ids;
  const float* gates;
  const uint16_t* x;
  int64_t ld_x;
  uint16_t* y;
  int64_t ld_y;
  int32_t* status;
  uint32_t flags;
};
// Launch plan of the GEMV (csrc/int4.cu), made on the host.
struct Int4Plan {
  int warps;         // streaming warps per CTA
  uint32_t nch;      // chunks of 128 blocks per weight row
  uint32_t np;       // tasks per output (COMBINE: slot pairs)
  int64_t outputs;
  uint32_t acc_off, ring_off;  // shared-memory offsets
  uint32_t polls;    // bound of every wait
  uint32_t sbulk;    // 1: scales travel with the codes in the bulk copies (K % 256 == 0, aligned)
};
size_t int4_gemv_smem_bytes(int nx, int64_t K, int warps);
int int4_gemv_warps(int nx, int64_t K);
int int4_gemv_max_slots();
cudaError_t launch_int4_gemv(const Int4Gemv& p, cudaStream_t st, int sms);
cudaError_t launch_quantize_int4(const float* w, int64_t nblocks, uint8_t* codes, uint16_t* scales,
                                 cudaStream_t st, int sms);
cudaError_t launch_gptq_repack(const int32_t* qweight, const uint16_t* gscales, int64_t E, int64_t N, int64_t K,
                               uint8_t* codes, uint16_t* scales, cudaStream_t st);

// ----------------------------------------------- MXFP4 block-scaled path
// (csrc/mx_native.cu)
// Routed rows per tile of the block-scaled GEMM, and the unit the activation
// rows of each expert are padded to.
constexpr int kMxRowBlock = 112;
// Upper bound on the rows of the padded activation layout: R routed rows,
// each active expert's rows rounded up to a multiple of kMxRowBlock.
int64_t mx_padded_rows_max(int64_t R, int64_t E);
// Prepared copy of one MXFP4 stack (see e4b_mxfp4_native_prepare).
cudaError_t launch_mx_prepare(const uint8_t* blocks, const uint8_t* scales, int E, int64_t Nm, int nmat,
                              int64_t K, int layout, uint8_t* out_codes, uint8_t* out_sf, cudaStream_t st,
                              int sms);
// bf16 rows -> e4m3 terms + e8m0 scales. Layer layouts: padded rows (expert
// e's rows from poff[e], a multiple of kMxRowBlock), elems [nterms][rows][Kp],
// sf chunks [nterms][rows/kMxRowBlock][Kp/128][512]; rows = the padded bound. perm set:
// padded row -> source row perm[p] / top_k (x); null: source row = padded row
// (h). plain: rows [rows][K] -> elems [rows][K], sf [rows][K/32], one term.
struct MxActArgs {
  const uint16_t* src;
  int64_t ld_src;
  const int32_t* perm;
  int32_t top_k;
  const int64_t* offsets;
  int32_t E;
  int64_t K;
  int64_t rows;
  uint8_t* elems;
  uint8_t* sf;
  int nterms;  // 1 = OCP MXFP8 rule, 2 = exact two-term split
  bool plain;
};
cudaError_t launch_mx_act_quant(const MxActArgs& a, cudaStream_t st, int sms);
// One projection on the block-scaled tensor cores: gate_up (two matrices,
// gated activation into bf16 h in padded rows) or down (one matrix, the
// gate-weighted fp32 row of every routed row).
struct MxGemmArgs {
  bool gated_rows;
  int nterms;
  int E, top_k;
  int64_t Nm, K, Rp_max;
  const uint8_t* codes;
  const uint8_t* sfa;
  const uint8_t* act;
  const uint8_t* sfb;
  const int64_t* offsets;
  const int32_t* perm;
  const float* gates;
  void* out;
  int64_t ldo;
  int layout, act_fn;
  float alpha, limit;
  const float* bias;
  int32_t* status;
  uint32_t flags;
};
cudaError_t launch_mx_gemm(const MxGemmArgs& a, cudaStream_t st, int sms);

}  // namespace e4b
