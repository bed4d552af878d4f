/*
 * e4b.h -- packed-4-bit Mixture-of-Experts layer for B200 (sm_100a), C ABI.
 *
 * One MoE layer run directly on 4-bit-packed fused expert stacks:
 * gate_up_proj [E, 2I, H] and down_proj [E, H, I] stored as NF4 (16-level
 * NormalFloat codebook, two codes per byte, fp32 absmax per 64 weights along
 * the input dimension, every expert quantised on its own) or as MXFP4 (OCP
 * e2m1 codes, one e8m0 scale per 32 weights). One launch covers all active
 * experts of a projection; weights are decoded on the fly through a 16-entry
 * per-block table; products accumulate in fp32; no bf16 copy of a weight
 * stack is ever written to memory.
 *
 * Sources (page titles; sections):
 *   [G]  "grouped-nf4-gemm" README: intro (one launch for all active experts,
 *        LUT decode, blockwise scaling, fp32 accumulation, bf16 epilogue; NF4
 *        on the bitsandbytes gemm_4bit layout; MXFP4 as OCP e2m1 + e8m0);
 *        "Try it on CPU right now" blocks 1-2 (quantize_pack_nf4 -> packed
 *        [N, K/2] u8 + absmax [N, K/64] f32; quantize_pack_mxfp4 -> blocks
 *        [N, K/32, 16] u8 + scales [N, K/32] u8); "Which entry point?" table.
 *   [P]  bitsandbytes PR #1984 "Experts4bit": Summary and Design (per-expert
 *        quantisation with per-expert absmax, per-expert dequantise loop,
 *        gated SiLU / SwiGLU activation).
 *   [Q]  "experts4bit-qlora" README: fused gate_up_proj / down_proj stacks
 *        (transformers v5 layout).
 *   [S]  "How do I run a single-token INT4 decode GEMV over routed MoE
 *        experts, and pack calibrated (GPTQ) weights for it?" (grouped-nf4-gemm
 *        solutions page): the int4-b32 decode GEMV and the GPTQ packer.
 *
 * Conventions for every entry point
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless
 *     its comment says "host". The library allocates and frees nothing and
 *     keeps no pointer after a call returns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Every
 *     call only enqueues work on that stream and returns without waiting,
 *     except the few marked "synchronises".
 *   - Argument errors are returned before anything is enqueued. Errors the
 *     GPU detects (an expert id outside [0, E), a bounded wait that gave up)
 *     are recorded in the workspace's status word; read it with
 *     e4b_read_device_status.
 *   - Element counts and offsets are 64-bit. bf16 values are passed as their
 *     16-bit patterns (uint16_t).
 *   - There is no fallback: a shape the kernels do not support returns
 *     E4B_ERR_UNSUPPORTED.
 */
#ifndef E4B_H_
#define E4B_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  E4B_OK = 0,
  E4B_ERR_INVALID_ARG = 1,         /* null pointer, negative size, k > E ... */
  E4B_ERR_UNSUPPORTED = 2,         /* shape outside what the kernels handle */
  E4B_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below the *_workspace_size query */
  E4B_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
  E4B_ERR_DEVICE_TIMEOUT = 5,      /* (device) a bounded wait gave up */
  E4B_ERR_BAD_EXPERT_ID = 6,       /* (device) an id outside [0, E); the slot is dropped */
  E4B_ERR_MISALIGNED = 7,          /* a pointer or row stride breaks 16-byte alignment */
  E4B_ERR_EXCEEDS_STATIC_SCRATCH = 8 /* e4b_moe_forward_noalloc: the call needs more than its
                                        16 MiB static scratch */
} e4b_status;

/* E4B_FMT_INT4B32: int4-b32 stacks (see e4b_gemv_int4_b32); only
 * e4b_moe_forward / e4b_moe_workspace_size take it, as the batch-1 decode path. */
typedef enum { E4B_FMT_NF4 = 0, E4B_FMT_MXFP4 = 1, E4B_FMT_INT4B32 = 2 } e4b_format;

/* Which kernel family ran last (e4b_last_path). */
typedef enum {
  E4B_PATH_NONE = 0,
  E4B_PATH_GEMV = 1,   /* small-M: register-fed mma.sync streaming the packed bytes */
  E4B_PATH_TCGEN05 = 2, /* large-M: TMA + on-the-fly decode + tcgen05 MMA into TMEM */
  E4B_PATH_INT4_GEMV = 3, /* the int4-b32 decode GEMV (dp4a, exact integer block sums) */
  E4B_PATH_TCGEN05_MX = 4 /* large-M MXFP4: e2m1 codes straight into the block-scaled MMA */
} e4b_path;

/* Flags for e4b_moe_forward / e4b_grouped_gemm. */
#define E4B_FLAG_FORCE_GEMV 0x1u     /* use the small-M path whatever the shape */
#define E4B_FLAG_FORCE_TCGEN05 0x2u  /* use the tcgen05 path whatever the shape */
#define E4B_FLAG_TEST_TIMEOUT 0x4u   /* bounded waits give up at once (tests the error path) */
/* Small-M layer path, NF4: decode every weight to bf16_rne(fp32(level *
 * absmax)) before the MMA, the operand the tcgen05 path and e4b_grouped_gemm
 * use. Without the flag the small-M layer path takes bf16_rne(level) as the
 * operand and applies the fp32 absmax to each 64-weight block's fp32 partial
 * sum, i.e. its decoded weight is bf16_rne(level) * absmax, exactly. The two
 * decodes differ by at most one bf16 rounding of each weight (both are within
 * 2^-8 relative of level * absmax); the default needs half the shared-memory
 * table traffic and is the faster one. */
#define E4B_FLAG_NF4_PRODUCT_DECODE 0x8u
/* e4b_gemv_int4_b32: the expert ids and gates are not written by the work
 * queued just before the call on the stream (they are ready when the call is
 * enqueued), so the kernel reads them and sets up its work before that work
 * completes. It still waits for it before reading x (and streams weights only
 * after quantising x). */
#define E4B_FLAG_IDS_READY 0x10u
/* MXFP4 layers with prepared stacks (e4b_moe_weights.*_mx_*), large-M path:
 * each activation row enters the block-scaled MMA as ONE e4m3 term per value
 * with an e8m0 scale per 32 (the OCP MXFP8 rule: shared exponent
 * floor(log2 amax) - 8, round to nearest even, saturating at 448), at half the
 * MMA count. The results are those of the layer on MXFP8-rounded x and h, not
 * of the bf16 layer. Without the flag every bf16 activation value is split
 * into two e4m3 terms x1 + x2 (exponents floor(log2 amax) - 7 of the block
 * and of its residual), which reproduces it exactly except for values below
 * ~2^-13 of their block's largest magnitude. */
#define E4B_FLAG_MX_ACT_E4M3 0x20u
/* MXFP4 layers with prepared stacks: take the decode-to-bf16 tcgen05 path
 * anyway on large-M shapes (for comparisons). */
#define E4B_FLAG_MX_DECODE 0x40u
/* Large-M tcgen05 projections and e4b_grouped_dgrad: run on the one-SM
 * kernel (M = 128 weight rows per MMA) instead of SM pairs
 * (tcgen05.mma.cta_group::2, M = 256 over two SMs of a cluster); for
 * comparisons. Gathered activation rows always take the one-SM kernel. */
#define E4B_FLAG_TC_SINGLE_SM 0x80u

/* NF4 block size (weights per absmax) and MXFP4 block size (weights per scale). */
#define E4B_NF4_BLOCK 64
#define E4B_MXFP4_BLOCK 32

/*
 * A layer's packed expert stacks [Q, G].
 *   NF4:   gate_up_codes  uint8 [E, 2I, H/2]  (two codes per byte, the earlier
 *                                              weight in the high nibble)
 *          gate_up_scales float [E, 2I, H/64] (absmax per 64 weights)
 *          down_codes     uint8 [E, H, I/2]
 *          down_scales    float [E, H, I/64]
 *   MXFP4: gate_up_codes  uint8 [E, 2I, H/32, 16] (the earlier weight in the low nibble)
 *          gate_up_scales uint8 [E, 2I, H/32]     (e8m0: value 2^(byte-127))
 *          down_codes     uint8 [E, H, I/32, 16]
 *          down_scales    uint8 [E, H, I/32]
 * With the default layout, rows 0..I-1 of gate_up are the gate projection and
 * rows I..2I-1 the up projection. All four arrays must be 16-byte aligned.
 *
 * Expert variant ("experts4bit-qlora" README, Scope: gpt-oss MXFP4 experts
 * with per-expert biases and a clamped GLU); all fields zero = the plain
 * layer. The pages name the variant without its layout or constants; this
 * library follows the released gpt-oss expert definition:
 *   gate_up_layout  E4B_GATE_UP_HALVES (default) or E4B_GATE_UP_INTERLEAVED
 *                   (gate = row 2n, up = row 2n+1 of gate_up)
 *   activation      E4B_ACT_SWIGLU: h = silu(g) * u (default), or
 *                   E4B_ACT_CLAMPED_GLU: g' = min(g, limit),
 *                   u' = clamp(u, -limit, limit), h = (u' + 1) * g' * sigmoid(alpha * g')
 *   glu_alpha, glu_limit   the clamped GLU's constants (released model: 1.702, 7)
 *   gate_up_bias    fp32 [E, 2I] in gate_up row order, added to g and u; or null
 *   down_bias       fp32 [E, H], added to each expert's down output before the
 *                   gate weighting; or null
 * Both biases must be 16-byte aligned. Unknown layout or activation codes, or
 * a clamped GLU whose limit is negative or NaN, return E4B_ERR_INVALID_ARG.
 */
typedef enum { E4B_GATE_UP_HALVES = 0, E4B_GATE_UP_INTERLEAVED = 1 } e4b_gate_up_layout;
typedef enum { E4B_ACT_SWIGLU = 0, E4B_ACT_CLAMPED_GLU = 1 } e4b_activation;

typedef struct {
  int32_t fmt; /* e4b_format */
  int32_t E, H, I;
  const uint8_t* gate_up_codes;
  const void* gate_up_scales;
  const uint8_t* down_codes;
  const void* down_scales;
  int32_t gate_up_layout; /* e4b_gate_up_layout */
  int32_t activation;     /* e4b_activation */
  float glu_alpha, glu_limit;
  const float* gate_up_bias;
  const float* down_bias;
  /* MXFP4 only, optional: the stacks prepared for the block-scaled FP4 MMA
   * by e4b_mxfp4_native_prepare (gate_up with nmat = 2, down with nmat = 1);
   * all four set, or all null. With them the large-M path multiplies the
   * e2m1 codes directly (E4B_PATH_TCGEN05_MX); without them it decodes to
   * bf16. Codes 32-byte aligned, scale chunks 16-byte aligned. */
  const uint8_t* gate_up_mx_codes;
  const uint8_t* gate_up_mx_sf;
  const uint8_t* down_mx_codes;
  const uint8_t* down_mx_sf;
} e4b_moe_weights;

/* ---------------------------------------------------------------- formats */

/*
 * e4b_quantize_nf4 -- [G] CPU block 1 (quantize_pack_nf4), [P] Summary.
 * w: float [E, N, K] row-major. For each expert, row and block of
 * `blocksize` weights along K: absmax = max|w|; every weight gets the index of
 * the NF4 level nearest to fp32(w / absmax) (ties to the lower index; an
 * all-zero block gets the zero level, index 7). Writes codes uint8
 * [E, N, K/2] (earlier weight in the high nibble) and absmax float
 * [E, N, K/blocksize]. blocksize must be 64; K % 64 == 0.
 */
e4b_status e4b_quantize_nf4(const float* w, int64_t E, int64_t N, int64_t K, int32_t blocksize,
                            uint8_t* codes, float* absmax, void* stream);

/*
 * e4b_quantize_mxfp4 -- [G] intro and CPU block 2 (quantize_pack_mxfp4),
 * OCP Microscaling v1.0. w: float [E, N, K], K % 32 == 0. Per 32-weight
 * block: scale exponent e = floor(log2 max|w|) - 2 clamped to [-127, 127]
 * (byte e + 127; an all-zero block gets byte 0 and zero codes); each weight
 * w / 2^e rounds to the nearest e2m1 value (ties to even, saturating at 6),
 * sign bit copied from w. Writes blocks uint8 [E, N, K/32, 16] (earlier
 * weight in the low nibble) and scales uint8 [E, N, K/32].
 */
e4b_status e4b_quantize_mxfp4(const float* w, int64_t E, int64_t N, int64_t K,
                              uint8_t* blocks, uint8_t* scales, void* stream);

/*
 * e4b_dequantize -- [G] CPU block 1 (dequant_ref) / block 2 (dequant_mxfp4).
 * Decodes a packed stack [E, N, K] to bf16 out [E, N, K] with exactly the
 * per-block table the GEMM kernels use: NF4 weight = bf16_rne(fp32(level) *
 * absmax), MXFP4 weight = sign * e2m1 * 2^(scale-127) (exact in bf16). For
 * tests of the decode; the layer never calls it.
 */
e4b_status e4b_dequantize(int32_t fmt, const uint8_t* codes, const void* scales, int64_t E,
                          int64_t N, int64_t K, uint16_t* out, void* stream);

/*
 * MXFP4 stacks for the block-scaled FP4 MMA ([G] intro: MXFP4 as OCP e2m1 +
 * e8m0 on the released bytes; Blackwell's tcgen05.mma kind::mxf8f6f4 reads
 * e2m1 codes with one e8m0 scale per 32 elements of K). The tensor memory
 * access that feeds those codes to the MMA needs rows padded to a multiple of
 * 128 elements, and the MMA takes its scales as 512-byte chunks of 128 rows x
 * 4 blocks, so a stack is prepared once into a second copy of its bytes:
 *   codes uint8 [E][nmat][Np][Kp/2]      the same nibbles (earlier weight low),
 *                                        rows past rows_per_mat and K zero
 *   sf    uint8 [E][nmat][Np/128][Kp/128][512]  row r of a 128-row block =
 *                                        32 m1 + m0, 32-block b of a 128-wide
 *                                        K chunk: byte 16 m0 + 4 m1 + b; pads 0
 * with Np, Kp = rows_per_mat and K rounded up to multiples of 128. gate_up
 * stacks are prepared with nmat = 2 (matrix 0 = the gate rows, matrix 1 = the
 * up rows, de-interleaved according to gate_up_layout), down stacks with
 * nmat = 1 (gate_up_layout ignored). The source stack is [E, nmat *
 * rows_per_mat, K/32, 16] codes + [E, nmat * rows_per_mat, K/32] scales as in
 * e4b_moe_weights; K % 32 == 0; blocks 16-byte aligned; codes_out 32-byte
 * aligned; sf_out 16-byte aligned. The prepared copy is read-only afterwards.
 */
e4b_status e4b_mxfp4_native_size(int32_t E, int64_t rows_per_mat, int64_t K, int32_t nmat,
                                 size_t* codes_bytes, size_t* sf_bytes);
e4b_status e4b_mxfp4_native_prepare(const uint8_t* blocks, const uint8_t* scales, int32_t E,
                                    int64_t rows_per_mat, int64_t K, int32_t nmat,
                                    int32_t gate_up_layout, uint8_t* codes_out, uint8_t* sf_out,
                                    void* stream);

/*
 * e4b_quantize_mxfp8 -- OCP Microscaling v1.0 MXFP8 with E4M3 elements (the
 * activations of the block-scaled MMA under E4B_FLAG_MX_ACT_E4M3; the pages do
 * not name an activation precision). x: bf16 [R, K] (16-byte aligned, K % 32
 * == 0). Per 32 values along K: amax = max|x|, X = floor(log2 amax) - 8
 * clamped to [-127, 127], scales[r, b] = X + 127 (0 for an all-zero block),
 * elems[r, k] = E4M3 bits of x / 2^X rounded to nearest even, saturating at
 * +-448. elems uint8 [R, K] (8-byte aligned), scales uint8 [R, K/32].
 */
e4b_status e4b_quantize_mxfp8(const uint16_t* x, int64_t R, int64_t K, uint8_t* elems, uint8_t* scales,
                              void* stream);

/* Host: copies the library's 16 NF4 levels (fp32, ascending) into out[16]. */
e4b_status e4b_nf4_codebook(float* out_host);

/* ---------------------------------------------------------------- routing */

/* Host: bytes of workspace e4b_route needs for these sizes (always > 0):
 * the status words, plus, for T*top_k >= 16384 slots, the scratch that lets
 * the pass run over many CTAs (two launches instead of one; same result). A
 * workspace of only the status words still routes any size, on one CTA. */
e4b_status e4b_route_workspace_size(int64_t T, int32_t top_k, int32_t E, size_t* bytes);

/*
 * e4b_route -- [G] intro (one launch over all active experts needs the
 * routed rows grouped by expert). ids: int32 [T, top_k] expert per slot
 * (slot s = t*top_k + j). Writes counts int32 [E] (slots per expert),
 * offsets int64 [E+1] (exclusive prefix sum), perm int32 [T*top_k] (perm[p]
 * = the slot at expert-ordered position p; within an expert slots keep
 * increasing order) and inv_perm int32 [T*top_k] (position of each slot).
 * An id outside [0, E) sets E4B_ERR_BAD_EXPERT_ID in ws's status word and
 * its slot is left out (offsets[E] then counts the valid slots; inv_perm of a
 * dropped slot is -1). ws: device scratch of e4b_route_workspace_size bytes.
 * Requires E <= 1024 and T*top_k < 2^31.
 */
e4b_status e4b_route(const int32_t* ids, int64_t T, int32_t top_k, int32_t E, int32_t* counts,
                     int64_t* offsets, int32_t* perm, int32_t* inv_perm, void* ws,
                     size_t ws_bytes, void* stream);

/* ------------------------------------------------------------ grouped GEMM */

typedef enum {
  E4B_EPI_STORE = 0,   /* out bf16 [R, N]: row p = A_p . W_e^T */
  E4B_EPI_SWIGLU = 1,  /* out bf16 [R, N/2]: silu(gate) * up, gate = rows [0, N/2) */
  E4B_EPI_COMBINE = 2  /* out fp32 [T, N] += gates[s] * (A_p . W_e^T), s = row_slot[p],
                          t = s / top_k; the caller zeroes out beforehand */
} e4b_epilogue;

/*
 * One projection of all experts in one launch ([G] intro: the grouped GEMM
 * over all active experts on packed weights, fp32 accumulation, bf16
 * epilogue). Rows of expert e are [offsets[e], offsets[e+1]); row p multiplies
 * the bf16 activation row a[(a_row_slot ? a_row_slot[p] / top_k : p) * lda ..
 * + K) with the decoded weight stack W [E, N, K] (codes / scales laid out as
 * in e4b_moe_weights). R = offsets[E] rows are produced.
 *   STORE:   out bf16, row p at out + p*ldo, N values.
 *   SWIGLU:  out bf16, row p at out + p*ldo, N/2 values silu(g)*u with g the
 *            row's first N/2 outputs (weight rows 0..N/2-1), u the rest.
 *   COMBINE: out fp32 [T, ldo]; with s = out_row_slot[p] (p if NULL) and
 *            t = s / top_k: out[t, n] += gates[s] * (row p output n). The
 *            caller zeroes out first; the sum order over slots is not fixed.
 * N must be a multiple of 16 (32 for SWIGLU), K of 64 (NF4) or 32 (MXFP4),
 * lda and ldo multiples of 8; a, codes and out 16-byte aligned.
 */
typedef struct {
  int32_t fmt;      /* e4b_format */
  int32_t epilogue; /* e4b_epilogue */
  int32_t E;
  int32_t top_k;    /* slots per token (1 when rows are not routing slots) */
  int64_t N, K;     /* weight rows and inner dimension */
  int64_t R_max;    /* upper bound on offsets[E], i.e. rows of the row buffers */
  const uint8_t* codes;        /* [E, N, K/2] */
  const void* scales;          /* NF4 float [E, N, K/64]; MXFP4 uint8 [E, N, K/32] */
  const uint16_t* a;           /* bf16 activations */
  int64_t lda;                 /* elements between activation rows */
  const int32_t* a_row_slot;   /* optional [R_max]: gather map for activation rows */
  const int32_t* out_row_slot; /* COMBINE, optional [R_max]: routing slot of each row */
  const int64_t* offsets;      /* [E+1] */
  const float* gates;          /* COMBINE: [T*top_k] weight of each slot */
  void* out;
  int64_t ldo;                 /* elements between output rows */
  /* expert variant (zero = plain), as in e4b_moe_weights: SWIGLU reads
   * gate_up_layout and activation; bias is per weight row, fp32 [E, N], added
   * to the accumulator before the epilogue (null = none) */
  int32_t gate_up_layout;
  int32_t activation;
  float glu_alpha, glu_limit;
  const float* bias;
} e4b_gemm_args;

e4b_status e4b_grouped_gemm(const e4b_gemm_args* args, uint32_t flags, void* stream);

/*
 * e4b_grouped_dgrad -- [G] entry table (the NF4 grouped GEMM's backward,
 * dgrad_4bit_grouped): the input gradient through the packed weights, in one
 * launch over all active experts. For routed row p of expert e (offsets[e] <=
 * p < offsets[e+1]):  dx[p] = dy[p] . W_e  (the contraction over the weight's
 * rows), fp32 accumulation, bf16 output. W_e is decoded as in e4b_grouped_gemm
 * (NF4 bf16_rne(fp32(level * absmax)), MXFP4 exact); no bf16 weight tensor is
 * stored. Runs on the tcgen05 path (E <= 256), on SM pairs; flags: 0 or
 * E4B_FLAG_TC_SINGLE_SM (the one-SM kernel; E4B_FLAG_FORCE_GEMV returns
 * E4B_ERR_UNSUPPORTED). Shapes: K % 64 == 0 (NF4) or K % 32 == 0
 * (MXFP4); N any. dy, codes, dx 16-byte aligned; ld_dy >= N and ld_dx >= K,
 * both multiples of 8. Rows p >= offsets[E] of dx are not written.
 */
typedef struct {
  int32_t fmt; /* e4b_format */
  int32_t E;
  int64_t N, K;          /* each expert's weight W_e is [N, K], packed along K (as the forward) */
  int64_t R_max;         /* bound on offsets[E] (rows of dy and dx) */
  const uint8_t* codes;  /* the packed stack [E, N, ...] as in e4b_gemm_args */
  const void* scales;
  const uint16_t* dy;    /* bf16 [R, N], rows in expert order */
  int64_t ld_dy;         /* elements between rows of dy */
  const int64_t* offsets; /* [E+1] */
  uint16_t* dx;          /* bf16 [R, K] */
  int64_t ld_dx;         /* elements between rows of dx */
} e4b_dgrad_args;

e4b_status e4b_grouped_dgrad(const e4b_dgrad_args* args, uint32_t flags, void* stream);

/* ---------------------------------------------------- int4-b32 (decode) */
/*
 * [S] "How do I run a single-token INT4 decode GEMV over routed MoE experts,
 * and pack calibrated (GPTQ) weights for it?" (grouped-nf4-gemm solutions
 * page): the batch-1 int4-b32 decode GEMV with exact integer accumulation and
 * the packer of calibrated weights onto the same bytes; [G] README table row
 * "int4-b32 decode GEMV, dense M=1". The pages do not print the encoding;
 * the library's reading:
 *   stack [E, N, K] as codes uint8 [E, N, K/2] (signed 4-bit q in [-8, 7],
 *   two's complement, the earlier weight in the LOW nibble) and scales fp16
 *   (bit patterns, uint16_t) [E, N, K/32]; weight = s * q. K % 32 == 0.
 */
#define E4B_INT4_BLOCK 32
#define E4B_INT4_MAX_SLOTS 64

/*
 * e4b_quantize_int4_b32 -- fp32 w [E, N, K] (16-byte aligned, K % 32 == 0)
 * -> codes [E, N, K/2] (16-byte aligned) and scales [E, N, K/32]: per 32
 * weights along K, s = fp16_rne(fp32(absmax / 7)) and q = clamp(rint(fp32(w /
 * s)), -8, 7), ties to even (q = 0 where s is 0). Weights must be finite.
 */
e4b_status e4b_quantize_int4_b32(const float* w, int64_t E, int64_t N, int64_t K, uint8_t* codes,
                                 uint16_t* scales, void* stream);

/*
 * e4b_gptq_pack_int4_b32 -- [S] the GPTQ packer. Input: symmetric GPTQ tensors
 * of each expert's W [N, K], group size 32, no act-order: qweight int32
 * [E, K/8, N] (eight unsigned 4-bit values u along K per word, value i in bits
 * 4i..4i+3, zero point 8: q = u - 8) and scales fp16 [E, K/32, N]. Output: the
 * int4-b32 stack above (codes [E, N, K/2], scales [E, N, K/32]), the same
 * values moved into row-major bytes. qweight and codes 4-byte aligned; buffers
 * must not overlap. Asymmetric zero points and act-order (g_idx) are not
 * accepted inputs.
 */
e4b_status e4b_gptq_pack_int4_b32(const int32_t* qweight, const uint16_t* gptq_scales, int64_t E,
                                  int64_t N, int64_t K, uint8_t* codes, uint16_t* scales,
                                  void* stream);

/*
 * e4b_gemv_int4_b32 -- [S] the decode GEMV: one token against its n_slots
 * routed experts e_j = expert_ids[j] of an int4-b32 stack, in one launch.
 * Every CTA quantises the token row(s) to int8 with one fp32 scale per row:
 * amax = max|x|, sx = fp32(amax / 127), r = fp32(127 / amax),
 * xq = clamp(rint(fp32(x * r)), -127, 127), ties to even (a row whose r is
 * not finite -- all zero, or amax below 127 / FLT_MAX -- gets sx = 0 and
 * xq = 0); per 32-weight block the products q * xq are summed exactly in
 * int32; then
 *   acc[j, n] = sx_j * sum_b s[e_j, n, b] * D[e_j, n, b]   (fp32)
 * and the epilogue writes bf16:
 *   E4B_EPI_STORE    y [n_slots, N] (row stride ld_y >= N):  bf16(acc[j, n])
 *   E4B_EPI_SWIGLU   y [n_slots, N/2] (ld_y >= N/2, N even): bf16(silu(acc[j, i])
 *                    * acc[j, N/2 + i]) -- gate rows first, up rows second
 *   E4B_EPI_COMBINE  y [N]: bf16(sum_j gates[j] * acc[j, n]) -- no accumulator,
 *                    one warp owns a row across all slots
 * x: bf16 rows of K values (16-byte aligned). ld_x == 0: every slot reads the
 * one row x (the gate_up GEMV); ld_x > 0 (>= K, multiple of 8): slot j reads
 * x + j * ld_x (the down GEMV, h of each slot), each row with its own sx.
 * 1 <= n_slots <= 64; the rows of x (ld_x == 0: 1, else n_slots) times K must
 * fit in shared memory (<= 200 KiB), else E4B_ERR_UNSUPPORTED. An expert id
 * outside [0, E) drops that slot (its STORE/SWIGLU rows are written as 0) and
 * records E4B_ERR_BAD_EXPERT_ID in *status when status is not NULL. x must
 * be finite. Weight rows stream through shared memory in bulk copies whose
 * waits are bounded; a wait that gives up records E4B_ERR_DEVICE_TIMEOUT in
 * *status and leaves y unwritten. The kernel is launched as a programmatic
 * dependent of the work before it on the stream: it waits for that work to
 * complete before it reads x (and, without E4B_FLAG_IDS_READY, the ids and
 * gates) or writes y. flags: any of E4B_FLAG_IDS_READY (see above) and
 * E4B_FLAG_TEST_TIMEOUT (every wait gives up at once: tests that error path).
 */
typedef struct {
  int32_t epilogue;           /* E4B_EPI_STORE, E4B_EPI_SWIGLU or E4B_EPI_COMBINE */
  int32_t E;
  int64_t N, K;               /* each expert's W is [N, K] */
  int32_t n_slots;
  const uint8_t* codes;       /* [E, N, K/2], 16-byte aligned */
  const uint16_t* scales;     /* fp16 [E, N, K/32] */
  const int32_t* expert_ids;  /* [n_slots] */
  const float* gates;         /* [n_slots], COMBINE only (else may be NULL) */
  const uint16_t* x;          /* bf16, see ld_x */
  int64_t ld_x;               /* 0 = one row for every slot, else elements between slot rows */
  uint16_t* y;                /* bf16 output, see epilogue */
  int64_t ld_y;               /* elements between output rows (STORE / SWIGLU) */
  int32_t* status;            /* optional device int32 that records a bad expert id */
} e4b_int4_gemv_args;

e4b_status e4b_gemv_int4_b32(const e4b_int4_gemv_args* args, uint32_t flags, void* stream);

/* ------------------------------------------------------ expert parallel */
/*
 * Expert parallelism over G ranks, one process per GPU (the pages describe one
 * GPU; this split is the library's own): rank r holds the experts
 * [r * epr, (r + 1) * epr) of the layer. A rank routes its tokens' slots by
 * destination rank (e4b_ep_dest, then e4b_route with E = G), packs the routed
 * rows in that order (e4b_ep_pack), exchanges them with an all-to-all (the
 * caller's NCCL), runs its experts on the rows it received with
 * e4b_moe_forward (one slot a row: ids = the local expert ids, gates = the
 * slot gates), sends the outputs back and sums each token's rows
 * (e4b_ep_combine). Every slot's output is rounded to bf16 before the sum, so
 * y differs from the one-GPU layer by at most top_k bf16 roundings.
 */

/* dest[i] = ids[i] / epr for ids[i] in [0, E), else -1 (the routing pass then
 * drops the slot and records E4B_ERR_BAD_EXPERT_ID). ids, dest: int32 [n]. */
e4b_status e4b_ep_dest(const int32_t* ids, int64_t n, int32_t E, int32_t epr, int32_t* dest, void* stream);

/* For every position p < offsets[G] of the destination order (perm and
 * offsets from e4b_route over dest with E = G): xs[p] = x[perm[p] / top_k]
 * (bf16 [R_max, H]), local_ids[p] = ids[perm[p]] % epr, local_gates[p] =
 * gates[perm[p]]. x and xs 16-byte aligned, H % 8 == 0. Positions from
 * offsets[G] to R_max are not written. */
e4b_status e4b_ep_pack(const uint16_t* x, int64_t H, const int32_t* ids, const float* gates, int32_t top_k,
                       const int32_t* perm, const int64_t* offsets, int32_t G, int64_t R_max, int32_t epr,
                       uint16_t* xs, int32_t* local_ids, float* local_gates, void* stream);

/* y[t] = bf16(sum_j ys[inv_perm[t * top_k + j]]) with fp32 sums; slots whose
 * inv_perm is -1 are left out (a token with none gets 0). ys bf16 [R, H] in
 * the destination order, y bf16 [T, H]; 16-byte aligned, H % 8 == 0. */
e4b_status e4b_ep_combine(const uint16_t* ys, int64_t H, const int32_t* inv_perm, int64_t T, int32_t top_k,
                          uint16_t* y, void* stream);

/* ---------------------------------------------------------- whole layer */

/* Host: workspace bytes for e4b_moe_forward with T tokens and top_k slots.
 * The workspace holds the status word, the routing arrays, h, one fp32 region
 * (the small-M path's partial sums [ceil(I/2048)][T*top_k][H] of its down
 * passes, or the large-M path's gate-weighted rows [T*top_k, H]) and last a
 * staging copy of the routed rows of x in expert order ([T*top_k, H] bf16)
 * that the large-M path uses. A smaller workspace
 * that holds everything the chosen path needs but the staging copy is
 * accepted; the large-M path then gathers the rows inside its kernel (same
 * results, slower). */
e4b_status e4b_moe_workspace_size(const e4b_moe_weights* w, int64_t T, int32_t top_k,
                                  size_t* bytes);

/*
 * e4b_moe_forward -- the MoE layer ([P] Design: per-expert gate_up GEMM,
 * gated SiLU, down GEMM, weighted sum over the chosen experts; [G] intro: one
 * launch per projection over all active experts on the packed bytes).
 *   x     bf16 [T, H] (16-byte aligned rows: H % 8 == 0)
 *   ids   int32 [T, top_k] expert of each slot (duplicates allowed)
 *   gates float [T, top_k] weight of each slot
 *   y     bf16 [T, H] output: y[t] = bf16( sum_j gates[t,j] * down_e(
 *         bf16(silu(gate_e(x[t])) * up_e(x[t])) ) ), e = ids[t,j]
 *   ws    device scratch of e4b_moe_workspace_size bytes (routing, the bf16
 *         intermediate h [T*top_k, I], an fp32 accumulator [T, H], status,
 *         the optional staging copy of the routed rows)
 *   flags E4B_FLAG_* (0 = choose the path from the shape)
 * The path is chosen on the host from T*top_k/E with no device sync, so the
 * call is graph-capturable. T == 0 is a no-op. Limits: E <= 1024 and
 * T*top_k < 2^31; the large-M (tcgen05) path takes E <= 256, so with E > 256
 * the small-M path runs whatever T (E4B_FLAG_FORCE_TCGEN05 then returns
 * E4B_ERR_UNSUPPORTED).
 * With w->fmt == E4B_FMT_INT4B32 (stacks as in e4b_gemv_int4_b32: scales fp16)
 * the layer runs the batch-1 int4-b32 decode GEMVs token by token: for each
 * token the gate_up GEMV with the SwiGLU epilogue into h [top_k, I] in ws,
 * then the down GEMV with the combine epilogue into y[t] (2 launches a
 * token; the intermediate h and the activations are quantised as described
 * there). The expert variant must be the plain one (halves, SwiGLU, no
 * biases), top_k <= 64, H % 32 == 0 and I % 32 == 0; flags: 0 or
 * E4B_FLAG_TEST_TIMEOUT. Otherwise E4B_ERR_UNSUPPORTED.
 * MXFP4 weights with prepared stacks (gate_up_mx_codes ...) take, on the
 * large-M path, the block-scaled FP4 MMA: x and h are split into e4m3 terms
 * (see E4B_FLAG_MX_ACT_E4M3) in padded per-expert row blocks inside ws
 * (e4b_moe_workspace_size then includes them), 6 launches. On every path each
 * routed row's output (small-M: each 2048-wide K slice's partial sum) is
 * written once and each token's rows are summed in a fixed order, so repeated
 * calls give the same bits. Launches: small-M 3 (routing, the layer kernel,
 * the combine), large-M 5 (4 without the staging copy); from 16384 routed rows
 * on the large-M paths the routing takes 2 launches instead of 1.
 */
e4b_status e4b_moe_forward(const e4b_moe_weights* w, const uint16_t* x, int64_t T, int32_t top_k,
                           const int32_t* ids, const float* gates, uint16_t* y, void* ws,
                           size_t ws_bytes, uint32_t flags, void* stream);

/*
 * e4b_moe_forward_noalloc -- the layer forward of e4b_moe_forward for callers
 * that cannot allocate device memory. The pages describe no such entry
 * point; it exists for callers that get no allocator: code running while a
 * stream is being captured into a CUDA graph under a framework that forbids
 * allocation there, runtimes that hand every byte of HBM to their own pool,
 * and host plug-in interfaces that pass only input and output buffers. A
 * cudaMalloc in such a place either fails, synchronises the device, or takes
 * memory its owner did not budget for.
 *
 * Same arguments and results as e4b_moe_forward, without ws / ws_bytes: the
 * scratch (routing arrays, bf16 intermediate, fp32 accumulator, status word)
 * lives in a 16 MiB array in the library's device memory, which every GPU
 * that loads the library keeps until the process exits. A call whose
 * required scratch exceeds 16 MiB returns E4B_ERR_EXCEEDS_STATIC_SCRATCH and
 * enqueues nothing. The required scratch is, for NF4 and MXFP4 stacks,
 * the part of e4b_moe_workspace_size the chosen path needs (without the
 * optional staging copy; a layer with E=8, H=4096, I=14336 and top-2 routing
 * fits up to 58 tokens on the small-M path it takes up to 64 tokens, and up to
 * 186 tokens on the large-M path it takes from 65 tokens on; the staging copy
 * is used while it also fits), and for int4-b32 stacks
 * e4b_moe_workspace_size itself, which does not grow with T. Nothing is
 * allocated or freed.
 *   - The first call on each device looks up that device's copy of the
 *     array (set-up, once per device); make that first call before any stream
 *     capture begins. The address found belongs to the device's context as it
 *     was then: after a cudaDeviceReset on that device, do not call this
 *     entry point again in the same process.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents; each call re-clears what must start at zero. Calls whose GPU
 *     work overlaps (different streams, or graphs replayed concurrently) race
 *     on the array: order them on one stream.
 *   - The device status word is inside the array and is not readable with
 *     e4b_read_device_status; use e4b_moe_forward with a workspace when the
 *     status is needed.
 */
e4b_status e4b_moe_forward_noalloc(const e4b_moe_weights* w, const uint16_t* x, int64_t T,
                                   int32_t top_k, const int32_t* ids, const float* gates,
                                   uint16_t* y, uint32_t flags, void* stream);

/* Synchronises `stream`, then reads and clears the device status word that
 * e4b_route / e4b_moe_forward keep at the start of ws. *status_host receives
 * an e4b_status (E4B_OK if the GPU reported nothing). */
e4b_status e4b_read_device_status(void* ws, int32_t* status_host, void* stream);

/*
 * Host: instrumentation for benchmarks. With n == 5, every later
 * e4b_moe_forward call on this thread records events[0..4] (cudaEvent_t,
 * created by the caller) on its stream before the routing kernel, before the
 * gate_up kernel, before the down kernel, before the output conversion and
 * after it. n == 0 switches recording off. The library does not own the events.
 */
e4b_status e4b_set_timing_events(void* const* events, int32_t n);

/* Host: the path the most recent e4b_moe_forward / e4b_grouped_gemm call on
 * this thread enqueued (an e4b_path). */
int32_t e4b_last_path(void);

/* Host: number of kernels the most recent e4b_moe_forward call on this thread
 * enqueued. */
int32_t e4b_last_launch_count(void);

/* Host: a static string naming the status. */
const char* e4b_status_string(int32_t status);

/* Host: library version, e.g. "e4b 0.1.0 sm_100a". */
const char* e4b_version(void);

#ifdef __cplusplus
}
#endif

#endif /* E4B_H_ */
