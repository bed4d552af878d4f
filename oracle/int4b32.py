"""Oracle: the int4-b32 format and its decode GEMV (test infrastructure only).

Definitions followed ("grouped-nf4-gemm" README, "How do I run a single-token
INT4 decode GEMV over routed MoE experts, and pack calibrated (GPTQ) weights
for it?": gemv_int4_b32 runs the batch-1 int4-b32 decode GEMV with exact
integer accumulation, and gptq_pack_int4_b32 packs calibrated weights onto the
same bytes; measured row: "int4-b32 decode GEMV, dense M=1"). The pages name
the format and the accumulation, not the encoding. Readings (plainest ones
that give exact integer accumulation):

* Weights, per row and per block of 32 weights along K: a signed 4-bit
  integer q in [-8, 7] per weight (two's complement, two per byte, the earlier
  weight in the LOW nibble) and one fp16 scale s per block; the weight value is
  s * q. Quantising an fp32 row: s = fp16(absmax / 7) (absmax / 7 in fp32, then
  rounded to fp16); q = clamp(round_half_even(fp32(w / float(s))), -8, 7); an
  all-zero block (or one whose scale rounds to 0) gets s = 0 and q = 0.
* Activation (one token): amax = max |x|; the dequantisation scale is
  sx = fp32(amax / 127) and the quantisation multiplier r = fp32(127 / amax)
  (both IEEE fp32 divisions); xq = clamp(round_half_even(fp32(x * r)), -127,
  127) as int8, so that every value is decided by one fp32 product. A token
  whose r is not finite (amax = 0, or amax below 127 / FLT_MAX) has sx = 0 and
  xq = 0.
* Output, for weight row n: y[n] = sx * sum_b s[n, b] * D[n, b] with the block
  dot products D[n, b] = sum over the block of q * xq, exact integers. Here the
  sum over blocks is taken in fp64 and y is rounded once to bf16, after the
  epilogue: none, the SwiGLU of the gate and up halves (the layer's gated SiLU,
  as in the NF4 path), or the gate-weighted sum over the routed slots.
* The down GEMV of a decode step reads one activation row per routed slot
  (that slot's h = bf16 SwiGLU output); each row is quantised with its own sx.
* GPTQ packing (symmetric, group size 32): GPTQ's packed int32 tensors hold
  unsigned 4-bit values u in [0, 15] with zero point 8, i.e. q = u - 8:
  ``qweight [K/8, N]`` int32 with 8 values along K per word (value i in bits
  4i..4i+3), ``scales [K/32, N]`` fp16. Packing onto int4-b32 moves the same
  values and scales into the row-major byte layout above.

Parity pins (tests/test_oracle_int4b32.py): hand-worked bytes of the nibble
packing and of a GPTQ word; the quantisers within half a step of their inputs,
with the block maximum on +-7; the block dot products against a pure-Python
integer loop; the GEMV against the dequantised fp64 matrix times sx * xq (a
different route to the same number); each epilogue against explicit loops;
the GPTQ pack against GPTQ's own dequantisation formula; a zero token and a
zero block.
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_round
from .moe import swiglu_ref

BLOCK = 32


def _rne(v: np.ndarray) -> np.ndarray:
    """Round half to even (numpy's rint) of float32 values, as int64."""
    return np.rint(v).astype(np.int64)


def quantize_int4b32(w) -> tuple[np.ndarray, np.ndarray]:
    """fp32 [..., N, K] -> (codes uint8 [..., N, K/2], scales fp16 [..., N, K/32])."""
    w = np.asarray(w, np.float32)
    K = w.shape[-1]
    assert K % BLOCK == 0
    blk = w.reshape(w.shape[:-1] + (K // BLOCK, BLOCK))
    amax = np.max(np.abs(blk), axis=-1)
    s16 = (amax / np.float32(7.0)).astype(np.float32).astype(np.float16)
    s32 = s16.astype(np.float32)
    safe = np.where(s32 > 0, s32, np.float32(1.0))
    q = _rne((blk / safe[..., None]).astype(np.float32))
    q = np.clip(q, -8, 7)
    q = np.where((s32 > 0)[..., None], q, 0)
    return pack_int4(q.reshape(w.shape)), s16


def pack_int4(q) -> np.ndarray:
    """Signed ints in [-8, 7], [..., K] -> bytes [..., K/2], earlier in the low nibble."""
    u = (np.asarray(q, np.int64) & 15).astype(np.uint8)
    return (u[..., 0::2] | (u[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(codes) -> np.ndarray:
    """bytes [..., K/2] -> signed ints [..., K]."""
    c = np.asarray(codes, np.uint8)
    lo = (c & 15).astype(np.int64)
    hi = (c >> 4).astype(np.int64)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return np.where(out >= 8, out - 16, out)


def dequant_int4b32(codes, scales) -> np.ndarray:
    """The weight values s * q as fp64 [..., N, K]."""
    q = unpack_int4(codes).astype(np.float64)
    s = np.repeat(np.asarray(scales, np.float16).astype(np.float64), BLOCK, axis=-1)
    return q * s


def quantize_token(x) -> tuple[np.ndarray, np.float32]:
    """One token (values as fp32 [K]) -> (xq int8 [K] as int64, sx fp32)."""
    x = np.asarray(x, np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0.0)
    with np.errstate(divide="ignore", over="ignore"):
        r = np.float32(np.float32(127.0) / amax) if amax > 0 else np.float32(np.inf)
    if not np.isfinite(r):
        return np.zeros(x.shape, np.int64), np.float32(0.0)
    sx = np.float32(amax / np.float32(127.0))
    xq = np.clip(_rne((x * r).astype(np.float32)), -127, 127)
    return xq, sx


def block_dots(codes, xq, rows=None, chunk: int = 1024) -> np.ndarray:
    """Exact integer block dot products D [n, K/32] of one expert's rows (all,
    or the listed `rows`) with the token's int8 values xq [K]; rows are taken
    `chunk` at a time to bound memory."""
    codes = np.asarray(codes, np.uint8)
    rows = np.arange(codes.shape[0]) if rows is None else np.asarray(rows, np.int64)
    K = codes.shape[1] * 2
    xb = np.asarray(xq, np.int64).reshape(1, K // BLOCK, BLOCK)
    out = np.empty((len(rows), K // BLOCK), np.int64)
    for r0 in range(0, len(rows), chunk):
        q = unpack_int4(codes[rows[r0:r0 + chunk]])
        out[r0:r0 + chunk] = (q.reshape(-1, K // BLOCK, BLOCK) * xb).sum(axis=-1)
    return out


def gemv_int4b32_acc(x, expert_ids, codes, scales, rows=None) -> np.ndarray:
    """acc[j, n] = sx_j * sum_b s_e[n, b] * D_e[n, b] in fp64, e = expert_ids[j].

    x holds the tokens' values: [K] (one token for every routed slot) or
    [n_slots, K] (slot j reads row j, each row quantised with its own scale).
    codes [E, N, K/2] uint8, scales [E, N, K/32] fp16; `rows` restricts n."""
    x = np.asarray(x, np.float32)
    ids = [int(e) for e in expert_ids]
    xs = [x] * len(ids) if x.ndim == 1 else [x[j] for j in range(len(ids))]
    out = []
    for j, e in enumerate(ids):
        xq, sx = quantize_token(xs[j])
        D = block_dots(codes[e], xq, rows).astype(np.float64)
        s = np.asarray(scales[e], np.float16).astype(np.float64)
        if rows is not None:
            s = s[np.asarray(rows, np.int64)]
        out.append(np.float64(sx) * np.sum(s * D, axis=-1))
    return np.array(out).reshape(len(ids), -1)


def gemv_int4b32_ref(x, expert_ids, codes, scales, epilogue: str = "store", gates=None,
                     rows=None) -> np.ndarray:
    """The batch-1 decode GEMV over routed experts, with its epilogues. With
    acc from gemv_int4b32_acc (fp64, never rounded before the epilogue):
      "store"    y[j, n] = bf16(acc[j, n])                       [n_slots, N]
      "swiglu"   h[j, i] = bf16(silu(acc[j, i]) * acc[j, N/2 + i]) [n_slots, N/2]
                 (gate rows first, up rows second, as the fused gate_up stack)
      "combine"  y[n] = bf16(sum_j gates[j] * acc[j, n])          [N]
    `rows` (store / combine: output rows; swiglu: output columns i) computes
    only those outputs. Returns fp64 holding bf16 values."""
    if epilogue == "store":
        return bf16_round(gemv_int4b32_acc(x, expert_ids, codes, scales, rows))
    if epilogue == "swiglu":
        half = np.asarray(codes).shape[1] // 2
        cols = np.arange(half) if rows is None else np.asarray(rows, np.int64)
        g = gemv_int4b32_acc(x, expert_ids, codes, scales, cols)
        u = gemv_int4b32_acc(x, expert_ids, codes, scales, cols + half)
        return bf16_round(swiglu_ref(g, u))
    if epilogue == "combine":
        acc = gemv_int4b32_acc(x, expert_ids, codes, scales, rows)
        g = np.asarray(gates, np.float32).astype(np.float64).reshape(-1, 1)
        return bf16_round(np.sum(g * acc, axis=0))
    raise ValueError(epilogue)


def int4b32_decode_layer_ref(x, expert_ids, gates, gu_codes, gu_scales, dn_codes, dn_scales,
                             rows=None) -> np.ndarray:
    """One token through the MoE layer on int4-b32 stacks: the gate_up GEMV with
    the SwiGLU epilogue gives h [k, I] (bf16); each slot's h row is quantised on
    its own for the down GEMV, whose combine epilogue gives y [H] (bf16).
    `rows` restricts the output rows of y (h is always computed in full)."""
    h = gemv_int4b32_ref(x, expert_ids, gu_codes, gu_scales, "swiglu")
    return gemv_int4b32_ref(h, expert_ids, dn_codes, dn_scales, "combine", gates, rows)


def gptq_pack_int4b32_ref(qweight, gscales) -> tuple[np.ndarray, np.ndarray]:
    """Symmetric GPTQ tensors of one matrix W [N, K] (qweight int32 [K/8, N],
    8 unsigned values along K per word; scales fp16 [K/32, N]) -> (codes uint8
    [N, K/2], scales fp16 [N, K/32]) in int4-b32."""
    qw = np.asarray(qweight).astype(np.int64) & 0xFFFFFFFF
    K8, N = qw.shape
    u = np.empty((K8 * 8, N), np.int64)
    for i in range(8):
        u[i::8] = (qw >> (4 * i)) & 15
    q = (u - 8).T  # [N, K]
    return pack_int4(q), np.ascontiguousarray(np.asarray(gscales, np.float16).T)
