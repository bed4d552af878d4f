"""Oracle: routing permutation and the MoE layer forward (test infrastructure only).

Definitions followed
--------------------
* Routing ("grouped-nf4-gemm" README intro: one launch covers all active
  experts; the decode glue's router epilogue and combine): the layer receives
  top-k expert ids [T, k] and gate weights [T, k]. Slots ``s = t*k + j`` are
  ordered expert by expert; within an expert, slots keep increasing ``s``
  (a stable order). ``counts[e]`` = slots routed to e, ``offsets`` = the
  exclusive prefix sum (E+1 entries, int64), ``perm[p]`` = the slot at
  expert-ordered position p, ``inv_perm[s]`` = the position of slot s.
* Layer (bitsandbytes PR #1984 Design: per-expert dequantise loop with a gated
  SiLU activation; "experts4bit-qlora" README: fused ``gate_up_proj
  [E, 2I, H]`` and ``down_proj [E, H, I]``; "grouped-nf4-gemm" README: the
  fused kernel computes what dequantise-then-matmul computes):

      [G | U]  = X_e . D(W_gu[e])^T      gate = rows 0..I-1, up = rows I..2I-1
      h        = bf16_rne(silu(G) * U)
      O        = h . D(W_d[e])^T
      y[t]     = bf16_rne( sum_j gates[t, j] * O[slot t*k + j] )   (slot order)

  where D is the parity-contract decode (``dequant_ref`` for NF4,
  ``dequant_mxfp4`` for MXFP4) and everything else is fp64. The oracle rounds h
  to bf16 because the fused layer stores h as bf16 between its two GEMMs.

* Expert variant ("experts4bit-qlora" README, Scope: gpt-oss MXFP4 experts
  with per-expert biases and a clamped GLU). The pages name the variant but
  print neither its row layout nor its activation. Reading, from the released
  gpt-oss expert definition: gate and up rows interleaved (gate = row 2n, up =
  row 2n+1 of gate_up), fp32 biases added to each projection's output, and

      g' = min(G, limit),  u' = clamp(U, -limit, limit)
      h  = bf16_rne((u' + 1) * g' * sigmoid(alpha * g'))

  with alpha and limit parameters of the call (the released model uses 1.702
  and 7). Bias rows follow the weight rows (gate_up bias [E, 2I] in the
  gate_up row order, down bias [E, H]).

* Grouped projection and its input gradient ("grouped-nf4-gemm" README,
  intro and entry table: the grouped GEMM and, for training, its backward
  ``dgrad_4bit_grouped``): for routed row p of expert e,
      out[p] = a[p] . D(W_e)^T        (grouped_projection_ref)
      dx[p]  = dy[p] . D(W_e)         (grouped_dgrad_ref, the contraction over
                                       the weight's rows: its adjoint)
  fp64, rounded once to bf16.

Parity pins (tests): routing invariants and a brute-force loop; the E=1, k=1,
gate=1 case reduces to a dense SwiGLU MLP checked against torch on CPU; a
pure-Python loop agrees with this module on tiny shapes. Variant: interleaved
rows equal the halves layout after a row permutation; the clamped GLU with
alpha = 1 and no clamp reduces to (U + 1) * silu(G) (checked against torch's
silu); saturation beyond the limit; biases shift the output linearly.
Projection and dgrad: the adjoint identity <dgrad(dy), a> = <dy, proj(a)>
before rounding, a brute-force loop on tiny shapes, and empty experts.
"""

from __future__ import annotations

import numpy as np

from .mxfp8 import mxfp8_round_trip
from .formats import (
    bf16_round,
    dequant_ref,
    dequant_ref_exact,
    dequant_ref_level,
    dequant_mxfp4,
)


def route_ref(ids, E: int):
    """Stable expert-contiguous order of the T*k routing slots.

    ids: int [T, k] with values in [0, E). Returns (counts int32 [E],
    offsets int64 [E+1], perm int32 [T*k], inv_perm int32 [T*k]).
    """
    flat = np.asarray(ids).reshape(-1).astype(np.int64)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id out of range")
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return counts, offsets, perm, inv


def swiglu_ref(G, U):
    """silu(G) * U in fp64."""
    G = np.asarray(G, np.float64)
    return G / (1.0 + np.exp(-G)) * np.asarray(U, np.float64)


def clamped_glu_ref(G, U, alpha: float, limit: float):
    """(clamp(U, -limit, limit) + 1) * g' * sigmoid(alpha * g'), g' = min(G, limit), in fp64."""
    g = np.minimum(np.asarray(G, np.float64), np.float64(limit))
    u = np.clip(np.asarray(U, np.float64), -np.float64(limit), np.float64(limit))
    return (u + 1.0) * g / (1.0 + np.exp(-np.float64(alpha) * g))


def split_gate_up(GU, layout: str):
    """Gate and up columns of a gate_up projection output [R, 2I]: the two
    halves, or the even and odd rows (interleaved)."""
    if layout == "halves":
        I = GU.shape[-1] // 2
        return GU[..., :I], GU[..., I:]
    if layout == "interleaved":
        return GU[..., 0::2], GU[..., 1::2]
    raise ValueError(layout)


def activation_ref(G, U, act: str, alpha: float = 1.702, limit: float = 7.0):
    if act == "swiglu":
        return swiglu_ref(G, U)
    if act == "clamped_glu":
        return clamped_glu_ref(G, U, alpha, limit)
    raise ValueError(act)


NF4_DECODES = ("product", "level", "exact")


def _decode(fmt, codes, scales, N, K, nf4_decode="product"):
    if fmt == "nf4":
        if nf4_decode == "exact":
            return dequant_ref_exact(codes, scales, N, K)
        if nf4_decode == "level":
            return dequant_ref_level(codes, scales, N, K)
        if nf4_decode == "product":
            return dequant_ref(codes, scales, N, K).astype(np.float64)
        raise ValueError(nf4_decode)
    if fmt == "mxfp4":
        return dequant_mxfp4(codes, scales).reshape(N, K).astype(np.float64)
    raise ValueError(fmt)


def expert_tokens(ids, tokens=None):
    """For each expert, the (slot, token) pairs routed to it, in slot order,
    restricted to ``tokens`` when given."""
    ids = np.asarray(ids)
    T, k = ids.shape
    sel = np.arange(T) if tokens is None else np.asarray(tokens)
    out = {}
    for t in sel:
        for j in range(k):
            out.setdefault(int(ids[t, j]), []).append((int(t) * k + j, int(t)))
    for e in out:
        out[e].sort()
    return out


def moe_forward_ref(fmt, x, ids, gates, gu_codes, gu_scales, dn_codes, dn_scales,
                    E, H, I, tokens=None, exact_decode=False, return_h=False,
                    layout="halves", act="swiglu", alpha=1.702, limit=7.0,
                    gu_bias=None, dn_bias=None, nf4_decode="product", act_quant=None):
    """The MoE layer forward (per-expert dequantise-then-matmul loop).

    x: bf16 values as any float array [T, H]; ids int [T, k]; gates fp32
    [T, k]. Weights per expert: NF4 codes [E, 2I, H/2] + absmax [E, 2I, H/64]
    and [E, H, I/2] + [E, H, I/64]; MXFP4 blocks [E, 2I, H/32, 16] + scales
    [E, 2I, H/32] and [E, H, I/32, 16] + [E, H, I/32].

    tokens: optional subset of token indices; only their outputs are computed
    (an expert's weights are decoded only if a selected token uses it).
    Returns y as fp64 holding bf16 values, [len(tokens) or T, H]; with
    return_h, also {slot: h row (fp64 holding bf16 values)}.

    Expert variant: ``layout`` "halves" | "interleaved", ``act`` "swiglu" |
    "clamped_glu" (alpha, limit), ``gu_bias`` [E, 2I] and ``dn_bias`` [E, H]
    fp32 or None.

    nf4_decode: the NF4 weight value, "product" (bf16_rne(fp32(level *
    absmax)), dequant_ref), "level" (bf16_rne(level) * absmax exactly,
    dequant_ref_level) or "exact" (level * absmax, fidelity only; also
    selected by exact_decode=True).

    act_quant: None (bf16 activations), or "mxfp8": the x rows and the bf16
    intermediate h are replaced by their MXFP8 decode (oracle.mxfp8: E4M3
    elements, one e8m0 scale per 32 along K) before the matmul that reads
    them -- the activations a block-scaled FP4 tensor-core MMA multiplies.
    """
    x = np.asarray(x, dtype=np.float64)
    ids = np.asarray(ids)
    gates = np.asarray(gates, dtype=np.float32)
    T, k = ids.shape
    sel = np.arange(T) if tokens is None else np.asarray(tokens)
    row_of = {int(t): i for i, t in enumerate(sel)}
    acc = np.zeros((len(sel), H), dtype=np.float64)
    # O for every selected slot, kept so the combine can run in slot order
    O_slot = {}
    h_slot = {}
    for e, pairs in sorted(expert_tokens(ids, sel).items()):
        mode = "exact" if exact_decode else nf4_decode
        Wgu = _decode(fmt, gu_codes[e], gu_scales[e], 2 * I, H, mode)
        Wd = _decode(fmt, dn_codes[e], dn_scales[e], H, I, mode)
        X = x[[t for _, t in pairs]]
        if act_quant == "mxfp8":
            X = mxfp8_round_trip(X)
        elif act_quant is not None:
            raise ValueError(act_quant)
        GU = X @ Wgu.T
        if gu_bias is not None:
            GU = GU + np.asarray(gu_bias[e], np.float64)
        G, U = split_gate_up(GU, layout)
        h = bf16_round(activation_ref(G, U, act, alpha, limit))
        O = (mxfp8_round_trip(h) if act_quant == "mxfp8" else h) @ Wd.T
        if dn_bias is not None:
            O = O + np.asarray(dn_bias[e], np.float64)
        for r, (s, _) in enumerate(pairs):
            O_slot[s] = O[r]
            h_slot[s] = h[r]
        del Wgu, Wd
    for t in sel:
        for j in range(k):
            s = int(t) * k + j
            acc[row_of[int(t)]] += np.float64(gates[t, j]) * O_slot[s]
    y = bf16_round(acc)
    if return_h:
        return y, h_slot
    return y


def grouped_projection_ref(fmt, a, offsets, codes, scales, N, K, nf4_decode="product"):
    """The grouped projection ("grouped-nf4-gemm" README, intro): routed row p
    of expert e (offsets[e] <= p < offsets[e+1]) times the decoded weight
    W_e [N, K]: out[p] = a[p] . W_e^T (a [R, K] -> out [R, N]), fp64 holding
    the bf16-rounded result."""
    a = np.asarray(a, np.float64)
    offsets = np.asarray(offsets)
    out = np.zeros((a.shape[0], N), np.float64)
    for e in range(len(offsets) - 1):
        p0, p1 = int(offsets[e]), int(offsets[e + 1])
        if p1 > p0:
            out[p0:p1] = a[p0:p1] @ _decode(fmt, codes[e], scales[e], N, K, nf4_decode).T
    return bf16_round(out)


def grouped_dgrad_ref(fmt, dy, offsets, codes, scales, N, K, nf4_decode="product"):
    """The input gradient through the packed weights ("grouped-nf4-gemm"
    README, entry table: the NF4 grouped GEMM's backward, dgrad_4bit_grouped):
    for routed row p of expert e, dx[p] = dy[p] . W_e, the contraction over the
    weight's rows (dy [R, N] -> dx [R, K]) -- the adjoint of
    grouped_projection_ref. fp64 holding the bf16-rounded result."""
    dy = np.asarray(dy, np.float64)
    offsets = np.asarray(offsets)
    out = np.zeros((dy.shape[0], K), np.float64)
    for e in range(len(offsets) - 1):
        p0, p1 = int(offsets[e]), int(offsets[e + 1])
        if p1 > p0:
            out[p0:p1] = dy[p0:p1] @ _decode(fmt, codes[e], scales[e], N, K, nf4_decode)
    return bf16_round(out)
