"""Oracle: the plain-C core (oracle_core.c) and the sampled full-size layer
(test infrastructure only).

The C functions restate the numpy definitions in ``formats`` as loops; the
CPU tests check them against the numpy oracle bit for bit before they are
used. ``moe_forward_sampled`` is ``moe.moe_forward_ref`` for a few tokens of
a full-size layer: the same per-expert quantise -> decode -> fp64 matmul ->
bf16(h) -> fp64 matmul -> weighted sum, with the heavy loops in C. It
quantises from the fp32 weights itself; nothing comes from the CUDA library.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .formats import bf16_round, nf4_codebook
from .moe import activation_ref, expert_tokens, split_gate_up
from .mxfp8 import mxfp8_round_trip

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "oracle_core.c")
LIB = os.path.join(_HERE, "_oracle_core.so")
_lib = None


def build(force: bool = False) -> str:
    """gcc -O2 without fast-math or FMA contraction (IEEE fp32/fp64 steps)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp"
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                        "-o", tmp, SRC, "-lm"], check=True)
        os.replace(tmp, LIB)
    return LIB


def _core():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        L.e4bref_nf4_quantize.argtypes = [vp, i64, i64, vp, vp, vp]
        L.e4bref_nf4_decode.argtypes = [vp, vp, i64, i64, vp, vp]
        L.e4bref_mxfp4_quantize.argtypes = [vp, i64, i64, vp, vp]
        L.e4bref_mxfp4_decode.argtypes = [vp, vp, i64, i64, vp]
        L.e4bref_nf4_decode_level.argtypes = [vp, vp, i64, i64, vp, vp]
        L.e4bref_matvec_f64.argtypes = [vp, i64, i64, vp, i64, vp]
        L.e4bref_matvec_f64w.argtypes = [vp, i64, i64, vp, i64, vp]
        for f in ("e4bref_nf4_quantize", "e4bref_nf4_decode", "e4bref_nf4_decode_level", "e4bref_mxfp4_quantize",
                  "e4bref_mxfp4_decode", "e4bref_matvec_f64", "e4bref_matvec_f64w"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.c_void_p)


def quantize(fmt: str, w: np.ndarray):
    """fp32 [N, K] -> (codes, scales) in the layouts of formats.quantize_pack_*."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    if fmt == "nf4":
        cb = nf4_codebook()
        codes = np.empty((N, K // 2), np.uint8)
        scales = np.empty((N, K // 64), np.float32)
        _core().e4bref_nf4_quantize(_p(w), N, K, _p(cb), _p(codes), _p(scales))
        return codes, scales
    codes = np.empty((N, K // 32, 16), np.uint8)
    scales = np.empty((N, K // 32), np.uint8)
    _core().e4bref_mxfp4_quantize(_p(w), N, K, _p(codes), _p(scales))
    return codes, scales


def decode(fmt: str, codes, scales, N: int, K: int, nf4_decode: str = "product") -> np.ndarray:
    """Decode to [N, K]: fp32 holding bf16 values (MXFP4, NF4 "product"), or
    fp64 for NF4 "level" (bf16_rne(level) * absmax exactly)."""
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    if fmt == "nf4" and nf4_decode == "level":
        out = np.empty((N, K), np.float64)
        _core().e4bref_nf4_decode_level(_p(codes), _p(scales), N, K, _p(nf4_codebook()), _p(out))
        return out
    if fmt == "nf4" and nf4_decode != "product":
        raise ValueError(nf4_decode)
    out = np.empty((N, K), np.float32)
    if fmt == "nf4":
        cb = nf4_codebook()
        _core().e4bref_nf4_decode(_p(codes), _p(scales), N, K, _p(cb), _p(out))
    else:
        _core().e4bref_mxfp4_decode(_p(codes), _p(scales), N, K, _p(out))
    return out


def matvec(W: np.ndarray, X: np.ndarray) -> np.ndarray:
    """fp64 X @ W^T for W fp32 or fp64 [rows, K], X fp64 [n, K]."""
    X = np.ascontiguousarray(X, np.float64)
    rows, K = W.shape
    n = X.shape[0]
    Y = np.empty((n, rows), np.float64)
    if W.dtype == np.float64:
        W = np.ascontiguousarray(W)
        _core().e4bref_matvec_f64w(_p(W), rows, K, _p(X), n, _p(Y))
    else:
        W = np.ascontiguousarray(W, np.float32)
        _core().e4bref_matvec_f64(_p(W), rows, K, _p(X), n, _p(Y))
    return Y


def expert_term(fmt, X, packed_gu, packed_dn, H, I, cols=None, variant=None, e=None, nf4_decode="product",
                act_quant=None):
    """One expert's contribution for the rows X (bf16 values, [n, H]):
    decode gate_up -> fp64 matmul (+ bias) -> bf16(activation(gate, up)) ->
    decode down -> fp64 matmul (+ bias). ``variant``: dict of moe_forward_ref's
    expert-variant arguments (layout, act, alpha, limit, gu_bias, dn_bias),
    the biases indexed by expert ``e``. ``nf4_decode`` as in moe_forward_ref
    ("product" or "level"); ``act_quant`` as in moe_forward_ref (None or
    "mxfp8"). Returns (O fp64 [n, len(cols)], h)."""
    v = variant or {}
    Wgu = decode(fmt, *packed_gu, 2 * I, H, nf4_decode)
    X = np.asarray(X, np.float64)
    if act_quant == "mxfp8":
        X = mxfp8_round_trip(X)
    elif act_quant is not None:
        raise ValueError(act_quant)
    GU = matvec(Wgu, X)
    del Wgu
    if v.get("gu_bias") is not None:
        GU = GU + np.asarray(v["gu_bias"][e], np.float64)
    G, U = split_gate_up(GU, v.get("layout", "halves"))
    h = bf16_round(activation_ref(G, U, v.get("act", "swiglu"), v.get("alpha", 1.702), v.get("limit", 7.0)))
    Wd = decode(fmt, *packed_dn, H, I, nf4_decode)
    if cols is not None:
        Wd = np.ascontiguousarray(Wd[cols])
    O = matvec(Wd, mxfp8_round_trip(h) if act_quant == "mxfp8" else h)
    if v.get("dn_bias") is not None:
        b = np.asarray(v["dn_bias"][e], np.float64)
        O = O + (b if cols is None else b[cols])
    return O, h


def moe_forward_sampled(fmt, x, ids, gates, weight_fn, E, H, I, tokens, down_rows=None,
                        packed_fn=None, variant=None, nf4_decode="product", workers=None, act_quant=None):
    """Outputs y[t, n] for the given tokens (and optionally only the given
    output columns n) of the layer whose fp32 expert weights weight_fn(which,
    e) returns ("gate_up" [2I, H], "down" [H, I]); with packed_fn(which, e)
    given instead, the experts arrive already packed (codes, scales).
    nf4_decode: the NF4 weight value as in moe_forward_ref.

    The experts are independent, so they are taken by `workers` threads
    (default: one per host core, at most one per expert); the C loops run
    without the interpreter lock. weight_fn / packed_fn are called under a
    lock, one at a time. Every expert's arithmetic is the serial one.

    Returns (y fp64 holding bf16 values [len(tokens), len(cols)], cols,
    packed) where packed[(which, e)] = (codes, scales) this function used.
    """
    import threading
    from concurrent.futures import ThreadPoolExecutor

    x = np.asarray(x, np.float64)
    ids = np.asarray(ids)
    gates = np.asarray(gates, np.float32)
    T, k = ids.shape
    cols = np.arange(H) if down_rows is None else np.asarray(down_rows)
    O_slot = {}
    packed = {}
    lock = threading.Lock()
    work = sorted(expert_tokens(ids, tokens).items())

    def one(item):
        e, pairs = item
        mine = {}
        for which in ("gate_up", "down"):
            with lock:
                src = packed_fn(which, e) if packed_fn is not None else weight_fn(which, e)
            mine[which] = src if packed_fn is not None else quantize(fmt, src)
            del src
        X = x[[t for _, t in pairs]]
        O, _ = expert_term(fmt, X, mine["gate_up"], mine["down"], H, I,
                           None if down_rows is None else cols, variant, e, nf4_decode, act_quant)
        return e, pairs, mine, O

    n = workers or min(len(work), os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=max(1, n)) as ex:
        for e, pairs, mine, O in ex.map(one, work):
            for which in ("gate_up", "down"):
                packed[(which, e)] = mine[which]
            for r, (slot, _) in enumerate(pairs):
                O_slot[slot] = O[r]
    y = np.zeros((len(tokens), len(cols)), np.float64)
    for i, t in enumerate(tokens):
        for j in range(k):
            y[i] += np.float64(gates[t, j]) * O_slot[int(t) * k + j]
    return bf16_round(y), cols, packed
