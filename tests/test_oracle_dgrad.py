"""Pins of the oracle's grouped projection and its input gradient
("grouped-nf4-gemm" README, entry table: the grouped GEMM's backward
dgrad_4bit_grouped). dgrad is the adjoint of the projection through the same
decoded weights: <dgrad(dy), a> = <dy, proj(a)> exactly before the final bf16
rounding; a pure-Python loop on tiny shapes; empty experts give no rows."""

import numpy as np
import pytest

import oracle
from oracle import moe as moe_mod


def _stack(fmt, E, N, K, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((E, N, K)) * 0.05).astype(np.float32)
    q = oracle.quantize_pack_nf4 if fmt == "nf4" else oracle.quantize_pack_mxfp4
    return q(w)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_dgrad_is_the_adjoint_of_the_projection(fmt):
    E, N, K = 3, 96, 128
    codes, scales = _stack(fmt, E, N, K, 1)
    offsets = np.array([0, 5, 5, 12])
    rng = np.random.default_rng(2)
    a = rng.standard_normal((12, K))
    dy = rng.standard_normal((12, N))
    # unrounded versions via the same decode
    proj = np.zeros((12, N))
    dg = np.zeros((12, K))
    for e in range(E):
        W = moe_mod._decode(fmt, codes[e], scales[e], N, K)
        p0, p1 = offsets[e], offsets[e + 1]
        proj[p0:p1] = a[p0:p1] @ W.T
        dg[p0:p1] = dy[p0:p1] @ W
    assert np.isclose(np.sum(dg * a), np.sum(dy * proj), rtol=1e-12, atol=1e-12)
    # the oracle functions round those once to bf16
    assert np.array_equal(oracle.grouped_dgrad_ref(fmt, dy, offsets, codes, scales, N, K), oracle.bf16_round(dg))
    assert np.array_equal(oracle.grouped_projection_ref(fmt, a, offsets, codes, scales, N, K),
                          oracle.bf16_round(proj))


def test_dgrad_brute_force_loop_nf4():
    E, N, K = 2, 8, 64
    codes, scales = _stack("nf4", E, N, K, 3)
    offsets = np.array([0, 2, 5])
    rng = np.random.default_rng(4)
    dy = oracle.bf16_round(rng.standard_normal((5, N)))
    cb = [float(v) for v in oracle.nf4_codebook()]
    levels = oracle.unpack_nf4_codes(codes)
    want = np.zeros((5, K))
    for p in range(5):
        e = 0 if p < 2 else 1
        for k in range(K):
            s = 0.0
            for n in range(N):
                wv = float(oracle.bf16_round(np.float32(np.float32(cb[levels[e, n, k]]) * scales[e, n, k // 64])))
                s += float(dy[p, n]) * wv
            want[p, k] = s
    got = oracle.grouped_dgrad_ref("nf4", dy, offsets, codes, scales, N, K)
    assert np.array_equal(got, oracle.bf16_round(want))


def test_empty_experts_and_no_rows():
    E, N, K = 3, 32, 64
    codes, scales = _stack("mxfp4", E, N, K, 5)
    dy = np.zeros((0, N))
    assert oracle.grouped_dgrad_ref("mxfp4", dy, np.zeros(E + 1, int), codes, scales, N, K).shape == (0, K)
    dy = np.ones((4, N))
    out = oracle.grouped_dgrad_ref("mxfp4", dy, np.array([0, 0, 4, 4]), codes, scales, N, K)
    W1 = oracle.dequant_mxfp4(codes[1], scales[1]).reshape(N, K).astype(np.float64)
    assert np.array_equal(out, oracle.bf16_round(np.tile(W1.sum(axis=0), (4, 1))))
