"""Pins of the oracle's expert variant ("experts4bit-qlora" README, Scope:
gpt-oss MXFP4 experts with per-expert biases and a clamped GLU): interleaved
gate/up rows, biases after each projection, the clamped GLU."""

import math

import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_e4b_b200 import synth


def _layer(fmt, E, H, I, seed, interleave=False, std=0.05):
    rng = np.random.default_rng(seed)
    wgu = (rng.standard_normal((E, 2 * I, H)) * std).astype(np.float32)
    wd = (rng.standard_normal((E, H, I)) * std).astype(np.float32)
    if interleave:  # gate row n -> 2n, up row n -> 2n+1
        wi = np.empty_like(wgu)
        wi[:, 0::2] = wgu[:, :I]
        wi[:, 1::2] = wgu[:, I:]
        wgu = wi
    q = oracle.quantize_pack_nf4 if fmt == "nf4" else oracle.quantize_pack_mxfp4
    return q(wgu) + q(wd)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_interleaved_rows_equal_halves_after_permutation(fmt):
    E, H, I, T, k = 3, 64, 128, 12, 2
    halves = _layer(fmt, E, H, I, seed=1)
    inter = _layer(fmt, E, H, I, seed=1, interleave=True)
    rng = np.random.default_rng(2)
    x = oracle.bf16_round(rng.standard_normal((T, H)))
    ids, gates = synth.random_ids(rng, T, k, E)
    bgu = rng.standard_normal((E, 2 * I)).astype(np.float32)
    bgu_i = np.empty_like(bgu)
    bgu_i[:, 0::2] = bgu[:, :I]
    bgu_i[:, 1::2] = bgu[:, I:]
    bd = rng.standard_normal((E, H)).astype(np.float32)
    kw = dict(act="clamped_glu", alpha=1.702, limit=7.0, dn_bias=bd)
    y_h = oracle.moe_forward_ref(fmt, x, ids, gates, *halves, E, H, I, layout="halves", gu_bias=bgu, **kw)
    y_i = oracle.moe_forward_ref(fmt, x, ids, gates, *inter, E, H, I, layout="interleaved", gu_bias=bgu_i, **kw)
    assert np.array_equal(y_h, y_i)


def test_clamped_glu_without_clamp_is_shifted_silu():
    # alpha = 1 and an infinite limit: (U + 1) * G * sigmoid(G) = (U + 1) * silu(G)
    rng = np.random.default_rng(3)
    G = rng.standard_normal(1000) * 6
    U = rng.standard_normal(1000) * 6
    got = oracle.clamped_glu_ref(G, U, 1.0, math.inf)
    want = ((torch.from_numpy(U) + 1) * torch.nn.functional.silu(torch.from_numpy(G))).numpy()
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


def test_clamped_glu_saturates_at_the_limit():
    alpha, limit = 1.702, 7.0
    big = np.array([7.0, 7.5, 30.0, 1e6])
    at = oracle.clamped_glu_ref(np.full(4, limit), np.full(4, limit), alpha, limit)
    assert np.array_equal(oracle.clamped_glu_ref(big, big, alpha, limit), at)
    # up is clamped from below too; gate only from above
    lo = oracle.clamped_glu_ref(np.array([2.0]), np.array([-50.0]), alpha, limit)
    assert lo[0] == (1.0 - limit) * 2.0 / (1.0 + math.exp(-alpha * 2.0))
    neg = oracle.clamped_glu_ref(np.array([-20.0]), np.array([0.0]), alpha, limit)
    assert neg[0] == -20.0 / (1.0 + math.exp(alpha * 20.0))


@pytest.mark.parametrize("layout", ["halves", "interleaved"])
def test_biases_with_zero_weights(layout):
    # all-zero weights decode to exact zeros, so GU is the gate_up bias, h the
    # activation of it, O the down bias and y the gate-weighted sum of biases
    fmt, E, H, I, T, k = "mxfp4", 2, 64, 32, 5, 2
    z = oracle.quantize_pack_mxfp4(np.zeros((E, 2 * I, H), np.float32)) + \
        oracle.quantize_pack_mxfp4(np.zeros((E, H, I), np.float32))
    rng = np.random.default_rng(4)
    x = oracle.bf16_round(rng.standard_normal((T, H)))
    ids, gates = synth.random_ids(rng, T, k, E)
    bgu = (rng.standard_normal((E, 2 * I)) * 8).astype(np.float32)
    bd = rng.standard_normal((E, H)).astype(np.float32)
    y, hs = oracle.moe_forward_ref(fmt, x, ids, gates, *z, E, H, I, layout=layout, act="clamped_glu",
                                   alpha=1.702, limit=7.0, gu_bias=bgu, dn_bias=bd, return_h=True)
    b = torch.from_numpy(bgu.astype(np.float64))
    gb, ub = (b[:, :I], b[:, I:]) if layout == "halves" else (b[:, 0::2], b[:, 1::2])
    g = torch.clamp(gb, max=7.0)
    u = torch.clamp(ub, -7.0, 7.0)
    h_want = oracle.bf16_round(((u + 1) * g * torch.sigmoid(1.702 * g)).numpy())
    for t in range(T):
        for j in range(k):
            assert np.array_equal(hs[t * k + j], h_want[ids[t, j]])
    y_want = oracle.bf16_round(np.stack([sum(np.float64(gates[t, j]) * bd[ids[t, j]].astype(np.float64)
                                             for j in range(k)) for t in range(T)]))
    assert np.array_equal(y, y_want)
