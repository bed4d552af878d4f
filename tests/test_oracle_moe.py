"""Pins for the oracle's routing and layer forward (CPU only)."""

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from bit_grouped_moe_e4b_b200 import synth
from bit_grouped_moe_e4b_b200.configs import TINY


def _quantised_layer(fmt, E, H, I, seed, std=0.02):
    rng = np.random.default_rng(seed)
    wgu = (rng.standard_normal((E, 2 * I, H)) * std).astype(np.float32)
    wd = (rng.standard_normal((E, H, I)) * std).astype(np.float32)
    q = oracle.quantize_pack_nf4 if fmt == "nf4" else oracle.quantize_pack_mxfp4
    gc, gs = q(wgu)
    dc, ds = q(wd)
    return gc, gs, dc, ds


def _decoded(fmt, codes, scales, N, K):
    if fmt == "nf4":
        return oracle.dequant_ref(codes, scales, N, K).astype(np.float64)
    return oracle.dequant_mxfp4(codes, scales).reshape(N, K).astype(np.float64)


# --------------------------------------------------------------- routing
def test_route_invariants_and_brute_force():
    rng = np.random.default_rng(2)
    for T, k, E in [(1, 1, 1), (5, 2, 8), (64, 8, 128), (33, 4, 3), (0, 2, 4)]:
        ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
        counts, offsets, perm, inv = oracle.route_ref(ids, E)
        assert counts.sum() == T * k and offsets[-1] == T * k
        assert np.array_equal(np.sort(perm), np.arange(T * k))
        assert np.array_equal(perm[inv], np.arange(T * k))
        flat = ids.reshape(-1)
        for e in range(E):
            seg = perm[offsets[e]:offsets[e + 1]]
            assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)  # stable
        bc, bo, bp, bi = brute.route_loops(ids.tolist(), E)
        assert counts.tolist() == bc and offsets.tolist() == bo
        assert perm.tolist() == bp and inv.tolist() == bi


def test_route_rejects_bad_ids():
    with pytest.raises(ValueError):
        oracle.route_ref(np.array([[0, 4]]), 4)
    with pytest.raises(ValueError):
        oracle.route_ref(np.array([[-1, 0]]), 4)


def test_synth_router_contract():
    ids, gates = synth.routing(TINY, 64)
    assert ids.shape == (64, 2) and gates.shape == (64, 2)
    assert np.all(ids[:, 0] != ids[:, 1])
    assert np.allclose(gates.sum(1), 1.0, atol=1e-6) and np.all(gates[:, 0] >= gates[:, 1])
    logits = np.zeros((1, 4), dtype=np.float32)  # all tied: lower index first
    i2, g2 = synth.topk_route(logits, 2)
    assert i2.tolist() == [[0, 1]] and np.allclose(g2, 0.5)


# ------------------------------------------------------------ the layer
@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_single_expert_reduces_to_dense_swiglu_mlp(fmt):
    # E=1, k=1, gate=1: y = bf16(Wd . bf16(silu(Wg x) * (Wu x))) with Wg the
    # first I rows of gate_up -- a textbook dense MLP, computed with torch.
    H, I, T = 64, 128, 5
    gc, gs, dc, ds = _quantised_layer(fmt, 1, H, I, seed=1)
    x = torch.randn(T, H, dtype=torch.float32).to(torch.bfloat16)
    ids = np.zeros((T, 1), np.int32)
    gates = np.ones((T, 1), np.float32)
    y = oracle.moe_forward_ref(fmt, x.float().numpy(), ids, gates, gc, gs, dc, ds, 1, H, I)
    Wgu = torch.from_numpy(_decoded(fmt, gc[0], gs[0], 2 * I, H))
    Wd = torch.from_numpy(_decoded(fmt, dc[0], ds[0], H, I))
    xd = x.double()
    g = torch.nn.functional.linear(xd, Wgu[:I])
    u = torch.nn.functional.linear(xd, Wgu[I:])
    h = torch.from_numpy(oracle.bf16_round((torch.nn.functional.silu(g) * u).numpy()))
    want = oracle.bf16_round(torch.nn.functional.linear(h, Wd).numpy())
    assert np.array_equal(y, want)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_layer_matches_pure_python_loops(fmt):
    E, H, I, T, k = 3, 64, 64, 4, 2
    gc, gs, dc, ds = _quantised_layer(fmt, E, H, I, seed=4, std=0.1)
    rng = np.random.default_rng(9)
    x = oracle.bf16_round(rng.standard_normal((T, H)))
    ids = np.array([[0, 2], [1, 1], [2, 0], [2, 1]], np.int32)  # a duplicate slot pair too
    gates = rng.random((T, k)).astype(np.float32)
    Wgu = [_decoded(fmt, gc[e], gs[e], 2 * I, H).tolist() for e in range(E)]
    Wd = [_decoded(fmt, dc[e], ds[e], H, I).tolist() for e in range(E)]
    y_loop, h_loop = brute.moe_loops(x.tolist(), ids.tolist(), gates.tolist(), Wgu, Wd, I)
    y, h = oracle.moe_forward_ref(fmt, x, ids, gates, gc, gs, dc, ds, E, H, I, return_h=True)
    for s, row in h_loop.items():
        assert np.array_equal(h[s], np.array(row))
    y_loop = np.array(y_loop)
    assert np.all(np.abs(y_loop - y) <= np.abs(y_loop) * 2 ** -8 + 1e-30)
    assert np.array_equal(oracle.bf16_round(y_loop), y)


def test_token_subset_equals_full_rows():
    E, H, I, T, k = 4, 64, 128, 12, 2
    gc, gs, dc, ds = _quantised_layer("nf4", E, H, I, seed=8)
    rng = np.random.default_rng(1)
    x = oracle.bf16_round(rng.standard_normal((T, H)))
    ids, gates = synth.random_ids(rng, T, k, E)
    full = oracle.moe_forward_ref("nf4", x, ids, gates, gc, gs, dc, ds, E, H, I)
    sub = oracle.moe_forward_ref("nf4", x, ids, gates, gc, gs, dc, ds, E, H, I, tokens=[3, 7, 11])
    assert np.array_equal(full[[3, 7, 11]], sub)


def test_gate_weights_scale_linearly_and_zero_gate_drops_expert():
    E, H, I, T, k = 4, 64, 64, 6, 2
    gc, gs, dc, ds = _quantised_layer("nf4", E, H, I, seed=3)
    rng = np.random.default_rng(5)
    x = oracle.bf16_round(rng.standard_normal((T, H)))
    ids, gates = synth.random_ids(rng, T, k, E)
    y1 = oracle.moe_forward_ref("nf4", x, ids, gates, gc, gs, dc, ds, E, H, I)
    y2 = oracle.moe_forward_ref("nf4", x, ids, gates * 2, gc, gs, dc, ds, E, H, I)
    assert np.array_equal(y1 * 2, y2)  # bf16 rounding commutes with x2
    g0 = gates.copy()
    g0[:, 1] = 0
    ids1 = ids.copy()
    ids1[:, 1] = (ids[:, 1] + 1) % E  # the dropped slot's expert does not matter
    a = oracle.moe_forward_ref("nf4", x, ids, g0, gc, gs, dc, ds, E, H, I)
    b = oracle.moe_forward_ref("nf4", x, ids1, g0, gc, gs, dc, ds, E, H, I)
    assert np.array_equal(a, b)


def test_planted_mistakes_are_caught(monkeypatch):
    """Each plausible slip in the layer, planted in the oracle, breaks a pin."""
    import oracle.moe as m

    H, I, T = 64, 128, 5
    gc, gs, dc, ds = _quantised_layer("nf4", 1, H, I, seed=1)
    x = torch.randn(T, H).to(torch.bfloat16).float().numpy()
    ids = np.zeros((T, 1), np.int32)
    gates = np.ones((T, 1), np.float32)
    good = oracle.moe_forward_ref("nf4", x, ids, gates, gc, gs, dc, ds, 1, H, I)

    # gate / up halves swapped
    monkeypatch.setattr(m, "swiglu_ref", lambda G, U: oracle.swiglu_ref(U, G))
    bad = m.moe_forward_ref("nf4", x, ids, gates, gc, gs, dc, ds, 1, H, I)
    assert not np.array_equal(bad, good)
    monkeypatch.undo()

    # a dropped absmax scale in the decode
    real = m.dequant_ref
    monkeypatch.setattr(m, "dequant_ref", lambda p, a, N, K: real(p, np.ones_like(a), N, K))
    bad = m.moe_forward_ref("nf4", x, ids, gates, gc, gs, dc, ds, 1, H, I)
    assert not np.array_equal(bad, good)
