"""The oracle's C core agrees with the numpy oracle (CPU only)."""

import numpy as np
import pytest

import oracle
from oracle import fast


@pytest.fixture(scope="module", autouse=True)
def _built():
    fast.build()


def _weights(seed, N, K):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[0, :64] = 0
    w[1, :64] = 0
    w[1, 5] = -0.25
    cb = oracle.nf4_codebook()
    w[2, :64] = 0
    w[2, 0] = 1.0
    w[2, 1] = cb[8] / 2  # exact tie
    w[2, 2] = cb[6] / 2
    w[3, :32] = np.array([4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0] * 4, np.float32)
    w[4, :64] *= 1e-33
    return w


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_c_quantise_and_decode_match_numpy(fmt):
    w = _weights(0, 64, 320)
    c, s = fast.quantize(fmt, w)
    if fmt == "nf4":
        cn, sn = oracle.quantize_pack_nf4(w)
        dn = oracle.dequant_ref(cn, sn, 64, 320)
    else:
        cn, sn = oracle.quantize_pack_mxfp4(w)
        dn = oracle.dequant_mxfp4(cn, sn)
    assert np.array_equal(c, cn) and np.array_equal(s, sn)
    d = fast.decode(fmt, c, s, 64, 320)
    assert np.array_equal(d.view(np.uint32), dn.view(np.uint32))


def test_c_matvec_matches_numpy():
    rng = np.random.default_rng(1)
    W = rng.standard_normal((33, 200)).astype(np.float32)
    X = rng.standard_normal((3, 200))
    assert np.allclose(fast.matvec(W, X), X @ W.astype(np.float64).T, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_sampled_layer_matches_oracle_layer(fmt):
    E, H, I, T, k = 4, 128, 192, 10, 2
    rng = np.random.default_rng(2)
    wgu = (rng.standard_normal((E, 2 * I, H)) * 0.05).astype(np.float32)
    wd = (rng.standard_normal((E, H, I)) * 0.05).astype(np.float32)
    q = oracle.quantize_pack_nf4 if fmt == "nf4" else oracle.quantize_pack_mxfp4
    gc, gs = q(wgu)
    dc, ds = q(wd)
    x = oracle.bf16_round(rng.standard_normal((T, H)))
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    gates = rng.random((T, k)).astype(np.float32)
    full = oracle.moe_forward_ref(fmt, x, ids, gates, gc, gs, dc, ds, E, H, I)
    toks = [1, 4, 9]
    fn = lambda which, e: wgu[e] if which == "gate_up" else wd[e]
    y, cols, packed = fast.moe_forward_sampled(fmt, x, ids, gates, fn, E, H, I, toks)
    assert np.array_equal(cols, np.arange(H))
    diff = np.abs(y - full[toks])
    # fp64 sums in another order: identical after bf16 rounding except at a
    # rounding boundary, where they may differ by one bf16 step
    assert np.all(diff <= np.abs(full[toks]) * 2 ** -7 + 1e-30)
    assert (diff == 0).mean() > 0.99
    for (which, e), (c, s) in packed.items():
        ref = (gc[e], gs[e]) if which == "gate_up" else (dc[e], ds[e])
        assert np.array_equal(c, ref[0]) and np.array_equal(s, ref[1])


def test_sampled_layer_matches_oracle_layer_for_the_expert_variant():
    # interleaved gate/up, biases and the clamped GLU through the C-backed path
    fmt, E, H, I, T, k = "mxfp4", 3, 96, 160, 8, 2
    rng = np.random.default_rng(5)
    wgu = (rng.standard_normal((E, 2 * I, H)) * 0.3).astype(np.float32)
    wd = (rng.standard_normal((E, H, I)) * 0.05).astype(np.float32)
    gc, gs = oracle.quantize_pack_mxfp4(wgu)
    dc, ds = oracle.quantize_pack_mxfp4(wd)
    x = oracle.bf16_round(rng.standard_normal((T, H)))
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    gates = rng.random((T, k)).astype(np.float32)
    v = dict(layout="interleaved", act="clamped_glu", alpha=1.702, limit=7.0,
             gu_bias=rng.standard_normal((E, 2 * I)).astype(np.float32),
             dn_bias=rng.standard_normal((E, H)).astype(np.float32))
    full = oracle.moe_forward_ref(fmt, x, ids, gates, gc, gs, dc, ds, E, H, I, **v)
    toks = [0, 3, 7]
    fn = lambda which, e: wgu[e] if which == "gate_up" else wd[e]
    y, _, _ = fast.moe_forward_sampled(fmt, x, ids, gates, fn, E, H, I, toks, variant=v)
    diff = np.abs(y - full[toks])
    assert np.all(diff <= np.abs(full[toks]) * 2 ** -7 + 1e-30)
    assert (diff == 0).mean() > 0.99
