"""Pins of the MXFP8 activation oracle (oracle/mxfp8.py): the E4M3 value set,
its rounding and saturation, the MXFP8 block rule on hand-worked blocks, and
the layer in the act_mxfp8 reading against pure-Python loops."""

import math
import os

import numpy as np
import torch

import oracle
from oracle import brute
from oracle import mxfp8 as mx

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp8_handworked.txt")


def test_e4m3_value_set_from_bit_fields():
    v = mx.e4m3_values()
    finite = v[np.isfinite(v)]
    assert finite.size == 254  # 256 patterns, two NaNs (S.1111.111)
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert finite.max() == 448.0 and finite.min() == -448.0
    pos = finite[finite > 0]
    assert pos.min() == 2.0 ** -9  # smallest subnormal
    assert v[0x08] == 2.0 ** -6    # smallest normal
    assert v[0x7E] == 448.0 and v[0x38] == 1.0
    # the independent construction in the brute-force module agrees
    b = dict((code, val) for val, code in brute.e4m3_finite_values())
    for code, val in b.items():
        assert v[code] == val


def test_e4m3_round_equals_nearest_search_with_even_ties():
    rng = np.random.default_rng(0)
    vals = e4 = mx.e4m3_values()
    pos = np.sort(np.unique(np.abs(e4[np.isfinite(e4)])))
    mids = (pos[:-1] + pos[1:]) / 2  # every tie between neighbours
    xs = np.concatenate([rng.standard_normal(3000) * 30, rng.standard_normal(500) * 0.01, mids, -mids,
                         pos, [0.0, 447.0, 448.0, 455.0, 464.0, 470.0, 1e6, -1e6, 2.0 ** -10, 3 * 2.0 ** -10]])
    got = mx.e4m3_round(xs)
    want = np.array([brute.e4m3_nearest(float(a)) for a in xs])
    assert np.array_equal(got, want)
    del vals


def test_e4m3_round_matches_torch_inside_the_finite_range():
    rng = np.random.default_rng(1)
    xs = np.concatenate([rng.standard_normal(20000) * 50, rng.standard_normal(2000) * 1e-3])
    xs = xs[np.abs(xs) <= 448.0].astype(np.float32)
    t = torch.from_numpy(xs).to(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(mx.e4m3_round(xs.astype(np.float64)), t)


def test_saturation_and_signs():
    assert np.array_equal(mx.e4m3_round([500.0, -1e30, 463.9, -0.0]), [448.0, -448.0, 448.0, -0.0])
    assert math.copysign(1.0, mx.e4m3_round([-1e-9])[0]) < 0  # negative values that round to 0 keep the sign


def _golden_blocks():
    blocks = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("block"):
            _, name, byte = line.split()
            blocks.append((name, int(byte), []))
        else:
            a, b = line.split()
            blocks[-1][2].append((float(a), float(b)))
    return blocks


def test_handworked_blocks():
    for name, byte, pairs in _golden_blocks():
        v = np.array([a for a, _ in pairs] or [0.0] * 32)
        want = np.array([b for _, b in pairs] or [0.0] * 32)
        elems, sb = mx.quantize_mxfp8(v[None])
        assert int(sb[0, 0]) == byte, name
        assert np.array_equal(mx.dequant_mxfp8(elems, sb)[0], want), name


def test_block_scale_rule():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((64, 256)) * np.exp2(rng.integers(-20, 20, size=(64, 1)))
    elems, sb = mx.quantize_mxfp8(v)
    amax = np.abs(v.reshape(64, 8, 32)).max(-1)
    X = sb.astype(np.int64) - 127
    r = amax / np.exp2(X)
    assert np.all((r >= 256) & (r < 512))  # the largest element lands in [256, 512) before saturation
    # elements are E4M3 values; the round trip is within half a quantum or saturated
    e4 = mx.e4m3_values()
    assert np.all(np.isin(elems, e4[np.isfinite(e4)]))
    back = mx.dequant_mxfp8(elems, sb)
    err = np.abs(back - v) / np.repeat(np.exp2(X), 32, axis=-1)
    assert np.all((err <= 16.0) | (np.abs(v) / np.repeat(np.exp2(X), 32, axis=-1) > 448))


def test_layer_act_mxfp8_against_loops():
    rng = np.random.default_rng(3)
    E, H, I, T, k = 3, 64, 64, 3, 2
    wgu = (rng.standard_normal((E, 2 * I, H)) * 0.2).astype(np.float32)
    wd = (rng.standard_normal((E, H, I)) * 0.2).astype(np.float32)
    gc, gs = oracle.quantize_pack_mxfp4(wgu)
    dc, ds = oracle.quantize_pack_mxfp4(wd)
    x = oracle.bf16_round(rng.standard_normal((T, H)))
    ids = np.array([[0, 2], [1, 1], [2, 0]], np.int32)
    gates = rng.random((T, k)).astype(np.float32)
    y = oracle.moe_forward_ref("mxfp4", x, ids, gates, gc, gs, dc, ds, E, H, I, act_quant="mxfp8")
    Wgu = oracle.dequant_mxfp4(gc, gs).reshape(E, 2 * I, H).astype(np.float64).tolist()
    Wd = oracle.dequant_mxfp4(dc, ds).reshape(E, H, I).astype(np.float64).tolist()
    yl = brute.moe_loops_mxfp8(x.tolist(), ids.tolist(), gates.tolist(), Wgu, Wd, I)
    assert np.array_equal(y, oracle.bf16_round(np.array(yl)))
    # and the reading differs from the bf16 layer (a planted omission of the
    # activation rounding would pass unnoticed otherwise)
    y0 = oracle.moe_forward_ref("mxfp4", x, ids, gates, gc, gs, dc, ds, E, H, I)
    assert not np.array_equal(y, y0)
