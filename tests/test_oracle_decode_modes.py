"""Pins of the oracle's two NF4 decode readings ("grouped-nf4-gemm" README,
intro: table decode to fp32, blockwise scale; the tensor cores take bf16
operands, so one bf16 rounding has to fall somewhere):
  "product"  bf16_rne(fp32(level * absmax))      (dequant_ref)
  "level"    bf16_rne(level) * absmax, exactly    (dequant_ref_level)
Both must lie within one bf16 rounding (2^-8 relative) of level * absmax,
agree exactly when absmax is a power of two, and the layer forward in the
"level" reading must be the per-block sum of bf16 levels times absmax."""

import numpy as np
import pytest

import oracle
from oracle import fast
from bit_grouped_moe_e4b_b200 import synth


def _packed(seed, N=64, K=256, std=0.05, pow2=False):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((N, K)) * std).astype(np.float32)
    codes, absmax = oracle.quantize_pack_nf4(w)
    if pow2:
        absmax = np.exp2(rng.integers(-6, 4, size=absmax.shape)).astype(np.float32)
    return codes, absmax


def test_level_equals_product_when_absmax_is_a_power_of_two():
    # bf16 rounding commutes with scaling by 2^k (no overflow or subnormals here)
    codes, absmax = _packed(1, pow2=True)
    lv = oracle.dequant_ref_level(codes, absmax, 64, 256)
    pr = oracle.dequant_ref(codes, absmax, 64, 256).astype(np.float64)
    assert np.array_equal(lv, pr)


def test_level_operands_are_bf16_rounded_levels():
    codes, absmax = _packed(2)
    lv = oracle.dequant_ref_level(codes, absmax, 64, 256)
    a = np.repeat(absmax.astype(np.float64), 64, axis=-1)
    operand = lv / a  # exact: the product of a bf16 value and a float32 is exact in float64
    allowed = oracle.bf16_round(oracle.nf4_codebook()).astype(np.float64)
    assert np.all(np.isin(operand, allowed))
    # and the operand is the rounded level of the stored code
    c = oracle.unpack_nf4_codes(codes)
    assert np.array_equal(operand, allowed[c])


@pytest.mark.parametrize("mode", ["level", "product"])
def test_both_readings_within_one_bf16_rounding_of_the_exact_product(mode):
    codes, absmax = _packed(3)
    exact = oracle.dequant_ref_exact(codes, absmax, 64, 256)
    dec = (oracle.dequant_ref_level(codes, absmax, 64, 256) if mode == "level"
           else oracle.dequant_ref(codes, absmax, 64, 256).astype(np.float64))
    bound = 2.0 ** -8 * np.abs(exact) * (1 + 2.0 ** -20)  # + the product's own fp32 rounding
    assert np.all(np.abs(dec - exact) <= bound)
    # zero levels stay zero
    assert np.all(dec[exact == 0] == 0)


def test_readings_differ_somewhere():
    # the two readings are distinct (otherwise one of the pins above is vacuous)
    codes, absmax = _packed(4)
    lv = oracle.dequant_ref_level(codes, absmax, 64, 256)
    pr = oracle.dequant_ref(codes, absmax, 64, 256).astype(np.float64)
    assert np.mean(lv != pr) > 0.05


def test_layer_level_reading_is_the_blockwise_sum():
    # y by explicit loops: per routed slot, per output row, per 64-block:
    # absmax * sum(bf16(level) * x), then the bf16 activation, the down
    # projection the same way, the gate-weighted combine and one bf16 rounding
    E, H, I, T, k = 2, 128, 64, 3, 2
    rng = np.random.default_rng(5)
    wgu = (rng.standard_normal((E, 2 * I, H)) * 0.05).astype(np.float32)
    wd = (rng.standard_normal((E, H, I)) * 0.05).astype(np.float32)
    gc, gs = oracle.quantize_pack_nf4(wgu)
    dc, ds = oracle.quantize_pack_nf4(wd)
    x = oracle.bf16_round(rng.standard_normal((T, H)))
    ids, gates = synth.random_ids(rng, T, k, E)
    lv = [float(v) for v in oracle.bf16_round(oracle.nf4_codebook())]

    def proj(codes, absmax, rows, K, v):
        c = oracle.unpack_nf4_codes(codes)
        out = []
        for r in range(rows):
            acc = 0.0
            for b in range(K // 64):
                part = 0.0
                for kk in range(64 * b, 64 * b + 64):
                    part += lv[c[r, kk]] * float(v[kk])
                acc += float(absmax[r, b]) * part
            out.append(acc)
        return np.array(out)

    y = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            gu = proj(gc[e], gs[e], 2 * I, H, x[t])
            g, u = gu[:I], gu[I:]
            h = oracle.bf16_round(g / (1 + np.exp(-g)) * u)
            y[t] += float(gates[t, j]) * proj(dc[e], ds[e], H, I, h)
    want = oracle.bf16_round(y)
    got = oracle.moe_forward_ref("nf4", x, ids, gates, gc, gs, dc, ds, E, H, I, nf4_decode="level")
    # identical up to the order of the fp64 additions (one bf16 rounding at the end)
    assert np.max(np.abs(got - want) / (1 + np.abs(want))) < 2.0 ** -7


def test_c_core_level_decode_and_sampled_layer_agree():
    fast.build()
    codes, absmax = _packed(6, N=96, K=320)
    assert np.array_equal(fast.decode("nf4", codes, absmax, 96, 320, "level"),
                          oracle.dequant_ref_level(codes, absmax, 96, 320))
    E, H, I, T, k = 3, 128, 128, 5, 2
    rng = np.random.default_rng(7)
    w = {("gate_up", e): (rng.standard_normal((2 * I, H)) * 0.05).astype(np.float32) for e in range(E)}
    w.update({("down", e): (rng.standard_normal((H, I)) * 0.05).astype(np.float32) for e in range(E)})
    x = oracle.bf16_round(rng.standard_normal((T, H)))
    ids, gates = synth.random_ids(rng, T, k, E)
    tokens = [0, 2, 4]
    y_fast, _, _ = fast.moe_forward_sampled("nf4", x, ids, gates, lambda which, e: w[(which, e)], E, H, I,
                                            tokens, nf4_decode="level")
    gc, gs = oracle.quantize_pack_nf4(np.stack([w[("gate_up", e)] for e in range(E)]))
    dc, ds = oracle.quantize_pack_nf4(np.stack([w[("down", e)] for e in range(E)]))
    y_ref = oracle.moe_forward_ref("nf4", x, ids, gates, gc, gs, dc, ds, E, H, I, tokens=tokens,
                                   nf4_decode="level")
    assert np.max(np.abs(y_fast - y_ref) / (1 + np.abs(y_ref))) < 2.0 ** -7
