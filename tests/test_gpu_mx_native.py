"""MXFP4 on the block-scaled FP4 tensor-core MMA: the prepared stacks (bit
for bit), the MXFP8 activation quantiser (bit for bit against the oracle),
and the layer on that path against the oracle in both activation readings:
the default two-term split against the plain (bf16-activation) layer, and
E4B_FLAG_MX_ACT_E4M3 against the oracle's act_mxfp8 reading."""

import numpy as np
import pytest
import torch

import oracle
from oracle import fast
from oracle import mxfp8 as mx
from bit_grouped_moe_e4b_b200 import e4b, synth
from bit_grouped_moe_e4b_b200.configs import MXFP4
from gpu_util import LAYER_MIN_RMS, TOL, assert_close, small_layer

pytestmark = pytest.mark.gpu


def _row_of(layout, Nm, m, n):
    return 2 * n + m if layout == "interleaved" else m * Nm + n


@pytest.mark.parametrize("nmat,layout", [(1, "halves"), (2, "halves"), (2, "interleaved")])
def test_prepared_stack_layout(nmat, layout):
    rng = np.random.default_rng(nmat * 7 + len(layout))
    E, Nm, K = 3, 200, 160  # neither a multiple of 128
    w = (rng.standard_normal((E, nmat * Nm, K)) * np.exp2(rng.integers(-3, 3, size=(E, nmat * Nm, 1)))
         ).astype(np.float32)
    blocks, scales = e4b.quantize("mxfp4", torch.from_numpy(w).cuda())
    codes_p, sf_p = e4b.mxfp4_native_prepare(blocks, scales, E, Nm, K, nmat, layout)
    torch.cuda.synchronize()
    Np, Kp = 256, 256
    cp = codes_p.cpu().numpy().reshape(E, nmat, Np, Kp // 2)
    sp = sf_p.cpu().numpy().reshape(E, nmat, Np // 128, Kp // 128, 512)
    b = blocks.cpu().numpy().reshape(E, nmat * Nm, K // 2)
    s = scales.cpu().numpy()
    want_c = np.zeros_like(cp)
    want_s = np.zeros_like(sp)
    for e in range(E):
        for m in range(nmat):
            for n in range(Nm):
                row = _row_of(layout, Nm, m, n) if nmat == 2 else n
                want_c[e, m, n, :K // 2] = b[e, row]
                r = n % 128
                for blk in range(K // 32):
                    want_s[e, m, n // 128, blk // 4, (r % 32) * 16 + (r // 32) * 4 + blk % 4] = s[e, row, blk]
    assert np.array_equal(cp, want_c)
    assert np.array_equal(sp, want_s)


def _e4m3_codes(values):
    table = mx.e4m3_values()
    lut = {}
    for code in range(256):
        v = table[code]
        if np.isfinite(v) and (v not in lut or (v == 0 and code == 0)):
            lut[v] = code
    out = np.empty(values.shape, np.uint8)
    flat = values.reshape(-1)
    o = out.reshape(-1)
    for i, v in enumerate(flat):
        o[i] = lut[v] if v != 0 else (0x80 if np.signbit(v) else 0)
    return out


def test_quantize_mxfp8_bit_exact():
    rng = np.random.default_rng(5)
    R, K = 37, 320
    x = rng.standard_normal((R, K)) * np.exp2(rng.integers(-30, 30, size=(R, 1)))
    x[3, 64:96] = 0.0                        # an all-zero block
    x[5, :32] = rng.standard_normal(32) * 1e-39  # tiny values (subnormal in fp32)
    x[7, 0] = 1.999 * 2.0 ** 20              # saturating elements next to it
    xb = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    elems, scales = e4b.quantize_mxfp8(xb.cuda())
    torch.cuda.synchronize()
    want_e, want_s = mx.quantize_mxfp8(xb.float().numpy().astype(np.float64))
    assert np.array_equal(scales.cpu().numpy(), want_s)
    assert np.array_equal(elems.cpu().numpy(), _e4m3_codes(want_e))


def _layer_case(fmt_layer, T, k, seed, skew=0.0):
    rng = np.random.default_rng(seed)
    x = torch.from_numpy(rng.standard_normal((T, fmt_layer.H)).astype(np.float32)).to(torch.bfloat16)
    ids, gates = synth.random_ids(rng, T, k, fmt_layer.E, skew=skew)
    return x, ids, gates


def _run(layer, x, ids, gates, flags):
    ids_d = torch.from_numpy(ids).cuda()
    g_d = torch.from_numpy(gates).cuda()
    ws = e4b.workspace(layer, ids.shape[0], ids.shape[1])
    y = e4b.moe_forward(layer, x.cuda(), ids_d, g_d, ws=ws, flags=flags)
    assert e4b.e4b_read_device_status(ws) == 0
    return y.float().cpu().numpy()


SHAPES = [
    (4, 160, 224, 300, 2),   # K tails on both projections, > 128 rows per expert
    (3, 288, 96, 97, 3),     # odd T, k = 3, one 128-block short K
    (6, 128, 256, 40, 1),    # some experts empty or with one row
]


@pytest.mark.parametrize("E,H,I,T,k", SHAPES)
def test_layer_exact_split_matches_plain_oracle(E, H, I, T, k):
    layer, ref = small_layer("mxfp4", E, H, I, seed=E * 31 + H)
    mxl = layer.prepare_mx()
    x, ids, gates = _layer_case(layer, T, k, seed=T)
    y = _run(mxl, x, ids, gates, e4b.FLAG_FORCE_TCGEN05)
    assert e4b.e4b_last_path() == e4b.E4B_PATH_TCGEN05_MX and e4b.e4b_last_launch_count() == 6
    y_ref = oracle.moe_forward_ref("mxfp4", x.float().numpy(), ids, gates, *ref, E, H, I)
    assert_close(y, y_ref, f"mx exact E={E} H={H} I={I} T={T}", min_rms=LAYER_MIN_RMS)


@pytest.mark.parametrize("E,H,I,T,k", SHAPES)
def test_layer_one_term_matches_act_mxfp8_oracle(E, H, I, T, k):
    layer, ref = small_layer("mxfp4", E, H, I, seed=E * 31 + H)
    mxl = layer.prepare_mx()
    x, ids, gates = _layer_case(layer, T, k, seed=T)
    y = _run(mxl, x, ids, gates, e4b.FLAG_FORCE_TCGEN05 | e4b.FLAG_MX_ACT_E4M3)
    assert e4b.e4b_last_path() == e4b.E4B_PATH_TCGEN05_MX
    xf = x.float().numpy()
    y_ref = oracle.moe_forward_ref("mxfp4", xf, ids, gates, *ref, E, H, I, act_quant="mxfp8")
    assert_close(y, y_ref, f"mx e4m3 E={E} H={H} I={I} T={T}", min_rms=LAYER_MIN_RMS)
    # the two activation readings are distinguishable on this data
    y_plain = oracle.moe_forward_ref("mxfp4", xf, ids, gates, *ref, E, H, I)
    assert np.max(np.abs(y_ref - y_plain)) > 0


def test_layer_variant_on_the_block_scaled_path():
    # interleaved gate/up rows, both biases, the clamped GLU
    E, H, I, T, k = 4, 192, 160, 150, 2
    layer, ref = small_layer("mxfp4", E, H, I, seed=17)
    rng = np.random.default_rng(18)
    gub = (rng.standard_normal((E, 2 * I)) * 0.5).astype(np.float32)
    dnb = (rng.standard_normal((E, H)) * 0.5).astype(np.float32)
    wgu = oracle.dequant_mxfp4(ref[0], ref[1])  # only to keep the layer's own weights
    del wgu
    import dataclasses
    # re-layout the same weights as interleaved rows
    g, u = ref[0][:, :I], ref[0][:, I:]
    gi = np.empty_like(ref[0]); gi[:, 0::2] = g; gi[:, 1::2] = u
    si = np.empty_like(ref[1]); si[:, 0::2] = ref[1][:, :I]; si[:, 1::2] = ref[1][:, I:]
    lay = dataclasses.replace(layer, gate_up_codes=torch.from_numpy(gi).cuda(), gate_up_scales=torch.from_numpy(si).cuda(),
                              layout="interleaved", act="clamped_glu", alpha=1.702, limit=7.0,
                              gate_up_bias=torch.from_numpy(gub).cuda(), down_bias=torch.from_numpy(dnb).cuda())
    mxl = lay.prepare_mx()
    x, ids, gates = _layer_case(layer, T, k, seed=19)
    y = _run(mxl, x, ids, gates, e4b.FLAG_FORCE_TCGEN05)
    assert e4b.e4b_last_path() == e4b.E4B_PATH_TCGEN05_MX
    y_ref = oracle.moe_forward_ref("mxfp4", x.float().numpy(), ids, gates, gi, si, ref[2], ref[3], E, H, I,
                                   layout="interleaved", act="clamped_glu", alpha=1.702, limit=7.0,
                                   gu_bias=gub, dn_bias=dnb)
    assert_close(y, y_ref, "mx variant", min_rms=LAYER_MIN_RMS)


def test_block_scaled_path_is_deterministic_and_decode_flag_switches_back():
    E, H, I, T, k = 8, 256, 256, 256, 4
    layer, ref = small_layer("mxfp4", E, H, I, seed=23)
    mxl = layer.prepare_mx()
    x, ids, gates = _layer_case(layer, T, k, seed=24)
    y0 = _run(mxl, x, ids, gates, e4b.FLAG_FORCE_TCGEN05)
    y1 = _run(mxl, x, ids, gates, e4b.FLAG_FORCE_TCGEN05)
    assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))
    yd = _run(mxl, x, ids, gates, e4b.FLAG_FORCE_TCGEN05 | e4b.FLAG_MX_DECODE)
    assert e4b.e4b_last_path() == e4b.E4B_PATH_TCGEN05
    y_ref = oracle.moe_forward_ref("mxfp4", x.float().numpy(), ids, gates, *ref, E, H, I)
    assert_close(y0, y_ref, "mx", min_rms=LAYER_MIN_RMS)
    assert_close(yd, y_ref, "decode path", min_rms=LAYER_MIN_RMS)


_full = {}


@pytest.mark.parametrize("T", [512, 8192])
@pytest.mark.parametrize("one_term", [False, True])
def test_mxfp4_workload_full_size(T, one_term):
    wl = MXFP4
    if "layer" not in _full:
        packed = []
        for which in ("gate_up", "down"):
            packed += list(e4b.quantize("mxfp4", synth.layer_weights(wl, which, "cuda")))
        _full["layer"] = e4b.PackedLayer("mxfp4", wl.E, wl.H, wl.I, *packed).prepare_mx()
    layer = _full["layer"]
    x = synth.tokens_bf16(wl, T)
    ids, gates = synth.routing(wl, T)
    flags = e4b.FLAG_MX_ACT_E4M3 if one_term else 0
    y = _run(layer, x, ids, gates, flags)
    assert e4b.e4b_last_path() == e4b.E4B_PATH_TCGEN05_MX
    rng = np.random.default_rng(T)
    tokens = sorted({0, T - 1} | set(int(t) for t in rng.integers(0, T, 30)))
    packed_fn = lambda which, e: (
        (layer.gate_up_codes if which == "gate_up" else layer.down_codes)[e].cpu().numpy(),
        (layer.gate_up_scales if which == "gate_up" else layer.down_scales)[e].cpu().numpy())
    y_ref, _, _ = fast.moe_forward_sampled("mxfp4", x.float().numpy(), ids, gates, None, wl.E, wl.H, wl.I, tokens,
                                           packed_fn=packed_fn, act_quant="mxfp8" if one_term else None)
    assert_close(y[tokens], y_ref, f"mxfp4 T={T} one_term={one_term}", min_rms=0.05)
