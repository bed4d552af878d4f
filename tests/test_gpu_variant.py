"""The expert variant ("experts4bit-qlora" README, Scope: gpt-oss MXFP4 experts
with per-expert biases and a clamped GLU) on the GPU against the oracle:
interleaved gate/up rows, both biases, the clamped GLU, on every kernel path
and both formats; the standalone grouped GEMM's epilogues with a bias; and the
gpt-oss-shaped MXFP4 layer at full size on sampled tokens."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from oracle import fast
from bit_grouped_moe_e4b_b200 import e4b, synth
from bit_grouped_moe_e4b_b200.configs import MXFP4
from gpu_util import assert_close, last_nf4_decode, run_layer, small_layer

pytestmark = pytest.mark.gpu

PATHS = {"gemv": e4b.FLAG_FORCE_GEMV, "tcgen05": e4b.FLAG_FORCE_TCGEN05,
         "tcgen05_gather": e4b.FLAG_FORCE_TCGEN05,
         "tcgen05_1sm": e4b.FLAG_FORCE_TCGEN05 | e4b.FLAG_TC_SINGLE_SM}
ALPHA, LIMIT = 1.702, 7.0


def _biases(E, H, I, seed, gu_std=4.0, dn_std=0.5):
    # gate_up biases large enough that the clamp at 7 decides a good share of
    # the gate and up values
    rng = np.random.default_rng(seed)
    bgu = (rng.standard_normal((E, 2 * I)) * gu_std).astype(np.float32)
    bd = (rng.standard_normal((E, H)) * dn_std).astype(np.float32)
    return bgu, bd


def _variant_layer(layer, layout, act, bgu, bd):
    return dataclasses.replace(layer, layout=layout, act=act, alpha=ALPHA, limit=LIMIT,
                               gate_up_bias=None if bgu is None else torch.from_numpy(bgu).cuda(),
                               down_bias=None if bd is None else torch.from_numpy(bd).cuda())


def _x(T, H, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16)


SHAPES = [
    ("mxfp4", 3, 256, 320, 300, 2),   # I tail (320 = 2.5 x 128), ~200 rows / expert
    ("nf4", 4, 320, 192, 60, 2),      # I tail (1.5 x 128), few rows per expert
    ("mxfp4", 2, 96, 160, 9, 2),      # K % 64 == 32 on gate_up, top_k = E
]


@pytest.mark.parametrize("path", ["gemv", "tcgen05", "tcgen05_gather", "tcgen05_1sm"])
@pytest.mark.parametrize("layout", ["halves", "interleaved"])
@pytest.mark.parametrize("fmt,E,H,I,T,k", SHAPES)
def test_clamped_glu_with_biases(fmt, E, H, I, T, k, layout, path):
    layer, ref = small_layer(fmt, E, H, I, seed=E * 10 + I, std=0.05)
    bgu, bd = _biases(E, H, I, seed=I)
    assert (np.abs(bgu) > LIMIT).mean() > 0.05
    vl = _variant_layer(layer, layout, "clamped_glu", bgu, bd)
    x = _x(T, H, seed=T)
    ids, gates = synth.random_ids(np.random.default_rng(T + k), T, k, E)
    y, status, _ = run_layer(vl, x, ids, gates, PATHS[path], staged=path != "tcgen05_gather")
    assert status == 0
    y_ref = oracle.moe_forward_ref(fmt, x.float().numpy(), ids, gates, *ref, E, H, I, layout=layout,
                                   act="clamped_glu", alpha=ALPHA, limit=LIMIT, gu_bias=bgu, dn_bias=bd,
                                   nf4_decode=last_nf4_decode())
    assert_close(y, y_ref, f"{fmt} {layout} {path}")


@pytest.mark.parametrize("path", ["gemv", "tcgen05", "tcgen05_1sm"])
@pytest.mark.parametrize("which", ["interleaved_swiglu", "halves_biases_only", "down_bias_only"])
def test_variant_parts(which, path):
    # each part of the variant alone: the interleaved rows with the plain
    # SwiGLU, the biases with the plain layer, the down bias alone
    fmt, E, H, I, T, k = "nf4", 3, 256, 192, 48, 2
    layer, ref = small_layer(fmt, E, H, I, seed=7, std=0.05)
    bgu, bd = _biases(E, H, I, seed=8, gu_std=1.0)
    layout, gb, db = {"interleaved_swiglu": ("interleaved", None, None),
                      "halves_biases_only": ("halves", bgu, bd),
                      "down_bias_only": ("halves", None, bd)}[which]
    vl = _variant_layer(layer, layout, "swiglu", gb, db)
    x = _x(T, H, seed=9)
    ids, gates = synth.random_ids(np.random.default_rng(10), T, k, E)
    y, status, _ = run_layer(vl, x, ids, gates, PATHS[path])
    assert status == 0
    y_ref = oracle.moe_forward_ref(fmt, x.float().numpy(), ids, gates, *ref, E, H, I, layout=layout,
                                   act="swiglu", gu_bias=gb, dn_bias=db, nf4_decode=last_nf4_decode())
    assert_close(y, y_ref, f"{which} {path}")


def test_down_bias_counted_once_across_k_slices():
    # I = 4608 > 2048: the small-M kernel splits the down projection into
    # three K slices; the down bias must join exactly one of them
    fmt, E, H, I, T, k = "mxfp4", 2, 128, 4608, 6, 2
    layer, ref = small_layer(fmt, E, H, I, seed=11, std=0.02)
    bd = (np.random.default_rng(12).standard_normal((E, H)) * 2.0).astype(np.float32)
    vl = _variant_layer(layer, "halves", "swiglu", None, bd)
    x = _x(T, H, seed=13)
    ids, gates = synth.random_ids(np.random.default_rng(14), T, k, E)
    for path in ("gemv", "tcgen05"):
        y, status, _ = run_layer(vl, x, ids, gates, PATHS[path])
        assert status == 0
        y_ref = oracle.moe_forward_ref(fmt, x.float().numpy(), ids, gates, *ref, E, H, I, dn_bias=bd,
                                       nf4_decode=last_nf4_decode())
        assert_close(y, y_ref, f"down bias, K split, {path}")


def test_invalid_variant_arguments():
    fmt, E, H, I = "nf4", 2, 64, 64
    layer, _ = small_layer(fmt, E, H, I, seed=15)
    x = _x(4, H, seed=16)
    ids, gates = synth.random_ids(np.random.default_rng(17), 4, 1, E)
    for bad in (dict(layout="halves", act="clamped_glu", limit=-1.0),
                dict(layout="halves", act="clamped_glu", limit=float("nan"))):
        vl = dataclasses.replace(layer, **bad)
        with pytest.raises(RuntimeError, match="E4B_ERR_INVALID_ARG"):
            run_layer(vl, x, ids, gates)
    # a bias that is not 16-byte aligned
    b = torch.zeros(E * 2 * I + 1, dtype=torch.float32, device="cuda")[1:].view(E, 2 * I)
    vl = dataclasses.replace(layer, gate_up_bias=b)
    with pytest.raises(RuntimeError, match="E4B_ERR_MISALIGNED"):
        run_layer(vl, x, ids, gates)


@pytest.mark.parametrize("flags", [e4b.FLAG_FORCE_GEMV, e4b.FLAG_FORCE_TCGEN05,
                                   e4b.FLAG_FORCE_TCGEN05 | e4b.FLAG_TC_SINGLE_SM])
@pytest.mark.parametrize("layout", ["halves", "interleaved"])
def test_grouped_gemm_gated_epilogue(layout, flags):
    # e4b_grouped_gemm alone: the gate_up projection with biases and the
    # clamped GLU, against decode -> fp64 matmul -> bias -> activation
    fmt, E, I, K = "mxfp4", 3, 144, 224
    N = 2 * I
    rng = np.random.default_rng(20)
    w = (rng.standard_normal((E, N, K)) * 0.06).astype(np.float32)
    codes, scales = e4b.quantize(fmt, torch.from_numpy(w).cuda())
    rc, rs = oracle.quantize_pack_mxfp4(w)
    assert np.array_equal(codes.cpu().numpy(), rc)
    counts = np.array([70, 0, 301])
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    R = int(offsets[-1])
    a = torch.from_numpy(rng.standard_normal((R, K)).astype(np.float32)).to(torch.bfloat16)
    bias = (rng.standard_normal((E, N)) * 4.0).astype(np.float32)
    wdec = oracle.dequant_mxfp4(rc, rs).astype(np.float64)
    want = []
    for e in range(E):
        GU = a[offsets[e]:offsets[e + 1]].double().numpy() @ wdec[e].T + bias[e].astype(np.float64)
        G, U = oracle.split_gate_up(GU, layout)
        want.append(oracle.activation_ref(G, U, "clamped_glu", ALPHA, LIMIT))
    want = oracle.bf16_round(np.concatenate(want))
    out = torch.empty((R, I), dtype=torch.bfloat16, device="cuda")
    e4b.e4b_grouped_gemm(fmt, e4b.E4B_EPI_SWIGLU, codes, scales, a.cuda(), torch.from_numpy(offsets).cuda(),
                         out, E=E, N=N, K=K, R_max=R, flags=flags, layout=layout, act="clamped_glu",
                         alpha=ALPHA, limit=LIMIT, bias=torch.from_numpy(bias).cuda())
    torch.cuda.synchronize()
    assert_close(out.float().cpu().numpy(), want, f"gated epilogue {layout} flags={flags}")


@pytest.mark.parametrize("flags", [e4b.FLAG_FORCE_GEMV, e4b.FLAG_FORCE_TCGEN05,
                                   e4b.FLAG_FORCE_TCGEN05 | e4b.FLAG_TC_SINGLE_SM])
def test_grouped_gemm_store_and_combine_bias(flags):
    fmt, E, N, K = "nf4", 2, 96, 192
    rng = np.random.default_rng(21)
    w = (rng.standard_normal((E, N, K)) * 0.05).astype(np.float32)
    codes, scales = e4b.quantize(fmt, torch.from_numpy(w).cuda())
    rc, rs = oracle.quantize_pack_nf4(w)
    wdec = np.stack([oracle.dequant_ref(rc[e], rs[e], N, K) for e in range(E)]).astype(np.float64)
    T, k = 40, 2
    ids, gates = synth.random_ids(rng, T, k, E)
    perm, offsets = _route_host(ids, E)
    R = T * k
    a = torch.from_numpy(rng.standard_normal((R, K)).astype(np.float32)).to(torch.bfloat16)
    bias = rng.standard_normal((E, N)).astype(np.float32)
    O = np.concatenate([a[offsets[e]:offsets[e + 1]].double().numpy() @ wdec[e].T + bias[e] for e in range(E)])
    out = torch.empty((R, N), dtype=torch.bfloat16, device="cuda")
    off_d = torch.from_numpy(offsets).cuda()
    b_d = torch.from_numpy(bias).cuda()
    e4b.e4b_grouped_gemm(fmt, e4b.E4B_EPI_STORE, codes, scales, a.cuda(), off_d, out, E=E, N=N, K=K,
                         R_max=R, flags=flags, bias=b_d)
    torch.cuda.synchronize()
    assert_close(out.float().cpu().numpy(), oracle.bf16_round(O), f"store bias flags={flags}")
    # combine: y[t] = sum over the token's slots of gate * (a_p W^T + b)
    acc = torch.zeros((T, N), dtype=torch.float32, device="cuda")
    e4b.e4b_grouped_gemm(fmt, e4b.E4B_EPI_COMBINE, codes, scales, a.cuda(), off_d, acc, E=E, N=N, K=K,
                         R_max=R, top_k=k, out_row_slot=torch.from_numpy(perm).cuda(),
                         gates=torch.from_numpy(gates.reshape(-1)).cuda(), flags=flags, bias=b_d)
    torch.cuda.synchronize()
    y = np.zeros((T, N))
    for p in range(R):
        s = int(perm[p])
        y[s // k] += np.float64(gates.reshape(-1)[s]) * O[p]
    assert_close(acc.cpu().numpy(), y, f"combine bias flags={flags}")


def _route_host(ids, E):
    # expert-contiguous slots, slot order inside an expert (a valid routing)
    flat = ids.reshape(-1)
    perm = np.concatenate([np.nonzero(flat == e)[0] for e in range(E)]).astype(np.int32)
    counts = np.bincount(flat, minlength=E)
    return perm, np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


_full = {}


@pytest.mark.parametrize("T", [16, 512])
def test_gpt_oss_shaped_mxfp4_layer_full_size(T):
    # the MXFP4 layer (E=32, H=I=2880, top-4) as the variant: interleaved
    # gate/up, both biases, clamped GLU; T=16 runs the small-M kernel, T=512
    # the tcgen05 one; sampled tokens against the oracle
    fast.build()
    wl = MXFP4
    if not _full:
        packed = []
        for which in ("gate_up", "down"):
            w = synth.layer_weights(wl, which, "cuda")
            packed += list(e4b.quantize(wl.fmt, w))
            del w
        bgu, bd = _biases(wl.E, wl.H, wl.I, seed=2880, gu_std=3.0, dn_std=0.5)
        _full["layer"] = e4b.PackedLayer(wl.fmt, wl.E, wl.H, wl.I, *packed)
        _full["b"] = (bgu, bd)
    bgu, bd = _full["b"]
    layer = _variant_layer(_full["layer"], "interleaved", "clamped_glu", bgu, bd)
    x = synth.tokens_bf16(wl, T)
    ids, gates = synth.routing(wl, T)
    ws = e4b.workspace(layer, T, wl.top_k)
    y = e4b.moe_forward(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(gates).cuda(), ws=ws)
    assert e4b.e4b_read_device_status(ws) == 0
    assert e4b.e4b_last_path() == (e4b.E4B_PATH_GEMV if T == 16 else e4b.E4B_PATH_TCGEN05)
    tokens = sorted({0, T // 2, T - 1})
    variant = dict(layout="interleaved", act="clamped_glu", alpha=ALPHA, limit=LIMIT, gu_bias=bgu, dn_bias=bd)
    # the oracle quantises the experts it needs from the same fp32 weights;
    # its codes must equal the GPU's bit for bit
    weight_fn = lambda which, e: synth.expert_weight(wl, which, e, "cuda").cpu().numpy()
    y_ref, _, packed = fast.moe_forward_sampled(wl.fmt, x.float().numpy(), ids, gates, weight_fn, wl.E, wl.H,
                                                wl.I, tokens, variant=variant)
    for (which, e), (c, sc) in packed.items():
        gc = layer.gate_up_codes if which == "gate_up" else layer.down_codes
        gs = layer.gate_up_scales if which == "gate_up" else layer.down_scales
        assert np.array_equal(gc[e].cpu().numpy(), c) and np.array_equal(gs[e].cpu().numpy(), sc), (which, e)
    assert_close(y.float().cpu().numpy()[tokens], y_ref, f"gpt-oss-shaped T={T}")
