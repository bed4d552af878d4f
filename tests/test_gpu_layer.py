"""The whole layer on the GPU against the oracle, at sizes the oracle finishes
in seconds: several tiles with ragged tails, both kernel paths, both formats,
and the degenerate routings."""

import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_e4b_b200 import e4b, synth
from bit_grouped_moe_e4b_b200.configs import TINY
from gpu_util import LAYER_MIN_RMS, assert_close, last_nf4_decode, oracle_layer, run_layer, scaled_err, small_layer

pytestmark = pytest.mark.gpu

PATHS = {"gemv": e4b.FLAG_FORCE_GEMV, "tcgen05": e4b.FLAG_FORCE_TCGEN05,
         "tcgen05_gather": e4b.FLAG_FORCE_TCGEN05,
         # the one-SM tcgen05 kernel on staged rows ("tcgen05" runs on SM pairs)
         "tcgen05_1sm": e4b.FLAG_FORCE_TCGEN05 | e4b.FLAG_TC_SINGLE_SM,
         # small-M with the NF4 product decode (the tcgen05 path's operands)
         "gemv_product": e4b.FLAG_FORCE_GEMV | e4b.FLAG_NF4_PRODUCT_DECODE}


def _run(layer, x, ids, gates, path):
    # "tcgen05_gather": a workspace without the staging copy of the routed
    # rows, so the tcgen05 kernel gathers them with four-row TMA copies
    return run_layer(layer, x, ids, gates, PATHS[path], staged=path != "tcgen05_gather")


def _x(T, H, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("path", ["auto", "gemv", "tcgen05"])
def test_tiny_workload(path):
    wl = TINY
    T = wl.T[0]
    wgu = synth.layer_weights(wl, "gate_up", "cuda")
    wd = synth.layer_weights(wl, "down", "cuda")
    gc_d, gs_d = e4b.quantize("nf4", wgu)
    dc_d, ds_d = e4b.quantize("nf4", wd)
    gc, gs = oracle.quantize_pack_nf4(wgu.cpu().numpy())
    dc, ds = oracle.quantize_pack_nf4(wd.cpu().numpy())
    assert np.array_equal(gc_d.cpu().numpy(), gc) and np.array_equal(gs_d.cpu().numpy(), gs)
    assert np.array_equal(dc_d.cpu().numpy(), dc) and np.array_equal(ds_d.cpu().numpy(), ds)
    layer = e4b.PackedLayer("nf4", wl.E, wl.H, wl.I, gc_d, gs_d, dc_d, ds_d)
    x = synth.tokens_bf16(wl, T)
    ids, gates = synth.routing(wl, T)
    y, status, _ = run_layer(layer, x, ids, gates, 0 if path == "auto" else PATHS[path])
    assert status == 0
    y_ref = oracle_layer("nf4", x, ids, gates, (gc, gs, dc, ds), wl.E, wl.H, wl.I)
    assert_close(y, y_ref, f"tiny workload, {path}")
    if path != "auto":
        assert e4b.e4b_last_path() == (e4b.E4B_PATH_GEMV if path == "gemv" else e4b.E4B_PATH_TCGEN05)
    # small-M: routing, the fused layer kernel, the fixed-order combine;
    # tcgen05: routing, staging of the routed rows, two GEMMs, the combine
    assert e4b.e4b_last_launch_count() == (3 if e4b.e4b_last_path() == e4b.E4B_PATH_GEMV else 5)


# shapes that span several tiles of both kernels and leave ragged tails:
# tcgen05 tiles are 128 weight rows x 256 routed rows x 64 K; the small-M
# kernel walks 16 rows x 256 K per warp step.
SHAPES = [
    ("nf4", 3, 256, 320, 300, 2),     # I tail (320 = 2.5 x 128), ~200 rows / expert
    ("nf4", 5, 384, 192, 97, 3),      # odd T, k=3
    ("mxfp4", 4, 96, 160, 70, 2),     # K % 64 == 32 on gate_up
    ("mxfp4", 2, 224, 288, 600, 1),   # > 256 rows on an expert
]


@pytest.mark.parametrize("path", ["gemv", "tcgen05", "tcgen05_gather", "tcgen05_1sm"])
@pytest.mark.parametrize("fmt,E,H,I,T,k", SHAPES)
def test_ragged_shapes(fmt, E, H, I, T, k, path):
    layer, ref = small_layer(fmt, E, H, I, seed=E * 100 + H)
    x = _x(T, H, seed=T)
    rng = np.random.default_rng(T + k)
    ids, gates = synth.random_ids(rng, T, k, E)
    y, status, _ = _run(layer, x, ids, gates, path)
    assert status == 0
    assert_close(y, oracle_layer(fmt, x, ids, gates, ref, E, H, I), f"{fmt} {E}x{H}x{I} T={T} {path}",
                 min_rms=LAYER_MIN_RMS)


_many = {}


@pytest.mark.parametrize("path", ["gemv", "tcgen05", "tcgen05_gather", "tcgen05_1sm"])
def test_many_tiles_per_cta(path):
    # 64 experts x 4 weight-row tiles per projection = 256 tcgen05 tiles, more
    # than one per SM, with 8 k-blocks each: the persistent kernels walk
    # several tiles per CTA and their staging rings wrap many times
    fmt, E, H, I, T, k = "nf4", 64, 512, 512, 256, 4
    if not _many:
        _many["layer"] = small_layer(fmt, E, H, I, seed=64)
        x = _x(T, H, seed=5)
        ids, gates = synth.random_ids(np.random.default_rng(6), T, k, E)
        _many["case"] = (x, ids, gates)
    layer, ref = _many["layer"]
    x, ids, gates = _many["case"]
    y, status, _ = _run(layer, x, ids, gates, path)
    assert status == 0
    key = ("ref", last_nf4_decode())
    if key not in _many:
        _many[key] = oracle_layer(fmt, x, ids, gates, ref, E, H, I)
    assert_close(y, _many[key], f"{fmt} {E}x{H}x{I} T={T} {path}", min_rms=LAYER_MIN_RMS)


@pytest.mark.parametrize("path", ["gemv", "gemv_product", "tcgen05", "tcgen05_1sm"])
@pytest.mark.parametrize("fmt,E,H,I,T,k", [("nf4", 3, 256, 320, 40, 2), ("mxfp4", 3, 288, 224, 40, 2),
                                           ("mxfp4", 2, 96, 160, 9, 1)])
def test_block_scales_and_large_outputs(fmt, E, H, I, T, k, path):
    # outputs of order 1-10 (where the tolerance is effectively relative) and
    # block scales that differ by powers of two between neighbouring 32-blocks
    # along K: a decode that applies one block's scale to another block's
    # weights fails here
    layer, ref = small_layer(fmt, E, H, I, seed=T + H, std=0.06, spread=True)
    x = _x(T, H, seed=2)
    rng = np.random.default_rng(4)
    ids, gates = synth.random_ids(rng, T, k, E)
    y, status, _ = run_layer(layer, x, ids, gates, PATHS[path])
    mode = last_nf4_decode()
    y_ref = oracle_layer(fmt, x, ids, gates, ref, E, H, I)
    assert status == 0 and 3.0 < np.abs(y_ref).max() < 100.0
    assert_close(y, y_ref, f"{fmt} spread {E}x{H}x{I} {path}")
    if fmt == "nf4":
        # the two NF4 readings differ visibly on this data: the kernel follows
        # the reading of its path, not the other one
        other = oracle_layer(fmt, x, ids, gates, ref, E, H, I, nf4_decode="product" if mode == "level" else "level")
        assert scaled_err(y, y_ref) < scaled_err(y, other), (path, mode)


@pytest.mark.parametrize("path", ["gemv", "tcgen05", "tcgen05_1sm"])
def test_mxfp4_special_scale_bytes(path):
    # e8m0 (OCP MX v1.0): byte 255 is NaN and byte 0 is 2^-127. One NaN block
    # in a down row makes exactly that output column NaN for the tokens routed
    # to the expert; one in an up row makes every output of the expert's
    # tokens NaN (through h). Byte-0 blocks stay finite.
    E, H, I, T, k = 3, 288, 224, 40, 2
    layer, (gc, gs, dc, ds) = small_layer("mxfp4", E, H, I, seed=11, std=0.06)
    gs, ds = gs.copy(), ds.copy()
    gs[0, 5, 1] = gs[0, 200, 0] = gs[0, 17, 8] = 0  # gate and up blocks of 2^-127
    ds[0, 100, 6] = 0
    ds[1, 7, 3] = 255  # output column 7 of expert 1
    gs[2, I + 76, 4] = 255  # up row 76 of expert 2
    layer.gate_up_scales.copy_(torch.from_numpy(gs))
    layer.down_scales.copy_(torch.from_numpy(ds))
    x = _x(T, H, seed=5)
    ids, gates = synth.random_ids(np.random.default_rng(6), T, k, E)
    to1, to2 = np.any(ids == 1, axis=1), np.any(ids == 2, axis=1)
    assert to1.any() and to2.any() and not (to1 | to2).all()
    y, status, _ = run_layer(layer, x, ids, gates, PATHS[path])
    y_ref = oracle_layer("mxfp4", x, ids, gates, (gc, gs, dc, ds), E, H, I)
    want_nan = to2[:, None] | (to1[:, None] & (np.arange(H) == 7)[None, :])
    assert status == 0
    assert np.array_equal(np.isnan(y_ref), want_nan)
    assert np.array_equal(np.isnan(y), want_nan), path
    fin = ~want_nan
    assert_close(y[fin], y_ref[fin], f"mxfp4 special scale bytes {path}")


EDGE = {
    "single_slot": (1, 1, lambda T, k, E: np.zeros((1, 1), np.int32)),
    "all_on_one_expert": (300, 2, lambda T, k, E: np.full((T, k), 3, np.int32)),
    "duplicate_slots": (40, 2, lambda T, k, E: np.repeat(np.arange(T, dtype=np.int32)[:, None] % E, k, 1)),
    "k_equals_E": (25, 4, lambda T, k, E: np.tile(np.arange(E, dtype=np.int32), (T, 1))),
    "mostly_empty": (5, 1, lambda T, k, E: np.array([[1], [1], [2], [1], [2]], np.int32)),
}


@pytest.mark.parametrize("path", ["gemv", "tcgen05", "tcgen05_gather", "tcgen05_1sm"])
@pytest.mark.parametrize("case", list(EDGE))
def test_degenerate_routing(case, path):
    E, H, I = 4, 128, 256
    if case == "mostly_empty":
        E = 16
    T, k, make = EDGE[case]
    layer, ref = small_layer("nf4", E, H, I, seed=7)
    x = _x(T, H, seed=3)
    ids = make(T, k, E)
    gates = np.random.default_rng(1).random((T, k)).astype(np.float32)
    y, status, _ = _run(layer, x, ids, gates, path)
    assert status == 0
    assert_close(y, oracle_layer("nf4", x, ids, gates, ref, E, H, I), f"{case} {path}", min_rms=LAYER_MIN_RMS)


@pytest.mark.parametrize("path", ["gemv", "tcgen05", "tcgen05_gather", "tcgen05_1sm"])
def test_bad_expert_ids_drop_only_their_slots(path):
    E, H, I, T = 4, 128, 128, 6
    layer, ref = small_layer("nf4", E, H, I, seed=11)
    x = _x(T, H, seed=5)
    ids = np.array([[0, 1], [9, 2], [3, -4], [1, 1], [2, 0], [3, 3]], np.int32)
    gates = np.random.default_rng(2).random((T, 2)).astype(np.float32)
    y, status, _ = _run(layer, x, ids, gates, path)
    assert status == 6
    g2 = gates.copy()
    ids2 = ids.copy()
    bad = (ids < 0) | (ids >= E)
    g2[bad] = 0.0
    ids2[bad] = 0
    assert_close(y, oracle_layer("nf4", x, ids2, g2, ref, E, H, I), "bad ids", min_rms=LAYER_MIN_RMS)


@pytest.mark.parametrize("path", ["gemv", "tcgen05", "tcgen05_1sm"])
def test_bounded_wait_reports_timeout_and_returns(path):
    # the test flag makes the kernels' bounded waits give up at once: the
    # kernel must record E4B_ERR_DEVICE_TIMEOUT and return (no hang, no trap)
    E, H, I, T = 2, 128, 128, 40
    layer, ref = small_layer("nf4", E, H, I, seed=12)
    x = _x(T, H, seed=6)
    ids = np.zeros((T, 1), np.int32)
    gates = np.ones((T, 1), np.float32)
    _, status, ws = run_layer(layer, x, ids, gates, PATHS[path] | e4b.FLAG_TEST_TIMEOUT)
    assert status == 5
    # the context is still usable: a normal call right after succeeds
    y, status, _ = run_layer(layer, x, ids, gates, PATHS[path])
    assert status == 0
    assert_close(y, oracle_layer("nf4", x, ids, gates, ref, E, H, I), f"after timeout {path}",
                 min_rms=LAYER_MIN_RMS)


def test_grouped_gemm_store_epilogue():
    # the standalone projection entry point, plain bf16 output
    fmt, E, N, K = "mxfp4", 3, 272, 320
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((E, N, K)) * 0.05).astype(np.float32)
    codes, scales = e4b.quantize(fmt, torch.from_numpy(w).cuda())
    rc, rs = oracle.quantize_pack_mxfp4(w)
    counts = np.array([5, 0, 300])
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    R = int(offsets[-1])
    a = torch.from_numpy(rng.standard_normal((R, K)).astype(np.float32)).to(torch.bfloat16)
    wdec = oracle.dequant_mxfp4(rc, rs).astype(np.float64)
    want = np.concatenate([a[offsets[e]:offsets[e + 1]].double().numpy() @ wdec[e].T for e in range(E)])
    want = oracle.bf16_round(want)
    for flags in (e4b.FLAG_FORCE_GEMV, e4b.FLAG_FORCE_TCGEN05):
        out = torch.empty((R, N), dtype=torch.bfloat16, device="cuda")
        e4b.e4b_grouped_gemm(fmt, e4b.E4B_EPI_STORE, codes, scales, a.cuda(),
                             torch.from_numpy(offsets).cuda(), out, E=E, N=N, K=K, R_max=R,
                             flags=flags)
        torch.cuda.synchronize()
        assert_close(out.float().cpu().numpy(), want, f"store flags={flags}")


@pytest.mark.parametrize("path", ["gemv", "tcgen05", "tcgen05_gather", "tcgen05_1sm"])
def test_combine_is_deterministic(path):
    # every path writes each routed row's output (small-M: each K slice's
    # partial sum) once and sums every token's rows in a fixed order:
    # repeated calls give the same bits
    fmt, E, H, I, T, k = "nf4", 16, 256, 384, 300, 8
    layer, ref = small_layer(fmt, E, H, I, seed=91)
    x = _x(T, H, seed=92)
    ids, gates = synth.random_ids(np.random.default_rng(93), T, k, E)
    y0, status, _ = _run(layer, x, ids, gates, path)
    assert status == 0
    for _ in range(3):
        y1, status, _ = _run(layer, x, ids, gates, path)
        assert status == 0
        assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))
    assert_close(y0, oracle_layer(fmt, x, ids, gates, ref, E, H, I), f"deterministic {path}",
                 min_rms=LAYER_MIN_RMS)
