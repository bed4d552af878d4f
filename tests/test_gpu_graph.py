"""The layer call inside a CUDA graph: e4b_moe_forward chooses its path on the
host with no device synchronisation and launches its kernels as programmatic
dependents, so a captured call replays. Each case captures one call, replays
it, replays it again after new inputs are copied into the same buffers, and
compares both results with eager calls on those inputs (the small-M and int4
combines add in an order that is not fixed, hence a tolerance)."""

import numpy as np
import pytest
import torch

import oracle
from oracle import int4b32 as q4
from bit_grouped_moe_e4b_b200 import e4b, synth
from gpu_util import LAYER_MIN_RMS, assert_close, small_layer

pytestmark = pytest.mark.gpu


def _inputs(rng, T, k, E, H):
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16).cuda()
    ids, gates = synth.random_ids(rng, T, k, E)
    return x, torch.from_numpy(ids).cuda(), torch.from_numpy(gates).cuda()


def _graph_vs_eager(layer, T, k, flags, seed, ref=None):
    """ref: the oracle's packed stacks; each replay is then also checked
    against the oracle's layer in the reading of the path that ran."""
    rng = np.random.default_rng(seed)
    x, ids, gates = _inputs(rng, T, k, layer.E, layer.H)
    ws = e4b.workspace(layer, T, k)
    y = torch.empty((T, layer.H), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # one call outside the capture first
        e4b.e4b_moe_forward(layer, x, ids, gates, y, ws, flags)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        e4b.e4b_moe_forward(layer, x, ids, gates, y, ws, flags)
    path = e4b.e4b_last_path()
    for rep in range(2):
        if rep:
            x2, ids2, gates2 = _inputs(rng, T, k, layer.E, layer.H)
            x.copy_(x2), ids.copy_(ids2), gates.copy_(gates2)
        g.replay()
        torch.cuda.synchronize()
        got = y.float().cpu().numpy()
        want = torch.empty_like(y)
        e4b.e4b_moe_forward(layer, x, ids, gates, want, e4b.workspace(layer, T, k), flags)
        torch.cuda.synchronize()
        assert_close(got, want.float().cpu().numpy(), f"graph replay {rep}", tol=2e-2)
        assert e4b.e4b_read_device_status(ws) == 0
        if ref is not None:
            mode = "level" if path == e4b.E4B_PATH_GEMV else "product"
            y_ref = oracle.moe_forward_ref(layer.fmt, x.float().cpu().numpy(), ids.cpu().numpy(),
                                           gates.cpu().numpy(), *ref, layer.E, layer.H, layer.I, nf4_decode=mode)
            assert_close(got, y_ref, f"graph replay {rep} vs oracle", min_rms=LAYER_MIN_RMS)
    del g
    return path


@pytest.mark.parametrize("flags,path", [(0, e4b.E4B_PATH_GEMV), (e4b.FLAG_FORCE_TCGEN05, e4b.E4B_PATH_TCGEN05)])
def test_nf4_layer_in_a_graph(flags, path):
    layer, ref = small_layer("nf4", 8, 256, 512, seed=31)
    assert _graph_vs_eager(layer, 16, 2, flags, seed=32, ref=ref) == path


def test_int4_layer_in_a_graph():
    rng = np.random.default_rng(33)
    E, H, I = 8, 512, 1024
    wgu = torch.from_numpy((rng.standard_normal((E, 2 * I, H)) * 0.02).astype(np.float32)).cuda()
    wd = torch.from_numpy((rng.standard_normal((E, H, I)) * 0.02).astype(np.float32)).cuda()
    gc, gs = e4b.quantize_int4_b32(wgu)
    dc, ds = e4b.quantize_int4_b32(wd)
    layer = e4b.PackedLayer("int4b32", E, H, I, gc, gs, dc, ds)
    assert _graph_vs_eager(layer, 2, 2, 0, seed=34) == e4b.E4B_PATH_INT4_GEMV
    # and the replayed values are the oracle's
    x = torch.from_numpy(rng.standard_normal((1, H)).astype(np.float32)).to(torch.bfloat16)
    ids = np.array([[4, 1]], np.int32)
    gates = np.array([[0.7, 0.3]], np.float32)
    y = e4b.moe_forward(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(gates).cuda())
    rgc, rgs = q4.quantize_int4b32(wgu.cpu().numpy())
    rdc, rds = q4.quantize_int4b32(wd.cpu().numpy())
    ref = q4.int4b32_decode_layer_ref(x.float().numpy()[0], [4, 1], gates[0], rgc, rgs, rdc, rds)
    assert_close(y[0].float().cpu().numpy(), ref, "int4 layer")
