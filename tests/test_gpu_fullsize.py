"""The five workloads at full size, in the launch configuration the bench
times (path chosen from the shape), plus the other kernel path: sampled
tokens checked against the oracle, which quantises the experts those tokens
use from the same fp32 weights and compares its codes with the GPU's bit for
bit. The sample holds at least 32 tokens and covers every active expert's
first and last routed row and the rows on both sides of each 256-row tile
boundary of the large-M kernel."""

import numpy as np
import pytest
import torch

from oracle import fast
from bit_grouped_moe_e4b_b200 import e4b, synth
from bit_grouped_moe_e4b_b200.configs import WORKLOADS
from gpu_util import TOL, TOL_NF4_ACROSS_PATHS, assert_close

pytestmark = pytest.mark.gpu

_layers = {}


def _layer(wl):
    if wl.layer not in _layers:
        _layers.clear()
        torch.cuda.empty_cache()
        packed = []
        for which in ("gate_up", "down"):
            w = synth.layer_weights(wl, which, "cuda")
            packed += list(e4b.quantize(wl.fmt, w))
            del w
        _layers[wl.layer] = e4b.PackedLayer(wl.fmt, wl.E, wl.H, wl.I, *packed)
    return _layers[wl.layer]


CASES = [(name, T) for name, wl in WORKLOADS.items() for T in wl.T]

TILE_ROWS = 256  # routed rows per tile of the large-M kernel


def sample_tokens(ids, E, n_min=32, seed=0):
    """Tokens whose routed rows include, for every active expert, its first
    and last row in expert order and the two rows on each side of every
    TILE_ROWS boundary inside it; then tokens 0, T/2 and T-1, and random
    tokens up to n_min (all tokens when T <= n_min)."""
    T, k = ids.shape
    flat = ids.ravel()
    perm = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    off = np.concatenate([[0], np.cumsum(counts)])
    rows = set()
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if b == a:
            continue
        rows.update((a, b - 1))
        for j in range(TILE_ROWS, b - a, TILE_ROWS):
            rows.update((a + j - 1, a + j))
    tokens = {int(perm[p]) // k for p in rows} | {0, T // 2, T - 1}
    if T <= n_min:
        return list(range(T))
    rng = np.random.default_rng(seed)
    while len(tokens) < n_min:
        tokens.add(int(rng.integers(T)))
    return sorted(tokens)


@pytest.mark.parametrize("name,T", CASES)
def test_workload_sampled_tokens(name, T):
    fast.build()
    wl = WORKLOADS[name]
    layer = _layer(wl)
    x = synth.tokens_bf16(wl, T)
    ids, gates = synth.routing(wl, T)
    ids_d = torch.from_numpy(ids).cuda()
    g_d = torch.from_numpy(gates).cuda()
    x_d = x.cuda()
    ws = e4b.workspace(layer, T, wl.top_k)
    y_auto = e4b.moe_forward(layer, x_d, ids_d, g_d, ws=ws)
    assert e4b.e4b_read_device_status(ws) == 0
    auto_path = e4b.e4b_last_path()
    other = e4b.FLAG_FORCE_TCGEN05 if auto_path == e4b.E4B_PATH_GEMV else e4b.FLAG_FORCE_GEMV
    y_other = e4b.moe_forward(layer, x_d, ids_d, g_d, ws=ws, flags=other)
    assert e4b.e4b_read_device_status(ws) == 0

    tokens = sample_tokens(ids, wl.E, seed=T)
    assert len(tokens) >= min(32, T)
    weight_fn = lambda which, e: synth.expert_weight(wl, which, e, "cuda").cpu().numpy()
    # NF4: the small-M path takes the "level" reading, tcgen05 the "product" one
    mode = {e4b.E4B_PATH_GEMV: "level", e4b.E4B_PATH_TCGEN05: "product"}
    auto_mode = mode[auto_path]
    other_mode = mode[e4b.E4B_PATH_TCGEN05 if auto_path == e4b.E4B_PATH_GEMV else e4b.E4B_PATH_GEMV]
    y_ref, cols, packed = fast.moe_forward_sampled(wl.fmt, x.float().numpy(), ids, gates, weight_fn,
                                                  wl.E, wl.H, wl.I, tokens, nf4_decode=auto_mode)
    for (which, e), (c, s) in packed.items():
        gc = layer.gate_up_codes if which == "gate_up" else layer.down_codes
        gs = layer.gate_up_scales if which == "gate_up" else layer.down_scales
        assert np.array_equal(gc[e].cpu().numpy(), c), (which, e)
        assert np.array_equal(gs[e].cpu().numpy().view(np.uint8), s.view(np.uint8)), (which, e)
    y_ref_other = y_ref
    if wl.fmt == "nf4" and other_mode != auto_mode:
        y_ref_other, _, _ = fast.moe_forward_sampled(wl.fmt, x.float().numpy(), ids, gates, None, wl.E, wl.H,
                                                     wl.I, tokens, packed_fn=lambda which, e: packed[(which, e)],
                                                     nf4_decode=other_mode)
    for y, ref, what in ((y_auto, y_ref, "auto"), (y_other, y_ref_other, "other path")):
        got = y.float().cpu().numpy()[tokens]
        # the workloads' N(0, 0.02) weights give output rms from ~0.02 (the
        # tiny layer) to ~2; the tolerance is relative to that scale, and the
        # guard only rules out a degenerate (all-zero) reference
        assert_close(got, ref, f"{name} T={T} {what}", min_rms=0.005)
    # rows not sampled: finite and equal across the two kernel paths within
    # tolerance (for NF4 the paths' readings differ by one bf16 rounding per
    # weight, far inside it on these N(0, 0.02) weights)
    assert torch.isfinite(y_auto.float()).all()
    assert_close(y_other.float().cpu().numpy(), y_auto.float().cpu().numpy(), f"{name} T={T} paths",
                 tol=TOL_NF4_ACROSS_PATHS if wl.fmt == "nf4" else TOL)
