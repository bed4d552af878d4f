"""The allocation-free layer forward (e4b_moe_forward_noalloc).

Some callers cannot allocate device memory: code that runs while a stream is
captured under a framework that forbids allocation, runtimes whose memory
pool owns all of HBM, plug-in hosts that hand over only input and output
buffers. For them the library keeps the layer's scratch in a fixed 16 MiB
device array. These tests call that entry point through the C ABI and check
it against the workspace-based e4b_moe_forward, twice in a row (the array
keeps the previous call's contents, so the second call checks that nothing
stale leaks in). This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

from bit_grouped_moe_e4b_b200 import e4b, synth
from bit_grouped_moe_e4b_b200.configs import DECODE, TINY
from gpu_util import assert_close, small_layer

pytestmark = pytest.mark.gpu


def _layer(wl):
    packed = []
    for which in ("gate_up", "down"):
        packed += list(e4b.quantize(wl.fmt, synth.layer_weights(wl, which, "cuda")))
    return e4b.PackedLayer(wl.fmt, wl.E, wl.H, wl.I, *packed)


@pytest.mark.parametrize("flags", [0, e4b.FLAG_FORCE_TCGEN05])
def test_noalloc_matches_workspace_forward_twice(flags):
    wl = TINY
    layer = _layer(wl)
    for T, seed_shift in ((wl.T[0], 0), (23, 1)):
        x = synth.tokens_bf16(wl, T).cuda()
        ids_h, gates_h = synth.routing(wl, T)
        ids = torch.from_numpy(ids_h).cuda()
        gates = torch.from_numpy(gates_h).cuda()
        ref = e4b.moe_forward(layer, x, ids, gates, flags=flags).float().cpu().numpy()
        for _ in range(2):
            y = torch.full((T, wl.H), float("nan"), dtype=torch.bfloat16, device="cuda")
            e4b.e4b_moe_forward_noalloc(layer, x, ids, gates, y, flags=flags)
            torch.cuda.synchronize()
            assert_close(y.float().cpu().numpy(), ref, f"noalloc T={T} flags={flags}")


def test_noalloc_decode_layer_and_size_limit():
    wl = DECODE
    layer = _layer(wl)
    for T in wl.T:
        x = synth.tokens_bf16(wl, T).cuda()
        ids_h, gates_h = synth.routing(wl, T)
        ids = torch.from_numpy(ids_h).cuda()
        gates = torch.from_numpy(gates_h).cuda()
        ref = e4b.moe_forward(layer, x, ids, gates).float().cpu().numpy()
        for _ in range(2):
            y = torch.empty((T, wl.H), dtype=torch.bfloat16, device="cuda")
            e4b.e4b_moe_forward_noalloc(layer, x, ids, gates, y)
            torch.cuda.synchronize()
            assert_close(y.float().cpu().numpy(), ref, f"noalloc decode T={T}")
    # the largest call that fits on the large-M path (the one this shape takes
    # from T = 65 on): the routing arrays, h and the gate-weighted fp32 rows
    # take the 16 MiB, the optional staging copy of the routed rows does not
    # fit, so the large-M kernel gathers the rows itself
    T = 186
    x = synth.tokens_bf16(wl, T).cuda()
    ids_h, gates_h = synth.routing(wl, T)
    ids = torch.from_numpy(ids_h).cuda()
    gates = torch.from_numpy(gates_h).cuda()
    ref = e4b.moe_forward(layer, x, ids, gates).float().cpu().numpy()
    assert e4b.e4b_last_launch_count() == 5  # staged rows with a full workspace
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device="cuda")
    e4b.e4b_moe_forward_noalloc(layer, x, ids, gates, y)
    torch.cuda.synchronize()
    assert e4b.e4b_last_launch_count() == 4  # rows gathered in the kernel
    assert_close(y.float().cpu().numpy(), ref, "noalloc decode T=186")
    # beyond the static scratch: a clear error, nothing enqueued
    T = 187
    x = torch.zeros((T, wl.H), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((T, 2), dtype=torch.int32, device="cuda")
    gates = torch.zeros((T, 2), dtype=torch.float32, device="cuda")
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(e4b.E4BError) as exc:
        e4b.e4b_moe_forward_noalloc(layer, x, ids, gates, y)
    assert exc.value.status == 8


@pytest.mark.parametrize("flags", [0, e4b.FLAG_FORCE_TCGEN05])
def test_noalloc_mxfp4_layer_twice(flags):
    layer, _ = small_layer("mxfp4", 8, 256, 512, seed=81)
    rng = np.random.default_rng(82)
    for T in (64, 7):
        x = torch.from_numpy(rng.standard_normal((T, 256)).astype(np.float32)).to(torch.bfloat16).cuda()
        ids_h, gates_h = synth.random_ids(rng, T, 2, 8)
        ids = torch.from_numpy(ids_h).cuda()
        gates = torch.from_numpy(gates_h).cuda()
        ref = e4b.moe_forward(layer, x, ids, gates, flags=flags).float().cpu().numpy()
        for _ in range(2):
            y = torch.full((T, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
            e4b.e4b_moe_forward_noalloc(layer, x, ids, gates, y, flags=flags)
            torch.cuda.synchronize()
            assert_close(y.float().cpu().numpy(), ref, f"noalloc mxfp4 T={T} flags={flags}", min_rms=0.5)


def test_noalloc_int4_layer_beyond_the_nf4_token_limit():
    # int4-b32 stacks need only the status words and h [top_k, I] whatever T,
    # so T = 256 (more than the 227 tokens an NF4 layer of this shape fits in
    # the static scratch) is accepted
    wl = DECODE
    gc, gs = e4b.quantize_int4_b32(synth.layer_weights(wl, "gate_up", "cuda"))
    dc, ds = e4b.quantize_int4_b32(synth.layer_weights(wl, "down", "cuda"))
    layer = e4b.PackedLayer("int4b32", wl.E, wl.H, wl.I, gc, gs, dc, ds)
    T = 256
    x = synth.tokens_bf16(wl, T).cuda()
    ids_h, gates_h = synth.routing(wl, T)
    ids = torch.from_numpy(ids_h).cuda()
    gates = torch.from_numpy(gates_h).cuda()
    ref = e4b.moe_forward(layer, x, ids, gates).float().cpu().numpy()
    for _ in range(2):
        y = torch.full((T, wl.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        e4b.e4b_moe_forward_noalloc(layer, x, ids, gates, y)
        torch.cuda.synchronize()
        assert e4b.e4b_last_path() == e4b.E4B_PATH_INT4_GEMV
        assert_close(y.float().cpu().numpy(), ref, f"noalloc int4 T={T}", min_rms=0.5)
