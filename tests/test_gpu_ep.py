"""Expert parallelism on the GPU through the library's kernels (e4b_ep_dest,
the routing pass by destination rank, e4b_ep_pack, e4b_moe_forward with one
slot a row, e4b_ep_combine): with a one-rank NCCL group (the all-to-alls are
then copies), and with two ranks' halves of the experts run in one process
(the exchange done by slicing, no collective). Both must match the one-GPU
layer within the per-slot bf16 rounding the split adds."""

import socket
from datetime import timedelta

import numpy as np
import pytest
import torch

from bit_grouped_moe_e4b_b200 import e4b, synth
from bit_grouped_moe_e4b_b200.ep import CudaOps, ExpertParallelLayer
from gpu_util import assert_close, small_layer

pytestmark = pytest.mark.gpu


def _inputs(seed, T, k, E, H):
    rng = np.random.default_rng(seed)
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16).cuda()
    ids, gates = synth.random_ids(rng, T, k, E)
    return x, torch.from_numpy(ids).cuda(), torch.from_numpy(gates).cuda()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_expert_parallel_one_rank_group():
    import torch.distributed as dist

    layer, _ = small_layer("nf4", 8, 256, 512, seed=51)
    x, ids, gates = _inputs(52, 24, 2, 8, 256)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=timedelta(seconds=120))
    try:
        y = ExpertParallelLayer(layer, 8).forward(x, ids, gates)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    want = e4b.moe_forward(layer, x, ids, gates)
    assert_close(y.float().cpu().numpy(), want.float().cpu().numpy(), "one-rank expert parallel", tol=2e-2)


def _halves(layer, G):
    epr = layer.E // G
    out = []
    for r in range(G):
        sl = slice(r * epr, (r + 1) * epr)
        out.append(e4b.PackedLayer(layer.fmt, epr, layer.H, layer.I, layer.gate_up_codes[sl].contiguous(),
                                   layer.gate_up_scales[sl].contiguous(), layer.down_codes[sl].contiguous(),
                                   layer.down_scales[sl].contiguous()))
    return out


@pytest.mark.parametrize("fmt", ["nf4", "int4b32"])
def test_two_ranks_emulated_in_one_process(fmt):
    E, H, I, T, k, G = 8, 256, 512, 20, 2, 2
    if fmt == "nf4":
        layer, _ = small_layer("nf4", E, H, I, seed=53)
    else:
        rng = np.random.default_rng(53)
        gc, gs = e4b.quantize_int4_b32(torch.from_numpy((rng.standard_normal((E, 2 * I, H)) * 0.02)
                                                        .astype(np.float32)).cuda())
        dc, ds = e4b.quantize_int4_b32(torch.from_numpy((rng.standard_normal((E, H, I)) * 0.02)
                                                        .astype(np.float32)).cuda())
        layer = e4b.PackedLayer("int4b32", E, H, I, gc, gs, dc, ds)
    x, ids, gates = _inputs(54, T, k, E, H)
    ids[3, 1] = 99  # a bad expert id: the slot is dropped on both sides
    ops, epr = CudaOps(), E // G
    dest = ops.dest(ids, E, epr)
    counts, offsets, perm, inv = ops.route(dest, G)
    off = offsets.cpu().numpy()
    R = int(off[-1])
    assert R == T * k - 1 and int(inv.view(-1)[3 * k + 1]) == -1
    xs, lids, gs = ops.pack(x, ids, gates, perm, offsets, G, R, epr)
    # ranks' rows are the destination ranges; each runs its own experts
    parts = []
    for r, local in enumerate(_halves(layer, G)):
        a, b = int(off[r]), int(off[r + 1])
        parts.append(ops.local_forward(local, xs[a:b], lids[a:b], gs[a:b]))
    y = ops.combine(torch.cat(parts), inv, T, k, H, x)
    torch.cuda.synchronize()
    ok_ids = ids.clone()
    ok_gates = gates.clone()
    ok_ids[3, 1] = ok_ids[3, 0]
    ok_gates[3, 1] = 0.0  # the dropped slot contributes nothing
    want = e4b.moe_forward(layer, x, ok_ids, ok_gates)
    assert_close(y.float().cpu().numpy(), want.float().cpu().numpy(), f"{fmt} two emulated ranks", tol=2e-2)
