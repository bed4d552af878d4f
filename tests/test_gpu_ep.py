"""Expert parallelism on the GPU through the library's kernels (e4b_ep_dest,
the routing pass by destination rank, e4b_ep_pack, e4b_moe_forward with one
slot a row, e4b_ep_combine): with a one-rank NCCL group (the all-to-alls are
then copies), and with two ranks' halves of the experts run in one process
(the exchange done by slicing, no collective). Both are checked against the
oracle's layer taken one routed slot at a time: every slot's output is
rounded to bf16 (the local layer runs with one slot a row and the gate
applied), then the slots of a token are summed and rounded once more."""

import socket
from datetime import timedelta

import numpy as np
import pytest
import torch

import oracle
from oracle import int4b32 as q4
from bit_grouped_moe_e4b_b200 import e4b, synth
from bit_grouped_moe_e4b_b200.ep import CudaOps, ExpertParallelLayer
from gpu_util import LAYER_MIN_RMS, assert_close, small_layer

pytestmark = pytest.mark.gpu


def _inputs(seed, T, k, E, H):
    rng = np.random.default_rng(seed)
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16).cuda()
    ids, gates = synth.random_ids(rng, T, k, E)
    return x, torch.from_numpy(ids).cuda(), torch.from_numpy(gates).cuda()


def _per_slot_oracle(fmt, x, ids, gates, ref, E, H, I, nf4_decode="product"):
    """y[t] = bf16(sum_j bf16(g[t,j] * expert_j(x[t]))) with the oracle's
    layer run on each slot alone; slots whose id is outside [0, E) add 0."""
    xf = x.float().cpu().numpy()
    ids = ids.cpu().numpy().astype(np.int32)
    gates = gates.cpu().numpy().astype(np.float32)
    T, k = ids.shape
    bad = (ids < 0) | (ids >= E)
    ids1 = np.where(bad, 0, ids).reshape(-1, 1)
    g1 = np.where(bad, 0.0, gates).astype(np.float32).reshape(-1, 1)
    xr = np.repeat(xf, k, axis=0)
    if fmt == "int4b32":
        gc, gs, dc, ds = ref
        ys = np.stack([q4.int4b32_decode_layer_ref(xr[s], [int(ids1[s, 0])], g1[s], gc, gs, dc, ds)
                       for s in range(T * k)])
    else:
        gc, gs, dc, ds = ref
        ys = oracle.moe_forward_ref(fmt, xr, ids1, g1, gc, gs, dc, ds, E, H, I, nf4_decode=nf4_decode)
    ys = np.where(bad.reshape(-1, 1), 0.0, ys)
    return oracle.bf16_round(ys.reshape(T, k, H).astype(np.float64).sum(axis=1))


def _nf4_mode():
    # the NF4 reading of the local layer's path: "level" on small-M
    return "level" if e4b.e4b_last_path() == e4b.E4B_PATH_GEMV else "product"


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_expert_parallel_one_rank_group():
    import torch.distributed as dist

    layer, ref = small_layer("nf4", 8, 256, 512, seed=51)
    x, ids, gates = _inputs(52, 24, 2, 8, 256)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=timedelta(seconds=120))
    try:
        y = ExpertParallelLayer(layer, 8).forward(x, ids, gates)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    want = _per_slot_oracle("nf4", x, ids, gates, ref, 8, 256, 512, nf4_decode=_nf4_mode())
    assert_close(y.float().cpu().numpy(), want, "one-rank expert parallel", min_rms=LAYER_MIN_RMS)


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
        layer, ref = small_layer("nf4", E, H, I, seed=53)
    else:
        rng = np.random.default_rng(53)
        wgu = (rng.standard_normal((E, 2 * I, H)) * 1.5 / np.sqrt(H)).astype(np.float32)
        wd = (rng.standard_normal((E, H, I)) * 2.0 / np.sqrt(I)).astype(np.float32)
        gc, gs = e4b.quantize_int4_b32(torch.from_numpy(wgu).cuda())
        dc, ds = e4b.quantize_int4_b32(torch.from_numpy(wd).cuda())
        layer = e4b.PackedLayer("int4b32", E, H, I, gc, gs, dc, ds)
        rgc, rgs = q4.quantize_int4b32(wgu)
        rdc, rds = q4.quantize_int4b32(wd)
        assert np.array_equal(gc.cpu().numpy(), rgc) and np.array_equal(dc.cpu().numpy(), rdc)
        ref = (rgc, rgs, rdc, rds)
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
    mode = _nf4_mode()
    y = ops.combine(torch.cat(parts), inv, T, k, H, x)
    torch.cuda.synchronize()
    # the dropped slot contributes nothing
    want = _per_slot_oracle(fmt, x, ids, gates, ref, E, H, I, nf4_decode=mode)
    assert_close(y.float().cpu().numpy(), want, f"{fmt} two emulated ranks", min_rms=LAYER_MIN_RMS)
