"""Expert parallelism on CPU ranks (gloo; 2 and 4 ranks): ExpertParallelLayer's routing by
destination rank, the all-to-all exchanges of counts, rows, local ids and
gates, the return of the outputs and the combine, with the device steps taken
by a CPU double built on the oracle. Each rank's output must match the
oracle's one-device layer on that rank's tokens (within the per-slot bf16
rounding the split adds)."""

import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest
import torch

from conftest import ROOT


class _OracleOps:
    """The device steps of an expert-parallel call, on the CPU, from the oracle."""

    def dest(self, ids, E, epr):
        return torch.where((ids >= 0) & (ids < E), ids // epr, torch.full_like(ids, -1))

    def route(self, dest, G):
        import oracle

        counts, offsets, perm, inv = oracle.route_ref(dest.numpy(), G)
        return (torch.from_numpy(counts), torch.from_numpy(offsets), torch.from_numpy(perm),
                torch.from_numpy(inv))

    def pack(self, x, ids, gates, perm, offsets, G, R, epr):
        k = ids.shape[1]
        slots = perm[:R].long()
        return x[slots // k], (ids.reshape(-1)[slots] % epr).int(), gates.reshape(-1)[slots]

    def local_forward(self, layer, x_in, lids, gates):
        import oracle

        if x_in.shape[0] == 0:
            return torch.empty_like(x_in)
        gc, gs, dc, ds = layer.stacks
        y = oracle.moe_forward_ref("nf4", x_in.numpy().astype(np.float64), lids.numpy().reshape(-1, 1),
                                   gates.numpy().reshape(-1, 1), gc, gs, dc, ds, layer.E, layer.H, layer.I)
        return torch.from_numpy(y.astype(np.float32))

    def combine(self, ys, inv, T, k, H, like):
        import oracle

        y = np.zeros((T, H))
        ysn = ys.numpy().astype(np.float64)
        for s, p in enumerate(inv.numpy()):
            if p >= 0:
                y[s // k] += ysn[p]
        return torch.from_numpy(oracle.bf16_round(y).astype(np.float32))


class _Local:
    def __init__(self, E, H, I, stacks):
        self.E, self.H, self.I, self.stacks = E, H, I, stacks


def _layer(E, H, I):
    import oracle

    rng = np.random.default_rng(41)
    wgu = (rng.standard_normal((E, 2 * I, H)) * 0.05).astype(np.float32)
    wd = (rng.standard_normal((E, H, I)) * 0.05).astype(np.float32)
    gc, gs = oracle.quantize_pack_nf4(wgu)
    dc, ds = oracle.quantize_pack_nf4(wd)
    return gc, gs, dc, ds


def _rank(rank, world, port, q, local_only=False):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    import oracle
    from bit_grouped_moe_e4b_b200 import synth
    from bit_grouped_moe_e4b_b200.ep import ExpertParallelLayer

    E, H, I, k = 4, 128, 64, 2
    gc, gs, dc, ds = _layer(E, H, I)
    epr = E // world
    sl = slice(rank * epr, (rank + 1) * epr)
    local = _Local(epr, H, I, (gc[sl], gs[sl], dc[sl], ds[sl]))
    ep = ExpertParallelLayer(local, E, ops=_OracleOps())
    rng = np.random.default_rng(100 + rank)
    T = 5 + 3 * rank  # the ranks hold different numbers of tokens
    x = oracle.bf16_round(rng.standard_normal((T, H))).astype(np.float32)
    ids, gates = synth.random_ids(rng, T, k, E)
    if rank == 1:
        ids[2, 1] = ids[2, 0]  # a token sending both slots to one expert
    if local_only:  # every slot stays on its own rank: the cross-rank exchanges are empty
        ids = (ids % epr + rank * epr).astype(np.int32)
    y = ep.forward(torch.from_numpy(x), torch.from_numpy(ids), torch.from_numpy(gates)).numpy()
    ref = oracle.moe_forward_ref("nf4", x.astype(np.float64), ids, gates, gc, gs, dc, ds, E, H, I)
    err = float(np.max(np.abs(y - ref) / (1 + np.abs(ref))))
    q.put((rank, err, y.shape))
    dist.barrier()
    dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,local_only", [(2, False), (2, True), (4, False)])
def test_expert_parallel_layer_on_gloo_ranks(world, local_only):
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q, local_only)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[2] for g in got] == [(5 + 3 * r, 128) for r in range(world)]
    for rank, err, _ in got:
        assert err <= 1e-2, f"rank {rank}: max scaled error {err}"
