"""The multi-rank path of bench.py on CPU: every rank runs its own token batch
with no collective on the data path, the timings are reduced with a max over
ranks (world size 2, gloo), and the reference arm prints one line from rank 0
only while the other ranks exit 0 without work."""

import json
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest

from conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench

    q.put((rank, bench.max_over_ranks(1.5 + 2.0 * rank, dist, "cpu"), bench.max_over_ranks(7.0 - rank, dist, "cpu")))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, 3.5, 7.0), (1, 3.5, 7.0)]


def test_max_over_ranks_without_a_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(2.25, None, "cpu") == 2.25


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_from_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(_free_port()))
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
           "tiny_nf4_E8_H256_I512_top2", "--steps", "2", "--warmup", "1"]
    out = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    if rank == 0:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle" and d["value"] > 0
    else:
        assert lines == []
