"""GPU routing pass, bit for bit against the oracle."""

import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_e4b_b200 import e4b, synth
from bit_grouped_moe_e4b_b200.configs import WORKLOADS

pytestmark = pytest.mark.gpu


def _check(ids, E):
    counts, offsets, perm, inv, ws = e4b.route(torch.from_numpy(ids).cuda(), E)
    status = e4b.e4b_read_device_status(ws)
    rc, ro, rp, ri = oracle.route_ref(ids, E)
    assert status == 0
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    assert np.array_equal(inv.cpu().numpy(), ri)


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (1, 2, 8), (7, 3, 5), (64, 2, 8), (1000, 8, 128),
                                   (4096, 2, 8), (333, 4, 1024), (20000, 1, 3)])
def test_route_random_ids(T, k, E):
    rng = np.random.default_rng(T * 31 + k * 7 + E)
    _check(rng.integers(0, E, (T, k)).astype(np.int32), E)


def test_route_skewed_and_empty_experts():
    rng = np.random.default_rng(4)
    p = rng.dirichlet(np.full(64, 0.05))
    ids = rng.choice(64, size=(5000, 4), p=p).astype(np.int32)
    _check(ids, 64)
    _check(np.zeros((300, 2), np.int32), 16)  # everything on one expert


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_route_workload_ids(name):
    wl = WORKLOADS[name]
    for T in wl.T:
        ids, _ = synth.routing(wl, T)
        _check(ids, wl.E)


def test_route_bad_ids_are_dropped_and_reported():
    ids = np.array([[0, 1], [5, 2], [-1, 3], [2, 2]], np.int32)
    counts, offsets, perm, inv, ws = e4b.route(torch.from_numpy(ids).cuda(), 4)
    assert e4b.e4b_read_device_status(ws) == 6
    flat = ids.reshape(-1)
    ok = (flat >= 0) & (flat < 4)
    rc, ro, rp, _ = oracle.route_ref(np.where(ok, flat, 0)[ok].reshape(1, -1), 4)
    assert np.array_equal(counts.cpu().numpy(), rc)
    valid_slots = np.nonzero(ok)[0]
    assert np.array_equal(perm.cpu().numpy()[:ok.sum()], valid_slots[rp])
    inv_h = inv.cpu().numpy()
    assert np.all(inv_h[~ok] == -1)
    # after reading, the status word is clear
    assert e4b.e4b_read_device_status(ws) == 0
