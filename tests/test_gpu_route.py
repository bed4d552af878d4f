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


def _route_ws(ids, E, ws_bytes):
    ids_d = torch.from_numpy(ids).cuda()
    T, k = ids.shape
    dev = ids_d.device
    out = (torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E + 1, dtype=torch.int64, device=dev),
           torch.empty(T * k, dtype=torch.int32, device=dev), torch.empty(T * k, dtype=torch.int32, device=dev))
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    e4b.e4b_route(ids_d, E, *out, ws)
    launches = e4b.e4b_last_launch_count()
    return [o.cpu().numpy() for o in out], e4b.e4b_read_device_status(ws), launches


@pytest.mark.parametrize("T,k,E,skew", [(2500, 8, 1024, 0.0), (8192, 8, 128, 0.05), (4097, 4, 32, 0.0),
                                        (16384, 1, 1, 0.0), (6000, 3, 7, 0.3)])
def test_route_many_ctas_equals_one_cta_and_oracle(T, k, E, skew):
    # from 16384 slots a workspace of e4b_route_workspace_size bytes routes
    # over many CTAs (two launches); a status-only workspace on one CTA
    rng = np.random.default_rng(T + E)
    if skew:
        ids = rng.choice(E, size=(T, k), p=rng.dirichlet(np.full(E, skew))).astype(np.int32)
    else:
        ids = rng.integers(0, E, (T, k)).astype(np.int32)
    full = e4b.e4b_route_workspace_size(T, k, E)
    assert full > 256
    many, st_m, l_m = _route_ws(ids, E, full)
    one, st_o, l_o = _route_ws(ids, E, 256)
    assert (l_m, l_o) == (2, 1) and st_m == 0 and st_o == 0
    ref = oracle.route_ref(ids, E)
    for a, b, r in zip(many, one, ref):
        assert np.array_equal(a, r) and np.array_equal(b, r)


def test_route_many_ctas_bad_ids():
    rng = np.random.default_rng(17)
    T, k, E = 9000, 2, 40
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    bad = rng.choice(T * k, 37, replace=False)
    ids.reshape(-1)[bad[:20]] = -3
    ids.reshape(-1)[bad[20:]] = E + 5
    (counts, offsets, perm, inv), status, launches = _route_ws(ids, E, e4b.e4b_route_workspace_size(T, k, E))
    assert launches == 2 and status == 6   # E4B_ERR_BAD_EXPERT_ID
    flat = ids.reshape(-1)
    ok = (flat >= 0) & (flat < E)
    rc, ro, rp, _ = oracle.route_ref(np.where(ok, flat, 0)[ok].reshape(1, -1), E)
    assert np.array_equal(counts, rc) and np.array_equal(offsets, ro)
    assert np.array_equal(perm[:ok.sum()], np.nonzero(ok)[0][rp])
    assert np.all(inv[~ok] == -1)
    assert np.array_equal(perm[inv[ok]], np.nonzero(ok)[0])
