"""bench.py's host arithmetic on CPU: the algorithmic bytes per kernel, the
roofline fields (which peak, which fraction), and the rule that DRAM traffic is
reported only while the kernel's sources are the ones it was captured on."""

import json
import os

import numpy as np
import pytest

from conftest import ROOT

import bench
from bit_grouped_moe_e4b_b200.configs import WORKLOADS


def test_decode_layer_bytes_are_the_packed_stacks_plus_activations():
    # decode NF4 (E=8, H=4096, I=14336, top-2) with every expert active: each
    # expert stores 3*H*I weights at 4 bits plus one fp32 absmax per 64, i.e.
    # 0.5625 bytes a weight = 99,090,432 bytes; x in and y out are bf16 [T, H];
    # ids and gates are 4 bytes each per routed slot
    wl = WORKLOADS["decode_nf4_E8_H4096_I14336_top2"]
    T = 16
    ids = np.arange(T * 2, dtype=np.int32).reshape(T, 2) % wl.E
    kb = bench.kernel_bytes(wl, T, ids)
    per_expert = 3 * 4096 * 14336 * 9 // 16
    assert per_expert == 99_090_432
    assert kb["active_experts"] == 8
    assert kb["layer"] == 8 * per_expert + 4 * T * 4096 + 8 * T * 2 == 792_985_856
    # the one-launch small-M kernel is charged both projections, each with x / y and the routing
    assert kb["smallm_layer"] == kb["gate_up"] + kb["down"]
    assert kb["gate_up"] == 8 * 2 * 14336 * 4096 * 0.5625 + 2 * T * 4096 + 4 * T * 2


def test_mxfp4_bytes_count_one_scale_byte_per_32_weights():
    wl = WORKLOADS["mxfp4_E32_H2880_I2880_top4"]
    ids = np.array([[0, 1, 2, 3]], np.int32)
    kb = bench.kernel_bytes(wl, 1, ids)
    assert kb["packed_bytes"] == 4 * 3 * 2880 * 2880 * (0.5 + 1 / 32)


def _tensor_roofline(power_capped):
    wl = WORKLOADS["prefill_nf4_E8_H4096_I14336_top2"]
    ids = np.zeros((4096, 2), np.int32)
    dur_s = 2.0e-3
    return bench._roofline(2, "gate_up", {}, dur_s, wl, ids, "no-such-key", 6546.9, 1658.4, 1375.3, "measured",
                           power_capped=power_capped), 2.0 * ids.size * 2 * wl.I * wl.H / dur_s / 1e12


@pytest.mark.parametrize("capped", [False, True])
def test_tensor_roofline_picks_the_peak_of_the_regime(capped):
    r, achieved = _tensor_roofline(capped)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(achieved)
    peak = 1375.3 if capped else 1658.4
    assert r["peak"] == peak
    assert r["frac"] == pytest.approx(achieved / peak)
    assert r["frac_burst"] == pytest.approx(achieved / 1658.4)
    assert r["traffic"] is None  # no record under that key


def test_hbm_roofline_is_bytes_over_time_against_the_copy_peak():
    wl = WORKLOADS["decode_nf4_E8_H4096_I14336_top2"]
    ids = np.arange(32, dtype=np.int32).reshape(16, 2) % 8
    kb = bench.kernel_bytes(wl, 16, ids)
    r = bench._roofline(1, "smallm_layer", kb, 0.2e-3, wl, ids, "no-such-key", 6546.9, 1658.4, 1375.3, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(kb["smallm_layer"] / 0.2e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6546.9)


def test_traffic_only_for_the_sources_it_was_captured_on(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        recs = {(k, kern): v for k, d in json.load(f).items() if not k.startswith("_") for kern, v in d.items()}
    assert recs
    for (key, kern), rec in recs.items():
        # every record names a kernel whose sources bench.py hashes
        assert kern in bench._KERNEL_SOURCES
        got = bench._traffic(key, kern)
        if rec["source_hash"] == bench._source_hash(kern):
            assert got == rec["dram_bytes_per_launch"]
        else:
            assert got is None
    # a change to the sources makes every record stale
    monkeypatch.setattr(bench, "_source_hash", lambda kernel: "0" * 16)
    assert all(bench._traffic(key, kern) is None for key, kern in recs)
