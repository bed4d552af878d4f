#!/usr/bin/env python
"""Benchmark of the packed-4-bit MoE layer forward on B200.

Default line: the prefill layer, NF4, E=8 experts, H=4096, I=14336, top-2,
T=4096 tokens (the largest single-GPU workload; weights N(0, 0.02) fp32 drawn
on the GPU and packed by the library's quantiser; x N(0, 1) in bf16; U[0, 1)
router logits, top-2 and a softmax over the chosen two). One step = one layer
forward: routing pass, gate_up grouped GEMM with SwiGLU, down grouped GEMM
with the weighted combine, bf16 output. The same line carries `per_config`:
every workload and token count, each timed as the median of 50 single-call
repetitions with the L2 flushed before each, launched on a stream and
replayed from a CUDA graph, with the spread between two independent medians
of the same call (self-pair).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl e4b|reference]
                    [--workload NAME] [--T T] [--sweep] [--no-per-config]

Prints one JSON line (rank 0). Under torchrun (N > 1) every rank runs its own
batch of T tokens on its own GPU with replicated weights and no collective on
the data path (weak scaling); the timed region is bracketed by barriers and
the max over ranks is reported. --impl reference times the CPU oracle on the
host cores instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and packed-weight HBM GB/s (% roofline) on 1 B200"
DEFAULT_WORKLOAD = "prefill_nf4_E8_H4096_I14336_top2"
DEFAULT_T = 4096
PER_CONFIG_REPS = 50
L2_BYTES = 126 * 2 ** 20


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["e4b", "reference"], default="e4b")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--sweep", action="store_true",
                    help="print one line per workload and token count (no cpu baseline)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-workload table of the default line")
    ap.add_argument("--mx", choices=["off", "exact", "e4m3"], default="off",
                    help="MXFP4 workloads: run the block-scaled FP4 MMA path on the prepared stacks, with the "
                         "bf16-exact two-term activations or one e4m3 term (OCP MXFP8)")
    ap.add_argument("--reps", type=int, default=PER_CONFIG_REPS,
                    help="repetitions per median in the per-workload table")
    ap.add_argument("--op", choices=["forward", "dgrad", "int4"], default="forward",
                    help="dgrad: time e4b_grouped_dgrad, the input gradients of both projections "
                         "(one JSON line, TFLOP/s); int4: the int4-b32 decode GEMVs of one token "
                         "through the workload's layer (one JSON line, packed-weight GB/s)")
    return ap.parse_args()


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# The sources a kernel is compiled from: its own file and the device headers.
# (the layer's large-M projections run on the SM-pair kernel, dispatched from
# the one-SM kernel's launcher)
_KERNEL_SOURCES = {
    "smallm_layer": ("smallm.cu",), "gate_up": ("tc_pair.cu", "tc_gemm.cu"), "down": ("tc_pair.cu", "tc_gemm.cu"),
    "int4_gemv_gate_up": ("int4.cu",), "int4_gemv_down": ("int4.cu",),
}
_DEVICE_HEADERS = ("common.cuh", "sm100.cuh", "launch.h", "tmap.h")


def _source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_grouped_moe_e4b_b200", "csrc")
    for name in _KERNEL_SOURCES[kernel] + _DEVICE_HEADERS:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(key: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel's current sources; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        rec = d[key][kernel]
        if rec.get("source_hash") != _source_hash(kernel):
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(value: float, dist, device) -> float:
    """The largest of every rank's value (the slowest rank sets a multi-GPU
    time); `value` itself without a process group."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ GPU arm
def build_layer(wl, device):
    import torch
    from bit_grouped_moe_e4b_b200 import e4b, synth

    packed = []
    for which in ("gate_up", "down"):
        w = synth.layer_weights(wl, which, device)
        packed += list(e4b.quantize(wl.fmt, w))
        del w
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return e4b.PackedLayer(wl.fmt, wl.E, wl.H, wl.I, *packed)


def _roofline(path, kernel, kb, dur_s, wl, ids, key, hbm, bf16, bf16_sus, peak_src, power_capped=False):
    """Roofline of the dominant kernel: HBM bytes for the small-M layer kernel,
    dense bf16 FLOPs for a tcgen05 projection. The tensor peak is the burst
    figure (a kernel timed alone) unless the clock samples of the timed region
    saw sw_power_cap: the kernel then ran in the power-capped regime the
    sustained figure measures, and is held against that one ("frac_burst"
    keeps the ratio to the burst figure)."""
    if path in (2, 4) and kernel in ("gate_up", "down", "quant_h+down"):
        R = ids.size
        flops = 2.0 * R * (2 * wl.I * wl.H if kernel == "gate_up" else wl.H * wl.I)
        achieved = flops / dur_s / 1e12
        # the block-scaled FP4 MMA runs at the f8f6f4 rate: the measured bf16
        # peak times 2, the nominal ratio of the dense fp8 and bf16 peaks
        scale = 2.0 if path == 4 else 1.0
        burst, sustained = bf16 * scale, bf16_sus * scale
        peak = sustained if power_capped else burst
        which = ("sustained: sw_power_cap was active in the timed region" if power_capped else "burst")
        return {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "frac_burst": achieved / burst,
                "peak_source": peak_src + (" bf16 x 2 (f8f6f4)" if path == 4 else " bf16") + f", {which}",
                "peak_burst": burst, "peak_sustained": sustained,
                "traffic": _traffic(key, kernel) if path == 2 else None, "algorithmic_flops": flops}
    achieved = kb[kernel] / dur_s / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "peak_source": peak_src, "traffic": _traffic(key, kernel),
            "algorithmic_bytes": kb[kernel]}


def kernel_bytes(wl, T, ids):
    """Algorithmic bytes per launch of each kernel: the packed bytes of the active experts plus the
    activation rows in and out, and the routing ids and gates."""
    # storage per weight: 4-bit code + fp32 absmax per 64 (NF4) or one e8m0 byte per 32 (MXFP4)
    bpw = 0.5 + (4.0 / 64 if wl.fmt == "nf4" else 1.0 / 32)
    active = len(np.unique(ids))
    R = ids.size
    gu = active * 2 * wl.I * wl.H * bpw + 2 * T * wl.H + 4 * R
    dn = active * wl.H * wl.I * bpw + 2 * T * wl.H + 4 * R
    return {"gate_up": gu, "down": dn, "smallm_layer": gu + dn, "combine": 4 * ids.size * wl.H + 2 * T * wl.H,
            "active_experts": active,
            "packed_bytes": active * 3 * wl.H * wl.I * bpw,
            "layer": active * 3 * wl.H * wl.I * bpw + 4 * T * wl.H + 8 * R}


def run_gpu(wl, T, steps, warmup, rank, world, dist, layer=None, flags=0):
    import torch
    from bit_grouped_moe_e4b_b200 import e4b, synth

    dev = torch.device("cuda", torch.cuda.current_device())
    if layer is None:
        layer = build_layer(wl, dev)
    x_h = synth.tokens_bf16(wl, T)
    ids_h, gates_h = synth.routing(wl, T)
    x = x_h.to(dev)
    ids = torch.from_numpy(ids_h).to(dev)
    gates = torch.from_numpy(gates_h).to(dev)
    ws = e4b.workspace(layer, T, wl.top_k, dev)
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(warmup):
        e4b.e4b_moe_forward(layer, x, ids, gates, y, ws, flags)
    torch.cuda.synchronize()
    status = e4b.e4b_read_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    path = e4b.e4b_last_path()
    launches_per_step = e4b.e4b_last_launch_count()

    # timed region: inputs resident in HBM
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for row in ev:  # torch creates the CUDA event on first record
        for e_ in row:
            e_.record(stream)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device())
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    # the steps run back to back with nothing between the launches (each is a
    # programmatic dependent of the one before); the per-kernel times come
    # from a second loop with the library's events between its launches
    t0.record(stream)
    for i in range(steps):
        e4b.e4b_moe_forward(layer, x, ids, gates, y, ws, flags)
    t1.record(stream)
    torch.cuda.synchronize()
    for i in range(steps):
        e4b.e4b_set_timing_events(ev[i])
        e4b.e4b_moe_forward(layer, x, ids, gates, y, ws, flags)
    torch.cuda.synchronize()
    e4b.e4b_set_timing_events(None)
    clk = clocks.stop()
    barrier()
    ms = t0.elapsed_time(t1)
    path = e4b.e4b_last_path()
    if path == e4b.E4B_PATH_GEMV:  # routing, the fused small-M layer kernel, the combine
        spans = (("route", 0, 1), ("smallm_layer", 1, 3), ("combine", 3, 4))
    elif path == e4b.E4B_PATH_TCGEN05_MX:  # routing + x terms, gate_up, h terms + down, combine
        spans = (("route+quant_x", 0, 1), ("gate_up", 1, 2), ("quant_h+down", 2, 3), ("combine", 3, 4))
    else:
        # routing (+ the staging copy of the routed rows when the workspace
        # holds it), the two tcgen05 projections, the bf16 conversion
        # 5 or 6 launches with the staging copy (routing takes 2 launches from
        # 16384 routed rows), 4 without
        first = "route+stage" if launches_per_step >= 5 else "route"
        spans = ((first, 0, 1), ("gate_up", 1, 2), ("down", 2, 3), ("combine", 3, 4))
    phases = {name: float(np.mean([ev[i][a].elapsed_time(ev[i][b]) for i in range(steps)]))
              for name, a, b in spans}
    phases["_note"] = "each launch alone (events between launches); the timed steps overlap them"
    ms = max_over_ranks(ms, dist, dev)

    # end-to-end through the C ABI with host buffers (pinned), copies inside
    x_pin = x_h.pin_memory()
    ids_pin = torch.from_numpy(ids_h).pin_memory()
    g_pin = torch.from_numpy(gates_h).pin_memory()
    y_pin = torch.empty((T, wl.H), dtype=torch.bfloat16).pin_memory()
    x_d = torch.empty_like(x)
    ids_d = torch.empty_like(ids)
    g_d = torch.empty_like(gates)
    for _ in range(warmup):
        x_d.copy_(x_pin, non_blocking=True)
        e4b.e4b_moe_forward(layer, x_d, ids_d.copy_(ids_pin, non_blocking=True),
                            g_d.copy_(g_pin, non_blocking=True), y, ws, flags)
        y_pin.copy_(y, non_blocking=True)
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        x_d.copy_(x_pin, non_blocking=True)
        ids_d.copy_(ids_pin, non_blocking=True)
        g_d.copy_(g_pin, non_blocking=True)
        e4b.e4b_moe_forward(layer, x_d, ids_d, g_d, y, ws, flags)
        y_pin.copy_(y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_serial_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)

    # the same calls pipelined the way a serving loop runs them: step i's
    # inputs go up on one copy stream while step i-1 computes, and step i's
    # output comes down on another while step i+1 computes (two device
    # buffers of each; every step's bytes still cross PCIe inside the timed
    # region, which opens before the first upload and closes after the last
    # download)
    nb = 2
    xs = [x_d] + [torch.empty_like(x) for _ in range(nb - 1)]
    idss = [ids_d] + [torch.empty_like(ids) for _ in range(nb - 1)]
    gs_ = [g_d] + [torch.empty_like(gates) for _ in range(nb - 1)]
    ys = [y] + [torch.empty_like(y) for _ in range(nb - 1)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    uploaded = [torch.cuda.Event() for _ in range(nb)]
    computed = [torch.cuda.Event() for _ in range(nb)]
    downloaded = [torch.cuda.Event() for _ in range(nb)]
    for e_ in uploaded + computed + downloaded:  # created on first record
        e_.record(stream)

    def pipelined(n):
        for i in range(n):
            b = i % nb
            up.wait_event(computed[b])  # step i - nb no longer reads buffer b
            with torch.cuda.stream(up):
                xs[b].copy_(x_pin, non_blocking=True)
                idss[b].copy_(ids_pin, non_blocking=True)
                gs_[b].copy_(g_pin, non_blocking=True)
            uploaded[b].record(up)
            stream.wait_event(uploaded[b])
            stream.wait_event(downloaded[b])  # y of step i - nb has left buffer b
            e4b.e4b_moe_forward(layer, xs[b], idss[b], gs_[b], ys[b], ws, flags, stream=stream)
            computed[b].record(stream)
            down.wait_event(computed[b])
            with torch.cuda.stream(down):
                y_pin.copy_(ys[b], non_blocking=True)
            downloaded[b].record(down)
        for b in range(nb):
            stream.wait_event(downloaded[b])

    pipelined(warmup)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    up.wait_event(e0)
    pipelined(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    if e4b.e4b_read_device_status(ws) != 0:
        raise RuntimeError("device status set during the timed loops")
    return {
        "ms": ms, "phases": phases, "clocks": clk, "path": path,
        "launches": launches_per_step * steps, "e2e_ms": e2e_ms, "e2e_serial_ms": e2e_serial_ms,
        "h2d": x_h.numel() * 2 + ids_h.nbytes + gates_h.nbytes, "d2h": T * wl.H * 2,
        "ids": ids_h, "layer": layer, "x": x_h, "gates": gates_h,
    }


# ------------------------------------------------------- per-config table
def _bound_label(t_bytes, t_flops):
    r = t_bytes / t_flops
    return "ridge" if 0.5 <= r <= 2.0 else ("hbm" if r > 1 else "tensor")


def _median_ms(fn, flush, reps, stream):
    """Median over `reps` single calls of fn, each timed alone with CUDA events
    on `stream`, with the L2 flushed (a write of 4x its size) before each."""
    import torch

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in ev]))


def per_config_entry(wl, T, layer, reps, flush, hbm, bf16, peak_src, flags=0, variant=""):
    """One workload and token count: the layer call (stream-launched and
    replayed from a CUDA graph), each the median of `reps` calls with the L2
    flushed before each; a second independent stream median for the
    self-pair spread; per-kernel medians from the library's timing events
    (a separate loop: events between launches stop their overlap)."""
    import torch
    from bit_grouped_moe_e4b_b200 import e4b, synth

    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    x = synth.tokens_bf16(wl, T).to(dev)
    ids_h, gates_h = synth.routing(wl, T)
    ids = torch.from_numpy(ids_h).to(dev)
    gates = torch.from_numpy(gates_h).to(dev)
    ws = e4b.workspace(layer, T, wl.top_k, dev)
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device=dev)

    def call():
        e4b.e4b_moe_forward(layer, x, ids, gates, y, ws, flags)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    if e4b.e4b_read_device_status(ws) != 0:
        raise RuntimeError(f"device status set: {wl.name} T={T}")
    path = e4b.e4b_last_path()
    launches = e4b.e4b_last_launch_count()
    ms_a = _median_ms(call, flush, reps, stream)
    ms_b = _median_ms(call, flush, reps, stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    g.replay()
    torch.cuda.synchronize()
    ms_g = _median_ms(g.replay, flush, reps, stream)
    del g
    # per-kernel medians
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(reps)]
    for row in evs:  # torch creates the CUDA event on its first record
        for e_ in row:
            e_.record(stream)
    torch.cuda.synchronize()
    for row in evs:
        flush.zero_()
        e4b.e4b_set_timing_events(row)
        call()
    e4b.e4b_set_timing_events(None)
    torch.cuda.synchronize()
    if e4b.e4b_read_device_status(ws) != 0:
        raise RuntimeError(f"device status set in the timed loops: {wl.name} T={T}")
    if path == e4b.E4B_PATH_GEMV:
        spans = (("route", 0, 1), ("smallm_layer", 1, 3), ("combine", 3, 4))
    elif path == e4b.E4B_PATH_TCGEN05_MX:
        # routing + x split into e4m3 terms, gate_up, h split + down, combine
        spans = (("route+quant_x", 0, 1), ("gate_up", 1, 2), ("quant_h+down", 2, 3), ("combine", 3, 4))
    else:
        spans = (("route+stage" if launches >= 5 else "route", 0, 1), ("gate_up", 1, 2), ("down", 2, 3),
                 ("combine", 3, 4))
    phases = {n: float(np.median([r[a].elapsed_time(r[b]) for r in evs])) for n, a, b in spans}
    kb = kernel_bytes(wl, T, ids_h)
    kb["quant_h+down"] = kb["down"]
    R = ids_h.size
    flops = 2.0 * R * 3 * wl.H * wl.I
    kflops = {"gate_up": 2.0 * R * 2 * wl.I * wl.H, "down": 2.0 * R * wl.H * wl.I, "smallm_layer": flops}
    kflops["quant_h+down"] = kflops["down"]
    ms = ms_a
    # the block-scaled path runs at the f8f6f4 rate: the measured bf16 peak x 2
    # (the nominal ratio of the dense fp8 and bf16 peaks)
    peak = bf16 * (2.0 if path == e4b.E4B_PATH_TCGEN05_MX else 1.0)
    t_bytes = kb["layer"] / (hbm * 1e9)
    t_flops = flops / (peak * 1e12)
    dom = max((n for n in phases if n in kflops), key=lambda n: phases[n])
    k_bytes = kb[dom] / (hbm * 1e9)
    k_flops = kflops[dom] / (peak * 1e12)
    entry = {
        "workload": wl.name, "T": T, "format": wl.fmt,
        "path": ["none", "gemv", "tcgen05", "int4", "tcgen05_mx"][path] + variant,
        "tensor_peak_tflops": peak,
        "active_experts": kb["active_experts"], "reps": reps,
        "ms": ms, "ms_graph": ms_g, "self_pair_ms": [ms_a, ms_b],
        "self_pair_spread": abs(ms_a - ms_b) / min(ms_a, ms_b),
        "tokens_s": T / (ms * 1e-3), "tokens_s_graph": T / (ms_g * 1e-3),
        "tflops": flops / (ms * 1e-3) / 1e12, "packed_gbs": kb["packed_bytes"] / (ms * 1e-3) / 1e9,
        "bound": _bound_label(t_bytes, t_flops),
        "roofline_frac": max(t_bytes, t_flops) / (ms * 1e-3),
        "roofline_frac_graph": max(t_bytes, t_flops) / (ms_g * 1e-3),
        "dominant_kernel": dom, "dominant_ms": phases[dom],
        "dominant_bound": _bound_label(k_bytes, k_flops),
        "dominant_frac": max(k_bytes, k_flops) / (phases[dom] * 1e-3),
        "phases_ms": phases, "launches_per_call": launches,
    }
    return entry


def per_config_table(args, hbm, bf16, peak_src, layers, dev):
    """Every workload and token count of the build's configs, one entry each."""
    import torch
    from bit_grouped_moe_e4b_b200.configs import WORKLOADS

    flush = torch.empty(4 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    out = []
    for wl in WORKLOADS.values():
        layer = layers.get(wl.layer)
        if layer is None:
            layers.clear()
            torch.cuda.empty_cache()
            layer = layers[wl.layer] = build_layer(wl, dev)
        for T in wl.T:
            out.append(per_config_entry(wl, T, layer, args.reps, flush, hbm, bf16, peak_src))
        if wl.fmt == "mxfp4":
            # the same layer on the block-scaled FP4 MMA, at the token counts
            # that take the large-M path: two-term (bf16-exact) and one-term
            # (OCP MXFP8) activations
            from bit_grouped_moe_e4b_b200 import e4b

            mxl = layer.prepare_mx()
            plain = {r["T"]: r["path"] for r in out if r["workload"] == wl.name}
            for T in wl.T:
                if plain[T] != "tcgen05":
                    continue
                out.append(per_config_entry(wl, T, mxl, args.reps, flush, hbm, bf16, peak_src, 0, ""))
                out.append(per_config_entry(wl, T, mxl, args.reps, flush, hbm, bf16, peak_src,
                                            e4b.FLAG_MX_ACT_E4M3, "_e4m3"))
            del mxl
    del flush
    torch.cuda.empty_cache()
    return {"peaks": {"hbm_gbs": hbm, "bf16_tflops": bf16, "source": peak_src + " (burst)"},
            "timing": f"median of {args.reps} single calls, L2 flushed before each (a {4 * L2_BYTES >> 20} MiB "
                      "write); stream-launched and CUDA-graph replayed; self-pair = two independent stream "
                      "medians; roofline_frac = max(algorithmic bytes / HBM, FLOP / bf16 peak) / time",
            "rows": out}


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def oracle_tokens_sample(wl, T, ids, gates, x_h, tokens, packed=None):
    """Times the CPU oracle's layer (oracle.fast.moe_forward_sampled: per
    expert decode, fp64 matmuls, bf16 h, fp64 weighted sum) on `tokens` of the
    batch, with one thread per expert those tokens use, up to the host's cores.
    The experts are packed by the oracle before timing (pass `packed` to reuse
    them). Returns (seconds, threads, packed)."""
    import torch
    from oracle import fast
    from bit_grouped_moe_e4b_b200 import synth

    fast.build()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    need = sorted({int(ids[t, j]) for t in tokens for j in range(wl.top_k)})
    packed = dict(packed or {})
    for e in need:
        for which in ("gate_up", "down"):
            if (which, e) not in packed:
                packed[(which, e)] = fast.quantize(wl.fmt, synth.expert_weight(wl, which, e, dev).cpu().numpy())
    threads = min(len(need), host_cores())
    xf = x_h.float().numpy()
    t = time.perf_counter()
    fast.moe_forward_sampled(wl.fmt, xf, ids, gates, None, wl.E, wl.H, wl.I, list(tokens),
                             packed_fn=lambda which, e: packed[(which, e)], workers=threads)
    return time.perf_counter() - t, threads, packed


# ------------------------------------------------------------ CPU oracle
def run_dgrad(wl, T, steps, warmup, bf16, bf16_sus, peak_src):
    """Times the input gradients through the packed weights of both
    projections of the workload's layer on its routed rows (expert order):
    gate_up: dx [R, H] = dGU [R, 2I] . W_gu;  down: dh [R, I] = dO [R, H] . W_d.
    dy values are N(0, 1) rounded to bf16. Returns one JSON-ready dict."""
    import torch
    from bit_grouped_moe_e4b_b200 import e4b, synth

    dev = torch.device("cuda", torch.cuda.current_device())
    layer = build_layer(wl, dev)
    ids_h, _ = synth.routing(wl, T)
    _, offsets, _, _, _ = e4b.route(torch.from_numpy(ids_h).to(dev), wl.E)
    R = ids_h.size
    g = torch.Generator(device=dev).manual_seed(wl.seed + 7)
    d_gu = torch.randn((R, 2 * wl.I), generator=g, device=dev).to(torch.bfloat16)
    d_dn = torch.randn((R, wl.H), generator=g, device=dev).to(torch.bfloat16)
    dx = torch.empty((R, wl.H), dtype=torch.bfloat16, device=dev)
    dh = torch.empty((R, wl.I), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        e4b.e4b_grouped_dgrad(wl.fmt, layer.gate_up_codes, layer.gate_up_scales, d_gu, offsets, dx, E=wl.E,
                              N=2 * wl.I, K=wl.H, R_max=R)
        if ev:
            ev[1].record(stream)
        e4b.e4b_grouped_dgrad(wl.fmt, layer.down_codes, layer.down_scales, d_dn, offsets, dh, E=wl.E,
                              N=wl.H, K=wl.I, R_max=R)
        if ev:
            ev[2].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        step(ev[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / steps
    gu_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    dn_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))
    f_gu = 2.0 * R * 2 * wl.I * wl.H
    f_dn = 2.0 * R * wl.H * wl.I
    dom, dom_ms, dom_f = ("gate_up_dgrad", gu_ms, f_gu) if gu_ms >= dn_ms else ("down_dgrad", dn_ms, f_dn)
    achieved = dom_f / (dom_ms * 1e-3) / 1e12
    return {
        "metric": "grouped dgrad TFLOP/s (input gradients of both projections, packed weights)",
        "value": (f_gu + f_dn) / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": steps,
        "warmup": warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "T": T, "routed_rows": R, "format": wl.fmt, "E": wl.E, "H": wl.H,
                   "I": wl.I, "op": "dgrad", "l2": "no flush: packed weights exceed the 126 MB L2"},
        "phases_ms": {"gate_up_dgrad": gu_ms, "down_dgrad": dn_ms},
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
                     "frac": achieved / bf16, "peak_source": peak_src + " (burst)", "peak_sustained": bf16_sus,
                     "traffic": None, "algorithmic_flops": dom_f},
        "clocks": clk,
        "gpu_launches": 2 * steps,
    }


def run_int4(wl, steps, warmup, hbm, peak_src, cpu_baseline=True):
    """Times one token through the workload's layer on int4-b32 stacks (the
    same N(0, 0.02) fp32 weights, packed by e4b_quantize_int4_b32): the gate_up
    GEMV with the SwiGLU epilogue, then the down GEMV with the combine. Step i
    routes the token to the i-th of four disjoint expert pairs, so consecutive
    steps read different weights (no L2 reuse across steps). Returns one
    JSON-ready dict."""
    import torch
    from bit_grouped_moe_e4b_b200 import e4b, synth

    dev = torch.device("cuda", torch.cuda.current_device())
    E, H, I = wl.E, wl.H, wl.I
    stacks = []
    for which in ("gate_up", "down"):
        w = synth.layer_weights(wl, which, dev)
        stacks += list(e4b.quantize_int4_b32(w))
        del w
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    gc, gs, dc, ds = stacks
    x_h = synth.tokens_bf16(wl, 1)[0].contiguous()
    pairs = [[(2 * i + 1) % E, (2 * i) % E] for i in range(E // 2)]
    gates_h = np.array([0.62, 0.38], np.float32)
    ids_d = [torch.tensor(p, dtype=torch.int32, device=dev) for p in pairs]
    g_d = torch.from_numpy(gates_h).to(dev)
    x = x_h.to(dev)
    h = torch.empty((2, I), dtype=torch.bfloat16, device=dev)
    y = torch.empty((H,), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step(i, ev=None, xin=x, ids=None):
        ids = ids_d[i % len(ids_d)] if ids is None else ids
        if ev:
            ev[0].record(stream)
        e4b.e4b_gemv_int4_b32("swiglu", gc, gs, ids, xin, h, E=E, N=2 * I, K=H, ld_y=I)
        if ev:
            ev[1].record(stream)
        e4b.e4b_gemv_int4_b32("combine", dc, ds, ids, h, y, E=E, N=H, K=I, gates=g_d, ld_x=I,
                              flags=e4b.FLAG_IDS_READY)
        if ev:
            ev[2].record(stream)

    for i in range(max(warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for row in ev:
        for e_ in row:
            e_.record(stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    # a step takes less GPU time than its two host calls: a sleep kernel ahead
    # of the timed region lets the host queue every step first, so the events
    # time the GPU, not the host (the e2e number below keeps the host in).
    # The steps run back to back with no event between the launches (each
    # launch is a programmatic dependent of the one before); the per-kernel
    # times come from a second loop with events around each launch.
    torch.cuda._sleep(int(5e7))
    t0.record(stream)
    for i in range(steps):
        step(i)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    torch.cuda._sleep(int(5e7))
    for i in range(steps):
        step(i, ev[i])
    torch.cuda.synchronize()
    clk = clocks.stop()
    gu_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    dn_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))
    bpw = 0.5 + 2.0 / 32
    gu_bytes = 2 * 2 * I * H * bpw + 2 * H + 2 * 2 * I      # two experts' gate_up, x in, h out
    dn_bytes = 2 * H * I * bpw + 2 * 2 * I + 2 * H          # two experts' down, h in, y out
    dom, dom_ms, dom_b = ("int4_gemv_gate_up", gu_ms, gu_bytes) if gu_ms >= dn_ms else \
        ("int4_gemv_down", dn_ms, dn_bytes)
    achieved = dom_b / (dom_ms * 1e-3) / 1e9

    # end to end through the public layer call (e4b_moe_forward on the int4-b32
    # stacks, one call a step) with host buffers: x, ids and gates in from
    # pinned memory, y out, every step
    layer = e4b.PackedLayer("int4b32", E, H, I, gc, gs, dc, ds)
    ws = e4b.workspace(layer, 1, 2, dev)
    x_pin = x_h.reshape(1, H).pin_memory()
    ids_pin = [torch.tensor([p], dtype=torch.int32).pin_memory() for p in pairs]
    g_pin = torch.from_numpy(gates_h.reshape(1, 2)).pin_memory()
    y_pin = torch.empty((1, H), dtype=torch.bfloat16).pin_memory()
    xd = torch.empty((1, H), dtype=torch.bfloat16, device=dev)
    idd = torch.empty((1, 2), dtype=torch.int32, device=dev)
    gd = torch.empty((1, 2), dtype=torch.float32, device=dev)
    yd = torch.empty((1, H), dtype=torch.bfloat16, device=dev)

    def e2e_step(i):
        xd.copy_(x_pin, non_blocking=True)
        idd.copy_(ids_pin[i % len(ids_pin)], non_blocking=True)
        gd.copy_(g_pin, non_blocking=True)
        e4b.e4b_moe_forward(layer, xd, idd, gd, yd, ws)
        y_pin.copy_(yd, non_blocking=True)

    for i in range(max(warmup, 3)):
        e2e_step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / steps
    if e4b.e4b_read_device_status(ws) != 0:
        raise RuntimeError("device status set during the end-to-end loop")
    line = {
        "metric": "int4-b32 decode: packed-weight HBM GB/s of one token through the MoE layer (GEMVs)",
        "value": (gu_bytes + dn_bytes) / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": 1, "steps": steps,
        "warmup": max(warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8xint4->int32", "data": "synthetic",
        "tokens_per_s": 1.0 / (ms * 1e-3),
        "config": {"workload": wl.name + "_int4b32_T1", "format": "int4-b32 (fp16 scale per 32)", "E": E, "H": H,
                   "I": I, "top_k": 2, "op": "int4",
                   "routing": "step i: the i-th of four disjoint expert pairs, gates 0.62/0.38",
                   "l2": "no flush: each step reads two experts not read by the step before "
                         f"({(gu_bytes + dn_bytes) / 2 ** 20:.0f} MiB a step, 4 steps before a pair repeats)"},
        "phases_ms": {"int4_gemv_gate_up": gu_ms, "int4_gemv_down": dn_ms,
                      "_note": "each launch alone (events around it); the step overlaps them"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "peak_source": peak_src, "traffic": _traffic(wl.name + "_int4", dom),
                     "algorithmic_bytes": dom_b},
        "clocks": clk,
        "e2e": {"value": (gu_bytes + dn_bytes) / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "tokens_per_s": 1.0 / (e2e_ms * 1e-3),
                "h2d_bytes_per_step": x_h.numel() * 2 + 8 + 8, "d2h_bytes_per_step": H * 2},
        "gpu_launches": 2 * steps,
    }
    if cpu_baseline:
        from oracle import int4b32 as q4

        e_pair = pairs[0]
        gcs, gss, dcs, dss = [], [], [], []
        for e in e_pair:
            a, b = q4.quantize_int4b32(synth.expert_weight(wl, "gate_up", e, dev).cpu().numpy())
            gcs.append(a), gss.append(b)
            a, b = q4.quantize_int4b32(synth.expert_weight(wl, "down", e, dev).cpu().numpy())
            dcs.append(a), dss.append(b)
        gcs, gss, dcs, dss = np.stack(gcs), np.stack(gss), np.stack(dcs), np.stack(dss)
        tc = time.perf_counter()
        q4.int4b32_decode_layer_ref(x_h.float().numpy(), [0, 1], gates_h, gcs, gss, dcs, dss)
        secs = time.perf_counter() - tc
        line["cpu_baseline"] = {"value": (gu_bytes + dn_bytes) / secs / 1e9, "unit": "GB/s",
                                "tokens_per_s": 1.0 / secs, "cores": 1, "kind": "oracle",
                                "sample": "one token through the layer on one expert pair (numpy oracle, "
                                          "weights packed before timing)"}
    return line


def run_reference(args, wl, T):
    """The oracle as it stands, on the host cores: each step runs the layer on
    a sample of the batch's tokens (oracle_tokens_sample), the experts packed
    once before timing."""
    from bit_grouped_moe_e4b_b200 import synth

    x_h = synth.tokens_bf16(wl, T)
    ids, gates = synth.routing(wl, T)
    n = REF_TOKENS_PER_STEP.get(wl.name, 4)
    sample = lambda i: [(i * n + j) % T for j in range(n)]
    packed = None
    for i in range(args.warmup):
        _, threads, packed = oracle_tokens_sample(wl, T, ids, gates, x_h, sample(i), packed)
    # pack every expert before the timed steps
    all_tokens = sorted({t for i in range(args.warmup, args.warmup + args.steps) for t in sample(i)})
    need = sorted({int(ids[t, j]) for t in all_tokens for j in range(wl.top_k)})
    from oracle import fast
    import torch

    dev = "cuda" if torch.cuda.is_available() else "cpu"
    packed = dict(packed or {})
    for e in need:
        for which in ("gate_up", "down"):
            if (which, e) not in packed:
                packed[(which, e)] = fast.quantize(wl.fmt, synth.expert_weight(wl, which, e, dev).cpu().numpy())
    secs, thr = 0.0, 1
    for i in range(args.warmup, args.warmup + args.steps):
        dt, t_used, packed = oracle_tokens_sample(wl, T, ids, gates, x_h, sample(i), packed)
        secs += dt
        thr = max(thr, t_used)
    tokens = n * args.steps
    value = tokens / secs
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "T": T, "format": wl.fmt, "E": wl.E, "H": wl.H, "I": wl.I,
                   "top_k": wl.top_k},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                         "host_cores": host_cores(), "cpu": cpu_model(),
                         "sample": f"{n} tokens of the batch a step (every routed slot of each: decode of the "
                                   "experts they use, fp64 matmuls, bf16 h, fp64 weighted sum), one thread per "
                                   "expert (C core, no BLAS), weights packed before timing"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# tokens per reference step: a bounded sample (each step decodes every expert
# its tokens use, seconds of host work at the large shapes)
REF_TOKENS_PER_STEP = {"tiny_nf4_E8_H256_I512_top2": 64, "prefill_nf4_E8_H4096_I14336_top2": 4,
                       "decode_nf4_E8_H4096_I14336_top2": 4, "skewed_nf4_E128_H2048_I768_top8": 8,
                       "mxfp4_E32_H2880_I2880_top4": 8}
# tokens in the cpu_baseline sample of the default line
CPU_BASELINE_TOKENS = 32


def main():
    args = _args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from bit_grouped_moe_e4b_b200.configs import WORKLOADS

    wl = WORKLOADS[args.workload]
    T = args.T or (DEFAULT_T if args.workload == DEFAULT_WORKLOAD else wl.T[-1])

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl, T)
        return

    import torch
    from bit_grouped_moe_e4b_b200 import build as builder

    builder.build()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    hbm, bf16, bf16_sus, peak_src = _peaks()

    if args.op == "dgrad":
        line = run_dgrad(wl, T, args.steps, args.warmup, bf16, bf16_sus, peak_src)
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    if args.op == "int4":
        line = run_int4(wl, args.steps, args.warmup, hbm, peak_src,
                        cpu_baseline=not args.no_cpu_baseline and rank == 0)
        if rank == 0:
            print(json.dumps(line), flush=True)
        return

    cases = [(wl, T)]
    if args.sweep:
        cases = [(w, t) for w in WORKLOADS.values() for t in w.T]
    layers = {}
    dev = torch.device("cuda", local)
    for wl_i, T_i in cases:
        if wl_i.layer not in layers:
            layers.clear()
            torch.cuda.empty_cache()
            layers[wl_i.layer] = build_layer(wl_i, dev)
        flags = 0
        lay = layers[wl_i.layer]
        if args.mx != "off" and wl_i.fmt == "mxfp4":
            from bit_grouped_moe_e4b_b200 import e4b as _e4b

            lay = lay.prepare_mx()
            flags = _e4b.FLAG_FORCE_TCGEN05 | (_e4b.FLAG_MX_ACT_E4M3 if args.mx == "e4m3" else 0)
        r = run_gpu(wl_i, T_i, args.steps, args.warmup, rank, world, dist, layer=lay, flags=flags)
        kb = kernel_bytes(wl_i, T_i, r["ids"])
        dominant = max((k for k in r["phases"] if not k.startswith("route") and not k.startswith("_")),
                       key=lambda k: r["phases"][k])
        dur_s = r["phases"][dominant] * 1e-3
        step_s = r["ms"] * 1e-3 / args.steps
        tokens_s = world * T_i / step_s
        flops = 2.0 * r["ids"].size * 3 * wl_i.H * wl_i.I
        key = f"{wl_i.name}_T{T_i}"
        line = {
            "metric": METRIC, "value": tokens_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl_i.name, "T": T_i, "format": wl_i.fmt, "E": wl_i.E,
                       "H": wl_i.H, "I": wl_i.I, "top_k": wl_i.top_k,
                       "active_experts": kb["active_experts"],
                       "path": ["none", "gemv", "tcgen05", "int4", "tcgen05_mx"][r["path"]]
                       + ("_e4m3" if args.mx == "e4m3" and r["path"] == 4 else ""),
                       "weights": "N(0,0.02) fp32 packed on the GPU by e4b_quantize_*",
                       "l2": "no flush: packed weights of the active experts "
                             f"({kb['packed_bytes'] / 2 ** 20:.0f} MiB) exceed the 126 MB L2",
                       "parallelism": f"replicas x{world}, token batches per GPU"},
            "packed_gbs": kb["packed_bytes"] / step_s / 1e9,
            "layer_frac_of_hbm": (kb["layer"] / step_s / 1e9) / hbm,
            "tflops": flops / step_s / 1e12,
            "phases_ms": r["phases"],
            "roofline": _roofline(r["path"], dominant, kb, dur_s, wl_i, r["ids"], key, hbm,
                                  bf16, bf16_sus, peak_src,
                                  power_capped="sw_power_cap" in r["clocks"].get("reasons", [])),
            "clocks": r["clocks"],
            "e2e": {"value": world * T_i / (r["e2e_ms"] * 1e-3 / args.steps), "unit": "tokens/s",
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                    "copies": "pipelined: step i+1's upload and step i-1's download overlap step i "
                              "(two copy streams, double-buffered device inputs and outputs)",
                    "serial_value": world * T_i / (r["e2e_serial_ms"] * 1e-3 / args.steps)},
            "gpu_launches": r["launches"],
        }
        if not args.sweep and not args.no_per_config and world == 1:
            line["per_config"] = per_config_table(args, hbm, bf16, peak_src, layers, dev)
        if (not args.sweep and rank == 0 and world == 1 and not args.no_cpu_baseline):
            ntok = min(CPU_BASELINE_TOKENS, T_i)
            secs, threads, _ = oracle_tokens_sample(wl_i, T_i, r["ids"], r["gates"], r["x"], list(range(ntok)))
            line["cpu_baseline"] = {
                "value": ntok / secs, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                "host_cores": host_cores(), "cpu": cpu_model(), "seconds": secs,
                "sample": f"tokens 0..{ntok - 1} of the batch (all their routed slots: decode of the experts "
                          "they use, fp64 matmuls, bf16 h, fp64 weighted sum); one thread per expert, "
                          "C core without BLAS; weights packed before timing"}
        if rank == 0:
            print(json.dumps(line), flush=True)
        del r
        torch.cuda.empty_cache()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
