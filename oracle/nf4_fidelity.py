"""Fidelity of the two NF4 decode readings against the exact decode (test
infrastructure: plain numpy, CPU only, imports nothing from the CUDA side).

The tensor cores take bf16 operands, so a bf16 rounding has to fall
somewhere in the NF4 decode ("grouped-nf4-gemm" README, intro: table decode,
blockwise scaling; its measured table row "Fidelity, fused vs
dequantise-to-bf16"). The oracle implements both readings:
  "product"  bf16_rne(fp32(level * absmax))
  "level"    bf16_rne(level) * absmax (exact)
and the exact value level * absmax ("exact", fp64). This script measures how
far each reading's decoded weights, and the layer outputs computed from them,
lie from the exact decode:

  python -m oracle.nf4_fidelity [--full]

Weight level: relative RMS error and maximum relative error over nonzero
weights, on N(0, 0.02) weights [512, 4096]. Layer level: max |y - y_exact| /
(1 + |y_exact|) and RMS(y - y_exact) / RMS(y_exact) on (a) the block-scale
test layer (E=3, H=256, I=320, weights N(0, 0.06) with power-of-two block
spread, 40 tokens, top-2), (b) an O(1)-output test layer (E=8, H=256, I=512,
64 tokens, top-2) and, with --full, (c) the decode workload (E=8, H=4096,
I=14336, top-2, T=16; CPU-drawn weights of the same distribution).
"""

from __future__ import annotations

import argparse
import sys

import numpy as np

from .formats import (bf16_round, dequant_ref, dequant_ref_exact, dequant_ref_level, quantize_pack_nf4)
from .moe import moe_forward_ref

MODES = ("level", "product")


def weight_errors(seed: int = 0, N: int = 512, K: int = 4096, std: float = 0.02) -> dict:
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((N, K)) * std).astype(np.float32)
    codes, absmax = quantize_pack_nf4(w)
    ex = dequant_ref_exact(codes, absmax, N, K)
    dec = {"level": dequant_ref_level(codes, absmax, N, K),
           "product": dequant_ref(codes, absmax, N, K).astype(np.float64)}
    nz = ex != 0
    out = {}
    for m in MODES:
        rel = (dec[m] - ex)[nz] / ex[nz]
        out[m] = {"rel_rms": float(np.sqrt(np.mean(rel ** 2))), "rel_max": float(np.abs(rel).max())}
    return out


def _spread(rng, w):
    E, N, K = w.shape
    f = np.exp2(rng.integers(-2, 3, size=(E, N, K // 32))).astype(np.float32)
    return (w.reshape(E, N, K // 32, 32) * f[..., None]).reshape(E, N, K)


def _random_routing(rng, T, k, E):
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    g = rng.random((T, k))
    return ids, (g / g.sum(1, keepdims=True)).astype(np.float32)


def layer_errors(E, H, I, T, k, seed, std_gu, std_dn, spread=False, weights=None) -> dict:
    rng = np.random.default_rng(seed)
    if weights is None:
        wgu = (rng.standard_normal((E, 2 * I, H)) * std_gu).astype(np.float32)
        wd = (rng.standard_normal((E, H, I)) * std_dn).astype(np.float32)
        if spread:
            wgu, wd = _spread(rng, wgu), _spread(rng, wd)
    else:
        wgu, wd = weights
    gc, gs = quantize_pack_nf4(wgu)
    dc, ds = quantize_pack_nf4(wd)
    x = bf16_round(rng.standard_normal((T, H)))
    ids, gates = _random_routing(rng, T, k, E)
    y = {m: moe_forward_ref("nf4", x, ids, gates, gc, gs, dc, ds, E, H, I, nf4_decode=m)
         for m in ("exact",) + MODES}
    ex = y["exact"]
    r = float(np.sqrt(np.mean(ex ** 2)))
    out = {"rms_y": r}
    for m in MODES:
        d = y[m] - ex
        out[m] = {"max_scaled": float(np.max(np.abs(d) / (1.0 + np.abs(ex)))),
                  "rel_rmse": float(np.sqrt(np.mean(d ** 2)) / r)}
    d = y["level"] - y["product"]
    out["level_vs_product_max_scaled"] = float(np.max(np.abs(d) / (1.0 + np.abs(y["product"]))))
    return out


def decode_workload_errors() -> dict:
    import torch

    sys.path.insert(0, __file__.rsplit("/oracle/", 1)[0])
    from bit_grouped_moe_e4b_b200 import synth
    from bit_grouped_moe_e4b_b200.configs import DECODE

    wl = DECODE
    wgu = synth.layer_weights(wl, "gate_up", "cpu").numpy()
    wd = synth.layer_weights(wl, "down", "cpu").numpy()
    del torch
    return layer_errors(wl.E, wl.H, wl.I, 16, wl.top_k, seed=16, std_gu=None, std_dn=None, weights=(wgu, wd))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--full", action="store_true", help="also the decode workload at full size (minutes)")
    a = ap.parse_args(argv)
    print("weights N(0,0.02) [512,4096]:", weight_errors())
    print("block-scale layer E3 H256 I320 T40:",
          layer_errors(3, 256, 320, 40, 2, seed=42, std_gu=0.06, std_dn=0.06, spread=True))
    print("O(1) layer E8 H256 I512 T64:",
          layer_errors(8, 256, 512, 64, 2, seed=7, std_gu=1.5 / 16, std_dn=2.0 / np.sqrt(512)))
    if a.full:
        print("decode workload E8 H4096 I14336 T16:", decode_workload_errors())


if __name__ == "__main__":
    main()
