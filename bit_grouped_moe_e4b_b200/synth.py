"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no quantisation, decode, routing permutation, GEMM or
activation). Token-side streams are numpy PCG64 generators keyed by
SeedSequence([seed, T, stream]); weights come from torch's generator seeded
from SeedSequence([hash(layer), stream, expert]), so one expert's weights can
be regenerated on their own, on the device that uses them.

Streams: 0 = x, 1 = router logits, 2 = per-expert logit bias, 3 = gate_up
weights, 4 = down weights.

The router's top-k choice and its softmax over the chosen k logits belong to
the model's router, not to this layer: the layer takes expert ids and gate
weights as inputs. They are produced here so that both sides receive the
same ids and gates.
"""

from __future__ import annotations

import zlib

import numpy as np
import torch

from .configs import Workload

X_STREAM, LOGIT_STREAM, BIAS_STREAM, GATE_UP_STREAM, DOWN_STREAM = 0, 1, 2, 3, 4


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _layer_key(layer: str) -> int:
    return zlib.crc32(layer.encode())


def _weight_seed(wl: Workload, stream: int, e: int) -> int:
    ss = np.random.SeedSequence([_layer_key(wl.layer), stream, e])
    return int(ss.generate_state(1, np.uint64)[0] & np.uint64(0x7FFFFFFFFFFFFFFF))


def expert_weight(wl: Workload, which: str, e: int, device="cpu") -> torch.Tensor:
    """fp32 weights of expert e: "gate_up" [2I, H] or "down" [H, I], N(0, std).

    Drawn by torch's seeded generator on `device` (Philox on a GPU), so
    full-size stacks are generated where they are used; a test hands the
    oracle a host copy of the very same tensor. The values depend on the
    device's generator, not only on the seed."""
    if which == "gate_up":
        shape, stream = (2 * wl.I, wl.H), GATE_UP_STREAM
    elif which == "down":
        shape, stream = (wl.H, wl.I), DOWN_STREAM
    else:
        raise ValueError(which)
    g = torch.Generator(device=device)
    g.manual_seed(_weight_seed(wl, stream, e))
    w = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return w * wl.weight_std


def layer_weights(wl: Workload, which: str, device="cpu") -> torch.Tensor:
    """The stacked fp32 weights [E, ...] of one projection."""
    return torch.stack([expert_weight(wl, which, e, device) for e in range(wl.E)])


def tokens_bf16(wl: Workload, T: int) -> torch.Tensor:
    """x [T, H]: N(0, 1) drawn in fp32, rounded to bf16 (CPU tensor)."""
    g = _rng(wl.seed, T, X_STREAM)
    x = g.standard_normal((T, wl.H), dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16)


def router_logits(wl: Workload, T: int) -> np.ndarray:
    g = _rng(wl.seed, T, LOGIT_STREAM)
    if wl.logits == "normal":
        logits = g.standard_normal((T, wl.E), dtype=np.float32)
    elif wl.logits == "uniform":
        logits = g.random((T, wl.E), dtype=np.float32)
    else:
        raise ValueError(wl.logits)
    if wl.bias_sigma:
        b = _rng(wl.seed, BIAS_STREAM).standard_normal(wl.E, dtype=np.float32)
        logits = logits + b * np.float32(wl.bias_sigma)
    return logits


def topk_route(logits: np.ndarray, k: int):
    """Router stand-in: the k largest logits per token (ties to the lower
    expert index, slots in descending logit order) and a softmax over those k
    logits (fp64, stored fp32). Returns (ids int32 [T, k], gates fp32 [T, k])."""
    T, E = logits.shape
    order = np.argsort(-logits.astype(np.float64), axis=1, kind="stable")[:, :k]
    chosen = np.take_along_axis(logits.astype(np.float64), order, axis=1)
    z = np.exp(chosen - chosen.max(axis=1, keepdims=True))
    gates = (z / z.sum(axis=1, keepdims=True)).astype(np.float32)
    return order.astype(np.int32), gates


def routing(wl: Workload, T: int):
    return topk_route(router_logits(wl, T), wl.top_k)


def random_ids(rng: np.random.Generator, T: int, k: int, E: int, skew: float = 0.0):
    """Arbitrary ids (duplicates within a token allowed) and positive gates,
    for edge-case tests of the layer beyond what a router produces."""
    if skew:
        p = rng.dirichlet(np.full(E, skew))
        ids = rng.choice(E, size=(T, k), p=p)
    else:
        ids = rng.integers(0, E, size=(T, k))
    gates = rng.random((T, k), dtype=np.float32)
    return ids.astype(np.int32), gates
