"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no quantisation, decode, routing permutation, GEMM or
activation). Every stream is a numpy PCG64 generator keyed by
SeedSequence([seed, T, stream]) for token-side data and
SeedSequence([hash(layer), stream, expert]) for weights, so one expert's
weights can be regenerated on their own.

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


def expert_weight(wl: Workload, which: str, e: int) -> np.ndarray:
    """fp32 weights of expert e: "gate_up" [2I, H] or "down" [H, I], N(0, std)."""
    if which == "gate_up":
        shape, stream = (2 * wl.I, wl.H), GATE_UP_STREAM
    elif which == "down":
        shape, stream = (wl.H, wl.I), DOWN_STREAM
    else:
        raise ValueError(which)
    g = _rng(_layer_key(wl.layer), stream, e)
    return g.standard_normal(shape, dtype=np.float32) * np.float32(wl.weight_std)


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
