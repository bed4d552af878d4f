"""The five synthetic MoE-layer workloads: shapes, formats and input recipes.

Each entry fixes the expert stack (E experts, hidden H, intermediate I,
top-k), the 4-bit format, the token counts to run and how router logits are
drawn. Weights are N(0, 0.02) fp32 quantised per expert; x is N(0, 1) rounded
to bf16. Workloads that share a ``layer`` name share their weights.
"""

from dataclasses import dataclass, field
from typing import List


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int  # seeds the token / router streams
    layer: str  # seeds the weight streams; equal names share weights
    fmt: str  # "nf4" or "mxfp4"
    E: int
    H: int
    I: int
    top_k: int
    T: List[int] = field(default_factory=list)
    logits: str = "normal"  # "normal" N(0,1) or "uniform" U[0,1)
    bias_sigma: float = 0.0  # per-expert logit bias N(0, sigma), 0 = none
    weight_std: float = 0.02

    @property
    def weights_per_expert(self) -> int:
        return 3 * self.H * self.I


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_nf4_E8_H256_I512_top2", 1, "nf4_E8_H256_I512", "nf4", 8, 256, 512, 2, [64]),
        Workload("decode_nf4_E8_H4096_I14336_top2", 2, "nf4_E8_H4096_I14336", "nf4", 8, 4096, 14336, 2,
                 [1, 4, 16]),
        Workload("prefill_nf4_E8_H4096_I14336_top2", 3, "nf4_E8_H4096_I14336", "nf4", 8, 4096, 14336, 2,
                 [4096], logits="uniform"),
        Workload("skewed_nf4_E128_H2048_I768_top8", 4, "nf4_E128_H2048_I768", "nf4", 128, 2048, 768, 8,
                 [8192], bias_sigma=1.5),
        Workload("mxfp4_E32_H2880_I2880_top4", 5, "mxfp4_E32_H2880_I2880", "mxfp4", 32, 2880, 2880, 4,
                 [16, 512, 8192]),
    ]
}

TINY = WORKLOADS["tiny_nf4_E8_H256_I512_top2"]
DECODE = WORKLOADS["decode_nf4_E8_H4096_I14336_top2"]
PREFILL = WORKLOADS["prefill_nf4_E8_H4096_I14336_top2"]
SKEWED = WORKLOADS["skewed_nf4_E128_H2048_I768_top8"]
MXFP4 = WORKLOADS["mxfp4_E32_H2880_I2880_top4"]
