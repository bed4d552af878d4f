"""CPU oracle for the packed-4-bit MoE layer (NF4 / MXFP4 fused expert stacks).

TEST INFRASTRUCTURE ONLY. This package is the plain, slow, obviously correct
reference that the CUDA library is checked against. Only the test suite, the
smoke check in ``__graft_entry__`` and the ``cpu_baseline`` / ``--impl
reference`` legs of ``bench.py`` may import it. The product path (the C-ABI
library and its Python binding) never imports, calls or links anything here,
and nothing here imports the product path: the two share no code, no tables
and no constants. Inputs common to both come from the seeded generators in
``bit_grouped_moe_e4b_b200.synth``, which hold none of the method's arithmetic.

Everything is numpy, in fp64 unless a step is defined in fp32 (the NF4
normalisation ``w / absmax`` and the decoded-weight product, which the method
performs in fp32).

Sources (page titles; sections):
  * "grouped-nf4-gemm" README, intro and "Try it on CPU right now" blocks 1-2:
    NF4 pack/decode (``quantize_pack_nf4``, ``dequant_ref``), MXFP4 pack/decode
    (``quantize_pack_mxfp4``, ``dequant_mxfp4``), the one-launch grouped GEMM
    over all active experts with LUT decode, blockwise scale, fp32
    accumulation and bf16 epilogue.
  * bitsandbytes PR #1984 "Experts4bit", Summary / Design / Benchmark Results:
    per-expert quantisation with per-expert absmax, the per-expert dequantise
    loop, the gated SiLU (SwiGLU) activation, MAE / RMSE of NF4.
  * "How do I run a single-token INT4 decode GEMV over routed MoE experts, and
    pack calibrated (GPTQ) weights for it?" (grouped-nf4-gemm solutions page):
    the int4-b32 decode GEMV with exact integer accumulation and the GPTQ
    packer (module ``int4b32``).
  * OCP Microscaling v1.0 MXFP8 (E4M3 elements, e8m0 scale per 32): the
    activations of the layer on the block-scaled FP4 MMA (module ``mxfp8``,
    ``moe_forward_ref(..., act_quant="mxfp8")``).
  * "experts4bit-qlora" README: fused ``gate_up_proj [E, 2I, H]`` and
    ``down_proj [E, H, I]`` expert stacks (transformers v5 layout).

Parity status per function is stated in each module's header.
"""

from .formats import (
    NF4_BLOCK,
    MXFP4_BLOCK,
    E2M1_MAGNITUDES,
    bf16_round,
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    nf4_codebook,
    quantize_pack_nf4,
    unpack_nf4_codes,
    dequant_ref,
    dequant_ref_exact,
    dequant_ref_level,
    quantize_pack_mxfp4,
    unpack_mxfp4_codes,
    dequant_mxfp4,
    packed_bytes_per_weight,
)
from .moe import (route_ref, moe_forward_ref, swiglu_ref, expert_tokens, clamped_glu_ref,
                  split_gate_up, activation_ref, grouped_projection_ref, grouped_dgrad_ref)
from . import int4b32
from . import mxfp8

__all__ = [
    "NF4_BLOCK", "MXFP4_BLOCK", "E2M1_MAGNITUDES",
    "bf16_round", "bf16_bits_from_f32", "f32_from_bf16_bits",
    "nf4_codebook", "quantize_pack_nf4", "unpack_nf4_codes", "dequant_ref",
    "dequant_ref_exact", "dequant_ref_level", "quantize_pack_mxfp4", "unpack_mxfp4_codes",
    "dequant_mxfp4", "packed_bytes_per_weight",
    "route_ref", "moe_forward_ref", "swiglu_ref", "expert_tokens", "clamped_glu_ref", "split_gate_up",
    "activation_ref", "grouped_projection_ref", "grouped_dgrad_ref", "int4b32", "mxfp8",
]
