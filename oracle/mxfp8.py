"""Oracle: MXFP8 activations (OCP e4m3 elements, one e8m0 scale per 32 along
K) for the layer run on Blackwell's block-scaled FP4 MMA (test
infrastructure only).

Why it exists: the "grouped-nf4-gemm" README (intro) takes MXFP4 as OCP e2m1
codes with e8m0 scales; a native block-scaled tensor-core MMA multiplies
those codes directly, and its other operand must be an 8-, 6- or 4-bit
block-scaled format too -- bf16 activations are not accepted. The pages say
nothing of activation precision, so the plainest reading (and the only
one this module implements) is the OCP Microscaling v1.0 MXFP8 format with
E4M3 elements:

  * E4M3 (OCP 8-bit Floating Point Specification, E4M3): sign, 4 exponent
    bits with bias 7, 3 mantissa bits. Normal values (1 + m/8) * 2^(e-7) for
    e = 1..15, except the pattern S.1111.111, which is NaN; subnormals
    (m/8) * 2^-6. Largest finite magnitude 448, smallest 2^-9. No infinity.
  * conversion of a real v: to the nearest E4M3 value, ties to the even
    mantissa; magnitudes beyond 448 saturate to 448 (the saturating
    conversion of the MX spec's "clamp" option); the sign of v is kept.
  * MXFP8 block of 32 consecutive values along K: amax = max |v|; shared
    exponent X = floor(log2 amax) - 8 (8 = the largest E4M3 exponent),
    clamped to [-127, 127]; scale byte X + 127; element i = e4m3(v_i / 2^X).
    amax == 0: scale byte 0 and zero elements.
  * decoded value: element * 2^(byte - 127).

The layer in this reading (``moe.moe_forward_ref(..., act_quant="mxfp8")``):
x rows are replaced by their MXFP8 decode before the gate_up matmul, and the
bf16 intermediate h by its MXFP8 decode before the down matmul; everything
else is the plain layer.

Parity pins (tests/test_oracle_mxfp8.py): the E4M3 value set built from the
bit fields (254 finite values, 448, 2^-6, 2^-9); the rounding against a
nearest-value search over that set with ties to the even code, and against
torch's float8_e4m3fn conversion inside the finite range; the saturation;
hand-worked MXFP8 blocks (tests/golden/mxfp8_handworked.txt); the layer
against pure-Python loops (oracle/brute.py) on tiny shapes.
"""

from __future__ import annotations

import numpy as np

MXFP8_BLOCK = 32
E4M3_MAX = 448.0
E4M3_EMAX = 8


def e4m3_values() -> np.ndarray:
    """The 256 E4M3 bit patterns decoded (fp64; NaN for S.1111.111)."""
    out = np.empty(256, np.float64)
    for b in range(256):
        s = -1.0 if b & 0x80 else 1.0
        e = (b >> 3) & 0xF
        m = b & 0x7
        if e == 0xF and m == 0x7:
            out[b] = np.nan
        elif e == 0:
            out[b] = s * (m / 8.0) * 2.0 ** -6
        else:
            out[b] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


def e4m3_round(v) -> np.ndarray:
    """Nearest E4M3 value of each entry (fp64 in, fp64 out), ties to the even
    mantissa, saturating at +-448; signs kept."""
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    # quantum: 2^(e - 3) in the binade [2^e, 2^(e+1)) for e >= -6, else 2^-9
    _, ex = np.frexp(np.where(a > 0, a, 1.0))  # a = f 2^ex, f in [0.5, 1)
    e = ex - 1
    q = np.exp2(np.maximum(e, -6) - 3)
    r = np.rint(a / q) * q  # a / q is exact (q is a power of two); rint ties to even
    r = np.minimum(r, E4M3_MAX)
    r = np.where(a > 0, r, 0.0)
    return np.copysign(r, v)


def quantize_mxfp8(v):
    """[..., K] (K % 32 == 0) -> (elements fp64 [..., K] holding E4M3 values,
    scale bytes uint8 [..., K/32])."""
    v = np.asarray(v, np.float64)
    K = v.shape[-1]
    assert K % MXFP8_BLOCK == 0
    b = v.reshape(*v.shape[:-1], K // MXFP8_BLOCK, MXFP8_BLOCK)
    amax = np.abs(b).max(axis=-1)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))
    X = np.clip(ex - 1 - E4M3_EMAX, -127, 127)
    elems = e4m3_round(b / np.exp2(X)[..., None])
    elems = np.where((amax > 0)[..., None], elems, 0.0)
    byte = np.where(amax > 0, X + 127, 0).astype(np.uint8)
    return elems.reshape(v.shape), byte


def dequant_mxfp8(elems, scale_bytes) -> np.ndarray:
    e = np.asarray(elems, np.float64)
    K = e.shape[-1]
    s = np.exp2(np.asarray(scale_bytes, np.float64) - 127.0)
    return (e.reshape(*e.shape[:-1], K // MXFP8_BLOCK, MXFP8_BLOCK) * s[..., None]).reshape(e.shape)


def mxfp8_round_trip(v) -> np.ndarray:
    """The MXFP8 decode of the MXFP8 quantisation of v (fp64)."""
    return dequant_mxfp8(*quantize_mxfp8(v))
