"""Oracle: the two 4-bit weight formats and bf16 rounding (test infrastructure only).

Definitions followed
--------------------
NF4 ("grouped-nf4-gemm" README, intro: "NF4 on the bitsandbytes gemm_4bit
layout"; CPU block 1: ``quantize_pack_nf4(w) -> packed [N, K/2] uint8,
absmax [N, K/64] fp32`` and ``dequant_ref(packed, absmax, N, K)``;
bitsandbytes PR #1984, Summary/Design: every expert quantised on its own with
per-expert fp32 absmax):

  * codebook: the 16-value NormalFloat table of the QLoRA paper (Dettmers et
    al. 2023, Sec. 3 "4-bit NormalFloat"), built here from its construction:
    8 positive levels are the standard-normal quantiles at 9 evenly spaced
    probabilities from ``offset`` down to 0.5 (the last, 0.5, dropped), 7
    negative levels are minus the quantiles at 8 such probabilities (last
    dropped), plus an exact zero; sorted and divided by the largest value.
    Reading: the offset is the printed 0.9677083 and the grid points are
    fp32 (this reproduces the published fp32 table bit for bit; the exact
    offset 1 - (1/30 + 1/32)/2 does not).
  * quantise, per row and per 64-weight block along K: ``a = max |w|``;
    ``s = fp32(w / a)``; code = the codebook index nearest to ``s`` (exact
    distance; ties go to the lower index). ``a == 0`` gives code 7 (the zero
    level) for the whole block. Pack two codes per byte, the first element of
    each pair in the HIGH nibble.
  * decode (the README's kernel decodes to fp32 in registers and applies the
    blockwise scale; the tensor cores take bf16 operands, so the reading
    fixes where the one bf16 rounding falls -- two ways, both within 2^-8
    relative of ``c[code] * a``):
      - ``dequant_ref`` ("product"): ``bf16_rne(fp32(c[code]) * a)`` (the
        product rounded to fp32, then once to bf16);
      - ``dequant_ref_level`` ("level"): ``bf16_rne(c[code]) * a``, the exact
        product of the bf16-rounded level and the fp32 absmax (the operand is
        the rounded level; the scale multiplies the block's partial sum).
    ``dequant_ref_exact`` returns ``c[code] * a`` in fp64, used for fidelity
    reports only.

MXFP4 (README intro: "MXFP4 (OCP e2m1 + e8m0)"; CPU block 2:
``quantize_pack_mxfp4(w) -> blocks [N, K/32, 16] u8, scales [N, K/32] u8``;
the OCP Microscaling Formats v1.0 spec fixes e2m1 and e8m0):

  * per 32-weight block along K: ``amax = max |w|``; shared exponent
    ``e = floor(log2 amax) - 2`` clamped to [-127, 127]; scale byte
    ``e + 127``; each element ``w / 2^e`` rounded to the nearest e2m1
    magnitude {0, .5, 1, 1.5, 2, 3, 4, 6} with ties to the even code,
    saturating at 6; the sign bit copies the sign bit of w (so -0.0 and
    negative values that round to zero keep it). ``amax == 0`` gives scale byte 0
    and all-zero codes. Pack two codes per byte, first element in the LOW
    nibble.
  * decode: ``sign * magnitude * 2^(byte - 127)``; byte 255 is NaN (e8m0).
    These values are exact in bf16, so one decode serves parity and
    fidelity.

bf16 rounding: IEEE round-to-nearest-even to 8 significant bits, with bf16's
subnormals (quantum 2^-133) and overflow to infinity.

Parity pins (tests, ``-m "not gpu"``): the codebook equals the published
QLoRA table bit for bit; NF4 MAE / RMSE on N(0,1) at block 64 match PR
#1984's 0.073 / 0.092; round-trip relative errors match the README's ~0.09 /
~0.12; the example shapes; re-pack idempotence; byte accounting 0.5625
B/weight (~28% of fp16); hand-worked MXFP4 blocks; brute-force quantisers.
Unpinned by the pages (readings, listed above): the nibble orders, the
tie-breaks, the MXFP4 scale rule beyond the OCP spec.
"""

from __future__ import annotations

import numpy as np
from scipy.stats import norm

NF4_BLOCK = 64
MXFP4_BLOCK = 32
NF4_OFFSET = 0.9677083

# e2m1 magnitudes indexed by the 3-bit magnitude code (OCP MX v1.0, FP4 E2M1).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)

_BF16_MAX = float.fromhex("0x1.fep127")  # largest finite bf16


# --------------------------------------------------------------------------
# bf16 rounding
# --------------------------------------------------------------------------
def bf16_round(v) -> np.ndarray:
    """Round real values (any float dtype, taken exactly as fp64) to bf16.

    Round-to-nearest-even at 8 significant bits; below 2^-126 the quantum is
    fixed at 2^-133 (bf16 subnormals); results beyond the largest finite bf16
    become +-inf. Returns fp64 holding the bf16 values.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.empty_like(v)
    finite = np.isfinite(v)
    out[~finite] = v[~finite]
    vf = v[finite]
    _, e = np.frexp(vf)  # vf = m * 2^e with 0.5 <= |m| < 1
    q = np.maximum(e, -125) - 8  # exponent of the bf16 quantum at this magnitude
    r = np.rint(np.ldexp(vf, -q))  # np.rint rounds half to even
    res = np.ldexp(r, q)
    res = np.where(np.abs(res) > _BF16_MAX, np.copysign(np.inf, vf), res)
    out[finite] = res
    return out


def bf16_bits_from_f32(x) -> np.ndarray:
    """bf16 bit patterns (uint16) of fp32 values rounded to nearest even."""
    x = np.asarray(x, dtype=np.float32)
    r = bf16_round(x.astype(np.float64)).astype(np.float32)  # exact: bf16 is a subset of fp32
    bits = (r.view(np.uint32) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    bits[nan] = 0x7FC0
    return bits


def f32_from_bf16_bits(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# NF4
# --------------------------------------------------------------------------
def _fp32_grid(start: float, stop: float, n: int) -> np.ndarray:
    """n evenly spaced fp32 points from start to stop, each computed in fp32
    from whichever end is nearer (so both ends are hit exactly)."""
    a = np.float32(start)
    b = np.float32(stop)
    step = np.float32((b - a) / np.float32(n - 1))
    pts = []
    for i in range(n):
        if i < n // 2:
            pts.append(np.float32(a + step * np.float32(i)))
        else:
            pts.append(np.float32(b - step * np.float32(n - 1 - i)))
    return np.array(pts, dtype=np.float32)


def nf4_codebook() -> np.ndarray:
    """The 16 NormalFloat levels (fp32, ascending); index 7 is exactly 0."""
    pos = norm.ppf(_fp32_grid(NF4_OFFSET, 0.5, 9)[:-1].astype(np.float64))
    neg = -norm.ppf(_fp32_grid(NF4_OFFSET, 0.5, 8)[:-1].astype(np.float64))
    levels = np.concatenate([pos, [0.0], neg]).astype(np.float32)
    levels = np.sort(levels)
    return (levels / levels.max()).astype(np.float32)


def _nearest_nf4(s: np.ndarray, cb: np.ndarray) -> np.ndarray:
    """Index of the nearest codebook level to fp32 values s, ties to the lower
    index, decided exactly: s is nearer to c[i+1] than to c[i] iff
    2 s > c[i] + c[i+1], and fp64 holds that sum of two fp32 values exactly."""
    sums = cb[:-1].astype(np.float64) + cb[1:].astype(np.float64)
    two_s = 2.0 * s.astype(np.float64)
    # number of boundaries strictly below 2s
    return np.searchsorted(sums, two_s, side="left").astype(np.uint8)


def quantize_pack_nf4(w, blocksize: int = NF4_BLOCK):
    """Quantise fp32 weights [..., N, K] to NF4.

    Returns (packed uint8 [..., N, K/2], absmax fp32 [..., N, K/blocksize]).
    Blocks run along K and never straddle rows or experts.
    """
    w = np.asarray(w, dtype=np.float32)
    K = w.shape[-1]
    if K % blocksize or blocksize % 2:
        raise ValueError("K must be a multiple of the (even) blocksize")
    cb = nf4_codebook()
    wb = w.reshape(*w.shape[:-1], K // blocksize, blocksize)
    absmax = np.max(np.abs(wb), axis=-1)
    zero = absmax == 0
    safe = np.where(zero, np.float32(1), absmax).astype(np.float32)
    s = (wb / safe[..., None]).astype(np.float32)  # IEEE fp32 division
    codes = _nearest_nf4(s, cb)
    codes[zero] = 7
    codes = codes.reshape(w.shape)
    packed = ((codes[..., 0::2] << 4) | codes[..., 1::2]).astype(np.uint8)
    return packed, absmax.astype(np.float32)


def unpack_nf4_codes(packed) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] codes (high nibble is the earlier element)."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((*p.shape[:-1], p.shape[-1] * 2), dtype=np.uint8)
    out[..., 0::2] = p >> 4
    out[..., 1::2] = p & 0xF
    return out


def _expand_blocks(scale, K, blocksize):
    return np.repeat(scale, blocksize, axis=-1)[..., :K]


def dequant_ref(packed, absmax, N: int, K: int, blocksize: int = NF4_BLOCK) -> np.ndarray:
    """Decode NF4 to the parity-contract value bf16_rne(fp32(c[code]) * absmax).

    Returns fp32 [..., N, K] holding bf16-representable values.
    """
    codes = unpack_nf4_codes(packed)
    assert codes.shape[-2:] == (N, K)
    cb = nf4_codebook()
    a = _expand_blocks(np.asarray(absmax, np.float32), K, blocksize)
    prod = (cb[codes] * a).astype(np.float32)  # one fp32 rounding of the product
    return bf16_round(prod).astype(np.float32)


def dequant_ref_level(packed, absmax, N: int, K: int, blocksize: int = NF4_BLOCK) -> np.ndarray:
    """Decode NF4 as bf16_rne(c[code]) * absmax, the exact product (fp64)."""
    codes = unpack_nf4_codes(packed)
    assert codes.shape[-2:] == (N, K)
    cb = bf16_round(nf4_codebook()).astype(np.float64)
    a = _expand_blocks(np.asarray(absmax, np.float64), K, blocksize)
    return cb[codes] * a


def dequant_ref_exact(packed, absmax, N: int, K: int, blocksize: int = NF4_BLOCK) -> np.ndarray:
    """Decode NF4 as the exact product c[code] * absmax (fp64; fidelity only)."""
    codes = unpack_nf4_codes(packed)
    assert codes.shape[-2:] == (N, K)
    cb = nf4_codebook().astype(np.float64)
    a = _expand_blocks(np.asarray(absmax, np.float64), K, blocksize)
    return cb[codes] * a


# --------------------------------------------------------------------------
# MXFP4
# --------------------------------------------------------------------------
def _round_e2m1(mag: np.ndarray) -> np.ndarray:
    """Nearest e2m1 magnitude code (0..7) for |q| >= 0, ties to the even code,
    saturating at 6.0 (code 7). Decided exactly in fp64."""
    M = E2M1_MAGNITUDES
    lo = np.clip(np.searchsorted(M, mag, side="right") - 1, 0, 7)  # largest M[lo] <= mag
    hi = np.minimum(lo + 1, 7)
    d_lo = mag - M[lo]
    d_hi = M[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (lo % 2 == 1))
    code = np.where(pick_hi & (hi != lo), hi, lo)
    return code.astype(np.uint8)


def quantize_pack_mxfp4(w):
    """Quantise fp32 weights [..., N, K] (K % 32 == 0) to MXFP4.

    Returns (blocks uint8 [..., N, K/32, 16], scales uint8 [..., N, K/32]).
    """
    w = np.asarray(w, dtype=np.float32)
    K = w.shape[-1]
    if K % MXFP4_BLOCK:
        raise ValueError("K must be a multiple of 32")
    wb = w.reshape(*w.shape[:-1], K // MXFP4_BLOCK, MXFP4_BLOCK).astype(np.float64)
    amax = np.max(np.abs(wb), axis=-1)
    zero = amax == 0
    _, ex = np.frexp(np.where(zero, 1.0, amax))  # amax = m 2^ex, m in [0.5, 1)
    e = np.clip((ex - 1) - 2, -127, 127)  # floor(log2 amax) - emax(e2m1)
    q = np.ldexp(wb, -e[..., None])  # exact
    mag = _round_e2m1(np.abs(q))
    sign = np.signbit(wb).astype(np.uint8)
    codes = (sign << 3) | mag
    codes[zero] = 0
    scales = np.where(zero, 0, e + 127).astype(np.uint8)
    blocks = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return blocks, scales


def unpack_mxfp4_codes(blocks) -> np.ndarray:
    """[..., K/32, 16] bytes -> [..., K/32, 32] codes (low nibble first)."""
    b = np.asarray(blocks, dtype=np.uint8)
    out = np.empty((*b.shape[:-1], b.shape[-1] * 2), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def dequant_mxfp4(blocks, scales) -> np.ndarray:
    """Decode MXFP4 to fp32 [..., N, K]: sign * e2m1 * 2^(scale - 127).
    The values are exact in fp32 and in bf16 where they are in range; the
    few past fp32's largest value (scale byte 254 with magnitude >= 2, byte
    253 with magnitude 4 or 6) become +-inf."""
    codes = unpack_mxfp4_codes(blocks)
    mag = E2M1_MAGNITUDES[codes & 7]
    val = np.where(codes & 8, -mag, mag)
    s = np.asarray(scales).astype(np.int64)
    out = np.ldexp(val, (s - 127)[..., None])
    out = np.where((s == 255)[..., None], np.nan, out)
    out = out.reshape(*out.shape[:-2], out.shape[-2] * out.shape[-1])
    with np.errstate(over="ignore"):  # the out-of-range values above
        return out.astype(np.float32)


def packed_bytes_per_weight(fmt: str) -> float:
    """Storage per weight including scales: NF4 4 bits + fp32 per 64,
    MXFP4 4 bits + one byte per 32."""
    if fmt == "nf4":
        return 0.5 + 4.0 / NF4_BLOCK
    if fmt == "mxfp4":
        return 0.5 + 1.0 / MXFP4_BLOCK
    raise ValueError(fmt)
