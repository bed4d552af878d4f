"""Oracle cross-check: pure-Python loops for tiny shapes (test infrastructure only).

Independent restatements of the same definitions as ``formats`` and ``moe``,
written as explicit loops with no vectorised numpy and no BLAS, so that a
slip in the vectorised oracle (an index, an axis, a nibble order, a
tie-break) shows up as a disagreement. fp32 steps use numpy fp32 scalars,
which follow IEEE rounding; everything else is Python floats (fp64).
"""

from __future__ import annotations

import math
import numpy as np


def nearest_level(s: float, levels) -> int:
    """Index of the nearest level (exact distance), ties to the lower index."""
    best, best_d = 0, None
    for i, c in enumerate(levels):
        d = abs(float(s) - float(c))
        if best_d is None or d < best_d:
            best, best_d = i, d
    return best


def quantize_nf4_loops(w, levels, blocksize=64):
    """w: list of rows (fp32 values). Returns (packed rows of ints, absmax rows)."""
    packed, absmax = [], []
    for row in w:
        prow, arow = [], []
        codes = []
        for b0 in range(0, len(row), blocksize):
            blk = [np.float32(v) for v in row[b0:b0 + blocksize]]
            a = np.float32(0)
            for v in blk:
                if abs(v) > a:
                    a = np.float32(abs(v))
            arow.append(a)
            for v in blk:
                if a == 0:
                    codes.append(7)
                else:
                    codes.append(nearest_level(np.float32(v / a), levels))
        for j in range(0, len(codes), 2):
            prow.append((codes[j] << 4) | codes[j + 1])
        packed.append(prow)
        absmax.append(arow)
    return packed, absmax


def bf16_nearest(v: float) -> float:
    """bf16 rounding by search among neighbours (normal range only)."""
    if v == 0 or not math.isfinite(v):
        return v
    m, e = math.frexp(abs(v))  # |v| = m 2^e
    q = 2.0 ** (e - 8)
    lo = math.floor(abs(v) / q) * q
    hi = lo + q
    if abs(v) - lo < hi - abs(v):
        r = lo
    elif abs(v) - lo > hi - abs(v):
        r = hi
    else:
        r = lo if (lo / q) % 2 == 0 else hi
    return math.copysign(r, v)


def decode_nf4_loops(packed, absmax, levels, blocksize=64):
    out = []
    for prow, arow in zip(packed, absmax):
        codes = []
        for byte in prow:
            codes.append(byte >> 4)
            codes.append(byte & 15)
        row = []
        for i, c in enumerate(codes):
            p = np.float32(np.float32(levels[c]) * np.float32(arow[i // blocksize]))
            row.append(bf16_nearest(float(p)))
        out.append(row)
    return out


def quantize_mxfp4_loops(w):
    """w: list of rows. Returns (blocks rows [K/32][16], scale rows [K/32])."""
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    blocks, scales = [], []
    for row in w:
        brow, srow = [], []
        for b0 in range(0, len(row), 32):
            blk = [float(np.float32(v)) for v in row[b0:b0 + 32]]
            amax = max(abs(v) for v in blk)
            if amax == 0:
                srow.append(0)
                brow.append([0] * 16)
                continue
            e = math.floor(math.log2(amax))
            # log2 of a float may round; correct it exactly
            while 2.0 ** e > amax:
                e -= 1
            while 2.0 ** (e + 1) <= amax:
                e += 1
            e = max(-127, min(127, e - 2))
            srow.append(e + 127)
            codes = []
            for v in blk:
                q = abs(v) / 2.0 ** e
                best, best_d = 0, None
                for i, m in enumerate(mags):
                    d = abs(q - m)
                    if best_d is None or d < best_d or (d == best_d and i % 2 == 0 and best % 2 == 1):
                        best, best_d = i, d
                codes.append((8 if math.copysign(1.0, v) < 0 else 0) | best)
            brow.append([codes[2 * j] | (codes[2 * j + 1] << 4) for j in range(16)])
        blocks.append(brow)
        scales.append(srow)
    return blocks, scales


def moe_loops(x, ids, gates, Wgu, Wd, I):
    """Dense per-slot loops. x [T][H]; Wgu[e] [2I][H]; Wd[e] [H][I] (decoded).
    Returns y [T][H] as Python floats BEFORE the final bf16 rounding, and h
    per slot (after its bf16 rounding)."""
    T = len(x)
    k = len(ids[0])
    H = len(x[0])
    y = [[0.0] * H for _ in range(T)]
    hs = {}
    for t in range(T):
        for j in range(k):
            e = ids[t][j]
            g = [sum(x[t][c] * Wgu[e][r][c] for c in range(H)) for r in range(2 * I)]
            h = []
            for i in range(I):
                G, U = g[i], g[I + i]
                h.append(bf16_nearest(G / (1.0 + math.exp(-G)) * U))
            hs[t * k + j] = h
            for n in range(H):
                o = sum(h[i] * Wd[e][n][i] for i in range(I))
                y[t][n] += float(np.float32(gates[t][j])) * o
    return y, hs


def route_loops(ids, E):
    flat = [e for row in ids for e in row]
    counts = [0] * E
    for e in flat:
        counts[e] += 1
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    fill = list(offsets[:-1])
    perm = [0] * len(flat)
    for s, e in enumerate(flat):
        perm[fill[e]] = s
        fill[e] += 1
    inv = [0] * len(flat)
    for p, s in enumerate(perm):
        inv[s] = p
    return counts, offsets, perm, inv


def e4m3_finite_values():
    """(value, code) for every finite E4M3 pattern, decoded from the bit fields
    (sign, 4 exponent bits with bias 7, 3 mantissa bits; S.1111.111 is NaN)."""
    out = []
    for b in range(256):
        e, m = (b >> 3) & 15, b & 7
        if e == 15 and m == 7:
            continue
        mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        out.append((-mag if b & 0x80 else mag, b))
    return out


def e4m3_nearest(v: float) -> float:
    """Nearest finite E4M3 value by search, ties to the even code, magnitudes
    beyond 448 saturated to 448."""
    if abs(v) >= 448.0:
        return math.copysign(448.0, v)
    best, best_code, best_d = 0.0, 0, None
    for val, code in e4m3_finite_values():
        if code & 0x80:
            continue  # search magnitudes, then restore the sign
        d = abs(abs(v) - val)
        if best_d is None or d < best_d or (d == best_d and code % 2 == 0 and best_code % 2 == 1):
            best, best_code, best_d = val, code, d
    return math.copysign(best, v)


def mxfp8_row_loops(row):
    """One row (length % 32 == 0) through MXFP8 and back, block by block."""
    out = []
    for b0 in range(0, len(row), 32):
        blk = [float(v) for v in row[b0:b0 + 32]]
        amax = max(abs(v) for v in blk)
        if amax == 0:
            out.extend([0.0] * 32)
            continue
        e = math.floor(math.log2(amax))
        while 2.0 ** e > amax:
            e -= 1
        while 2.0 ** (e + 1) <= amax:
            e += 1
        X = max(-127, min(127, e - 8))
        out.extend(e4m3_nearest(v / 2.0 ** X) * 2.0 ** X for v in blk)
    return out


def moe_loops_mxfp8(x, ids, gates, Wgu, Wd, I):
    """moe_loops with the x rows and the bf16 h rows replaced by their MXFP8
    decode before the matmuls that read them."""
    T = len(x)
    k = len(ids[0])
    H = len(x[0])
    y = [[0.0] * H for _ in range(T)]
    for t in range(T):
        xq = mxfp8_row_loops(x[t])
        for j in range(k):
            e = ids[t][j]
            g = [sum(xq[c] * Wgu[e][r][c] for c in range(H)) for r in range(2 * I)]
            h = []
            for i in range(I):
                G, U = g[i], g[I + i]
                h.append(bf16_nearest(G / (1.0 + math.exp(-G)) * U))
            hq = mxfp8_row_loops(h)
            for n in range(H):
                o = sum(hq[i] * Wd[e][n][i] for i in range(I))
                y[t][n] += float(np.float32(gates[t][j])) * o
    return y
