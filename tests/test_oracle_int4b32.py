"""Pins of the int4-b32 oracle ("How do I run a single-token INT4 decode GEMV
over routed MoE experts, and pack calibrated (GPTQ) weights for it?": the
batch-1 int4-b32 decode GEMV with exact integer accumulation, and the GPTQ
packer onto the same bytes). The readings they pin (signed nibbles, earlier
weight low, fp16 scale per 32 weights, int8 token with one fp32 scale, GPTQ
symmetric with zero point 8) are stated in the oracle module's header.

Each pin checks the oracle against something other than itself: bytes worked
out by hand, the quantisers' error bound, pure-Python integer loops, the
dequantised matrix (another route to the same sum) and GPTQ's own
dequantisation formula."""

import math

import numpy as np
import pytest

from oracle import int4b32 as q4
from oracle import bf16_round


def _u32_to_i32(v: int) -> int:
    return v - (1 << 32) if v >= (1 << 31) else v


def test_nibble_packing_handworked():
    # q -> 4-bit two's complement nibbles (8, 7, 0, 15, 1, 14, 3, 5), pairs
    # (earlier low, later high): 0x78, 0xF0, 0xE1, 0x53
    q = np.array([-8, 7, 0, -1, 1, -2, 3, 5])
    assert q4.pack_int4(q).tolist() == [0x78, 0xF0, 0xE1, 0x53]
    assert q4.unpack_int4(np.array([0x78, 0xF0, 0xE1, 0x53], np.uint8)).tolist() == q.tolist()


def test_gptq_word_handworked():
    # one column, K = 32: four words, value i of a word in bits 4i..4i+3,
    # unsigned with zero point 8 (q = u - 8)
    words = [0x76543210, 0xFEDCBA98, 0x88888888, 0x0000000F]
    qweight = np.array([[_u32_to_i32(w)] for w in words], np.int32)  # [K/8, N=1]
    scales = np.array([[0.5]], np.float16)                             # [K/32, N=1]
    codes, s = q4.gptq_pack_int4b32_ref(qweight, scales)
    # word 0: q = -8..-1 -> nibble pairs (8,9) (10,11) (12,13) (14,15)
    # word 1: q = 0..7   -> (0,1) (2,3) (4,5) (6,7)
    # word 2: q = 0 (all) ; word 3: q0 = 7, the rest -8
    want = [0x98, 0xBA, 0xDC, 0xFE, 0x10, 0x32, 0x54, 0x76, 0, 0, 0, 0, 0x87, 0x88, 0x88, 0x88]
    assert codes.shape == (1, 16) and codes[0].tolist() == want
    assert s.shape == (1, 1) and float(s[0, 0]) == 0.5


def test_quantize_weights_within_half_a_step():
    rng = np.random.default_rng(11)
    w = (rng.standard_normal((48, 256)) * 0.02).astype(np.float32)
    w[3] *= 40.0  # a row far from the others: scales are per block
    w[5, 32:64] = rng.standard_t(2, 32) * 0.05  # heavy-tailed block
    codes, s = q4.quantize_int4b32(w)
    assert codes.shape == (48, 128) and codes.dtype == np.uint8
    assert s.shape == (48, 8) and s.dtype == np.float16
    q = q4.unpack_int4(codes)
    assert q.min() >= -8 and q.max() <= 7
    sf = np.repeat(s.astype(np.float64), 32, axis=1)
    err = np.abs(w.astype(np.float64) - sf * q)
    # half a step, plus the fp32 rounding of w / s (|w / s| <= 7.01)
    assert np.all(err <= sf * (0.5 + 8 * 2.0 ** -24))
    # the block maximum lands on +-7 (amax / s is 7 up to the fp16 rounding of s)
    blk = w.reshape(48, 8, 32)
    idx = np.argmax(np.abs(blk), axis=-1)
    qb = q.reshape(48, 8, 32)
    top = np.take_along_axis(qb, idx[..., None], -1)[..., 0]
    sign = np.sign(np.take_along_axis(blk, idx[..., None], -1)[..., 0])
    assert np.array_equal(top, (7 * sign).astype(np.int64))
    # scale = fp16(absmax / 7)
    amax = np.max(np.abs(blk), axis=-1)
    assert np.array_equal(s, (amax / np.float32(7)).astype(np.float16))


def test_zero_block_and_zero_token():
    w = np.zeros((2, 64), np.float32)
    w[1, 32:] = 0.25
    codes, s = q4.quantize_int4b32(w)
    assert float(s[0, 0]) == 0 and float(s[0, 1]) == 0 and float(s[1, 0]) == 0
    assert np.all(codes[0] == 0) and np.all(codes[1, :16] == 0)
    assert np.all(q4.unpack_int4(codes[1, 16:]) == 7)
    xq, sx = q4.quantize_token(np.zeros(64, np.float32))
    assert sx == 0 and np.all(xq == 0)
    y = q4.gemv_int4b32_ref(np.zeros(64, np.float32), [0], codes[None], s[None])
    assert np.all(y == 0)


def test_quantize_token_within_half_a_step():
    rng = np.random.default_rng(12)
    x = bf16_round(rng.standard_normal(512)).astype(np.float32)
    xq, sx = q4.quantize_token(x)
    amax = np.float32(np.max(np.abs(x)))
    assert sx == np.float32(amax / np.float32(127))
    assert np.max(np.abs(xq)) == 127 and np.min(xq) >= -127
    # x * fp32(127 / amax) is within 2^-21 relative of x / sx: half a step and a hair
    assert np.all(np.abs(x - np.float64(sx) * xq) <= np.float64(sx) * (0.5 + 2.0 ** -12))
    assert xq[np.argmax(np.abs(x))] == 127 * np.sign(x[np.argmax(np.abs(x))])
    # each value is decided by one fp32 product with r = fp32(127 / amax)
    r = np.float32(np.float32(127) / amax)
    for i in range(0, 512, 37):
        t = float(np.float32(x[i] * r))
        lo = np.floor(t)
        want = lo + 1 if (t - lo > 0.5 or (t - lo == 0.5 and lo % 2 == 1)) else lo
        assert xq[i] == int(want)


def test_quantize_token_tiny_and_tie_values():
    # a token so small that 127 / amax overflows is treated as zero
    xq, sx = q4.quantize_token(np.array([1e-38, -2e-38], np.float32))
    assert sx == 0 and np.all(xq == 0)
    # exact ties of x * r round to even: amax = 127 gives r = 1
    x = np.array([127.0, 0.5, 1.5, 2.5, -0.5, -1.5, -126.5], np.float32)
    xq, sx = q4.quantize_token(x)
    assert sx == 1.0 and xq.tolist() == [127, 0, 2, 2, 0, -2, -126]


def test_block_dots_against_integer_loops():
    rng = np.random.default_rng(13)
    N, K = 3, 96
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    xq = rng.integers(-127, 128, size=K)
    got = q4.block_dots(codes, xq)
    for n in range(N):
        for b in range(K // 32):
            acc = 0
            for k in range(32 * b, 32 * b + 32):
                byte = int(codes[n, k // 2])
                nib = (byte & 15) if k % 2 == 0 else (byte >> 4)
                val = nib - 16 if nib >= 8 else nib
                acc += val * int(xq[k])
            assert got[n, b] == acc
    # a subset of rows, taken in small chunks, gives the same integers
    assert np.array_equal(q4.block_dots(codes, xq, rows=[2, 0], chunk=1), got[[2, 0]])


def test_gemv_equals_dequantised_matrix_times_quantised_token():
    rng = np.random.default_rng(14)
    E, N, K = 3, 40, 160
    w = (rng.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    codes, s = q4.quantize_int4b32(w)
    x = bf16_round(rng.standard_normal(K)).astype(np.float32)
    ids = [2, 0]
    acc = q4.gemv_int4b32_acc(x, ids, codes, s)
    xq, sx = q4.quantize_token(x)
    for j, e in enumerate(ids):
        want = np.float64(sx) * (q4.dequant_int4b32(codes[e], s[e]) @ xq.astype(np.float64))
        assert np.allclose(acc[j], want, rtol=1e-12, atol=1e-15)
    # and the dequantised weights are near the fp32 weights they came from
    assert np.max(np.abs(q4.dequant_int4b32(codes, s) - w)) < 0.02
    # sampled rows are the same numbers as the full output
    assert np.array_equal(q4.gemv_int4b32_acc(x, ids, codes, s, rows=[5, 39]), acc[:, [5, 39]])


def _acc_loop(xrow, e, codes, s, n):
    """acc for one (slot, row) by explicit loops over blocks, from the bytes."""
    xq, sx = q4.quantize_token(xrow)
    K = codes.shape[-1] * 2
    total = 0.0
    for b in range(K // 32):
        d = 0
        for k in range(32 * b, 32 * b + 32):
            byte = int(codes[e, n, k // 2])
            nib = (byte & 15) if k % 2 == 0 else (byte >> 4)
            d += (nib - 16 if nib >= 8 else nib) * int(xq[k])
        total += float(s[e, n, b]) * d
    return float(sx) * total


def test_epilogues_against_loops():
    rng = np.random.default_rng(15)
    E, I, K = 4, 6, 64
    codes, s = q4.quantize_int4b32((rng.standard_normal((E, 2 * I, K)) * 0.02).astype(np.float32))
    x = bf16_round(rng.standard_normal(K)).astype(np.float32)
    ids = [3, 1]
    gates = np.array([0.7, 0.3], np.float32)
    # store
    y = q4.gemv_int4b32_ref(x, ids, codes, s, "store")
    for j, e in enumerate(ids):
        for n in range(2 * I):
            assert y[j, n] == bf16_round(_acc_loop(x, e, codes, s, n))
    # swiglu: gate rows [0, I), up rows [I, 2I)
    h = q4.gemv_int4b32_ref(x, ids, codes, s, "swiglu")
    assert h.shape == (2, I)
    for j, e in enumerate(ids):
        for i in range(I):
            g, u = _acc_loop(x, e, codes, s, i), _acc_loop(x, e, codes, s, I + i)
            want = bf16_round(g / (1.0 + math.exp(-g)) * u)
            assert abs(h[j, i] - want) <= 2.0 ** -8 * abs(want) + 1e-30
    # combine, one activation row per slot (each with its own scale)
    xs = bf16_round(rng.standard_normal((2, K)) * np.array([[1.0], [30.0]])).astype(np.float32)
    yc = q4.gemv_int4b32_ref(xs, ids, codes, s, "combine", gates)
    assert yc.shape == (2 * I,)
    for n in range(2 * I):
        want = sum(float(gates[j]) * _acc_loop(xs[j], e, codes, s, n) for j, e in enumerate(ids))
        assert abs(yc[n] - bf16_round(want)) <= 2.0 ** -8 * abs(want) + 1e-30


def test_decode_layer_is_the_composition():
    rng = np.random.default_rng(16)
    E, H, I = 3, 64, 96
    gc, gs = q4.quantize_int4b32((rng.standard_normal((E, 2 * I, H)) * 0.05).astype(np.float32))
    dc, ds = q4.quantize_int4b32((rng.standard_normal((E, H, I)) * 0.05).astype(np.float32))
    x = bf16_round(rng.standard_normal(H)).astype(np.float32)
    ids, gates = [2, 0], np.array([0.6, 0.4], np.float32)
    y = q4.int4b32_decode_layer_ref(x, ids, gates, gc, gs, dc, ds)
    h = np.array([[bf16_round(_swiglu(_acc_loop(x, e, gc, gs, i), _acc_loop(x, e, gc, gs, I + i)))
                   for i in range(I)] for e in ids], np.float32)
    for n in range(0, H, 7):
        want = sum(float(gates[j]) * _acc_loop(h[j], e, dc, ds, n) for j, e in enumerate(ids))
        assert abs(y[n] - bf16_round(want)) <= 2.0 ** -8 * abs(want) + 1e-30
    assert np.array_equal(q4.int4b32_decode_layer_ref(x, ids, gates, gc, gs, dc, ds, rows=[1, 9]),
                          y[[1, 9]])


def _swiglu(g, u):
    return g / (1.0 + math.exp(-g)) * u


def test_gptq_pack_matches_gptq_dequantisation():
    rng = np.random.default_rng(17)
    K, N = 96, 5
    u = rng.integers(0, 16, size=(K, N))
    gscales = (rng.random((K // 32, N)) * 0.01 + 1e-3).astype(np.float16)
    qweight = np.zeros((K // 8, N), np.int32)
    for w in range(K // 8):
        for n in range(N):
            word = 0
            for i in range(8):
                word |= int(u[8 * w + i, n]) << (4 * i)
            qweight[w, n] = _u32_to_i32(word)
    codes, s = q4.gptq_pack_int4b32_ref(qweight, gscales)
    assert codes.shape == (N, K // 2) and s.shape == (N, K // 32) and s.dtype == np.float16
    W = q4.dequant_int4b32(codes, s)
    for n in range(N):
        for k in range(K):
            assert W[n, k] == (int(u[k, n]) - 8) * float(gscales[k // 32, n])


@pytest.mark.parametrize("K", [32, 1024])
def test_integer_range_is_exact_in_int32(K):
    # the worst block dot product, 32 * 8 * 127, sits far inside int32; the
    # oracle's integer result equals the product bound exactly
    codes = q4.pack_int4(np.full(K, -8))[None]
    xq = np.full(K, 127)
    assert np.all(q4.block_dots(codes, xq) == -32 * 8 * 127)
