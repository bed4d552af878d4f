"""Pins for the oracle's weight formats (CPU only).

Each test ties the oracle to something outside itself: values the pages print
(MAE / RMSE, round-trip errors, example shapes, idempotence, memory ratio),
the published NF4 table, hand-worked blocks, torch's bf16 conversion, and
pure-Python brute force.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from golden_io import read_cases, read_floats


# ---------------------------------------------------------------- codebook
def test_codebook_equals_published_table_bit_for_bit():
    pub = np.array(read_floats("nf4_codebook_qlora.txt"), dtype=np.float32)
    cb = oracle.nf4_codebook()
    assert cb.dtype == np.float32 and cb.shape == (16,)
    assert np.array_equal(cb.view(np.uint32), pub.view(np.uint32))


def test_codebook_shape_facts():
    cb = oracle.nf4_codebook()
    assert np.all(np.diff(cb) > 0)
    assert cb[0] == -1.0 and cb[7] == 0.0 and cb[15] == 1.0
    assert (cb < 0).sum() == 7 and (cb > 0).sum() == 8


# ---------------------------------------------------- pages' printed numbers
def test_nf4_mae_rmse_match_pr1984():
    # bitsandbytes PR #1984, Benchmark Results (NF4): MAE 0.073, RMSE 0.092.
    rng = np.random.default_rng(1984)
    w = rng.standard_normal((1024, 4096), dtype=np.float32)
    packed, absmax = oracle.quantize_pack_nf4(w)
    wq = oracle.dequant_ref_exact(packed, absmax, *w.shape)
    err = wq - w.astype(np.float64)
    assert round(float(np.abs(err).mean()), 3) == 0.073
    assert round(float(np.sqrt((err ** 2).mean())), 3) == 0.092


def test_readme_cpu_block_1_nf4_roundtrip():
    # "grouped-nf4-gemm" README, CPU block 1: w [256,512] -> packed [256,256]
    # uint8, absmax [256,8] fp32; rel-err ~0.09; re-pack idempotent: True.
    rng = np.random.default_rng(0)
    w = rng.standard_normal((256, 512), dtype=np.float32)
    packed, absmax = oracle.quantize_pack_nf4(w)
    assert packed.shape == (256, 256) and packed.dtype == np.uint8
    assert absmax.shape == (256, 8) and absmax.dtype == np.float32
    for wq in (oracle.dequant_ref_exact(packed, absmax, 256, 512),
               oracle.dequant_ref(packed, absmax, 256, 512)):
        rel = np.linalg.norm(wq - w) / np.linalg.norm(w)
        assert round(float(rel), 2) == 0.09
        assert np.array_equal(oracle.quantize_pack_nf4(wq.astype(np.float32))[0], packed)


def test_readme_cpu_block_2_mxfp4_roundtrip():
    # README CPU block 2: w [128,256] -> blocks [128,8,16] u8, scales [128,8]
    # u8 (e8m0); rel-err ~0.12.
    rng = np.random.default_rng(0)
    w = rng.standard_normal((128, 256), dtype=np.float32)
    blocks, scales = oracle.quantize_pack_mxfp4(w)
    assert blocks.shape == (128, 8, 16) and blocks.dtype == np.uint8
    assert scales.shape == (128, 8) and scales.dtype == np.uint8
    wq = oracle.dequant_mxfp4(blocks, scales)
    assert wq.shape == (128, 256)
    rel = np.linalg.norm(wq - w) / np.linalg.norm(w)
    assert 0.10 <= rel <= 0.125
    b2, s2 = oracle.quantize_pack_mxfp4(wq)
    assert np.array_equal(b2, blocks) and np.array_equal(s2, scales)


def test_memory_ratio_matches_pr1984():
    # PR #1984, Memory Savings: 4-bit uses ~28% of fp16 memory (72% reduction).
    bpw = oracle.packed_bytes_per_weight("nf4")
    assert bpw == 0.5625
    assert round(100 * bpw / 2.0) == 28
    w = np.ones((4, 640), dtype=np.float32)
    p, a = oracle.quantize_pack_nf4(w)
    assert (p.nbytes + a.nbytes) / w.size == bpw
    assert oracle.packed_bytes_per_weight("mxfp4") == 0.53125


# ----------------------------------------------------------- hand-worked
def test_nf4_handworked_block():
    (case,) = read_cases("nf4_handworked.txt")
    w = np.zeros((1, 64), dtype=np.float32)
    for i, v in case["in"].items():
        w[0, i] = v
    packed, absmax = oracle.quantize_pack_nf4(w)
    assert absmax[0, 0] == np.float32(case["absmax"])
    codes = oracle.unpack_nf4_codes(packed)[0]
    want = np.full(64, 7)
    for i, c in case["codes"].items():
        want[i] = c
    assert np.array_equal(codes, want)
    for i, b in case["bytes"].items():
        assert packed[0, i] == b
    assert np.all(packed[0, 5:] == 0x77)


def test_mxfp4_handworked_blocks():
    for case in read_cases("mxfp4_handworked.txt"):
        w = np.zeros((1, 32), dtype=np.float32)
        for i, v in case.get("in", {}).items():
            w[0, i] = v
        blocks, scales = oracle.quantize_pack_mxfp4(w)
        assert scales[0, 0] == int(case["scale"]), case["name"]
        codes = oracle.unpack_mxfp4_codes(blocks)[0, 0]
        want = np.zeros(32, dtype=int)
        for i, c in case.get("codes", {}).items():
            want[i] = c
        assert np.array_equal(codes, want), case["name"]


def test_mxfp4_low_nibble_first():
    w = np.zeros((1, 32), dtype=np.float32)
    w[0, 0], w[0, 1] = 6.0, -1.0  # e = 0: codes 7 and 8|2
    blocks, _ = oracle.quantize_pack_mxfp4(w)
    assert blocks[0, 0, 0] == (7 | (10 << 4))


# ------------------------------------------------------------- invariants
@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_idempotence_and_membership(fmt):
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    w[3, :64] = 0.0  # an all-zero block
    w[5, :64] = 0.0
    w[5, 10] = -0.5  # a single nonzero
    if fmt == "nf4":
        p, a = oracle.quantize_pack_nf4(w)
        ex = oracle.dequant_ref_exact(p, a, 64, 256)
        cb = oracle.nf4_codebook().astype(np.float64)
        blk = np.repeat(a.astype(np.float64), 64, axis=1)
        ratio = np.where(blk > 0, ex / np.where(blk > 0, blk, 1), 0)
        assert np.all(np.isin(ratio, cb))
        assert np.all(ex[3, :64] == 0) and np.all(oracle.unpack_nf4_codes(p)[3, :64] == 7)
        assert ex[5, 10] == -0.5 and a[5, 0] == np.float32(0.5)
        for dec in (ex, oracle.dequant_ref(p, a, 64, 256)):
            assert np.array_equal(oracle.quantize_pack_nf4(dec.astype(np.float32))[0], p)
    else:
        b, s = oracle.quantize_pack_mxfp4(w)
        d = oracle.dequant_mxfp4(b, s)
        scale = np.ldexp(1.0, s.astype(int) - 127)
        q = d.reshape(64, 8, 32) / scale[..., None]
        assert np.all(np.isin(np.abs(q), oracle.E2M1_MAGNITUDES))
        assert np.all(d[3, :64] == 0) and np.all(s[3, :2] == 0)
        assert d[5, 10] == -0.5
        b2, s2 = oracle.quantize_pack_mxfp4(d)
        assert np.array_equal(b2, b) and np.array_equal(s2, s)


def test_dequant_ref_is_bf16_of_fp32_product():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((8, 128)) * 0.02).astype(np.float32)
    p, a = oracle.quantize_pack_nf4(w)
    d = oracle.dequant_ref(p, a, 8, 128)
    codes = oracle.unpack_nf4_codes(p)
    cb = torch.tensor(oracle.nf4_codebook())
    prod = cb[torch.from_numpy(codes.astype(np.int64))] * torch.from_numpy(np.repeat(a, 64, axis=1))
    want = prod.to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(d, want)


# ------------------------------------------------------------------ bf16
def test_bf16_round_matches_torch_on_fp32():
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2 ** 32, size=200000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    specials = np.array([0.0, -0.0, 1.0, 1.00390625, 1.0078125, 1.005859375, 3.3895313892515355e38,
                         3.3961775292304767e38, 1e-40, -1e-45, 2 ** -133, 2 ** -134, 3 * 2 ** -135],
                        dtype=np.float32)
    x = np.concatenate([x, specials])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_bits_from_f32(x)
    assert np.array_equal(got, want)


def test_bf16_round_fp64_against_neighbour_search():
    rng = np.random.default_rng(12)
    v = rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000)
    # exact midpoints between bf16 neighbours must go to the even one
    v = np.concatenate([v, [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8)]])
    got = oracle.bf16_round(v)
    want = np.array([brute.bf16_nearest(float(t)) for t in v])
    assert np.array_equal(got, want)
    assert got[-3] == 1.0 and got[-2] == 1.0 + 2 ** -6 and got[-1] == -1.0


# ------------------------------------------------------------ brute force
def test_nf4_quantiser_matches_brute_force():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((6, 128)) * 0.02).astype(np.float32)
    cb = oracle.nf4_codebook()
    # plant exact ties: w / absmax equal to a midpoint between two levels
    w[0, :64] = 0
    w[0, 0] = 1.0
    w[0, 1] = np.float32(cb[8]) / 2  # tie between levels 7 and 8
    w[0, 2] = np.float32(cb[6]) / 2  # tie between levels 6 and 7
    p, a = oracle.quantize_pack_nf4(w)
    pb, ab = brute.quantize_nf4_loops(w.tolist(), cb)
    assert np.array_equal(p, np.array(pb, dtype=np.uint8))
    assert np.array_equal(a, np.array(ab, dtype=np.float32))
    d = oracle.dequant_ref(p, a, 6, 128)
    db = brute.decode_nf4_loops(pb, ab, cb)
    assert np.array_equal(d.astype(np.float64), np.array(db))


def test_mxfp4_quantiser_matches_brute_force():
    rng = np.random.default_rng(6)
    w = (rng.standard_normal((5, 96)) * 0.02).astype(np.float32)
    w[1, :32] = np.array([4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0] * 4, dtype=np.float32)
    w[2, :32] *= 1e-30
    b, s = oracle.quantize_pack_mxfp4(w)
    bb, sb = brute.quantize_mxfp4_loops(w.tolist())
    assert np.array_equal(b, np.array(bb, dtype=np.uint8))
    assert np.array_equal(s, np.array(sb, dtype=np.uint8))
