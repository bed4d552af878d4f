"""GPU quantisers and the table decode, bit for bit against the oracle."""

import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_e4b_b200 import e4b
from golden_io import read_cases

pytestmark = pytest.mark.gpu


def _edge_weights(N, K, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    cb = oracle.nf4_codebook()
    w[0, :64] = 0.0                      # zero block
    w[1, :64] = 0.0
    w[1, 17] = -3.5                      # single nonzero
    w[2, :64] = 0.0
    w[2, 0] = 1.0
    w[2, 1] = cb[8] / 2                  # NF4 tie between levels 7 and 8
    w[2, 2] = cb[6] / 2                  # tie between levels 6 and 7
    w[2, 3] = (cb[12] + cb[13]) / 2      # midpoint rounded to fp32
    w[3, :32] = np.array([4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0] * 4, np.float32)  # e2m1 ties
    w[3, 32:64] = -w[3, :32]
    w[4, :64] *= np.float32(1e-35)       # subnormal-range blocks
    w[5, :64] *= np.float32(1e30)        # large blocks
    w[6, :64] = -0.0
    return w


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
@pytest.mark.parametrize("shape", [(1, 8, 64), (3, 40, 320), (2, 256, 2880)])
def test_quantise_bit_exact(fmt, shape):
    E, N, K = shape
    if fmt == "nf4" and K % 64:
        pytest.skip("NF4 needs K % 64 == 0")
    w = np.stack([_edge_weights(N, K, s) if N >= 8 else
                  (np.random.default_rng(s).standard_normal((N, K)) * 0.02).astype(np.float32)
                  for s in range(E)])
    codes, scales = e4b.quantize(fmt, torch.from_numpy(w).cuda())
    if fmt == "nf4":
        rc, rs = oracle.quantize_pack_nf4(w)
    else:
        rc, rs = oracle.quantize_pack_mxfp4(w)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint8), rs.view(np.uint8))


def test_mxfp4_handworked_blocks_on_gpu():
    cases = read_cases("mxfp4_handworked.txt")
    w = np.zeros((1, len(cases), 32), np.float32)
    for i, case in enumerate(cases):
        for j, v in case.get("in", {}).items():
            w[0, i, j] = v
    blocks, scales = e4b.quantize("mxfp4", torch.from_numpy(w).cuda())
    codes = oracle.unpack_mxfp4_codes(blocks.cpu().numpy())[0]
    for i, case in enumerate(cases):
        assert scales[0, i, 0].item() == int(case["scale"]), case["name"]
        want = np.zeros(32, int)
        for j, c in case.get("codes", {}).items():
            want[j] = c
        assert np.array_equal(codes[i, 0], want), case["name"]


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_table_decode_bit_exact(fmt):
    E, N, K = 2, 48, 640 if fmt == "nf4" else 608
    w = np.stack([_edge_weights(N, K, 10 + e) for e in range(E)])
    if fmt == "nf4":
        rc, rs = oracle.quantize_pack_nf4(w)
        want = oracle.dequant_ref(rc, rs, N, K)
    else:
        rc, rs = oracle.quantize_pack_mxfp4(w)
        want = oracle.dequant_mxfp4(rc, rs)
    out = e4b.dequantize(fmt, torch.from_numpy(rc).cuda(), torch.from_numpy(rs).cuda(), E, N, K)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, oracle.bf16_bits_from_f32(want))


def test_mxfp4_decode_every_code_and_scale():
    # every scale byte 0..254 with every code: exact e2m1 * 2^(s-127)
    scales = np.arange(255, dtype=np.uint8).reshape(1, 255, 1)
    codes = np.tile(np.array([0x10 * (2 * i + 1) + 2 * i for i in range(8)], np.uint8), 2)
    blocks = np.broadcast_to(codes, (1, 255, 1, 16)).copy()
    want = oracle.dequant_mxfp4(blocks, scales)
    out = e4b.dequantize("mxfp4", torch.from_numpy(blocks).cuda(), torch.from_numpy(scales).cuda(),
                         1, 255, 32)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, oracle.bf16_bits_from_f32(want))
