"""The input gradient through the packed weights (e4b_grouped_dgrad, the
grouped GEMM's backward in the grouped-nf4-gemm README's entry table) on the
GPU against the oracle's grouped_dgrad_ref: both formats, weight rows and
columns with ragged tails, empty experts, experts with several 256-row tiles,
and rows past offsets[E] left untouched."""

import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_e4b_b200 import e4b
from gpu_util import assert_close

pytestmark = pytest.mark.gpu


def _stack(fmt, E, N, K, seed, std=0.05):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((E, N, K)) * std).astype(np.float32)
    codes, scales = e4b.quantize(fmt, torch.from_numpy(w).cuda())
    q = oracle.quantize_pack_nf4 if fmt == "nf4" else oracle.quantize_pack_mxfp4
    rc, rs = q(w)
    assert np.array_equal(codes.cpu().numpy(), rc)
    return codes, scales, rc, rs


CASES = [
    ("nf4", 3, 256, 256, [70, 0, 301]),     # tiles of 128 columns, rows in 64-row jobs, an empty expert
    ("nf4", 2, 200, 192, [5, 260]),         # N and K tails (200 = 3 x 64 + 8 rows, 192 = 1.5 x 128 columns)
    ("mxfp4", 4, 96, 160, [1, 33, 0, 513]),  # K % 64 == 32, > 2 tiles of 256 rows
    ("mxfp4", 1, 1000, 64, [17]),           # K < 128
]


@pytest.mark.parametrize("flags", [0, e4b.FLAG_TC_SINGLE_SM], ids=["sm_pairs", "one_sm"])
@pytest.mark.parametrize("fmt,E,N,K,counts", CASES)
def test_dgrad_matches_oracle(fmt, E, N, K, counts, flags):
    codes, scales, rc, rs = _stack(fmt, E, N, K, seed=N + K)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    R = int(offsets[-1])
    rng = np.random.default_rng(K)
    dy = torch.from_numpy(rng.standard_normal((R + 3, N)).astype(np.float32)).to(torch.bfloat16)
    dx = torch.full((R + 3, K), 7.0, dtype=torch.bfloat16, device="cuda")
    e4b.e4b_grouped_dgrad(fmt, codes, scales, dy.cuda(), torch.from_numpy(offsets).cuda(), dx, E=E, N=N, K=K,
                          R_max=R, flags=flags)
    torch.cuda.synchronize()
    assert e4b.e4b_last_path() == e4b.E4B_PATH_TCGEN05
    want = oracle.grouped_dgrad_ref(fmt, dy.float().numpy()[:R], offsets, rc, rs, N, K)
    got = dx.float().cpu().numpy()
    assert_close(got[:R], want, f"dgrad {fmt} E={E} N={N} K={K}")
    assert np.all(got[R:] == 7.0)  # rows past offsets[E] untouched


def test_dgrad_is_the_adjoint_of_the_forward_projection():
    # <dgrad(dy), a> = <dy, proj(a)> through the same packed weights, both
    # computed by the library (the STORE projection and the dgrad)
    fmt, E, N, K = "nf4", 2, 256, 320
    codes, scales, rc, rs = _stack(fmt, E, N, K, seed=3)
    offsets = np.array([0, 300, 512], np.int64)
    rng = np.random.default_rng(4)
    a = torch.from_numpy(rng.standard_normal((512, K)).astype(np.float32)).to(torch.bfloat16)
    dy = torch.from_numpy(rng.standard_normal((512, N)).astype(np.float32)).to(torch.bfloat16)
    off = torch.from_numpy(offsets).cuda()
    proj = torch.empty((512, N), dtype=torch.bfloat16, device="cuda")
    e4b.e4b_grouped_gemm(fmt, e4b.E4B_EPI_STORE, codes, scales, a.cuda(), off, proj, E=E, N=N, K=K, R_max=512,
                         flags=e4b.FLAG_FORCE_TCGEN05)
    dx = torch.empty((512, K), dtype=torch.bfloat16, device="cuda")
    e4b.e4b_grouped_dgrad(fmt, codes, scales, dy.cuda(), off, dx, E=E, N=N, K=K, R_max=512)
    torch.cuda.synchronize()
    lhs = float((dx.double() * a.cuda().double()).sum())
    rhs = float((dy.cuda().double() * proj.double()).sum())
    # both sides carry one bf16 rounding per output element
    assert abs(lhs - rhs) <= 2e-2 * (abs(lhs) + abs(rhs) + 1.0)
