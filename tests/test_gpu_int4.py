"""The int4-b32 decode GEMV, its quantiser and the GPTQ repack on the GPU,
called through the C ABI, against the oracle (oracle/int4b32.py): codes,
scales and repacked bytes bit-exact; GEMV outputs within 1e-2 * (1 + |y|)
for every epilogue, with ragged rows, ragged lane blocks, several chunk rounds
along K, duplicate and odd slot counts, per-slot activation rows, a dropped
(bad) expert id, a zero token; the two-launch decode layer at a mid size and at
the full decode shape (E=8, H=4096, I=14336, top-2) on sampled outputs."""

import numpy as np
import pytest
import torch

from oracle import int4b32 as q4
from bit_grouped_moe_e4b_b200 import e4b, synth
from bit_grouped_moe_e4b_b200.configs import DECODE
from gpu_util import assert_close

pytestmark = pytest.mark.gpu


def _weights(rng, shape, std=0.02):
    w = (rng.standard_normal(shape) * std).astype(np.float32)
    flat = w.reshape(-1, w.shape[-1])
    flat[0, :32] = 0.0                                    # an all-zero block
    if flat.shape[-1] >= 64:
        flat[-1, 32:64] = rng.standard_t(2, 32) * 0.1     # heavy-tailed block
    return w


def _stack(rng, E, N, K):
    w = _weights(rng, (E, N, K))
    codes, scales = e4b.quantize_int4_b32(torch.from_numpy(w).cuda())
    rc, rs = q4.quantize_int4b32(w)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    return codes, scales, rc, rs


def _bf16(rng, shape, scale=1.0):
    x = torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32)).to(torch.bfloat16)
    return x, x.float().numpy()


@pytest.mark.parametrize("E,N,K", [(3, 70, 160), (2, 33, 4096), (1, 5, 32)])
def test_quantizer_bit_exact(E, N, K):
    _stack(np.random.default_rng(N + K), E, N, K)


@pytest.mark.parametrize("E,N,K", [(2, 70, 96), (1, 300, 2048 + 256), (3, 1, 32)])
def test_gptq_repack_bit_exact(E, N, K):
    rng = np.random.default_rng(7 + N)
    qweight = rng.integers(-(2 ** 31), 2 ** 31, size=(E, K // 8, N), dtype=np.int64).astype(np.int32)
    gsc = (rng.random((E, K // 32, N)) * 0.02).astype(np.float16)
    codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((E, N, K // 32), dtype=torch.float16, device="cuda")
    e4b.e4b_gptq_pack_int4_b32(torch.from_numpy(qweight).cuda(), torch.from_numpy(gsc).cuda(), codes, scales,
                               E=E, N=N, K=K)
    for e in range(E):
        rc, rs = q4.gptq_pack_int4b32_ref(qweight[e], gsc[e])
        assert np.array_equal(codes[e].cpu().numpy(), rc)
        assert np.array_equal(scales[e].cpu().numpy().view(np.uint16), rs.view(np.uint16))


# (E, N, K, ids): ragged row pairs (odd N), lanes with unequal block counts
# (K/32 not a multiple of 32), several chunk rounds (K/32 > 128), duplicates
STORE_CASES = [
    (4, 333, 1216, [2, 0, 2]),
    (2, 64, 5120, [1]),
    (8, 31, 96, [7, 3, 5, 1, 0]),
]


@pytest.mark.parametrize("E,N,K,ids", STORE_CASES)
@pytest.mark.parametrize("per_slot", [False, True])
def test_store_matches_oracle(E, N, K, ids, per_slot):
    rng = np.random.default_rng(N * 7 + K)
    codes, scales, rc, rs = _stack(rng, E, N, K)
    k = len(ids)
    x, xf = _bf16(rng, (k, K) if per_slot else (K,), 1.0)
    if per_slot:
        x[1 % k] *= 40.0  # rows with different scales
        xf = x.float().numpy()
    y = torch.full((k, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    idt = torch.tensor(ids, dtype=torch.int32, device="cuda")
    e4b.e4b_gemv_int4_b32("store", codes, scales, idt, x.cuda(), y, E=E, N=N, K=K, ld_x=K if per_slot else 0)
    assert e4b.e4b_last_path() == e4b.E4B_PATH_INT4_GEMV and e4b.e4b_last_launch_count() == 1
    ref = q4.gemv_int4b32_ref(xf, ids, rc, rs, "store")
    assert_close(y.float().cpu().numpy(), ref, f"store E={E} N={N} K={K}")


@pytest.mark.parametrize("E,I,K,ids", [(4, 200, 5120, [3, 1]), (3, 17, 1024, [0, 0, 2]), (2, 96, 2880 - 32 * 2, [1])])
def test_swiglu_matches_oracle(E, I, K, ids):
    rng = np.random.default_rng(I + K)
    codes, scales, rc, rs = _stack(rng, E, 2 * I, K)
    x, xf = _bf16(rng, (K,))
    y = torch.empty((len(ids), I + 8), dtype=torch.bfloat16, device="cuda")  # ld_y > I
    y.fill_(float("nan"))
    e4b.e4b_gemv_int4_b32("swiglu", codes, scales, torch.tensor(ids, dtype=torch.int32, device="cuda"), x.cuda(),
                          y, E=E, N=2 * I, K=K, ld_y=I + 8)
    ref = q4.gemv_int4b32_ref(xf, ids, rc, rs, "swiglu")
    out = y.float().cpu().numpy()
    assert_close(out[:, :I], ref, "swiglu")
    assert np.all(np.isnan(out[:, I:]))  # padding past N/2 untouched


@pytest.mark.parametrize("E,N,K,ids", [(8, 256, 4608, [5, 2]), (6, 77, 1280, [1, 4, 1]), (4, 40, 64, [3, 0, 1, 2])])
@pytest.mark.parametrize("per_slot", [True, False])
def test_combine_matches_oracle(E, N, K, ids, per_slot):
    rng = np.random.default_rng(E * N + K)
    codes, scales, rc, rs = _stack(rng, E, N, K)
    k = len(ids)
    x, xf = _bf16(rng, (k, K) if per_slot else (K,), 0.5)
    g = rng.random(k).astype(np.float32)
    g /= g.sum()
    y = torch.empty((N,), dtype=torch.bfloat16, device="cuda")
    e4b.e4b_gemv_int4_b32("combine", codes, scales, torch.tensor(ids, dtype=torch.int32, device="cuda"), x.cuda(), y,
                          E=E, N=N, K=K, gates=torch.from_numpy(g).cuda(), ld_x=K if per_slot else 0)
    ref = q4.gemv_int4b32_ref(xf, ids, rc, rs, "combine", g)
    assert_close(y.float().cpu().numpy(), ref, "combine")


def test_bad_expert_id_is_dropped_and_recorded():
    rng = np.random.default_rng(3)
    E, N, K = 3, 40, 256
    codes, scales, rc, rs = _stack(rng, E, N, K)
    x, xf = _bf16(rng, (K,))
    ids = [1, 9]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.full((2, N), 1.0, dtype=torch.bfloat16, device="cuda")
    e4b.e4b_gemv_int4_b32("store", codes, scales, torch.tensor(ids, dtype=torch.int32, device="cuda"), x.cuda(), y,
                          E=E, N=N, K=K, status=status)
    assert int(status.item()) == 6  # E4B_ERR_BAD_EXPERT_ID
    out = y.float().cpu().numpy()
    assert_close(out[0], q4.gemv_int4b32_ref(xf, [1], rc, rs, "store")[0], "kept slot")
    assert np.all(out[1] == 0)
    g = torch.tensor([0.25, 0.75], device="cuda")
    yc = torch.empty((N,), dtype=torch.bfloat16, device="cuda")
    e4b.e4b_gemv_int4_b32("combine", codes, scales, torch.tensor(ids, dtype=torch.int32, device="cuda"), x.cuda(), yc,
                          E=E, N=N, K=K, gates=g)
    ref = q4.gemv_int4b32_ref(xf, [1], rc, rs, "combine", np.array([0.25], np.float32))
    assert_close(yc.float().cpu().numpy(), ref, "combine without the dropped slot")


def test_zero_token_gives_zeros():
    rng = np.random.default_rng(4)
    codes, scales, _, _ = _stack(rng, 2, 20, 128)
    y = torch.full((1, 20), 1.0, dtype=torch.bfloat16, device="cuda")
    e4b.e4b_gemv_int4_b32("store", codes, scales, torch.tensor([1], dtype=torch.int32, device="cuda"),
                          torch.zeros(128, dtype=torch.bfloat16, device="cuda"), y, E=2, N=20, K=128)
    assert torch.all(y == 0)


def test_decode_layer_mid_size():
    rng = np.random.default_rng(5)
    E, H, I = 8, 1024, 2048
    gc, gs, rgc, rgs = _stack(rng, E, 2 * I, H)
    dc, ds, rdc, rds = _stack(rng, E, H, I)
    x, xf = _bf16(rng, (H,))
    ids, g = [6, 1], np.array([0.7, 0.3], np.float32)
    y = e4b.int4_decode_layer(x.cuda(), torch.tensor(ids, dtype=torch.int32, device="cuda"), torch.from_numpy(g).cuda(),
                              gc, gs, dc, ds, E=E, H=H, I=I)
    ref = q4.int4b32_decode_layer_ref(xf, ids, g, rgc, rgs, rdc, rds)
    assert_close(y.float().cpu().numpy(), ref, "int4 decode layer")


def _quantize_rows_oracle(w: np.ndarray, chunk=2048):
    codes = np.empty((w.shape[0], w.shape[1] // 2), np.uint8)
    scales = np.empty((w.shape[0], w.shape[1] // 32), np.float16)
    for r in range(0, w.shape[0], chunk):
        codes[r:r + chunk], scales[r:r + chunk] = q4.quantize_int4b32(w[r:r + chunk])
    return codes, scales


def test_decode_layer_full_size_sampled():
    # the decode shape the bench times: E=8, H=4096, I=14336, top-2, one token
    wl = DECODE
    E, H, I = wl.E, wl.H, wl.I
    dev = "cuda"
    gu = torch.stack([synth.expert_weight(wl, "gate_up", e, device=dev) for e in range(E)])
    gc, gs = e4b.quantize_int4_b32(gu)
    del gu
    dn = torch.stack([synth.expert_weight(wl, "down", e, device=dev) for e in range(E)])
    dc, ds = e4b.quantize_int4_b32(dn)
    del dn
    rng = np.random.default_rng(11)
    x, xf = _bf16(rng, (H,))
    ids, g = [5, 2], np.array([0.62, 0.38], np.float32)
    y = e4b.int4_decode_layer(x.to(dev), torch.tensor(ids, dtype=torch.int32, device=dev), torch.from_numpy(g).to(dev),
                              gc, gs, dc, ds, E=E, H=H, I=I)
    rows = np.sort(rng.choice(H, 48, replace=False))
    # the oracle quantises the routed experts' fp32 weights itself (same
    # generator, host copy): all gate_up rows (h needs them), sampled down rows
    rgc, rgs, rdc, rds = {}, {}, {}, {}
    for e in ids:
        rgc[e], rgs[e] = _quantize_rows_oracle(synth.expert_weight(wl, "gate_up", e, device=dev).cpu().numpy())
        w = synth.expert_weight(wl, "down", e, device=dev)[torch.from_numpy(rows).to(dev)].cpu().numpy()
        rdc[e], rds[e] = _quantize_rows_oracle(w)
        # the GPU codes of those rows are the oracle's bytes
        assert np.array_equal(gc[e].cpu().numpy(), rgc[e])
        assert np.array_equal(dc[e][torch.from_numpy(rows).to(dev)].cpu().numpy(), rdc[e])
    remap = {e: j for j, e in enumerate(ids)}
    gcs = np.stack([rgc[e] for e in ids]); gss = np.stack([rgs[e] for e in ids])
    dcs = np.stack([rdc[e] for e in ids]); dss = np.stack([rds[e] for e in ids])
    lids = [remap[e] for e in ids]
    h = q4.gemv_int4b32_ref(xf, lids, gcs, gss, "swiglu")
    ref = q4.gemv_int4b32_ref(h, lids, dcs, dss, "combine", g)
    assert_close(y.float().cpu().numpy()[rows], ref, "full-size int4 decode layer (sampled rows)")


def test_timeout_path_records_status_and_returns():
    # every bounded wait gives up at once: the kernel drains its copies,
    # records E4B_ERR_DEVICE_TIMEOUT, writes no output, and the context stays usable
    rng = np.random.default_rng(6)
    codes, scales, rc, rs = _stack(rng, 2, 64, 1024)
    x, xf = _bf16(rng, (1024,))
    ids = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.full((2, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    e4b.e4b_gemv_int4_b32("store", codes, scales, ids, x.cuda(), y, E=2, N=64, K=1024, status=status,
                          flags=e4b.FLAG_TEST_TIMEOUT)
    assert int(status.item()) == 5  # E4B_ERR_DEVICE_TIMEOUT
    assert torch.all(y == 3.0)
    y2 = torch.empty((2, 64), dtype=torch.bfloat16, device="cuda")
    e4b.e4b_gemv_int4_b32("store", codes, scales, ids, x.cuda(), y2, E=2, N=64, K=1024)
    assert_close(y2.float().cpu().numpy(), q4.gemv_int4b32_ref(xf, [1, 0], rc, rs, "store"), "after a timeout")


def test_layer_forward_int4_through_moe_forward():
    # e4b_moe_forward on int4-b32 stacks: two decode GEMVs a token, in one call
    rng = np.random.default_rng(21)
    E, H, I, T, k = 8, 512, 1024, 3, 2
    gc, gs, rgc, rgs = _stack(rng, E, 2 * I, H)
    dc, ds, rdc, rds = _stack(rng, E, H, I)
    layer = e4b.PackedLayer("int4b32", E, H, I, gc, gs, dc, ds)
    x, xf = _bf16(rng, (T, H))
    ids = np.array([[3, 5], [0, 0], [7, 2]], np.int32)  # a duplicate expert in token 1
    gates = np.array([[0.6, 0.4], [0.5, 0.5], [0.9, 0.1]], np.float32)
    y = e4b.moe_forward(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(gates).cuda())
    torch.cuda.synchronize()
    assert e4b.e4b_last_path() == e4b.E4B_PATH_INT4_GEMV and e4b.e4b_last_launch_count() == 2 * T
    for t in range(T):
        ref = q4.int4b32_decode_layer_ref(xf[t], list(ids[t]), gates[t], rgc, rgs, rdc, rds)
        assert_close(y[t].float().cpu().numpy(), ref, f"int4 layer token {t}")
