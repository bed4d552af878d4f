"""Helpers for the GPU parity tests: build packed layers on both sides and
compare with the tolerance of the layer's fp outputs."""

import numpy as np
import torch

import oracle
from bit_grouped_moe_e4b_b200 import e4b

# max |y - y_ref| <= TOL * (s + |y_ref|), elementwise, with s = min(1,
# rms(y_ref)) (fp32 accumulation on the GPU, fp64 in the oracle, both with
# the same bf16 decode and bf16 h). For outputs of unit scale or larger this is
# the layer's stated tolerance max |y - y_ref| <= 1e-2 * (1 + |y_ref|); for
# outputs much smaller than 1 the absolute term shrinks with them, so that a
# wrong result cannot hide below the "1" (every source of error in the path
# -- bf16 rounding of weights, h and y, fp32 sums -- is relative to the
# output scale).
TOL = 1e-2


def rms(a) -> float:
    a = np.asarray(a, np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


def scaled_err(y, y_ref) -> float:
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    if not y.size:
        return 0.0
    s = min(1.0, max(rms(y_ref), 1e-30))
    return float(np.max(np.abs(y - y_ref) / (s + np.abs(y_ref))))


def assert_close(y, y_ref, what="", tol=TOL, min_rms=None):
    """min_rms: also require rms(y_ref) >= min_rms (the comparison runs at
    outputs of that scale, where the tolerance is the layer's own)."""
    err = scaled_err(y, y_ref)
    assert np.all(np.isfinite(y)), what
    if min_rms is not None:
        r = rms(y_ref)
        assert r >= min_rms, f"{what}: reference outputs too small to discriminate (rms {r:.3g} < {min_rms})"
    assert err <= tol, f"{what}: max scaled error {err:.4g} > {tol}"
    return err


# Layers built by small_layer() with the default weight scale give outputs of
# rms ~2 (median |y| ~1.4); comparisons on them assert at least this rms.
LAYER_MIN_RMS = 0.5


# Between the two kernel paths on NF4: their decode readings ("level" on
# small-M, "product" on tcgen05) differ by up to one bf16 rounding of every
# weight, which at full size moves outputs by a few 1e-2 of the scale; each
# path matches its own reading within TOL.
TOL_NF4_ACROSS_PATHS = 5e-2


def oracle_quantize(fmt, w: np.ndarray):
    if fmt == "nf4":
        return oracle.quantize_pack_nf4(w)
    return oracle.quantize_pack_mxfp4(w)


def _spread(rng, w):
    """Multiplies every 32-wide block along K by its own power of two in
    [2^-2, 2^2], so neighbouring blocks get different scales."""
    E, N, K = w.shape
    f = np.exp2(rng.integers(-2, 3, size=(E, N, K // 32))).astype(np.float32)
    return (w.reshape(E, N, K // 32, 32) * f[..., None]).reshape(E, N, K)


def small_layer(fmt, E, H, I, seed, std=None, spread=False):
    """Random layer quantised by the GPU and by the oracle; checks the codes
    agree bit for bit. Returns (PackedLayer, oracle tuple (gc, gs, dc, ds)).
    std=None draws gate_up with standard deviation 1.5/sqrt(H) and down with
    2/sqrt(I), so that x ~ N(0, 1) gives outputs of rms ~2; a number uses that
    standard deviation for both. spread=True varies the block scales along K
    by powers of two."""
    rng = np.random.default_rng(seed)
    std_gu = 1.5 / np.sqrt(H) if std is None else std
    std_dn = 2.0 / np.sqrt(I) if std is None else std
    wgu = (rng.standard_normal((E, 2 * I, H)) * std_gu).astype(np.float32)
    wd = (rng.standard_normal((E, H, I)) * std_dn).astype(np.float32)
    if spread:
        wgu = _spread(rng, wgu)
        wd = _spread(rng, wd)
    gc_d, gs_d = e4b.quantize(fmt, torch.from_numpy(wgu).cuda())
    dc_d, ds_d = e4b.quantize(fmt, torch.from_numpy(wd).cuda())
    gc, gs = oracle_quantize(fmt, wgu)
    dc, ds = oracle_quantize(fmt, wd)
    for got, want in ((gc_d, gc), (gs_d, gs), (dc_d, dc), (ds_d, ds)):
        assert np.array_equal(got.cpu().numpy(), want)
    layer = e4b.PackedLayer(fmt, E, H, I, gc_d, gs_d, dc_d, ds_d)
    return layer, (gc, gs, dc, ds)


_last = {"flags": 0}


def last_nf4_decode() -> str:
    """The NF4 decode reading the last layer call used: the small-M path's
    default "level" (bf16(level), absmax after the block's MMA) unless the
    product flag was given; "product" (bf16(fp32(level * absmax))) on tcgen05."""
    if e4b.e4b_last_path() == e4b.E4B_PATH_GEMV and not (_last["flags"] & e4b.FLAG_NF4_PRODUCT_DECODE):
        return "level"
    return "product"


def run_layer(layer, x_bf16: torch.Tensor, ids: np.ndarray, gates: np.ndarray, flags=0, staged=True):
    """staged=False hands the layer a workspace without room for the staging
    copy of the routed rows (the last [T*k, H] bf16 region), so the large-M
    path gathers the rows inside its kernel."""
    ids_d = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()
    g_d = torch.from_numpy(np.ascontiguousarray(gates, np.float32)).cuda()
    x_d = x_bf16.cuda()
    ws = e4b.workspace(layer, ids.shape[0], ids.shape[1])
    if not staged:
        ws = ws[: ws.numel() - (ids.size * layer.H * 2 + 255) // 256 * 256]
    _last["flags"] = flags
    y = e4b.moe_forward(layer, x_d, ids_d, g_d, ws=ws, flags=flags)
    status = e4b.e4b_read_device_status(ws)
    return y.float().cpu().numpy(), status, ws


def oracle_layer(fmt, x_bf16: torch.Tensor, ids, gates, ref, E, H, I, tokens=None, nf4_decode="last"):
    """The oracle's layer forward; nf4_decode "last" = the reading the last
    layer call used (last_nf4_decode)."""
    gc, gs, dc, ds = ref
    mode = last_nf4_decode() if nf4_decode == "last" else nf4_decode
    return oracle.moe_forward_ref(fmt, x_bf16.float().numpy(), ids, gates, gc, gs, dc, ds, E, H, I,
                                  tokens=tokens, nf4_decode=mode)
