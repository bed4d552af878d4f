"""ctypes binding of libe4b.so (include/e4b.h), argument marshalling only.

Every function named ``e4b_*`` here calls the C entry point of the same name
with device pointers taken from torch tensors and the current CUDA stream.
All compute happens in the library's kernels; a missing library raises
``E4BError`` on first use (there is no CPU fallback). Helpers without the
prefix allocate outputs with torch and then call the ``e4b_*`` function.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libe4b.so")

E4B_OK = 0
E4B_FMT_NF4, E4B_FMT_MXFP4, E4B_FMT_INT4B32 = 0, 1, 2
E4B_EPI_STORE, E4B_EPI_SWIGLU, E4B_EPI_COMBINE = 0, 1, 2
E4B_PATH_NONE, E4B_PATH_GEMV, E4B_PATH_TCGEN05, E4B_PATH_INT4_GEMV, E4B_PATH_TCGEN05_MX = 0, 1, 2, 3, 4
FLAG_FORCE_GEMV = 0x1
FLAG_FORCE_TCGEN05 = 0x2
FLAG_TEST_TIMEOUT = 0x4
FLAG_IDS_READY = 0x10  # e4b_gemv_int4_b32: ids and gates not written by the preceding work on the stream
FLAG_MX_ACT_E4M3 = 0x20  # native MXFP4 path: one e4m3 term per activation (OCP MXFP8 rule)
FLAG_MX_DECODE = 0x40  # MXFP4 with prepared stacks: the decode-to-bf16 tcgen05 path anyway
FLAG_TC_SINGLE_SM = 0x80  # large-M projections on the one-SM tcgen05 kernel instead of SM pairs
FLAG_NF4_PRODUCT_DECODE = 0x8  # small-M NF4: bf16(level * absmax) operands (the default is bf16(level), absmax after the block MMA)
STATUS_NAMES = {
    0: "E4B_OK", 1: "E4B_ERR_INVALID_ARG", 2: "E4B_ERR_UNSUPPORTED",
    3: "E4B_ERR_WORKSPACE_TOO_SMALL", 4: "E4B_ERR_CUDA", 5: "E4B_ERR_DEVICE_TIMEOUT",
    6: "E4B_ERR_BAD_EXPERT_ID", 7: "E4B_ERR_MISALIGNED", 8: "E4B_ERR_EXCEEDS_STATIC_SCRATCH",
}
FMT = {"nf4": E4B_FMT_NF4, "mxfp4": E4B_FMT_MXFP4, "int4b32": E4B_FMT_INT4B32}

# Every symbol include/e4b.h declares.
EXPORTED = [
    "e4b_quantize_nf4", "e4b_quantize_mxfp4", "e4b_dequantize", "e4b_nf4_codebook",
    "e4b_route_workspace_size", "e4b_route", "e4b_grouped_gemm", "e4b_grouped_dgrad", "e4b_moe_workspace_size",
    "e4b_moe_forward", "e4b_moe_forward_noalloc", "e4b_read_device_status", "e4b_set_timing_events", "e4b_last_path",
    "e4b_last_launch_count",
    "e4b_status_string", "e4b_version",
    "e4b_quantize_int4_b32", "e4b_gptq_pack_int4_b32", "e4b_gemv_int4_b32",
    "e4b_ep_dest", "e4b_ep_pack", "e4b_ep_combine",
    "e4b_mxfp4_native_size", "e4b_mxfp4_native_prepare", "e4b_quantize_mxfp8",
]
EPI = {"store": E4B_EPI_STORE, "swiglu": E4B_EPI_SWIGLU, "combine": E4B_EPI_COMBINE}


class E4BError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class MoeWeights(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32), ("E", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
        ("gate_up_codes", ctypes.c_void_p), ("gate_up_scales", ctypes.c_void_p),
        ("down_codes", ctypes.c_void_p), ("down_scales", ctypes.c_void_p),
        ("gate_up_layout", ctypes.c_int32), ("activation", ctypes.c_int32),
        ("glu_alpha", ctypes.c_float), ("glu_limit", ctypes.c_float),
        ("gate_up_bias", ctypes.c_void_p), ("down_bias", ctypes.c_void_p),
        ("gate_up_mx_codes", ctypes.c_void_p), ("gate_up_mx_sf", ctypes.c_void_p),
        ("down_mx_codes", ctypes.c_void_p), ("down_mx_sf", ctypes.c_void_p),
    ]


class GemmArgs(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32), ("epilogue", ctypes.c_int32), ("E", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
        ("R_max", ctypes.c_int64), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("a", ctypes.c_void_p), ("lda", ctypes.c_int64), ("a_row_slot", ctypes.c_void_p),
        ("out_row_slot", ctypes.c_void_p), ("offsets", ctypes.c_void_p), ("gates", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("ldo", ctypes.c_int64),
        ("gate_up_layout", ctypes.c_int32), ("activation", ctypes.c_int32),
        ("glu_alpha", ctypes.c_float), ("glu_limit", ctypes.c_float), ("bias", ctypes.c_void_p),
    ]


class DgradArgs(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32), ("E", ctypes.c_int32), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
        ("R_max", ctypes.c_int64), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("dy", ctypes.c_void_p), ("ld_dy", ctypes.c_int64), ("offsets", ctypes.c_void_p),
        ("dx", ctypes.c_void_p), ("ld_dx", ctypes.c_int64),
    ]


class Int4GemvArgs(ctypes.Structure):
    _fields_ = [
        ("epilogue", ctypes.c_int32), ("E", ctypes.c_int32), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
        ("n_slots", ctypes.c_int32), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("expert_ids", ctypes.c_void_p), ("gates", ctypes.c_void_p), ("x", ctypes.c_void_p),
        ("ld_x", ctypes.c_int64), ("y", ctypes.c_void_p), ("ld_y", ctypes.c_int64), ("status", ctypes.c_void_p),
    ]


# expert-variant codes (include/e4b.h)
LAYOUT = {"halves": 0, "interleaved": 1}
ACT = {"swiglu": 0, "clamped_glu": 1}


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libe4b.so (once). Raises E4BError-like RuntimeError if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m bit_grouped_moe_e4b_b200.build` (no CPU fallback exists)")
    L = ctypes.CDLL(LIB_PATH)
    i32, i64, vp, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    sig = {
        "e4b_quantize_nf4": [vp, i64, i64, i64, i32, vp, vp, vp],
        "e4b_quantize_mxfp4": [vp, i64, i64, i64, vp, vp, vp],
        "e4b_dequantize": [i32, vp, vp, i64, i64, i64, vp, vp],
        "e4b_nf4_codebook": [vp],
        "e4b_route_workspace_size": [i64, i32, i32, ctypes.POINTER(sz)],
        "e4b_route": [vp, i64, i32, i32, vp, vp, vp, vp, vp, sz, vp],
        "e4b_grouped_gemm": [ctypes.POINTER(GemmArgs), ctypes.c_uint32, vp],
        "e4b_grouped_dgrad": [ctypes.POINTER(DgradArgs), ctypes.c_uint32, vp],
        "e4b_moe_workspace_size": [ctypes.POINTER(MoeWeights), i64, i32, ctypes.POINTER(sz)],
        "e4b_moe_forward": [ctypes.POINTER(MoeWeights), vp, i64, i32, vp, vp, vp, vp, sz,
                            ctypes.c_uint32, vp],
        "e4b_moe_forward_noalloc": [ctypes.POINTER(MoeWeights), vp, i64, i32, vp, vp, vp,
                                    ctypes.c_uint32, vp],
        "e4b_read_device_status": [vp, ctypes.POINTER(i32), vp],
        "e4b_set_timing_events": [ctypes.POINTER(vp), i32],
        "e4b_last_path": [],
        "e4b_last_launch_count": [],
        "e4b_status_string": [i32],
        "e4b_version": [],
        "e4b_quantize_int4_b32": [vp, i64, i64, i64, vp, vp, vp],
        "e4b_gptq_pack_int4_b32": [vp, vp, i64, i64, i64, vp, vp, vp],
        "e4b_gemv_int4_b32": [ctypes.POINTER(Int4GemvArgs), ctypes.c_uint32, vp],
        "e4b_ep_dest": [vp, i64, i32, i32, vp, vp],
        "e4b_ep_pack": [vp, i64, vp, vp, i32, vp, vp, i32, i64, i32, vp, vp, vp, vp],
        "e4b_ep_combine": [vp, i64, vp, i64, i32, vp, vp],
        "e4b_mxfp4_native_size": [i32, i64, i64, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)],
        "e4b_mxfp4_native_prepare": [vp, vp, i32, i64, i64, i32, i32, vp, vp, vp],
        "e4b_quantize_mxfp8": [vp, i64, i64, vp, vp, vp],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_char_p if name in ("e4b_status_string", "e4b_version") else ctypes.c_int32
    _lib = L
    return L


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != E4B_OK:
        raise E4BError(status, where)


def _dev(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("e4b kernels take CUDA tensors")
        if t is not None and not t.is_contiguous():
            raise ValueError("e4b kernels take contiguous tensors")


# ------------------------------------------------------------------ formats
def e4b_quantize_nf4(w, codes, absmax, blocksize=64, stream=None):
    _dev(w, codes, absmax)
    E, N, K = w.shape
    _check(lib().e4b_quantize_nf4(_ptr(w), E, N, K, blocksize, _ptr(codes), _ptr(absmax),
                                  _stream(stream)), "e4b_quantize_nf4")


def e4b_quantize_mxfp4(w, blocks, scales, stream=None):
    _dev(w, blocks, scales)
    E, N, K = w.shape
    _check(lib().e4b_quantize_mxfp4(_ptr(w), E, N, K, _ptr(blocks), _ptr(scales), _stream(stream)),
           "e4b_quantize_mxfp4")


def e4b_dequantize(fmt, codes, scales, E, N, K, out, stream=None):
    _dev(codes, scales, out)
    _check(lib().e4b_dequantize(FMT.get(fmt, fmt), _ptr(codes), _ptr(scales), E, N, K, _ptr(out),
                                _stream(stream)), "e4b_dequantize")


def e4b_nf4_codebook():
    import numpy as np
    out = (ctypes.c_float * 16)()
    _check(lib().e4b_nf4_codebook(ctypes.cast(out, ctypes.c_void_p)), "e4b_nf4_codebook")
    return np.array(out[:], dtype=np.float32)


def quantize(fmt: str, w: torch.Tensor):
    """Packs fp32 weights [E, N, K] on the GPU; returns (codes, scales)."""
    E, N, K = w.shape
    if fmt == "nf4":
        codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=w.device)
        scales = torch.empty((E, N, K // 64), dtype=torch.float32, device=w.device)
        e4b_quantize_nf4(w, codes, scales)
    else:
        codes = torch.empty((E, N, K // 32, 16), dtype=torch.uint8, device=w.device)
        scales = torch.empty((E, N, K // 32), dtype=torch.uint8, device=w.device)
        e4b_quantize_mxfp4(w, codes, scales)
    return codes, scales


def dequantize(fmt: str, codes, scales, E, N, K):
    out = torch.empty((E, N, K), dtype=torch.bfloat16, device=codes.device)
    e4b_dequantize(fmt, codes, scales, E, N, K, out)
    return out


def e4b_mxfp4_native_size(E, rows_per_mat, K, nmat):
    c, f = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib().e4b_mxfp4_native_size(E, rows_per_mat, K, nmat, ctypes.byref(c), ctypes.byref(f)),
           "e4b_mxfp4_native_size")
    return c.value, f.value


def mxfp4_native_prepare(blocks, scales, E, rows_per_mat, K, nmat, layout="halves", stream=None):
    """The prepared copy of an MXFP4 stack for the block-scaled FP4 MMA (see
    e4b.h); returns (codes uint8, scale chunks uint8), flat."""
    _dev(blocks, scales)
    cb, fb = e4b_mxfp4_native_size(E, rows_per_mat, K, nmat)
    codes = torch.empty(cb, dtype=torch.uint8, device=blocks.device)
    sf = torch.empty(fb, dtype=torch.uint8, device=blocks.device)
    _check(lib().e4b_mxfp4_native_prepare(_ptr(blocks), _ptr(scales), E, rows_per_mat, K, nmat, LAYOUT[layout],
                                          _ptr(codes), _ptr(sf), _stream(stream)), "e4b_mxfp4_native_prepare")
    return codes, sf


def quantize_mxfp8(x: torch.Tensor, stream=None):
    """bf16 [R, K] -> (E4M3 bytes uint8 [R, K], e8m0 scale bytes uint8 [R, K/32])."""
    _dev(x)
    R, K = x.shape
    elems = torch.empty((R, K), dtype=torch.uint8, device=x.device)
    scales = torch.empty((R, K // 32), dtype=torch.uint8, device=x.device)
    _check(lib().e4b_quantize_mxfp8(_ptr(x), R, K, _ptr(elems), _ptr(scales), _stream(stream)),
           "e4b_quantize_mxfp8")
    return elems, scales


# ------------------------------------------------------------------ routing
# ------------------------------------------------------------- int4-b32
def e4b_quantize_int4_b32(w, codes, scales, stream=None):
    """fp32 w [E, N, K] -> codes uint8 [E, N, K/2], scales fp16 [E, N, K/32]."""
    _dev(w, codes, scales)
    E, N, K = w.shape
    _check(lib().e4b_quantize_int4_b32(_ptr(w), E, N, K, _ptr(codes), _ptr(scales), _stream(stream)),
           "e4b_quantize_int4_b32")


def e4b_gptq_pack_int4_b32(qweight, gptq_scales, codes, scales, *, E, N, K, stream=None):
    """GPTQ qweight int32 [E, K/8, N] + scales fp16 [E, K/32, N] -> int4-b32 codes/scales."""
    _dev(qweight, gptq_scales, codes, scales)
    _check(lib().e4b_gptq_pack_int4_b32(_ptr(qweight), _ptr(gptq_scales), E, N, K, _ptr(codes), _ptr(scales),
                                        _stream(stream)), "e4b_gptq_pack_int4_b32")


def e4b_gemv_int4_b32(epilogue, codes, scales, expert_ids, x, y, *, E, N, K, gates=None, ld_x=0, ld_y=None,
                      status=None, flags=0, stream=None):
    """The int4-b32 decode GEMV of one token over its routed experts (include/e4b.h)."""
    _dev(codes, scales, expert_ids, x, y, gates, status)
    epi = EPI.get(epilogue, epilogue)
    n_slots = expert_ids.numel()
    if ld_y is None:
        ld_y = N // 2 if epi == E4B_EPI_SWIGLU else N
    a = Int4GemvArgs(epi, E, N, K, n_slots, codes.data_ptr(), scales.data_ptr(), expert_ids.data_ptr(),
                     None if gates is None else gates.data_ptr(), x.data_ptr(), ld_x, y.data_ptr(), ld_y,
                     None if status is None else status.data_ptr())
    _check(lib().e4b_gemv_int4_b32(ctypes.byref(a), flags, _stream(stream)), "e4b_gemv_int4_b32")


def quantize_int4_b32(w: torch.Tensor):
    """Packs fp32 weights [E, N, K] into int4-b32 on the GPU; returns (codes, scales)."""
    E, N, K = w.shape
    codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((E, N, K // 32), dtype=torch.float16, device=w.device)
    e4b_quantize_int4_b32(w, codes, scales)
    return codes, scales


def int4_decode_layer(x, expert_ids, gates, gu_codes, gu_scales, dn_codes, dn_scales, *, E, H, I, h=None, y=None):
    """One token through the MoE layer on int4-b32 stacks: the gate_up GEMV
    with the SwiGLU epilogue (h [k, I]), then the down GEMV with the combine
    epilogue (y [H]). Two launches (the second a programmatic dependent of the
    first); returns y."""
    k = expert_ids.numel()
    if h is None:
        h = torch.empty((k, I), dtype=torch.bfloat16, device=x.device)
    if y is None:
        y = torch.empty((H,), dtype=torch.bfloat16, device=x.device)
    e4b_gemv_int4_b32("swiglu", gu_codes, gu_scales, expert_ids, x, h, E=E, N=2 * I, K=H, ld_y=I)
    # the ids and gates were read by the gate_up launch: the down launch may
    # start streaming its experts' weights while gate_up finishes
    e4b_gemv_int4_b32("combine", dn_codes, dn_scales, expert_ids, h, y, E=E, N=H, K=I, gates=gates, ld_x=I,
                      flags=FLAG_IDS_READY)
    return y


# ---------------------------------------------------------- expert parallel
def e4b_ep_dest(ids, E, epr, dest, stream=None):
    _dev(ids, dest)
    _check(lib().e4b_ep_dest(_ptr(ids), ids.numel(), E, epr, _ptr(dest), _stream(stream)), "e4b_ep_dest")


def e4b_ep_pack(x, ids, gates, perm, offsets, G, R_max, epr, xs, local_ids, local_gates, stream=None):
    _dev(x, ids, gates, perm, offsets, xs, local_ids, local_gates)
    _check(lib().e4b_ep_pack(_ptr(x), x.shape[1], _ptr(ids), _ptr(gates), ids.shape[1], _ptr(perm), _ptr(offsets),
                             G, R_max, epr, _ptr(xs), _ptr(local_ids), _ptr(local_gates), _stream(stream)),
           "e4b_ep_pack")


def e4b_ep_combine(ys, inv_perm, T, top_k, y, stream=None):
    _dev(ys, inv_perm, y)
    _check(lib().e4b_ep_combine(_ptr(ys), y.shape[1], _ptr(inv_perm), T, top_k, _ptr(y), _stream(stream)),
           "e4b_ep_combine")


def e4b_route_workspace_size(T, top_k, E) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().e4b_route_workspace_size(T, top_k, E, ctypes.byref(n)), "e4b_route_workspace_size")
    return n.value


def e4b_route(ids, E, counts, offsets, perm, inv_perm, ws, stream=None):
    _dev(ids, counts, offsets, perm, inv_perm, ws)
    T, k = ids.shape
    _check(lib().e4b_route(_ptr(ids), T, k, E, _ptr(counts), _ptr(offsets), _ptr(perm),
                           _ptr(inv_perm), _ptr(ws), ws.numel() * ws.element_size(),
                           _stream(stream)), "e4b_route")


def route(ids: torch.Tensor, E: int):
    T, k = ids.shape
    dev = ids.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int64, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    ws = torch.empty(e4b_route_workspace_size(T, k, E), dtype=torch.uint8, device=dev)
    e4b_route(ids, E, counts, offsets, perm, inv, ws)
    return counts, offsets, perm, inv, ws


# --------------------------------------------------------------- grouped GEMM
def e4b_grouped_dgrad(fmt, codes, scales, dy, offsets, dx, *, E, N, K, R_max, flags=0, stream=None):
    """dx[p] = dy[p] . W_e for the routed rows p of each expert (dy [R, N],
    dx [R, K], bf16, rows in expert order)."""
    _dev(codes, scales, dy, offsets, dx)
    args = DgradArgs(FMT.get(fmt, fmt), E, N, K, R_max, _ptr(codes), _ptr(scales), _ptr(dy), dy.shape[-1],
                     _ptr(offsets), _ptr(dx), dx.shape[-1])
    _check(lib().e4b_grouped_dgrad(ctypes.byref(args), flags, _stream(stream)), "e4b_grouped_dgrad")



def e4b_grouped_gemm(fmt, epilogue, codes, scales, a, offsets, out, *, E, N, K, R_max, top_k=1,
                     a_row_slot=None, out_row_slot=None, gates=None, flags=0, stream=None,
                     layout="halves", act="swiglu", alpha=1.702, limit=7.0, bias=None):
    _dev(codes, scales, a, offsets, out, a_row_slot, out_row_slot, gates, bias)
    args = GemmArgs(FMT.get(fmt, fmt), epilogue, E, top_k, N, K, R_max, _ptr(codes), _ptr(scales),
                    _ptr(a), a.shape[-1], _ptr(a_row_slot), _ptr(out_row_slot), _ptr(offsets),
                    _ptr(gates), _ptr(out), out.shape[-1], LAYOUT[layout], ACT[act], alpha, limit,
                    _ptr(bias))
    _check(lib().e4b_grouped_gemm(ctypes.byref(args), flags, _stream(stream)), "e4b_grouped_gemm")


# ---------------------------------------------------------------- the layer
@dataclass
class PackedLayer:
    """A layer's packed expert stacks on the GPU."""
    fmt: str
    E: int
    H: int
    I: int
    gate_up_codes: torch.Tensor
    gate_up_scales: torch.Tensor
    down_codes: torch.Tensor
    down_scales: torch.Tensor
    # expert variant (include/e4b.h): "halves" | "interleaved", "swiglu" | "clamped_glu"
    layout: str = "halves"
    act: str = "swiglu"
    alpha: float = 1.702
    limit: float = 7.0
    gate_up_bias: torch.Tensor | None = None  # fp32 [E, 2I]
    down_bias: torch.Tensor | None = None     # fp32 [E, H]
    # MXFP4 stacks prepared for the block-scaled FP4 MMA (prepare_mx())
    gate_up_mx_codes: torch.Tensor | None = None
    gate_up_mx_sf: torch.Tensor | None = None
    down_mx_codes: torch.Tensor | None = None
    down_mx_sf: torch.Tensor | None = None

    def c_struct(self) -> MoeWeights:
        _dev(self.gate_up_codes, self.gate_up_scales, self.down_codes, self.down_scales,
             self.gate_up_bias, self.down_bias, self.gate_up_mx_codes, self.gate_up_mx_sf,
             self.down_mx_codes, self.down_mx_sf)
        return MoeWeights(FMT[self.fmt], self.E, self.H, self.I, self.gate_up_codes.data_ptr(),
                          self.gate_up_scales.data_ptr(), self.down_codes.data_ptr(),
                          self.down_scales.data_ptr(), LAYOUT[self.layout], ACT[self.act],
                          self.alpha, self.limit, _ptr(self.gate_up_bias), _ptr(self.down_bias),
                          _ptr(self.gate_up_mx_codes), _ptr(self.gate_up_mx_sf), _ptr(self.down_mx_codes),
                          _ptr(self.down_mx_sf))

    def prepare_mx(self) -> "PackedLayer":
        """A copy of this MXFP4 layer with its stacks also prepared for the
        block-scaled FP4 MMA (e4b_mxfp4_native_prepare)."""
        import dataclasses
        if self.fmt != "mxfp4":
            raise ValueError("only MXFP4 stacks have a block-scaled MMA form")
        gc, gs = mxfp4_native_prepare(self.gate_up_codes, self.gate_up_scales, self.E, self.I, self.H, 2,
                                      self.layout)
        dc, ds = mxfp4_native_prepare(self.down_codes, self.down_scales, self.E, self.H, self.I, 1)
        return dataclasses.replace(self, gate_up_mx_codes=gc, gate_up_mx_sf=gs, down_mx_codes=dc, down_mx_sf=ds)

    def packed_bytes_per_expert(self) -> int:
        return (self.gate_up_codes[0].numel() + self.gate_up_scales[0].numel() * self.gate_up_scales.element_size()
                + self.down_codes[0].numel() + self.down_scales[0].numel() * self.down_scales.element_size())


def e4b_moe_workspace_size(layer: PackedLayer, T: int, top_k: int) -> int:
    n = ctypes.c_size_t(0)
    w = layer.c_struct()
    _check(lib().e4b_moe_workspace_size(ctypes.byref(w), T, top_k, ctypes.byref(n)),
           "e4b_moe_workspace_size")
    return n.value


def e4b_moe_forward(layer: PackedLayer, x, ids, gates, y, ws, flags=0, stream=None):
    _dev(x, ids, gates, y, ws)
    T, k = ids.shape
    w = layer.c_struct()
    _check(lib().e4b_moe_forward(ctypes.byref(w), _ptr(x), T, k, _ptr(ids), _ptr(gates), _ptr(y),
                                 _ptr(ws), ws.numel() * ws.element_size(), flags, _stream(stream)),
           "e4b_moe_forward")


def e4b_moe_forward_noalloc(layer: PackedLayer, x, ids, gates, y, flags=0, stream=None):
    """The layer forward with the library's static scratch instead of a
    workspace, for callers that cannot allocate device memory (see e4b.h)."""
    _dev(x, ids, gates, y)
    T, k = ids.shape
    w = layer.c_struct()
    _check(lib().e4b_moe_forward_noalloc(ctypes.byref(w), _ptr(x), T, k, _ptr(ids), _ptr(gates),
                                         _ptr(y), flags, _stream(stream)),
           "e4b_moe_forward_noalloc")


def e4b_read_device_status(ws, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(lib().e4b_read_device_status(_ptr(ws), ctypes.byref(v), _stream(stream)),
           "e4b_read_device_status")
    return v.value


def e4b_set_timing_events(events=None):
    """events: five torch.cuda.Event(enable_timing=True) or None to stop."""
    if not events:
        _check(lib().e4b_set_timing_events(None, 0), "e4b_set_timing_events")
        return
    arr = (ctypes.c_void_p * 5)(*[ev.cuda_event for ev in events])
    _check(lib().e4b_set_timing_events(arr, 5), "e4b_set_timing_events")


def e4b_last_path() -> int:
    return lib().e4b_last_path()


def e4b_last_launch_count() -> int:
    return lib().e4b_last_launch_count()


def e4b_status_string(s: int) -> str:
    return lib().e4b_status_string(s).decode()


def e4b_version() -> str:
    return lib().e4b_version().decode()


def workspace(layer: PackedLayer, T: int, top_k: int, device="cuda") -> torch.Tensor:
    return torch.empty(e4b_moe_workspace_size(layer, T, top_k), dtype=torch.uint8, device=device)


def moe_forward(layer: PackedLayer, x, ids, gates, ws=None, flags=0):
    """y = the MoE layer on x (bf16 [T, H]) with routing ids / gates [T, k]."""
    T, k = ids.shape
    if ws is None:
        ws = workspace(layer, T, k, x.device)
    y = torch.empty((T, layer.H), dtype=torch.bfloat16, device=x.device)
    e4b_moe_forward(layer, x, ids, gates, y, ws, flags)
    return y
