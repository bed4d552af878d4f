"""The C-ABI library without a GPU: it loads, exports every entry point that
include/e4b.h declares, and rejects bad arguments on the host before any
launch."""

import ctypes
import os
import re

import numpy as np
import pytest

from conftest import ROOT
from golden_io import read_floats
from bit_grouped_moe_e4b_b200 import e4b

HEADER = os.path.join(ROOT, "include", "e4b.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(e4b_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = e4b.lib()
    names = declared_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert sorted(e4b.EXPORTED) == names


def test_version_and_status_strings():
    assert "sm_100a" in e4b.e4b_version()
    assert e4b.e4b_status_string(0) == "ok"
    assert "expert id" in e4b.e4b_status_string(6)


def test_library_codebook_is_the_published_table():
    pub = np.array(read_floats("nf4_codebook_qlora.txt"), dtype=np.float32)
    assert np.array_equal(e4b.e4b_nf4_codebook().view(np.uint32), pub.view(np.uint32))


def _w(fmt=0, E=8, H=256, I=512, ptr=4096):
    return e4b.MoeWeights(fmt, E, H, I, ptr, ptr, ptr, ptr)


def test_host_argument_checks_return_before_launch():
    L = e4b.lib()
    n = ctypes.c_size_t(0)
    w = _w()
    assert L.e4b_moe_workspace_size(ctypes.byref(w), 64, 2, ctypes.byref(n)) == 0
    need = n.value
    assert need > 64 * 2 * 512 * 2  # holds at least h
    fwd = L.e4b_moe_forward
    p = ctypes.c_void_p(4096)
    # T == 0 is a no-op
    assert fwd(ctypes.byref(w), None, 0, 2, None, None, None, None, 0, 0, None) == 0
    # null pointers
    assert fwd(ctypes.byref(w), None, 4, 2, p, p, p, p, need, 0, None) == 1
    # top_k > E
    assert fwd(ctypes.byref(_w(E=2)), p, 4, 3, p, p, p, p, need, 0, None) == 1
    # unsupported shapes: NF4 needs H, I multiples of 64
    assert fwd(ctypes.byref(_w(H=96)), p, 4, 2, p, p, p, p, need, 0, None) == 2
    # misaligned
    assert fwd(ctypes.byref(w), ctypes.c_void_p(4098), 4, 2, p, p, p, p, need, 0, None) == 7
    # workspace too small: below the required part of the path taken. The size
    # query ends with one fp32 region (the small-M path's partial sums
    # [K slices][T*k][H], or the large-M path's gate-weighted rows [T*k, H];
    # one K slice here, I = 512) and an optional [T*k, H] bf16 staging copy,
    # each 256-byte aligned; both paths need everything but the staging copy.
    staging = (64 * 2 * 256 * 2 + 255) // 256 * 256
    assert fwd(ctypes.byref(w), p, 64, 2, p, p, p, p, need - staging - 1, 0, None) == 3
    assert fwd(ctypes.byref(w), p, 64, 2, p, p, p, p, need - staging - 1, e4b.FLAG_FORCE_TCGEN05, None) == 3
    # bad format
    assert fwd(ctypes.byref(_w(fmt=5)), p, 4, 2, p, p, p, p, need, 0, None) == 1
    # (every call above and below fails validation, so nothing is launched
    # even when a GPU is present: the pointers are not real allocations)
    # quantiser checks
    assert L.e4b_quantize_nf4(p, 1, 4, 96, 64, p, p, None) == 2
    assert L.e4b_quantize_nf4(p, 1, 4, 128, 32, p, p, None) == 2
    assert L.e4b_quantize_nf4(None, 1, 4, 128, 64, p, p, None) == 1
    assert L.e4b_quantize_mxfp4(p, 1, 4, 48, p, p, None) == 2
    # routing checks
    assert L.e4b_route(p, 4, 2, 2000, p, p, p, p, p, 256, None) == 2
    assert L.e4b_route(p, 4, 2, 8, p, p, p, p, p, 16, None) == 3
    ga = e4b.GemmArgs(0, 5, 8, 1, 256, 256, 64, 4096, 4096, 4096, 256, None, None, 4096, None, 4096, 256)
    assert L.e4b_grouped_gemm(ctypes.byref(ga), 0, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        e4b.e4b_quantize_nf4(torch.zeros(1, 4, 64), torch.zeros(1, 4, 32, dtype=torch.uint8),
                             torch.zeros(1, 4, 1))


def test_variant_argument_checks():
    L = e4b.lib()
    p = ctypes.c_void_p(4096)
    n = ctypes.c_size_t(0)
    w = _w()
    assert L.e4b_moe_workspace_size(ctypes.byref(w), 64, 2, ctypes.byref(n)) == 0
    fwd = L.e4b_moe_forward

    def variant(**kw):
        v = _w()
        v.glu_alpha, v.glu_limit = 1.702, 7.0
        for k, val in kw.items():
            setattr(v, k, val)
        return fwd(ctypes.byref(v), p, 64, 2, p, p, p, p, n.value, 0, None)

    assert variant(gate_up_layout=2) == 1
    assert variant(activation=-1) == 1
    assert variant(activation=1, glu_limit=-0.5) == 1
    assert variant(activation=1, glu_limit=float("nan")) == 1
    assert variant(gate_up_bias=4100) == 7
    assert variant(down_bias=4104) == 7
    ga = e4b.GemmArgs(0, 1, 8, 1, 256, 256, 64, 4096, 4096, 4096, 256, None, None, 4096, None, 4096, 128,
                      1, 1, 1.702, -1.0, None)
    assert L.e4b_grouped_gemm(ctypes.byref(ga), 0, None) == 1
    ga.glu_limit, ga.bias = 7.0, 4108
    assert L.e4b_grouped_gemm(ctypes.byref(ga), 0, None) == 7


def test_binding_structs_match_the_header(tmp_path):
    # sizes and field offsets of the two argument structs, as a C compiler
    # lays them out from include/e4b.h, against the ctypes mirrors
    structs = {"e4b_moe_weights": e4b.MoeWeights, "e4b_gemm_args": e4b.GemmArgs, "e4b_dgrad_args": e4b.DgradArgs,
               "e4b_int4_gemv_args": e4b.Int4GemvArgs}
    src = ["#include <stdio.h>", "#include <stddef.h>", '#include "e4b.h"', "int main(void) {"]
    for cname, py in structs.items():
        src.append(f'printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            src.append(f'printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    src += ["return 0; }"]
    c = tmp_path / "layout.c"
    c.write_text("\n".join(src))
    exe = tmp_path / "layout"
    import subprocess
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        s, f, v = line.split()
        got[(s, f)] = int(v)
    for cname, py in structs.items():
        assert got[(cname, "sizeof")] == ctypes.sizeof(py), cname
        for f, _ in py._fields_:
            assert got[(cname, f)] == getattr(py, f).offset, (cname, f)


def test_dgrad_argument_checks():
    L = e4b.lib()
    p = 4096

    def call(**kw):
        a = e4b.DgradArgs(0, 4, 256, 128, 64, p, p, p, 256, p, p, 128)
        for k, v in kw.items():
            setattr(a, k, v)
        return L.e4b_grouped_dgrad(ctypes.byref(a), 0, None)

    assert call(fmt=7) == 1
    assert call(K=96) == 2            # NF4 needs K % 64
    assert call(E=300) == 2           # tcgen05 table holds 256 experts
    assert call(dy=4100) == 7
    assert call(ld_dy=200) == 1       # ld_dy < N
    assert call(ld_dx=100) == 7       # not a multiple of 8
    assert call(dx=None) == 1
    a = e4b.DgradArgs(0, 4, 256, 128, 0, p, p, p, 256, p, p, 128)
    assert L.e4b_grouped_dgrad(ctypes.byref(a), 0, None) == 0  # no rows: nothing to do
    a = e4b.DgradArgs(0, 4, 256, 128, 64, p, p, p, 256, p, p, 128)
    assert L.e4b_grouped_dgrad(ctypes.byref(a), e4b.FLAG_FORCE_GEMV, None) == 2


def test_int4_argument_checks():
    L = e4b.lib()
    p = 4096

    def gemv(**kw):
        a = e4b.Int4GemvArgs(e4b.E4B_EPI_STORE, 8, 256, 512, 2, p, p, p, p, p, 0, p, 256, None)
        for k, v in kw.items():
            setattr(a, k, v)
        return L.e4b_gemv_int4_b32(ctypes.byref(a), 0, None)

    assert gemv(epilogue=5) == 1
    assert gemv(K=48) == 2                       # blocks of 32 along K
    assert gemv(n_slots=0) == 1
    assert gemv(n_slots=65) == 2                 # at most 64 routed slots
    assert gemv(epilogue=e4b.E4B_EPI_SWIGLU, N=255, ld_y=200) == 1  # SwiGLU needs N even
    assert gemv(epilogue=e4b.E4B_EPI_COMBINE, gates=None) == 1
    assert gemv(codes=p + 8) == 7
    assert gemv(x=p + 2) == 7
    assert gemv(ld_x=12) == 7                    # row stride not a multiple of 8
    assert gemv(ld_x=256) == 1                   # row stride below K
    assert gemv(ld_y=100) == 1                   # STORE rows need N
    assert gemv(x=None) == 1
    assert gemv(K=256 * 1024) == 2               # activation row beyond shared memory
    assert gemv(ld_x=64 * 1024, K=64 * 1024, n_slots=4) == 2
    a = e4b.Int4GemvArgs(0, 8, 256, 512, 2, p, p, p, p, p, 0, p, 256, None)
    assert L.e4b_gemv_int4_b32(ctypes.byref(a), 1, None) == 1  # only E4B_FLAG_TEST_TIMEOUT and E4B_FLAG_IDS_READY
    q = L.e4b_quantize_int4_b32
    assert q(p, 2, 4, 48, p, p, None) == 2
    assert q(p, -1, 4, 64, p, p, None) == 1
    assert q(None, 2, 4, 64, p, p, None) == 1
    assert q(p + 4, 2, 4, 64, p, p, None) == 7
    assert q(None, 0, 4, 64, None, None, None) == 0   # nothing to pack
    g = L.e4b_gptq_pack_int4_b32
    assert g(p, p, 2, 4, 48, p, p, None) == 2
    assert g(p + 2, p, 2, 4, 64, p, p, None) == 7
    assert g(None, p, 2, 4, 64, p, p, None) == 1
    assert g(None, None, 0, 4, 64, None, None, None) == 0


def test_int4_layer_argument_checks():
    # e4b_moe_forward with the int4-b32 format: the batch-1 decode path
    L = e4b.lib()
    p = 4096
    n = ctypes.c_size_t(0)
    w = e4b.MoeWeights(e4b.E4B_FMT_INT4B32, 8, 256, 512, p, p, p, p)
    assert L.e4b_moe_workspace_size(ctypes.byref(w), 3, 2, ctypes.byref(n)) == 0
    assert n.value >= 256 + 2 * 512 * 2          # status words and h [top_k, I]
    fwd = L.e4b_moe_forward
    q = ctypes.c_void_p(p)
    big = 1 << 20
    assert fwd(ctypes.byref(w), None, 0, 2, None, None, None, None, 0, 0, None) == 0  # T == 0
    assert fwd(ctypes.byref(w), q, 1, 2, q, q, None, q, big, 0, None) == 1            # null y
    assert fwd(ctypes.byref(w), q, 1, 2, q, q, q, q, 16, 0, None) == 3                # workspace too small
    assert fwd(ctypes.byref(w), q, 1, 2, q, q, q, q, big, e4b.FLAG_FORCE_GEMV, None) == 2
    bad = e4b.MoeWeights(e4b.E4B_FMT_INT4B32, 8, 256, 496, p, p, p, p)              # I % 32
    assert fwd(ctypes.byref(bad), q, 1, 2, q, q, q, q, big, 0, None) == 2
    var = e4b.MoeWeights(e4b.E4B_FMT_INT4B32, 8, 256, 512, p, p, p, p, 1)            # interleaved
    assert fwd(ctypes.byref(var), q, 1, 2, q, q, q, q, big, 0, None) == 2
    assert fwd(ctypes.byref(w), ctypes.c_void_p(p + 2), 1, 2, q, q, q, q, big, 0, None) == 7


def test_ep_argument_checks():
    L = e4b.lib()
    p = 4096
    assert L.e4b_ep_dest(p, 10, 8, 3, p, None) == 1            # 8 experts do not split over ranks of 3
    assert L.e4b_ep_dest(None, 0, 8, 4, None, None) == 0       # nothing to do
    assert L.e4b_ep_dest(None, 4, 8, 4, p, None) == 1
    pack = L.e4b_ep_pack
    assert pack(p, 100, p, p, 2, p, p, 2, 8, 4, p, p, p, None) == 2        # H % 8
    assert pack(p + 8, 128, p, p, 2, p, p, 2, 8, 4, p, p, p, None) == 7    # x not 16-byte aligned
    assert pack(p, 128, p, p, 2, p, p, 2, 0, 4, None, None, None, None) == 0
    assert pack(p, 128, None, p, 2, p, p, 2, 8, 4, p, p, p, None) == 1
    comb = L.e4b_ep_combine
    assert comb(p, 128, p, 4, 2, p + 4, None) == 7
    assert comb(p, 100, p, 4, 2, p, None) == 2                 # H % 8
    assert comb(None, 128, None, 0, 2, None, None) == 0


def test_expert_parallel_layer_rejects_a_bad_split():
    import torch.distributed as dist
    from bit_grouped_moe_e4b_b200.ep import ExpertParallelLayer

    class _L:
        E = 3

    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        with pytest.raises(ValueError):
            ExpertParallelLayer(_L(), 8)   # 8 experts on one rank, but the local layer holds 3
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (64, 2, 8), (8191, 2, 128), (8192, 2, 128), (4097, 4, 32),
                                   (8192, 8, 128), (65536, 1, 1024)])
def test_route_workspace_size_holds_the_many_cta_scratch(T, k, E):
    # the status words (256 bytes); from 16384 routed slots also one int32
    # histogram per 2048-slot chunk and expert, plus the chunk's bad-id count
    n = e4b.e4b_route_workspace_size(T, k, E)
    R = T * k
    chunks = -(-R // 2048)
    assert n == 256 + (chunks * (E + 1) * 4 if R >= 16384 else 0)
