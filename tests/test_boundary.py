"""The C-ABI library on the host: it loads, exports every entry point the
header declares, and turns every invalid argument into its status code before
launching anything (CPU only; no compute call is made without a GPU)."""
import ctypes as C
import os
import re

import pytest
import torch

import group_wise_affine_dequant_b200 as nvq
from group_wise_affine_dequant_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvq.h")


def declared_entry_points():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nv_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert declared_entry_points() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = nvq.lib()
    for name in declared_entry_points():
        assert hasattr(L, name), name


def test_status_strings():
    for s in range(5):
        txt = nvq.nv_status_string(s)
        assert txt.startswith(("NV_OK", "NV_ERR")), txt
    assert "unknown" in nvq.nv_status_string(99)


def _qmm(**kw):
    a = dict(x=16, dt=1, M=1, K=64, N=16, codes=16, scales=16, biases=16, gs=64, bits=4,
             transpose=1, row_exact=0, y=16, stream=None)
    a.update(kw)
    return nvq.lib().nv_qmm(a["x"], a["dt"], a["M"], a["K"], a["N"], a["codes"], a["scales"],
                            a["biases"], a["gs"], a["bits"], a["transpose"], a["row_exact"], a["y"],
                            a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(bits=3), B.NV_ERR_UNSUPPORTED),
    (dict(bits=5), B.NV_ERR_UNSUPPORTED),
    (dict(bits=6), B.NV_ERR_UNSUPPORTED),
    (dict(bits=1), B.NV_ERR_UNSUPPORTED),
    (dict(bits=7), B.NV_ERR_INVALID_ARG),
    (dict(gs=16), B.NV_ERR_INVALID_ARG),
    (dict(gs=96), B.NV_ERR_INVALID_ARG),
    (dict(dt=7), B.NV_ERR_UNSUPPORTED),
    (dict(M=-1), B.NV_ERR_INVALID_ARG),
    (dict(K=0), B.NV_ERR_INVALID_ARG),
    (dict(K=96), B.NV_ERR_INVALID_ARG),            # K not a multiple of the group size
    (dict(transpose=0, N=48), B.NV_ERR_INVALID_ARG),  # transpose=0 groups along N
    (dict(row_exact=1, M=9), B.NV_ERR_INVALID_ARG),
    (dict(x=0), B.NV_ERR_INVALID_ARG),
    (dict(y=0), B.NV_ERR_INVALID_ARG),
    (dict(codes=8), B.NV_ERR_INVALID_ARG),         # misaligned
    (dict(scales=18), B.NV_ERR_INVALID_ARG),
    (dict(M=0), B.NV_OK),                          # empty: nothing to launch
    (dict(N=0), B.NV_OK),
])
def test_qmm_argument_errors(kw, status):
    assert _qmm(**kw) == status


def test_quantize_argument_errors():
    q = nvq.lib().nv_quantize_affine
    assert q(16, 1, 4, 64, 64, 3, 16, 16, 16, None) == B.NV_ERR_UNSUPPORTED
    assert q(16, 1, 4, 96, 64, 4, 16, 16, 16, None) == B.NV_ERR_INVALID_ARG
    assert q(16, 1, -1, 64, 64, 4, 16, 16, 16, None) == B.NV_ERR_INVALID_ARG
    assert q(16, 1, 4, 64, 64, 4, 0, 16, 16, None) == B.NV_ERR_INVALID_ARG
    assert q(24, 1, 4, 64, 64, 4, 16, 16, 16, None) == B.NV_ERR_INVALID_ARG
    assert q(16, 1, 0, 64, 64, 4, 16, 16, 16, None) == B.NV_OK
    assert q(16, 1, 0, 64, 64, 1, 16, 16, 16, None) == B.NV_OK  # 1-bit codes: quantizer only
    assert q(16, 1, 4, 64, 64, 7, 16, 16, 16, None) == B.NV_ERR_INVALID_ARG


def test_dequantize_argument_errors():
    d = nvq.lib().nv_dequantize_affine
    # codes, scales, biases, dt, rows, cols, group_size, bits, w, stream
    assert d(16, 16, 16, 1, 4, 64, 64, 3, 16, None) == B.NV_ERR_UNSUPPORTED
    assert d(16, 16, 16, 1, 4, 64, 64, 7, 16, None) == B.NV_ERR_INVALID_ARG
    assert d(16, 16, 16, 7, 4, 64, 64, 4, 16, None) == B.NV_ERR_UNSUPPORTED
    assert d(16, 16, 16, 1, 4, 96, 64, 4, 16, None) == B.NV_ERR_INVALID_ARG   # cols % group
    assert d(16, 16, 16, 1, 4, 64, 48, 4, 16, None) == B.NV_ERR_INVALID_ARG   # group size
    assert d(16, 16, 16, 1, -1, 64, 64, 4, 16, None) == B.NV_ERR_INVALID_ARG
    assert d(0, 16, 16, 1, 4, 64, 64, 4, 16, None) == B.NV_ERR_INVALID_ARG
    assert d(16, 16, 16, 1, 4, 64, 64, 4, 0, None) == B.NV_ERR_INVALID_ARG
    assert d(24, 16, 16, 1, 4, 64, 64, 4, 16, None) == B.NV_ERR_INVALID_ARG  # misaligned
    assert d(16, 16, 16, 1, 0, 64, 64, 1, 16, None) == B.NV_OK                # empty


def test_gather_argument_errors():
    L = nvq.lib()
    R, E = 2048, 64
    need = L.nv_gather_qmm_workspace_size(R, E)
    assert need >= 4 * R

    def call(ws=16, ws_bytes=need, **kw):
        a = dict(x=16, dt=1, x_rows=512, K=2048, lhs=16, rhs=16, R=R, E=E, N=1536, codes=16,
                 scales=16, biases=16, gs=64, bits=4, transpose=1, sorted=0, row_exact=0, y=16)
        a.update(kw)
        return L.nv_gather_qmm(a["x"], a["dt"], a["x_rows"], a["K"], a["lhs"], a["rhs"], a["R"],
                               a["E"], a["N"], a["codes"], a["scales"], a["biases"], a["gs"],
                               a["bits"], a["transpose"], a["sorted"], a["row_exact"], ws,
                               ws_bytes, a["y"], None)

    assert call(ws_bytes=need - 1) == B.NV_ERR_WORKSPACE
    assert call(ws=0) == B.NV_ERR_WORKSPACE
    assert call(ws=8) == B.NV_ERR_WORKSPACE
    assert call(bits=5) == B.NV_ERR_UNSUPPORTED
    assert call(E=0) == B.NV_ERR_INVALID_ARG
    assert call(E=5000, ws_bytes=L.nv_gather_qmm_workspace_size(R, 5000)) == B.NV_ERR_UNSUPPORTED
    assert call(K=100) == B.NV_ERR_INVALID_ARG
    assert call(rhs=0) == B.NV_ERR_INVALID_ARG
    assert call(lhs=4) == B.NV_ERR_INVALID_ARG
    assert call(R=0, ws_bytes=L.nv_gather_qmm_workspace_size(0, E)) == B.NV_OK


def test_gather_mm_argument_errors():
    L = nvq.lib()
    R, E = 2048, 64
    need = L.nv_gather_qmm_workspace_size(R, E)

    def call(ws=16, ws_bytes=need, **kw):
        a = dict(x=16, dt=1, x_rows=512, K=2048, lhs=16, rhs=16, R=R, E=E, N=1536, w=16,
                 sorted=0, y=16)
        a.update(kw)
        return L.nv_gather_mm(a["x"], a["dt"], a["x_rows"], a["K"], a["lhs"], a["rhs"], a["R"],
                              a["E"], a["N"], a["w"], a["sorted"], ws, ws_bytes, a["y"], None)

    assert call(ws_bytes=need - 1) == B.NV_ERR_WORKSPACE
    assert call(ws=0) == B.NV_ERR_WORKSPACE
    assert call(ws=8) == B.NV_ERR_WORKSPACE
    assert call(dt=0) == B.NV_ERR_UNSUPPORTED        # fp32 experts: not implemented
    assert call(dt=7) == B.NV_ERR_UNSUPPORTED
    assert call(K=100) == B.NV_ERR_UNSUPPORTED       # K not a multiple of 64
    assert call(E=0) == B.NV_ERR_INVALID_ARG
    assert call(R=-1) == B.NV_ERR_INVALID_ARG
    assert call(E=5000, ws_bytes=L.nv_gather_qmm_workspace_size(R, 5000)) == B.NV_ERR_UNSUPPORTED
    assert call(rhs=0) == B.NV_ERR_INVALID_ARG
    assert call(w=0) == B.NV_ERR_INVALID_ARG
    assert call(w=24) == B.NV_ERR_INVALID_ARG        # misaligned
    assert call(lhs=4) == B.NV_ERR_INVALID_ARG
    assert call(R=0, ws_bytes=L.nv_gather_qmm_workspace_size(0, E)) == B.NV_OK
    assert call(x_rows=1 << 24) == B.NV_ERR_UNSUPPORTED  # x_rows * K = 2^35 elements


def test_flags_argument_errors():
    L = nvq.lib()
    assert L.nv_pipeline_error(0) == B.NV_ERR_INVALID_ARG
    assert L.nv_pipeline_selftest(0, None) == B.NV_ERR_INVALID_ARG       # no limit
    assert L.nv_pipeline_selftest(2000001, None) == B.NV_ERR_INVALID_ARG  # above 2 s
    flags = C.c_uint32(0)
    assert L.nv_gather_qmm_flags(0, C.addressof(flags), None) == B.NV_ERR_INVALID_ARG
    assert L.nv_gather_qmm_flags(16, 0, None) == B.NV_ERR_INVALID_ARG


def test_product_path_fails_loudly_without_library(tmp_path, monkeypatch):
    """The binding has no fallback: a missing library that cannot be built raises."""
    monkeypatch.setattr(B, "_LIB", None)
    monkeypatch.setattr(B._build, "LIB", str(tmp_path / "missing.so"))
    monkeypatch.setattr(B._build, "build", lambda *a, **k: None)
    with pytest.raises(RuntimeError, match="libnvq.so missing"):
        B.lib()


def test_split_k_routing_is_a_pure_function_of_the_shape():
    """Split-K only where the output tiles would leave most SMs idle and K is
    long; the matrix-vector sizes, fp32 and the transposed layout never split."""
    S = nvq.nv_qmm_splits
    assert S(64, 14336, 1024) > 1            # small N, long K
    assert S(20, 2432, 200) > 1
    assert S(2048, 4096, 14336) == 1         # prefill: tiles fill the GPU
    assert S(8, 14336, 1024) == 1            # matrix-vector rows
    assert S(64, 256, 1024) == 1             # K too short to split
    assert S(64, 14336, 1024, transpose=False) > 1    # weights [K, N]: the same split
    assert S(64, 14336, 1024, dtype=torch.float32) == 1
    assert S(64, 14336, 1024) == S(64, 14336, 1024)
    assert 2 <= S(64, 14336, 1024) <= 8


def test_batched_argument_errors():
    L = nvq.lib()

    def call(**kw):
        a = dict(x=16, dt=1, B=2, L=3, K=128, N=64, c=16, s=16, b=16, gs=64, bits=4, t=1, y=16)
        a.update(kw)
        return L.nv_qmm_batched(a["x"], a["dt"], a["B"], a["L"], a["K"], a["N"], a["c"], a["s"],
                                a["b"], a["gs"], a["bits"], a["t"], a["y"], None)

    assert call(B=-1) == B.NV_ERR_INVALID_ARG
    assert call(L=-1) == B.NV_ERR_INVALID_ARG
    assert call(K=100) == B.NV_ERR_INVALID_ARG       # K not a multiple of the group
    assert call(bits=3) == B.NV_ERR_UNSUPPORTED
    assert call(dt=5) == B.NV_ERR_UNSUPPORTED
    assert call(x=0) == B.NV_ERR_INVALID_ARG
    assert call(y=8) == B.NV_ERR_INVALID_ARG         # misaligned
    assert call(B=1 << 30, L=1 << 20) == B.NV_ERR_INVALID_ARG
    assert call(B=0) == B.NV_OK
    assert call(N=0) == B.NV_OK


def test_moe_swiglu_argument_errors():
    L = nvq.lib()
    T, topk, E, I, K = 8, 2, 4, 512, 512
    need = L.nv_moe_swiglu_workspace_size(T, topk, E, I, K)
    assert need > 0 and L.nv_moe_swiglu_workspace_size(T, 0, E, I, K) == 0

    def call(ws=16, ws_bytes=need, **kw):
        a = dict(x=16, dt=1, T=T, K=K, ids=16, rw=16, topk=topk, E=E, I=I, gs=64, bits=4, y=16)
        a.update(kw)
        p = 16
        return L.nv_moe_swiglu(a["x"], a["dt"], a["T"], a["K"], a["ids"], a["rw"], a["topk"],
                               a["E"], a["I"], p, p, p, p, p, p, p, p, p, a["gs"], a["bits"],
                               ws, ws_bytes, a["y"], None)

    assert call(ws_bytes=need - 1) == B.NV_ERR_WORKSPACE
    assert call(ws=0) == B.NV_ERR_WORKSPACE
    assert call(dt=0) == B.NV_ERR_UNSUPPORTED        # fp32 activations: not implemented
    assert call(bits=3) == B.NV_ERR_UNSUPPORTED
    assert call(bits=7) == B.NV_ERR_INVALID_ARG
    assert call(K=320) == B.NV_ERR_UNSUPPORTED       # K not a multiple of 128
    assert call(I=96) == B.NV_ERR_INVALID_ARG        # I not a multiple of the group size
    assert call(I=256) == B.NV_ERR_UNSUPPORTED       # I / group_size not a multiple of 8
    assert call(topk=0) == B.NV_ERR_INVALID_ARG
    assert call(E=5000) == B.NV_ERR_UNSUPPORTED
    assert call(x=0) == B.NV_ERR_INVALID_ARG
    assert call(rw=8) == B.NV_ERR_INVALID_ARG        # misaligned
    assert call(T=0) == B.NV_OK
