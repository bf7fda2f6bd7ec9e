"""Python binding of libnvq.so (include/nvq.h): argument marshalling only.

Every function here has the name of the C entry point it calls. It checks
nothing the library does not check itself beyond what torch needs (device,
contiguity, dtype of the output it allocates); every step of the computation
runs in the CUDA kernels behind the C ABI. There is no CPU fallback: if the
library is missing or a call fails, an exception says so.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import torch

from . import build as _build

NV_OK, NV_ERR_INVALID_ARG, NV_ERR_UNSUPPORTED, NV_ERR_WORKSPACE, NV_ERR_CUDA = range(5)
NV_F32, NV_BF16 = 0, 1
NV_ROW_INDEPENDENT_ROWS = 8
NV_FLAG_EXPERT_OUT_OF_RANGE = 0x1
NV_FLAG_NOT_SORTED = 0x2
NV_FLAG_TOKEN_OUT_OF_RANGE = 0x4

# Every entry point declared in include/nvq.h.
EXPORTS = ("nv_status_string", "nv_quantize_affine", "nv_dequantize_affine", "nv_qmm",
           "nv_qmm_batched", "nv_qmm_splits", "nv_moe_swiglu", "nv_moe_swiglu_workspace_size",
           "nv_gather_qmm_workspace_size", "nv_gather_mm",
           "nv_gather_qmm", "nv_gather_qmm_flags", "nv_pipeline_error", "nv_pipeline_selftest",
           "nv_last_cuda_error",
           "nv_gather_qmm_noalloc", "nv_quantize_fp", "nv_dequantize_fp", "nv_qmm_fp")
NV_FP_MODES = {"mxfp4": 1, "mxfp8": 2, "nvfp4": 3}
_FP_GROUP = {"mxfp4": 32, "mxfp8": 32, "nvfp4": 16}
_FP_BITS = {"mxfp4": 4, "mxfp8": 8, "nvfp4": 4}

_DT = {torch.float32: NV_F32, torch.bfloat16: NV_BF16}
_LOCK = threading.Lock()
_LIB = None

_p, _i64, _i, _sz = C.c_void_p, C.c_int64, C.c_int, C.c_size_t


class NvqError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn}: {text}")
        self.status = status


def lib_path() -> str:
    return _build.LIB


def lib():
    """The loaded C library (ctypes), built first if it is missing."""
    global _LIB
    with _LOCK:
        if _LIB is None:
            path = _build.LIB
            if not os.path.exists(path):
                _build.build()
            if not os.path.exists(path):
                raise RuntimeError(f"libnvq.so missing at {path}; the CUDA library is required")
            L = C.CDLL(path)
            L.nv_status_string.argtypes = [_i]
            L.nv_status_string.restype = C.c_char_p
            L.nv_quantize_affine.argtypes = [_p, _i, _i64, _i64, _i, _i, _p, _p, _p, _p]
            L.nv_quantize_affine.restype = _i
            L.nv_dequantize_affine.argtypes = [_p, _p, _p, _i, _i64, _i64, _i, _i, _p, _p]
            L.nv_dequantize_affine.restype = _i
            L.nv_qmm.argtypes = [_p, _i, _i64, _i64, _i64, _p, _p, _p, _i, _i, _i, _i, _p, _p]
            L.nv_qmm.restype = _i
            L.nv_qmm_batched.argtypes = [_p, _i, _i64, _i64, _i64, _i64, _p, _p, _p, _i, _i, _i,
                                         _p, _p]
            L.nv_qmm_batched.restype = _i
            L.nv_qmm_splits.argtypes = [_i64, _i64, _i64, _i, _i, _i, _i]
            L.nv_qmm_splits.restype = _i
            L.nv_gather_qmm_workspace_size.argtypes = [_i64, _i64]
            L.nv_gather_qmm_workspace_size.restype = _sz
            L.nv_gather_qmm.argtypes = [_p, _i, _i64, _i64, _p, _p, _i64, _i64, _i64, _p, _p, _p,
                                        _i, _i, _i, _i, _i, _p, _sz, _p, _p]
            L.nv_gather_qmm.restype = _i
            L.nv_gather_mm.argtypes = [_p, _i, _i64, _i64, _p, _p, _i64, _i64, _i64, _p, _i, _p,
                                       _sz, _p, _p]
            L.nv_gather_mm.restype = _i
            L.nv_moe_swiglu_workspace_size.argtypes = [_i64, _i64, _i64, _i64, _i64]
            L.nv_moe_swiglu_workspace_size.restype = _sz
            L.nv_moe_swiglu.argtypes = [_p, _i, _i64, _i64, _p, _p, _i, _i64, _i64, _p, _p, _p,
                                        _p, _p, _p, _p, _p, _p, _i, _i, _p, _sz, _p, _p]
            L.nv_moe_swiglu.restype = _i
            L.nv_gather_qmm_flags.argtypes = [_p, _p, _p]
            L.nv_gather_qmm_flags.restype = _i
            L.nv_gather_qmm_noalloc.argtypes = [_p, _i, _i64, _i64, _p, _p, _i64, _i64, _i64, _p,
                                                 _p, _p, _i, _i, _i, _i, _i, _p, _p]
            L.nv_gather_qmm_noalloc.restype = _i
            L.nv_last_cuda_error.argtypes = []
            L.nv_last_cuda_error.restype = C.c_char_p
            L.nv_pipeline_error.argtypes = [_p]
            L.nv_pipeline_error.restype = _i
            L.nv_pipeline_selftest.argtypes = [C.c_uint32, _p]
            L.nv_pipeline_selftest.restype = _i
            L.nv_quantize_fp.argtypes = [_p, _i, _i64, _i64, _i, _p, _p, _p]
            L.nv_quantize_fp.restype = _i
            L.nv_dequantize_fp.argtypes = [_p, _p, _i64, _i64, _i, _p, _p]
            L.nv_dequantize_fp.restype = _i
            L.nv_qmm_fp.argtypes = [_p, _i, _i64, _i64, _i64, _p, _p, _i, _p, _p]
            L.nv_qmm_fp.restype = _i
            _LIB = L
        return _LIB


def nv_status_string(status: int) -> str:
    return lib().nv_status_string(status).decode()


def _check(fn: str, status: int):
    if status != NV_OK:
        text = nv_status_string(status)
        if status == NV_ERR_CUDA:
            text += f" ({lib().nv_last_cuda_error().decode()})"
        raise NvqError(fn, status, text)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _ptr(t):
    return None if t is None else t.data_ptr()


def nv_quantize_affine(w: torch.Tensor, group_size: int = 64, bits: int = 4, stream=None):
    """Quantize w [..., cols] along its last axis. Returns (codes int32-as-uint32,
    scales, biases) with scales/biases in w's dtype."""
    _dev(w, "w")
    cols = w.shape[-1]
    rows = w.numel() // cols if cols else 0
    codes = torch.empty(*w.shape[:-1], cols * bits // 32, dtype=torch.int32, device=w.device)
    scales = torch.empty(*w.shape[:-1], max(cols // group_size, 0), dtype=w.dtype, device=w.device)
    biases = torch.empty_like(scales)
    st = lib().nv_quantize_affine(w.data_ptr(), _DT.get(w.dtype, -1), rows, cols, group_size, bits,
                                  codes.data_ptr(), scales.data_ptr(), biases.data_ptr(),
                                  _stream(stream))
    _check("nv_quantize_affine", st)
    return codes, scales, biases


def nv_dequantize_affine(codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
                         group_size: int = 64, bits: int = 4, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """w = scale * code + bias [..., rows, cols] in the scales' dtype, from the
    layout nv_quantize_affine writes (codes [..., rows, cols * bits / 32])."""
    for t, n in ((codes, "codes"), (scales, "scales"), (biases, "biases")):
        _dev(t, n)
    if scales.shape != biases.shape or scales.dtype != biases.dtype or codes.dim() < 1:
        raise ValueError("scales and biases must match, codes must have a last axis")
    cols = codes.shape[-1] * 32 // bits
    rows = codes.numel() // codes.shape[-1] if codes.shape[-1] else 0
    if tuple(scales.shape) != (*codes.shape[:-1], cols // group_size):
        raise ValueError(f"scales {tuple(scales.shape)} do not match codes {tuple(codes.shape)} "
                         f"at group_size {group_size}, bits {bits}")
    w = out if out is not None else torch.empty(*codes.shape[:-1], cols, dtype=scales.dtype,
                                                device=codes.device)
    if w.numel() != rows * cols or w.dtype != scales.dtype:
        raise ValueError("out has the wrong size or dtype")
    _dev(w, "out")
    st = lib().nv_dequantize_affine(codes.data_ptr(), scales.data_ptr(), biases.data_ptr(),
                                    _DT.get(scales.dtype, -1), rows, cols, group_size, bits,
                                    w.data_ptr(), _stream(stream))
    _check("nv_dequantize_affine", st)
    return w


def nv_qmm(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
           group_size: int = 64, bits: int = 4, transpose: bool = True, row_exact: bool = False,
           out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x . w^T (transpose, weights [N, K]) or x . w (weights [K, N]); y in x's dtype."""
    for t, n in ((x, "x"), (codes, "codes"), (scales, "scales"), (biases, "biases")):
        _dev(t, n)
    K = x.shape[-1]
    M = x.numel() // K if K else 0
    if codes.dim() != 2 or scales.shape != biases.shape or scales.dim() != 2:
        raise ValueError("codes, scales and biases must be 2-D and scales/biases alike")
    N = codes.shape[-2] if transpose else codes.shape[-1] * 32 // bits
    rows, cols = (N, K) if transpose else (K, N)
    if tuple(codes.shape) != (rows, cols * bits // 32) or \
            tuple(scales.shape) != (rows, cols // group_size):
        raise ValueError(f"weights do not match x: codes {tuple(codes.shape)}, scales "
                         f"{tuple(scales.shape)} for K={K}, N={N}, transpose={transpose}")
    y = out if out is not None else torch.empty(*x.shape[:-1], N, dtype=x.dtype, device=x.device)
    if y.numel() != M * N or y.dtype != x.dtype:
        raise ValueError("out has the wrong size or dtype")
    _dev(y, "out")
    if scales.dtype != x.dtype:
        raise NvqError("nv_qmm", NV_ERR_UNSUPPORTED, nv_status_string(NV_ERR_UNSUPPORTED))
    st = lib().nv_qmm(x.data_ptr(), _DT.get(x.dtype, -1), M, K, N, codes.data_ptr(),
                      scales.data_ptr(), biases.data_ptr(), group_size, bits, int(transpose),
                      int(row_exact), y.data_ptr(), _stream(stream))
    _check("nv_qmm", st)
    return y


def nv_qmm_batched(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                   biases: torch.Tensor, group_size: int = 64, bits: int = 4,
                   transpose: bool = True, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """x [B, L, K]: B items of L rows with the same weights; y [B, L, N]. Item b
    is bitwise equal to nv_qmm(x[b]) (routing and split-K per item)."""
    for t, n in ((x, "x"), (codes, "codes"), (scales, "scales"), (biases, "biases")):
        _dev(t, n)
    if x.dim() != 3:
        raise ValueError("x must be [B, L, K]")
    B, L, K = x.shape
    if codes.dim() != 2 or scales.shape != biases.shape or scales.dim() != 2:
        raise ValueError("codes, scales and biases must be 2-D and scales/biases alike")
    N = codes.shape[-2] if transpose else codes.shape[-1] * 32 // bits
    rows, cols = (N, K) if transpose else (K, N)
    if tuple(codes.shape) != (rows, cols * bits // 32) or \
            tuple(scales.shape) != (rows, cols // group_size):
        raise ValueError(f"weights do not match x: codes {tuple(codes.shape)}, scales "
                         f"{tuple(scales.shape)} for K={K}, N={N}, transpose={transpose}")
    y = out if out is not None else torch.empty(B, L, N, dtype=x.dtype, device=x.device)
    if y.numel() != B * L * N or y.dtype != x.dtype:
        raise ValueError("out has the wrong size or dtype")
    _dev(y, "out")
    if scales.dtype != x.dtype:
        raise NvqError("nv_qmm_batched", NV_ERR_UNSUPPORTED, nv_status_string(NV_ERR_UNSUPPORTED))
    st = lib().nv_qmm_batched(x.data_ptr(), _DT.get(x.dtype, -1), B, L, K, N, codes.data_ptr(),
                              scales.data_ptr(), biases.data_ptr(), group_size, bits,
                              int(transpose), y.data_ptr(), _stream(stream))
    _check("nv_qmm_batched", st)
    return y


def nv_qmm_splits(M: int, K: int, N: int, bits: int = 4, group_size: int = 64,
                  transpose: bool = True, dtype=torch.bfloat16) -> int:
    """K-partitions nv_qmm uses for an M-row product (1: no split)."""
    return int(lib().nv_qmm_splits(M, K, N, bits, group_size, int(transpose),
                                   _DT.get(dtype, -1)))


def nv_gather_qmm_workspace_size(R: int, E: int) -> int:
    return int(lib().nv_gather_qmm_workspace_size(R, E))


def nv_gather_qmm(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                  biases: torch.Tensor, rhs: torch.Tensor, lhs: torch.Tensor | None = None,
                  group_size: int = 64, bits: int = 4, transpose: bool = True,
                  sorted: bool = False, row_exact: bool = False,
                  workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """Row r of the result is x[lhs[r]] times expert rhs[r] (lhs None: row r).

    x [x_rows, K] (or [x_rows, 1, K]); codes/scales/biases [E, ...] as for nv_qmm;
    rhs, lhs int32 (uint32 values) [R]. Returns y [R, N] in x's dtype."""
    for t, n in ((x, "x"), (codes, "codes"), (scales, "scales"), (biases, "biases"), (rhs, "rhs")):
        _dev(t, n)
    if lhs is not None:
        _dev(lhs, "lhs")
    K = x.shape[-1]
    x_rows = x.numel() // K if K else 0
    E = codes.shape[0]
    if codes.dim() != 3 or scales.dim() != 3 or scales.shape != biases.shape:
        raise ValueError("codes, scales and biases must be [E, rows, ...] alike")
    N = codes.shape[1] if transpose else codes.shape[2] * 32 // bits
    rows, cols = (N, K) if transpose else (K, N)
    if tuple(codes.shape) != (E, rows, cols * bits // 32) or \
            tuple(scales.shape) != (E, rows, cols // group_size):
        raise ValueError(f"expert weights do not match x: codes {tuple(codes.shape)}, scales "
                         f"{tuple(scales.shape)} for K={K}, N={N}, transpose={transpose}")
    R = rhs.numel()
    if lhs is not None and lhs.numel() != R:
        raise ValueError("lhs and rhs differ in length")
    ws_bytes = nv_gather_qmm_workspace_size(R, E)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=x.device)
    y = out if out is not None else torch.empty(R, N, dtype=x.dtype, device=x.device)
    if y.numel() != R * N or y.dtype != x.dtype:
        raise ValueError("out has the wrong size or dtype")
    st = lib().nv_gather_qmm(x.data_ptr(), _DT.get(x.dtype, -1), x_rows, K, _ptr(lhs),
                             rhs.data_ptr(), R, E, N, codes.data_ptr(), scales.data_ptr(),
                             biases.data_ptr(), group_size, bits, int(transpose), int(sorted),
                             int(row_exact), workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), y.data_ptr(),
                             _stream(stream))
    _check("nv_gather_qmm", st)
    return y


def nv_gather_mm(x: torch.Tensor, w: torch.Tensor, rhs: torch.Tensor,
                 lhs: torch.Tensor | None = None, sorted: bool = False,
                 workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """Row r of the result is x[lhs[r]] times full-precision expert w[rhs[r]]
    (transposed: w [E, N, K] bf16, y[r] = x[lhs[r]] . w[rhs[r]]^T)."""
    for t, n in ((x, "x"), (w, "w"), (rhs, "rhs")):
        _dev(t, n)
    if lhs is not None:
        _dev(lhs, "lhs")
    K = x.shape[-1]
    x_rows = x.numel() // K if K else 0
    if w.dim() != 3 or w.shape[2] != K:
        raise ValueError(f"experts {tuple(w.shape)} do not match x (K={K})")
    E, N = w.shape[0], w.shape[1]
    if w.dtype != x.dtype:
        raise NvqError("nv_gather_mm", NV_ERR_UNSUPPORTED, nv_status_string(NV_ERR_UNSUPPORTED))
    R = rhs.numel()
    if lhs is not None and lhs.numel() != R:
        raise ValueError("lhs and rhs differ in length")
    ws_bytes = nv_gather_qmm_workspace_size(R, E)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=x.device)
    y = out if out is not None else torch.empty(R, N, dtype=x.dtype, device=x.device)
    if y.numel() != R * N or y.dtype != x.dtype:
        raise ValueError("out has the wrong size or dtype")
    st = lib().nv_gather_mm(x.data_ptr(), _DT.get(x.dtype, -1), x_rows, K, _ptr(lhs),
                            rhs.data_ptr(), R, E, N, w.data_ptr(), int(sorted),
                            workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                            y.data_ptr(), _stream(stream))
    _check("nv_gather_mm", st)
    return y


def nv_moe_swiglu_workspace_size(T: int, topk: int, E: int, I: int, K: int) -> int:
    return int(lib().nv_moe_swiglu_workspace_size(T, topk, E, I, K))


def nv_moe_swiglu(x: torch.Tensor, gate, up, down, ids: torch.Tensor, rw: torch.Tensor,
                  group_size: int = 64, bits: int = 4, workspace: torch.Tensor | None = None,
                  out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The routed SwiGLU block: y[t] = sum_j rw[t, j] down_e(silu(gate_e x[t]) *
    up_e x[t]). gate, up: (codes, scales, biases) of [E, I, K] weights; down:
    of [E, K, I]; ids int32 [T, topk]; rw fp32 [T, topk]. Returns y [T, K]."""
    (gc, gsc, gb), (uc, usc, ub), (dc, dsc, db) = gate, up, down
    for t, n in ((x, "x"), (gc, "gate codes"), (gsc, "gate scales"), (gb, "gate biases"),
                 (uc, "up codes"), (usc, "up scales"), (ub, "up biases"), (dc, "down codes"),
                 (dsc, "down scales"), (db, "down biases"), (ids, "ids"), (rw, "rw")):
        _dev(t, n)
    T, K = x.shape
    E, I = gc.shape[0], gc.shape[1]
    if tuple(gc.shape) != (E, I, K * bits // 32) or tuple(uc.shape) != tuple(gc.shape) or \
            tuple(dc.shape) != (E, K, I * bits // 32):
        raise ValueError("gate/up must be [E, I, K] and down [E, K, I] quantized weights")
    if ids.dim() != 2 or ids.shape[0] != T or tuple(rw.shape) != tuple(ids.shape) or \
            rw.dtype != torch.float32:
        raise ValueError("ids [T, topk] and fp32 rw [T, topk] expected")
    topk = ids.shape[1]
    need = nv_moe_swiglu_workspace_size(T, topk, E, I, K)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    y = out if out is not None else torch.empty(T, K, dtype=x.dtype, device=x.device)
    if y.numel() != T * K or y.dtype != x.dtype:
        raise ValueError("out has the wrong size or dtype")
    st = lib().nv_moe_swiglu(x.data_ptr(), _DT.get(x.dtype, -1), T, K, ids.data_ptr(),
                             rw.data_ptr(), topk, E, I, gc.data_ptr(), gsc.data_ptr(),
                             gb.data_ptr(), uc.data_ptr(), usc.data_ptr(), ub.data_ptr(),
                             dc.data_ptr(), dsc.data_ptr(), db.data_ptr(), group_size, bits,
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             y.data_ptr(), _stream(stream))
    _check("nv_moe_swiglu", st)
    return y


def nv_gather_qmm_flags(workspace: torch.Tensor, stream=None) -> int:
    flags = C.c_uint32(0)
    st = lib().nv_gather_qmm_flags(workspace.data_ptr(), C.addressof(flags), _stream(stream))
    _check("nv_gather_qmm_flags", st)
    return int(flags.value)


def nv_pipeline_error() -> int:
    """Read and clear the kernels' pipeline timeout word (0 = no wait gave up)."""
    code = C.c_uint32(0)
    st = lib().nv_pipeline_error(C.addressof(code))
    _check("nv_pipeline_error", st)
    return int(code.value)


def nv_pipeline_selftest(limit_us: int = 1000, stream=None) -> None:
    """Enqueue one wait on a barrier nothing completes; it gives up after
    limit_us and records code 0x5E (read it with nv_pipeline_error)."""
    st = lib().nv_pipeline_selftest(int(limit_us), _stream(stream))
    _check("nv_pipeline_selftest", st)


def _fp_mode(mode: str) -> int:
    if mode not in NV_FP_MODES:
        raise ValueError(f"mode must be one of {sorted(NV_FP_MODES)}")
    return NV_FP_MODES[mode]


def nv_quantize_fp(w: torch.Tensor, mode: str = "mxfp4", stream=None):
    """Codes [..., rows, cols * b / 32] (uint32 as int32) and uint8 scale codes
    [..., rows, cols / group] of w [..., rows, cols] in a floating-point mode
    ('mxfp4', 'mxfp8', 'nvfp4')."""
    m = _fp_mode(mode)
    _dev(w, "w")
    cols = w.shape[-1]
    rows = w.numel() // cols if cols else 0
    codes = torch.empty(*w.shape[:-1], cols * _FP_BITS[mode] // 32, dtype=torch.int32, device=w.device)
    scales = torch.empty(*w.shape[:-1], cols // _FP_GROUP[mode], dtype=torch.uint8, device=w.device)
    st = lib().nv_quantize_fp(w.data_ptr(), _DT.get(w.dtype, -1), rows, cols, m, codes.data_ptr(),
                              scales.data_ptr(), _stream(stream))
    _check("nv_quantize_fp", st)
    return codes, scales


def nv_dequantize_fp(codes: torch.Tensor, scales: torch.Tensor, mode: str = "mxfp4",
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bf16 [..., rows, cols]: element value times scale value."""
    m = _fp_mode(mode)
    _dev(codes, "codes")
    _dev(scales, "scales")
    cols = codes.shape[-1] * 32 // _FP_BITS[mode]
    rows = codes.numel() // codes.shape[-1] if codes.shape[-1] else 0
    if scales.dtype != torch.uint8 or tuple(scales.shape) != (*codes.shape[:-1], cols // _FP_GROUP[mode]):
        raise ValueError("scales must be uint8 [..., rows, cols / group]")
    w = out if out is not None else torch.empty(*codes.shape[:-1], cols, dtype=torch.bfloat16,
                                                device=codes.device)
    if w.numel() != rows * cols or w.dtype != torch.bfloat16:
        raise ValueError("out has the wrong size or dtype")
    _dev(w, "out")
    st = lib().nv_dequantize_fp(codes.data_ptr(), scales.data_ptr(), rows, cols, m, w.data_ptr(),
                                _stream(stream))
    _check("nv_dequantize_fp", st)
    return w


def nv_qmm_fp(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, mode: str = "mxfp4",
              out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x . w^T with floating-point-mode weights [N, K]; bf16 x and y."""
    m = _fp_mode(mode)
    for t, n in ((x, "x"), (codes, "codes"), (scales, "scales")):
        _dev(t, n)
    K = x.shape[-1]
    M = x.numel() // K if K else 0
    if codes.dim() != 2 or scales.dim() != 2 or scales.dtype != torch.uint8:
        raise ValueError("codes and uint8 scales must be 2-D")
    N = codes.shape[0]
    if tuple(codes.shape) != (N, K * _FP_BITS[mode] // 32) or tuple(scales.shape) != (N, K // _FP_GROUP[mode]):
        raise ValueError(f"weights do not match x: codes {tuple(codes.shape)}, scales {tuple(scales.shape)}")
    y = out if out is not None else torch.empty(*x.shape[:-1], N, dtype=x.dtype, device=x.device)
    if y.numel() != M * N or y.dtype != x.dtype:
        raise ValueError("out has the wrong size or dtype")
    _dev(y, "out")
    st = lib().nv_qmm_fp(x.data_ptr(), _DT.get(x.dtype, -1), M, K, N, codes.data_ptr(), scales.data_ptr(), m,
                         y.data_ptr(), _stream(stream))
    _check("nv_qmm_fp", st)
    return y
