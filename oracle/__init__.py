"""Host oracle for group-wise affine quantization and quantized products.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg call it; the CUDA library never does. The arithmetic
lives in ``oracle.cpp`` (plain C++, fp32 quantizer, fp64 products); this module
only marshals CPU torch tensors through ctypes.

Parity status: every function is pinned by tests/test_oracle_pins.py against
closed forms, hand-built integer groups and brute force (no function here is
"parity unpinned").
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import torch

from . import build as _build

_LOCK = threading.Lock()
_LIB = None

F32, BF16 = 0, 1
_DT = {torch.float32: F32, torch.bfloat16: BF16}
_TORCH = {F32: torch.float32, BF16: torch.bfloat16}

_p = C.c_void_p
_i64 = C.c_int64
_i = C.c_int


def load(path: str | None = None):
    """Load liboracle.so, compiling it first if it is missing or older than its source."""
    global _LIB
    with _LOCK:
        if path is not None:
            return _bind(C.CDLL(path))
        if _LIB is None:
            if _build.stale():
                _build.build()
            _LIB = _bind(C.CDLL(_build.LIB))
        return _LIB


def _bind(lib):
    lib.orc_threads.restype = _i
    lib.orc_set_threads.argtypes = [_i]
    lib.orc_cast_bf16.argtypes = [_p, _p, _i64]
    lib.orc_quantize_affine.argtypes = [_p, _i, _i64, _i64, _i, _i, _p, _p, _p]
    lib.orc_quantize_affine.restype = _i
    lib.orc_dequantize.argtypes = [_p, _p, _p, _i, _i64, _i64, _i, _i, _p]
    lib.orc_dequantize.restype = _i
    lib.orc_dequantize_stored.argtypes = [_p, _p, _p, _i, _i64, _i64, _i, _i, _p]
    lib.orc_dequantize_stored.restype = _i
    lib.orc_qmm.argtypes = [_p, _i, _i64, _i64, _i64, _p, _p, _p, _i, _i, _i, _i, _p, _p]
    lib.orc_qmm.restype = _i
    lib.orc_qmm_sampled.argtypes = [_p, _i, _i64, _i64, _i64, _p, _p, _p, _i, _i, _i, _i,
                                    _i64, _p, _p, _p, _p]
    lib.orc_qmm_sampled.restype = _i
    lib.orc_gather_qmm.argtypes = [_p, _i, _i64, _i64, _p, _p, _i64, _i64, _i64, _p, _p, _p,
                                   _i, _i, _i, _i, _p, _p]
    lib.orc_gather_qmm.restype = _i
    lib.orc_gather_qmm_sampled.argtypes = [_p, _i, _i64, _i64, _p, _p, _i64, _i64, _i64, _p,
                                           _p, _p, _i, _i, _i, _i, _i64, _p, _p, _p, _p]
    lib.orc_gather_qmm_sampled.restype = _i
    lib.orc_gather_mm.argtypes = [_p, _i, _i64, _i64, _p, _p, _i64, _i64, _i64, _p, _i, _p, _p]
    lib.orc_gather_mm.restype = _i
    lib.orc_moe_swiglu.argtypes = [_p, _i, _i64, _i64, _p, _p, _i, _i64, _i64,
                                   _p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _p, _p]
    lib.orc_moe_swiglu.restype = _i
    lib.orc_quantize_fp.argtypes = [_p, _i, _i64, _i64, _i, _p, _p]
    lib.orc_quantize_fp.restype = _i
    lib.orc_dequantize_fp.argtypes = [_p, _p, _i64, _i64, _i, _p]
    lib.orc_dequantize_fp.restype = _i
    lib.orc_qmm_fp.argtypes = [_p, _i, _i64, _i64, _i64, _p, _p, _i, _p, _p]
    lib.orc_qmm_fp.restype = _i
    lib.orc_fp_value.argtypes = [_i, C.c_uint32]
    lib.orc_fp_value.restype = C.c_double
    lib.orc_fp_nearest.argtypes = [_i, C.c_double]
    lib.orc_fp_nearest.restype = C.c_uint32
    return lib


def _cpu(t: torch.Tensor) -> torch.Tensor:
    assert t.device.type == "cpu", "the oracle reads host tensors only"
    return t.contiguous()


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments")


def threads() -> int:
    return load().orc_threads()


def set_threads(n: int):
    load().orc_set_threads(n)


def cast_bf16(x: torch.Tensor, lib=None) -> torch.Tensor:
    """fp32 -> bf16 by the oracle's own round-to-nearest-even on the bits."""
    lib = lib or load()
    x = _cpu(x.to(torch.float32))
    out = torch.empty(x.shape, dtype=torch.int16)
    lib.orc_cast_bf16(x.data_ptr(), out.data_ptr(), x.numel())
    return out.view(torch.bfloat16)


def quantize_affine(w: torch.Tensor, group_size: int, bits: int, lib=None):
    """Affine quantization of w [..., rows, cols] along cols.

    Returns (codes uint32-as-int32 [..., rows, cols*bits/32], scales, biases
    [..., rows, cols/group_size] in w's dtype)."""
    lib = lib or load()
    w = _cpu(w)
    cols = w.shape[-1]
    rows = w.numel() // cols
    codes = torch.zeros(*w.shape[:-1], cols * bits // 32, dtype=torch.int32)
    scales = torch.empty(*w.shape[:-1], cols // group_size, dtype=w.dtype)
    biases = torch.empty_like(scales)
    rc = lib.orc_quantize_affine(w.data_ptr(), _DT[w.dtype], rows, cols, group_size, bits,
                                 codes.data_ptr(), scales.data_ptr(), biases.data_ptr())
    _check(rc, "quantize_affine")
    return codes, scales, biases


def dequantize(codes, scales, biases, group_size: int, bits: int, lib=None) -> torch.Tensor:
    """fp64 w_hat = scale * code + bias, shape [..., rows, cols]."""
    lib = lib or load()
    codes, scales, biases = _cpu(codes), _cpu(scales), _cpu(biases)
    cols = codes.shape[-1] * 32 // bits
    rows = codes.numel() // codes.shape[-1]
    out = torch.empty(*codes.shape[:-1], cols, dtype=torch.float64)
    rc = lib.orc_dequantize(codes.data_ptr(), scales.data_ptr(), biases.data_ptr(),
                            _DT[scales.dtype], rows, cols, group_size, bits, out.data_ptr())
    _check(rc, "dequantize")
    return out


def dequantize_stored(codes, scales, biases, group_size: int, bits: int, lib=None) -> torch.Tensor:
    """The dequantized weights as stored in the scales' dtype ("Docs /
    Quantization", section "Affine": w ~= scale * code + bias; the nuvec crate
    docs, Quantized: scales in the weights' dtype).

    Reading (the pages fix no precision for this step): the exact value
    scale * code + bias rounded once, to nearest with ties to even, to the
    dtype. oracle.cpp computes that single rounding exactly (two-sum, then a
    rounding to odd at fp64 precision, then the dtype's rounding)."""
    lib = lib or load()
    codes, scales, biases = _cpu(codes), _cpu(scales), _cpu(biases)
    cols = codes.shape[-1] * 32 // bits
    rows = codes.numel() // codes.shape[-1]
    dt = scales.dtype
    out = torch.empty(*codes.shape[:-1], cols, dtype=torch.float32 if dt == torch.float32
                      else torch.int16)
    rc = lib.orc_dequantize_stored(codes.data_ptr(), scales.data_ptr(), biases.data_ptr(),
                                   _DT[dt], rows, cols, group_size, bits, out.data_ptr())
    _check(rc, "dequantize_stored")
    return out if dt == torch.float32 else out.view(torch.bfloat16)


def qmm(x, codes, scales, biases, group_size: int, bits: int, transpose: bool = True, lib=None):
    """fp64 (y, a) for x [M, K]; weights [N, K] (transpose) or [K, N].

    a = sum_k |x * w_hat| per output, the scale of the tolerance."""
    lib = lib or load()
    x, codes, scales, biases = _cpu(x), _cpu(codes), _cpu(scales), _cpu(biases)
    M, K = x.shape
    if transpose:
        N = codes.shape[0]
    else:
        N = codes.shape[1] * 32 // bits
    _check_weights(codes, scales, biases, K, N, group_size, bits, transpose)
    y = torch.empty(M, N, dtype=torch.float64)
    a = torch.empty(M, N, dtype=torch.float64)
    rc = lib.orc_qmm(x.data_ptr(), _DT[x.dtype], M, K, N, codes.data_ptr(), scales.data_ptr(),
                     biases.data_ptr(), _DT[scales.dtype], group_size, bits, int(transpose),
                     y.data_ptr(), a.data_ptr())
    _check(rc, "qmm")
    return y, a


def qmm_sampled(x, codes, scales, biases, group_size, bits, transpose, m_idx, n_idx, lib=None):
    """(y, a) at the positions (m_idx[s], n_idx[s]) only."""
    lib = lib or load()
    x, codes, scales, biases = _cpu(x), _cpu(codes), _cpu(scales), _cpu(biases)
    M, K = x.shape
    N = codes.shape[0] if transpose else codes.shape[1] * 32 // bits
    _check_weights(codes, scales, biases, K, N, group_size, bits, transpose)
    m_idx = _cpu(torch.as_tensor(m_idx, dtype=torch.int64))
    n_idx = _cpu(torch.as_tensor(n_idx, dtype=torch.int64))
    S = m_idx.numel()
    y = torch.empty(S, dtype=torch.float64)
    a = torch.empty(S, dtype=torch.float64)
    rc = lib.orc_qmm_sampled(x.data_ptr(), _DT[x.dtype], M, K, N, codes.data_ptr(),
                             scales.data_ptr(), biases.data_ptr(), _DT[scales.dtype], group_size,
                             bits, int(transpose), S, m_idx.data_ptr(), n_idx.data_ptr(),
                             y.data_ptr(), a.data_ptr())
    _check(rc, "qmm_sampled")
    return y, a


def _check_weights(codes, scales, biases, K, N, group_size, bits, transpose):
    rows, cols = (N, K) if transpose else (K, N)
    lead = tuple(codes.shape[:-2])
    if tuple(codes.shape[-2:]) != (rows, cols * bits // 32) or \
            tuple(scales.shape) != lead + (rows, cols // group_size) or scales.shape != biases.shape:
        raise ValueError(f"oracle: weights {tuple(codes.shape)}/{tuple(scales.shape)} do not "
                         f"match K={K}, N={N}, transpose={transpose}")


def _u32(t):
    if t is None:
        return None
    return _cpu(torch.as_tensor(t).to(torch.int64).to(torch.int32))


def gather_qmm(x, codes, scales, biases, lhs, rhs, group_size, bits, transpose=True, lib=None):
    """fp64 (y, a) [R, N]: row r = x[lhs[r]] times expert rhs[r] (lhs None: identity)."""
    lib = lib or load()
    x, codes, scales, biases = _cpu(x), _cpu(codes), _cpu(scales), _cpu(biases)
    x2 = x.reshape(-1, x.shape[-1])
    x_rows, K = x2.shape
    E = codes.shape[0]
    N = codes.shape[1] if transpose else codes.shape[2] * 32 // bits
    _check_weights(codes, scales, biases, K, N, group_size, bits, transpose)
    lhs_t, rhs_t = _u32(lhs), _u32(rhs)
    R = rhs_t.numel()
    y = torch.empty(R, N, dtype=torch.float64)
    a = torch.empty(R, N, dtype=torch.float64)
    rc = lib.orc_gather_qmm(x2.data_ptr(), _DT[x.dtype], x_rows, K,
                            None if lhs_t is None else lhs_t.data_ptr(), rhs_t.data_ptr(), R, E, N,
                            codes.data_ptr(), scales.data_ptr(), biases.data_ptr(),
                            _DT[scales.dtype], group_size, bits, int(transpose), y.data_ptr(),
                            a.data_ptr())
    _check(rc, "gather_qmm")
    return y, a


def gather_mm(x, w, lhs, rhs, lib=None):
    """fp64 (y, a) [R, N]: row r = x[lhs[r]] times full-precision expert
    w[rhs[r]] ([E, N, K], transposed product; lhs None: identity)."""
    lib = lib or load()
    x, w = _cpu(x), _cpu(w)
    x2 = x.reshape(-1, x.shape[-1])
    x_rows, K = x2.shape
    E, N = w.shape[0], w.shape[1]
    if w.dim() != 3 or w.shape[2] != K:
        raise ValueError(f"oracle: experts {tuple(w.shape)} do not match K={K}")
    lhs_t, rhs_t = _u32(lhs), _u32(rhs)
    R = rhs_t.numel()
    y = torch.empty(R, N, dtype=torch.float64)
    a = torch.empty(R, N, dtype=torch.float64)
    w = w.contiguous()
    rc = lib.orc_gather_mm(x2.contiguous().data_ptr(), _DT[x.dtype], x_rows, K,
                           None if lhs_t is None else lhs_t.data_ptr(), rhs_t.data_ptr(), R, E, N,
                           w.data_ptr(), _DT[w.dtype], y.data_ptr(), a.data_ptr())
    _check(rc, "gather_mm")
    return y, a


def moe_swiglu(x, gate, up, down, ids, rw, group_size, bits, lib=None):
    """fp64 (y, a) [T, K]: each token's top-k experts, weighted by rw, of the
    SwiGLU block down(silu(x . gate^T) * (x . up^T)). gate and up are quantized
    (codes, scales, biases) of [E, I, K] weights, down of [E, K, I]; ids and rw
    are [T, topk]."""
    lib = lib or load()
    x = _cpu(x).contiguous()
    T, K = x.shape
    (gc, gsc, gb), (uc, usc, ub), (dc, dsc, db) = [tuple(_cpu(t).contiguous() for t in q)
                                                    for q in (gate, up, down)]
    E, I = gc.shape[0], gc.shape[1]
    if tuple(dc.shape[:2]) != (E, K) or tuple(uc.shape) != tuple(gc.shape):
        raise ValueError("oracle: gate/up [E, I, K] and down [E, K, I] do not agree")
    ids_t = _u32(ids).reshape(T, -1).contiguous()
    rw_t = _cpu(torch.as_tensor(rw, dtype=torch.float32)).reshape(T, -1).contiguous()
    topk = ids_t.shape[1]
    y = torch.empty(T, K, dtype=torch.float64)
    a = torch.empty(T, K, dtype=torch.float64)
    rc = lib.orc_moe_swiglu(x.data_ptr(), _DT[x.dtype], T, K, ids_t.data_ptr(), rw_t.data_ptr(),
                            topk, E, I, gc.data_ptr(), gsc.data_ptr(), gb.data_ptr(), uc.data_ptr(),
                            usc.data_ptr(), ub.data_ptr(), dc.data_ptr(), dsc.data_ptr(),
                            db.data_ptr(), _DT[gsc.dtype], group_size, bits, y.data_ptr(),
                            a.data_ptr())
    _check(rc, "moe_swiglu")
    return y, a


def gather_qmm_sampled(x, codes, scales, biases, lhs, rhs, group_size, bits, transpose,
                       r_idx, n_idx, lib=None):
    lib = lib or load()
    x, codes, scales, biases = _cpu(x), _cpu(codes), _cpu(scales), _cpu(biases)
    x2 = x.reshape(-1, x.shape[-1])
    x_rows, K = x2.shape
    E = codes.shape[0]
    N = codes.shape[1] if transpose else codes.shape[2] * 32 // bits
    _check_weights(codes, scales, biases, K, N, group_size, bits, transpose)
    lhs_t, rhs_t = _u32(lhs), _u32(rhs)
    R = rhs_t.numel()
    r_idx = _cpu(torch.as_tensor(r_idx, dtype=torch.int64))
    n_idx = _cpu(torch.as_tensor(n_idx, dtype=torch.int64))
    S = r_idx.numel()
    y = torch.empty(S, dtype=torch.float64)
    a = torch.empty(S, dtype=torch.float64)
    rc = lib.orc_gather_qmm_sampled(x2.data_ptr(), _DT[x.dtype], x_rows, K,
                                    None if lhs_t is None else lhs_t.data_ptr(),
                                    rhs_t.data_ptr(), R, E, N, codes.data_ptr(),
                                    scales.data_ptr(), biases.data_ptr(), _DT[scales.dtype],
                                    group_size, bits, int(transpose), S, r_idx.data_ptr(),
                                    n_idx.data_ptr(), y.data_ptr(), a.data_ptr())
    _check(rc, "gather_qmm_sampled")
    return y, a


# Acceptance bounds of the products: |y - y_ref| <= rel * a + 1e-5 with
# rel = 4e-3 for bf16 activations and 1e-5 for fp32.
TOL_REL = {torch.bfloat16: 4e-3, torch.float32: 1e-5}
TOL_ABS = 1e-5


def within_tolerance(y, y_ref, a, dtype) -> torch.Tensor:
    """Element-wise acceptance mask of the product tolerance."""
    err = (y.to(torch.float64) - y_ref).abs()
    return err <= TOL_REL[dtype] * a + TOL_ABS


# ---- floating-point modes ("Docs / Quantization", section "Floating-point
# formats"): MXFP4 = E2M1 values with an E8M0 scale per 32, MXFP8 = E4M3
# values with an E8M0 scale per 32, NVFP4 = E2M1 values with an E4M3 scale per
# 16 (the published definitions of the names; the pages' own table of the
# formats did not survive extraction). Parity with MLX's quantizer is unpinned.
FP_MODES = {"mxfp4": 1, "mxfp8": 2, "nvfp4": 3}
FP_GROUP = {"mxfp4": 32, "mxfp8": 32, "nvfp4": 16}
FP_BITS = {"mxfp4": 4, "mxfp8": 8, "nvfp4": 4}


def quantize_fp(w: torch.Tensor, mode: str, lib=None):
    """Codes [rows, cols*bits/32] (uint32 as int32) and uint8 scale codes
    [rows, cols/group] of w [rows, cols] (fp32 or bf16) in a floating-point mode."""
    lib = lib or load()
    w = _cpu(w)
    cols = w.shape[-1]
    rows = w.numel() // cols
    codes = torch.zeros(*w.shape[:-1], cols * FP_BITS[mode] // 32, dtype=torch.int32)
    scales = torch.empty(*w.shape[:-1], cols // FP_GROUP[mode], dtype=torch.uint8)
    rc = lib.orc_quantize_fp(w.data_ptr(), _DT[w.dtype], rows, cols, FP_MODES[mode],
                             codes.data_ptr(), scales.data_ptr())
    _check(rc, "quantize_fp")
    return codes, scales


def dequantize_fp(codes, scales, mode: str, lib=None) -> torch.Tensor:
    """element value x scale value, as bf16 [rows, cols]."""
    lib = lib or load()
    codes, scales = _cpu(codes), _cpu(scales)
    cols = codes.shape[-1] * 32 // FP_BITS[mode]
    rows = codes.numel() // codes.shape[-1]
    out = torch.empty(*codes.shape[:-1], cols, dtype=torch.int16)
    rc = lib.orc_dequantize_fp(codes.data_ptr(), scales.data_ptr(), rows, cols, FP_MODES[mode],
                               out.data_ptr())
    _check(rc, "dequantize_fp")
    return out.view(torch.bfloat16)


def qmm_fp(x, codes, scales, mode: str, lib=None):
    """(y, a): y = x . w_hat^T in fp64 with weights [N, K] in a floating-point
    mode, and a = sum_k |x w_hat| (the tolerance's scale)."""
    lib = lib or load()
    x, codes, scales = _cpu(x), _cpu(codes), _cpu(scales)
    M, K = x.shape
    N = codes.shape[0]
    y = torch.empty(M, N, dtype=torch.float64)
    a = torch.empty(M, N, dtype=torch.float64)
    rc = lib.orc_qmm_fp(x.data_ptr(), _DT[x.dtype], M, K, N, codes.data_ptr(), scales.data_ptr(),
                        FP_MODES[mode], y.data_ptr(), a.data_ptr())
    _check(rc, "qmm_fp")
    return y, a


def fp_value(kind: str, code: int, lib=None) -> float:
    """Value of one code: kind 'e2m1', 'e4m3' (elements) or 'e8m0' (scales)."""
    lib = lib or load()
    return lib.orc_fp_value({"e2m1": 0, "e4m3": 1, "e8m0": 2}[kind], code)


def fp_nearest(kind: str, v: float, lib=None) -> int:
    """Nearest code of v in 'e2m1' or 'e4m3' (ties to even, saturating)."""
    lib = lib or load()
    return lib.orc_fp_nearest({"e2m1": 0, "e4m3": 1}[kind], v)
