"""Helpers shared by the GPU parity tests: run the oracle on host copies of the
same inputs the CUDA path receives, and compare element by element."""
from __future__ import annotations

import torch

import oracle as O


def tol_mask(y_gpu: torch.Tensor, y_ref: torch.Tensor, a: torch.Tensor, dtype) -> torch.Tensor:
    """|y - y_ref| <= rel * a + 1e-5, rel = 4e-3 (bf16 activations) or 1e-5 (fp32)."""
    return O.within_tolerance(y_gpu.detach().cpu().to(torch.float64), y_ref, a, dtype)


def assert_within(y_gpu, y_ref, a, dtype, what=""):
    ok = tol_mask(y_gpu, y_ref, a, dtype)
    if not bool(ok.all()):
        yg = y_gpu.detach().cpu().to(torch.float64)
        err = (yg - y_ref).abs()
        bad = (~ok).nonzero()
        i = tuple(bad[0].tolist())
        raise AssertionError(
            f"{what}: {int((~ok).sum())} of {ok.numel()} outside tolerance; first {i}: "
            f"gpu {float(yg[i])} ref {float(y_ref[i])} err {float(err[i])} a {float(a[i])}")


def worst_ratio(y_gpu, y_ref, a, dtype) -> float:
    """max |y - y_ref| / (rel * a + 1e-5): below 1 passes."""
    yg = y_gpu.detach().cpu().to(torch.float64)
    return float(((yg - y_ref).abs() / (O.TOL_REL[dtype] * a + O.TOL_ABS)).max())


def quantize_host(w: torch.Tensor, gs: int, bits: int):
    """Oracle codes, scales, biases of host weights (the inputs both sides use)."""
    return O.quantize_affine(w, gs, bits)


def to_dev(*ts, device="cuda"):
    return [t.to(device) for t in ts]


def integer_weights(rows, cols, gs, bits, gen):
    """Integer weights whose every group (along cols) holds 0 and 2^b - 1:
    scale 1, bias 0, code = weight."""
    hi = 2 ** bits - 1
    w = torch.randint(0, hi + 1, (rows, cols), generator=gen)
    for g in range(cols // gs):
        w[:, g * gs] = 0
        w[:, g * gs + 1] = hi
    return w
