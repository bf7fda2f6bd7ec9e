"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle.

This module only draws random numbers and casts them to the storage dtype. It
holds none of the quantization or product arithmetic, so both sides of every
parity check can read the same bytes without sharing any of the method.

Recipe (every workload):
  * ``torch.Generator('cpu').manual_seed(seed)`` then ``torch.randn`` in fp32,
    multiplied by the standard deviation, then cast round-to-nearest-even to
    the stored dtype (torch's own cast).
  * Weights use seed 0, activations seed 1, expert ids seed 2, except the tiny
    workload, which draws W then x from one generator seeded 0.
  * Expert ids: for each token, the first ``top_k`` entries of a seeded
    ``randperm(n_experts)``: uniform without replacement.

Shapes are the Llama/MoE shapes of the quantized-product workloads: 4096 and
14336 are the hidden and MLP sizes of an 8B-class model; the MoE layer has 64
experts of [1536, 2048].
"""
from __future__ import annotations

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def normal(shape, std: float, seed: int, dtype: str = "bf16",
           generator: torch.Generator | None = None) -> torch.Tensor:
    """N(0, std^2) fp32 draws cast round-to-nearest-even to ``dtype`` (CPU tensor)."""
    g = generator if generator is not None else torch.Generator().manual_seed(seed)
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t = t * std
    return t.to(DTYPES[dtype]).contiguous()


def expert_ids(tokens: int, n_experts: int, top_k: int, seed: int = 2) -> torch.Tensor:
    """[tokens, top_k] uint32-valued (int64 tensor) ids, distinct within each token."""
    g = torch.Generator().manual_seed(seed)
    rows = [torch.randperm(n_experts, generator=g)[:top_k] for _ in range(tokens)]
    return torch.stack(rows).to(torch.int64)


def flatten_pairs(ids: torch.Tensor):
    """Flatten [tokens, top_k] ids into (lhs, rhs) pair lists of length tokens*top_k.

    lhs[r] is the token (the row of x), rhs[r] the expert of pair r; pairs are in
    token-major order, which is the order of the output rows."""
    tokens, k = ids.shape
    lhs = torch.arange(tokens, dtype=torch.int64).repeat_interleave(k)
    rhs = ids.reshape(-1).clone()
    return lhs, rhs


def stable_sort_pairs(lhs: torch.Tensor, rhs: torch.Tensor):
    """Pairs stable-sorted by expert (the "sorted" run's input order)."""
    order = torch.sort(rhs, stable=True).indices
    return lhs[order].contiguous(), rhs[order].contiguous(), order


# ---------------------------------------------------------------------------
# The workloads. Each entry gives shapes and the quantization parameters;
# sizes follow the decode, few-row, prefill and mixture-of-experts shapes.
# ---------------------------------------------------------------------------
TINY = dict(name="tiny", N=256, K=512, M=4, dtype="f32", group_size=64, bits=4, seed=0)

DECODE = dict(name="decode", N=14336, K=4096, M=1, dtype="bf16", w_std=0.02)
FEWROW_SHAPES = [(4096, 4096), (14336, 4096)]      # (N, K)
FEWROW_M = [2, 4, 8]
PREFILL = dict(name="prefill", M=2048, N=14336, K=4096, dtype="bf16", w_std=0.02)
PREFILL_VARIANTS = [(4, 32), (4, 64), (4, 128), (2, 64), (8, 64)]  # (bits, group_size)
MOE = dict(name="moe", E=64, N=1536, K=2048, tokens=512, top_k=4, dtype="bf16",
           w_std=0.02, group_size=64, bits=4)


def tiny_inputs():
    """W [256,512] and x [4,512], fp32 ~N(0,1), one generator seeded 0 (W first)."""
    g = torch.Generator().manual_seed(TINY["seed"])
    w = normal((TINY["N"], TINY["K"]), 1.0, 0, "f32", generator=g)
    x = normal((TINY["M"], TINY["K"]), 1.0, 0, "f32", generator=g)
    return w, x


def decode_weight(N: int = 14336, K: int = 4096, std: float = 0.02, seed: int = 0):
    return normal((N, K), std, seed, "bf16")


def activations(M: int, K: int, seed: int = 1, dtype: str = "bf16"):
    return normal((M, K), 1.0, seed, dtype)
