"""gather_mm (mixture of experts with full-precision bf16 experts) on the GPU
against the oracle, through the C ABI ("Docs / Quantization", section
"Mixture of experts"; gather_mm beside gather_qmm in the nuvec crate docs).

Tolerance: |y - y_ref| <= 4e-3 * sum_k |x_k w_k| + 1e-5 (bf16 output);
integer inputs give exact integers, compared bit for bit.
"""
import pytest
import torch

import group_wise_affine_dequant_b200 as nvq
import oracle as O
from group_wise_affine_dequant_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16


def _gather_mm(x, w, rhs, lhs=None, sorted_=False):
    ws = torch.empty(nvq.nv_gather_qmm_workspace_size(rhs.numel(), w.shape[0]), dtype=torch.uint8,
                     device="cuda")
    y = nvq.nv_gather_mm(x.cuda(), w.cuda(), rhs.to(torch.int32).cuda(),
                         None if lhs is None else lhs.to(torch.int32).cuda(), sorted_, workspace=ws)
    flags = nvq.nv_gather_qmm_flags(ws)
    return y.cpu(), flags


def test_gather_mm_page_example_shapes():
    w = W.normal((8, 128, 256), 0.02, 0, "bf16")
    x = W.normal((4, 1, 256), 1.0, 1, "bf16")
    ids = torch.tensor([0, 0, 3, 5])
    y, flags = _gather_mm(x, w, ids, sorted_=True)
    assert flags == 0 and tuple(y.shape) == (4, 128)
    yr, a = O.gather_mm(x, w, None, ids)
    P.assert_within(y, yr, a, BF16, "page example shapes")


def test_gather_mm_ragged_and_deterministic():
    """37 pairs over 5 experts (one empty, one with 17), a random token map,
    N = 200 (a unit ending mid-tile): within tolerance; two runs give the same
    bits; the sorted run gives the same rows per pair."""
    g = torch.Generator().manual_seed(43)
    E, N, K = 5, 200, 512
    w = W.normal((E, N, K), 0.02, 2, "bf16")
    x = W.normal((23, K), 1.0, 3, "bf16")
    rhs = torch.tensor([0] * 9 + [2] * 17 + [3] * 4 + [4] * 7)[torch.randperm(37, generator=g)]
    lhs = torch.randint(0, 23, (37,), generator=g)
    y, flags = _gather_mm(x, w, rhs, lhs)
    assert flags == 0
    yr, a = O.gather_mm(x, w, lhs, rhs)
    P.assert_within(y, yr, a, BF16, "ragged gather_mm")
    y2, _ = _gather_mm(x, w, rhs, lhs)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    order = torch.sort(rhs, stable=True).indices
    ys, flags = _gather_mm(x, w, rhs[order], lhs[order], sorted_=True)
    assert flags == 0
    assert torch.equal(ys.view(torch.int16), y[order].view(torch.int16))


def test_gather_mm_many_pairs_per_expert():
    """600 pairs on one expert (several 64-pair passes) and N = 300."""
    E, N, K = 3, 300, 256
    w = W.normal((E, N, K), 0.02, 4, "bf16")
    x = W.normal((700, K), 1.0, 5, "bf16")
    g = torch.Generator().manual_seed(3)
    rhs = torch.cat([torch.full((600,), 1), torch.full((40,), 2), torch.full((5,), 0)])
    rhs = rhs[torch.randperm(645, generator=g)]
    lhs = torch.randint(0, 700, (645,), generator=g)
    y, flags = _gather_mm(x, w, rhs, lhs)
    assert flags == 0
    yr, a = O.gather_mm(x, w, lhs, rhs)
    P.assert_within(y, yr, a, BF16, "many pairs")


def test_gather_mm_integer_exact():
    """Integer experts in [-1, 1] and x in [-2, 2] over K = 128: every output is
    an integer of magnitude <= 256, which bf16 holds, and every partial sum is
    exact in fp32, so the GPU must equal the oracle exactly."""
    g = torch.Generator().manual_seed(47)
    E, N, K, T = 4, 96, 128, 10
    w = torch.randint(-1, 2, (E, N, K), generator=g).to(BF16)
    x = torch.randint(-2, 3, (T, K), generator=g).to(BF16)
    lhs = torch.randint(0, T, (30,), generator=g)
    rhs = torch.randint(0, E, (30,), generator=g)
    y, flags = _gather_mm(x, w, rhs, lhs)
    assert flags == 0
    yr, _ = O.gather_mm(x, w, lhs, rhs)
    assert yr.abs().max() <= 256
    assert torch.equal(y.to(torch.float64), yr)


def test_gather_mm_invalid_ids_get_zero_rows_and_flags():
    E, N, K = 4, 64, 128
    w = W.normal((E, N, K), 0.02, 2, "bf16")
    x = W.normal((6, K), 1.0, 3, "bf16")
    rhs = torch.tensor([0, 1, 9, 2, 1])
    lhs = torch.tensor([0, 7, 1, 5, 2])
    y, flags = _gather_mm(x, w, rhs, lhs)
    assert flags & B_EXPERT and flags & B_TOKEN
    assert (y[1] == 0).all() and (y[2] == 0).all()
    ok = torch.tensor([0, 3, 4])
    yr, a = O.gather_mm(x, w, lhs[ok], rhs[ok])
    P.assert_within(y[ok], yr, a, BF16, "valid pairs beside invalid ones")


B_EXPERT = 1  # NV_FLAG_EXPERT_OUT_OF_RANGE
B_TOKEN = 4   # NV_FLAG_TOKEN_OUT_OF_RANGE


def test_gather_mm_moe_config_sampled():
    """64 bf16 experts [1536, 2048], 512 tokens x top-4 (unsorted): 64 pairs
    checked against the oracle, every output column of each."""
    m = W.MOE
    w = W.normal((m["E"], m["N"], m["K"]), 0.02, 0, "bf16")
    x = W.normal((m["tokens"], m["K"]), 1.0, 1, "bf16")
    ids = W.expert_ids(m["tokens"], m["E"], m["top_k"], 2)
    lhs, rhs = W.flatten_pairs(ids)
    y, flags = _gather_mm(x, w, rhs, lhs)
    assert flags == 0 and tuple(y.shape) == (rhs.numel(), m["N"])
    pick = torch.randperm(rhs.numel(), generator=torch.Generator().manual_seed(9))[:64]
    yr, a = O.gather_mm(x, w, lhs[pick], rhs[pick])
    P.assert_within(y[pick], yr, a, BF16, "MoE config, sampled pairs")
