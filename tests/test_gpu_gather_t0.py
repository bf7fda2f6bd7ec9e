"""The grouped tensor-core route of gather_qmm with experts stored [E, K, N]
(transpose = 0, grouped along N; "Docs / Quantization", section "Mixture of
experts", and the product's transpose flag, section "Affine") against the
oracle: ragged experts, a unit of weight columns that ends inside the tile,
experts with more pairs than one pass holds, invalid ids, unit activations that
read out every dequantized weight exactly, and the mixture-of-experts shapes on
sampled outputs. Tolerance as in the other parity tests."""
import pytest
import torch

import group_wise_affine_dequant_b200 as nvq
import oracle as O
from group_wise_affine_dequant_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16
QUANTS = [(4, 32), (4, 64), (4, 128), (8, 32), (8, 64), (8, 128), (2, 32), (2, 64), (2, 128)]


def _gather(x, c, s, b, rhs, lhs, gs, bits, sorted_=False, ws=None):
    if ws is None:
        ws = torch.empty(max(nvq.nv_gather_qmm_workspace_size(rhs.numel(), c.shape[0]), 16),
                         dtype=torch.uint8, device="cuda")
    y = nvq.nv_gather_qmm(x.cuda(), c.cuda(), s.cuda(), b.cuda(), rhs.to(torch.int32).cuda(),
                          None if lhs is None else lhs.to(torch.int32).cuda(), gs, bits, False,
                          sorted_, False, workspace=ws)
    flags = nvq.nv_gather_qmm_flags(ws)
    assert nvq.nv_pipeline_error() == 0
    return y.cpu(), flags


@pytest.mark.parametrize("N", [384, 1024])
@pytest.mark.parametrize("bits,gs", QUANTS)
def test_ragged_experts(bits, gs, N):
    """37 pairs over 5 experts (one empty, one with 17 pairs); N = 384 is one
    full unit of 256 columns and one that ends half way, and its scale rows
    are read from global memory; N = 1024 has N / gs a multiple of 8, so the
    scales and biases come with the codes by TMA."""
    g = torch.Generator().manual_seed(70 + bits + gs)
    E, K, T = 5, 512, 23
    w = W.normal((E, K, N), 0.02, 71, "bf16")
    x = W.normal((T, K), 1.0, 72, "bf16")
    c, s, b = O.quantize_affine(w, gs, bits)
    rhs = torch.tensor([0] * 9 + [2] * 17 + [3] * 4 + [4] * 7)[torch.randperm(37, generator=g)]
    lhs = torch.randint(0, T, (37,), generator=g)
    y, flags = _gather(x, c, s, b, rhs, lhs, gs, bits)
    assert flags == 0
    yr, a = O.gather_qmm(x, c, s, b, lhs, rhs, gs, bits, False)
    P.assert_within(y, yr, a, BF16, f"transpose=0 ragged b{bits} g{gs}")


@pytest.mark.parametrize("spread", ["small", "wide"])
@pytest.mark.parametrize("bits", [4, 8, 2])
def test_unit_activations_read_out_the_weights(bits, spread):
    """x rows are unit vectors e_k: every output is one dequantized weight
    w_hat[k, n] times 1 plus exact zeros, so it must equal the oracle's stored
    (once-rounded) weight bit for bit. Covers every column of two units, the
    A-tile row order and the epilogue's column map. "small": N(0, 0.02)
    weights (scales below 2^-5); "wide": k-rows scaled by 10^u, u in [-5, 3],
    and a constant row (scale 0), so scales on both sides of 2^-5 and zero
    meet in the same stages."""
    E, K, N, gs = 3, 256, 512, 64
    w = W.normal((E, K, N), 0.02, 73, "bf16")
    if spread == "wide":
        g = torch.Generator().manual_seed(86)
        w = (w.float() * 10.0 ** (torch.rand(E, K, 1, generator=g) * 8 - 5)).to(BF16)
        w[:, 5, :] = 0.75
    c, s, b = O.quantize_affine(w, gs, bits)
    wh = O.dequantize_stored(c, s, b, gs, bits)  # [E, K, N] bf16
    g = torch.Generator().manual_seed(74)
    R = 96
    ks = torch.randint(0, K, (R,), generator=g)
    rhs = torch.randint(0, E, (R,), generator=g)
    x = torch.zeros(R, K, dtype=BF16)
    x[torch.arange(R), ks] = 1.0
    y, flags = _gather(x, c, s, b, rhs, None, gs, bits)
    assert flags == 0
    want = wh[rhs, ks]  # [R, N]
    bad = y.float() != want.float()
    assert not bad.any(), f"b{bits}: {int(bad.sum())} differ, first {bad.nonzero()[0].tolist()}"


def test_many_pairs_per_expert_and_deterministic():
    """One expert with 600 pairs (ten passes of 64), and a second call that
    must give the same bits."""
    E, K, N = 3, 256, 768
    w = W.normal((E, K, N), 0.02, 75, "bf16")
    x = W.normal((700, K), 1.0, 76, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    g = torch.Generator().manual_seed(77)
    rhs = torch.cat([torch.full((600,), 1), torch.full((40,), 2), torch.full((5,), 0)])
    rhs = rhs[torch.randperm(645, generator=g)]
    lhs = torch.randint(0, 700, (645,), generator=g)
    y, flags = _gather(x, c, s, b, rhs, lhs, 64, 4)
    y2, _ = _gather(x, c, s, b, rhs, lhs, 64, 4)
    assert flags == 0
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    yr, a = O.gather_qmm(x, c, s, b, lhs, rhs, 64, 4, False)
    P.assert_within(y, yr, a, BF16, "transpose=0 many pairs")


def test_invalid_ids_get_zero_rows():
    E, K, N = 4, 128, 256
    w = W.normal((E, K, N), 0.02, 78, "bf16")
    x = W.normal((6, K), 1.0, 79, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    rhs = torch.tensor([0, 1, 9, 2, 1])
    lhs = torch.tensor([0, 1, 2, 7, 5])
    y, flags = _gather(x, c, s, b, rhs, lhs, 64, 4)
    assert flags & nvq.binding.NV_FLAG_EXPERT_OUT_OF_RANGE
    assert flags & nvq.binding.NV_FLAG_TOKEN_OUT_OF_RANGE
    assert (y[2] == 0).all() and (y[3] == 0).all()
    ok = torch.tensor([0, 1, 4])
    yr, a = O.gather_qmm(x, c, s, b, lhs[ok], rhs[ok], 64, 4, False)
    P.assert_within(y[ok], yr, a, BF16, "transpose=0 valid rows")


def test_shapes_outside_the_tiles_take_the_general_route():
    """N * bits not a multiple of 128 (N = 96, 2-bit) and K not a multiple of
    64 (K = 96) still give the right products (the general kernel)."""
    g = torch.Generator().manual_seed(80)
    for K, N, bits in ((512, 96, 2), (96, 256, 4)):
        w = W.normal((3, K, N), 0.02, 81, "bf16")
        x = W.normal((9, K), 1.0, 82, "bf16")
        c, s, b = O.quantize_affine(w, 32, bits)
        rhs = torch.randint(0, 3, (20,), generator=g)
        lhs = torch.randint(0, 9, (20,), generator=g)
        y, flags = _gather(x, c, s, b, rhs, lhs, 32, bits)
        assert flags == 0
        yr, a = O.gather_qmm(x, c, s, b, lhs, rhs, 32, bits, False)
        P.assert_within(y, yr, a, BF16, f"transpose=0 general K={K} N={N} b{bits}")


def test_moe_shapes_sampled():
    """The mixture-of-experts workload's shapes with the experts stored
    [E, K, N]: 2048 pairs over 64 experts, K = 2048, N = 1536; sorted and
    unsorted pair orders give the same bits, sampled outputs match the oracle."""
    m = W.MOE
    w = W.normal((m["E"], m["K"], m["N"]), 0.02, 83, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    x = W.normal((m["tokens"], m["K"]), 1.0, 84, "bf16")
    ids = W.expert_ids(m["tokens"], m["E"], m["top_k"], 2)
    lhs, rhs = W.flatten_pairs(ids)
    lhs_s, rhs_s, order = W.stable_sort_pairs(lhs, rhs)
    y_u, f_u = _gather(x, c, s, b, rhs, lhs, 64, 4)
    y_s, f_s = _gather(x, c, s, b, rhs_s, lhs_s, 64, 4, sorted_=True)
    assert f_u == 0 and f_s == 0
    assert torch.equal(y_s.view(torch.int16), y_u[order].view(torch.int16))
    g = torch.Generator().manual_seed(85)
    R, N = rhs.numel(), m["N"]
    r_idx = torch.randint(0, R, (4096,), generator=g)
    n_idx = torch.randint(0, N, (4096,), generator=g)
    yr, a = O.gather_qmm_sampled(x, c, s, b, lhs, rhs, 64, 4, False, r_idx, n_idx)
    P.assert_within(y_u[r_idx, n_idx], yr, a, BF16, "transpose=0 moe sampled")


@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 64), (2, 32), (4, 128)])
def test_zero_weights_with_nonzero_bias_under_huge_activations(bits, gs):
    """Integer experts in [-(2^bits - 1), 0] with both ends in every group:
    scale 1 and bias -(2^bits - 1), so code 2^bits - 1 dequantizes to exactly
    0 while scale * code and bias are each large. k-rows S hold only such
    zeros (and each group's -max) and meet activations of +-2^60: a product
    that summed scale * code * x and bias * x apart would cancel 2^60-sized
    terms. The grouped kernel dequantizes first (the general form here, since
    the scales are 1)."""
    E, K, N, T = 3, 512, 512, 12
    hi = 2 ** bits - 1
    g = torch.Generator().manual_seed(95 + bits)
    S = torch.arange(3, K, 64)
    ws = []
    for _ in range(E):
        w = -torch.randint(0, hi + 1, (K, N), generator=g).to(torch.float32)
        w[:, ::gs] = -hi
        w[:, 1::gs] = 0.0
        w[S, :] = 0.0
        w[S.unsqueeze(1), torch.arange(0, N, gs).unsqueeze(0)] = -hi
        ws.append(w)
    w = torch.stack(ws).to(BF16)
    c, s, b = O.quantize_affine(w, gs, bits)
    assert (s.float() == 1).all() and (b.float() == -hi).all()
    x = torch.randn(T, K, generator=g)
    x[:, S] = 2.0 ** 60 * torch.where(torch.rand(len(S), generator=g) < 0.5, -1.0, 1.0)
    x = x.to(BF16)
    R = 40
    rhs = torch.randint(0, E, (R,), generator=g)
    lhs = torch.randint(0, T, (R,), generator=g)
    y, flags = _gather(x, c, s, b, rhs, lhs, gs, bits)
    assert flags == 0 and torch.isfinite(y.float()).all()
    yr, a = O.gather_qmm(x, c, s, b, lhs, rhs, gs, bits, False)
    P.assert_within(y, yr, a, BF16, f"transpose=0 cancelling bias b{bits} g{gs}")


@pytest.mark.parametrize("j", [-40, -7, 9, 50])
def test_power_of_two_scalings_are_exact(j):
    """y(2^j x) == 2^j y(x) bit for bit: every product and sum scales exactly
    (no value leaves the fp32 range) and so does the bf16 rounding."""
    E, K, N, T = 3, 256, 512, 10
    w = W.normal((E, K, N), 0.02, 96, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    x = W.normal((T, K), 1.0, 97, "bf16")
    g = torch.Generator().manual_seed(98)
    rhs = torch.randint(0, E, (24,), generator=g)
    lhs = torch.randint(0, T, (24,), generator=g)
    y1, _ = _gather(x, c, s, b, rhs, lhs, 64, 4)
    y2, _ = _gather((x.float() * 2.0 ** j).to(BF16), c, s, b, rhs, lhs, 64, 4)
    assert torch.equal((y1.float() * 2.0 ** j).to(BF16).view(torch.int16), y2.view(torch.int16)), j
