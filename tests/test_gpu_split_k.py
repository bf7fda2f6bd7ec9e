"""Split-K quantized products and batched products ("Docs / Quantization",
section "Products on the GPU": split-K when the output is small but the inner
dimension long; nuvec crate docs, section "Determinism": each batch item of a
quantized product gets its solo bits, the split-K partitions counted per
item), against the oracle through the C ABI."""
import pytest
import torch

import group_wise_affine_dequant_b200 as nvq
import oracle as O
from group_wise_affine_dequant_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu
BF16, F32 = torch.bfloat16, torch.float32


def _case(N, K, M, bits, gs, seed=70):
    w = W.normal((N, K), 0.02, seed, "bf16")
    x = W.normal((M, K), 1.0, seed + 1, "bf16")
    c, s, b = O.quantize_affine(w, gs, bits)
    return x, c, s, b


@pytest.mark.parametrize("bits,gs", [(4, 64), (4, 32), (4, 128), (2, 64), (8, 64), (8, 128), (2, 32)])
@pytest.mark.parametrize("M,N,K", [(20, 200, 2432), (130, 96, 4864), (9, 1000, 1280), (64, 448, 7680)])
def test_split_k_against_the_oracle(bits, gs, M, N, K):
    """Shapes whose tiles fill few SMs: K is split over a cluster (uneven
    k-ranges when the steps do not divide), ragged rows and columns."""
    assert nvq.nv_qmm_splits(M, K, N, bits, gs) > 1
    x, c, s, b = _case(N, K, M, bits, gs)
    y = nvq.nv_qmm(x.cuda(), c.cuda(), s.cuda(), b.cuda(), gs, bits, True).cpu()
    yr, a = O.qmm(x, c, s, b, gs, bits, True)
    P.assert_within(y, yr, a, BF16, f"split-K M={M} N={N} K={K} b{bits} g{gs}")


def test_split_k_deterministic_and_integer_exact():
    x, c, s, b = P.to_dev(*_case(200, 2432, 20, 4, 64))
    y1 = nvq.nv_qmm(x, c, s, b, 64, 4, True)
    y2 = nvq.nv_qmm(x, c, s, b, 64, 4, True)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    gen = torch.Generator().manual_seed(71)
    wi = P.integer_weights(160, 4096, 64, 4, gen)
    xi = torch.randint(-2, 3, (24, 4096), generator=gen)
    keep = torch.tensor([0, 511, 1024, 1600, 2100, 2600, 3100, 4095])  # spread over the splits
    mask = torch.zeros(4096, dtype=torch.bool)
    mask[keep] = True
    xi[:, ~mask] = 0  # |y| <= 8 * 2 * 15 = 240: exact in bf16
    ci, si, bi = O.quantize_affine(wi.to(BF16), 64, 4)
    assert nvq.nv_qmm_splits(24, 4096, 160, 4, 64) > 1
    y = nvq.nv_qmm(xi.to(BF16).cuda(), ci.cuda(), si.cuda(), bi.cuda(), 64, 4, True).cpu()
    yr, _ = O.qmm(xi.to(BF16), ci, si, bi, 64, 4, True)
    assert torch.equal(y.to(torch.float64), yr)


def test_split_k_small_n_long_k_workload():
    """x [64, 14336] . W[1024, 14336]^T, 4-bit g64 (the split-K bench shape):
    sampled outputs and whole rows against the oracle."""
    x, c, s, b = _case(1024, 14336, 64, 4, 64, seed=72)
    assert nvq.nv_qmm_splits(64, 14336, 1024, 4, 64) > 1
    y = nvq.nv_qmm(x.cuda(), c.cuda(), s.cuda(), b.cuda(), 64, 4, True).cpu()
    g = torch.Generator().manual_seed(73)
    mi = torch.randint(0, 64, (2000,), generator=g)
    ni = torch.randint(0, 1024, (2000,), generator=g)
    yr, a = O.qmm_sampled(x, c, s, b, 64, 4, True, mi, ni)
    P.assert_within(y[mi, ni], yr, a, BF16, "split-K 64x1024x14336 sampled")
    for m in (0, 63):
        yr, a = O.qmm(x[m:m + 1], c, s, b, 64, 4, True)
        P.assert_within(y[m:m + 1], yr, a, BF16, f"split-K 64x1024x14336 row {m}")


@pytest.mark.parametrize("transpose", [True, False])
@pytest.mark.parametrize("B,L", [(5, 20), (7, 3), (4, 1), (3, 9), (2, 64)])
def test_batch_items_get_their_solo_bits(B, L, transpose):
    """nv_qmm_batched on [B, L, K]: every item equals nv_qmm of that item alone,
    bit for bit, whether the batch is routed to the matrix-vector kernels
    (L <= 8), the tiled kernel with split-K (L > 8, small N) or the plain one."""
    N, K = (192, 3072) if transpose else (384, 1024)
    w = W.normal((N, K) if transpose else (K, N), 0.02, 74, "bf16")
    c, s, b = P.to_dev(*O.quantize_affine(w, 64, 4))
    x = W.normal((B, L, K), 1.0, 75, "bf16").cuda()
    yb = nvq.nv_qmm_batched(x, c, s, b, 64, 4, transpose)
    assert tuple(yb.shape) == (B, L, N)
    for i in range(B):
        yi = nvq.nv_qmm(x[i], c, s, b, 64, 4, transpose)
        assert torch.equal(yb[i].view(torch.int16), yi.view(torch.int16)), (B, L, i)
    if transpose and L > 8:
        assert nvq.nv_qmm_splits(L, K, N, 4, 64) > 1  # the items themselves split K
    yr, a = O.qmm(x.reshape(B * L, K).cpu(), c.cpu(), s.cpu(), b.cpu(), 64, 4, transpose)
    P.assert_within(yb.reshape(B * L, N), yr, a, BF16, f"batched B={B} L={L}")


def test_batch_fp32_items_get_their_solo_bits():
    w = W.normal((96, 256), 1.0, 76, "f32")
    c, s, b = P.to_dev(*O.quantize_affine(w, 64, 4))
    x = W.normal((3, 11, 256), 1.0, 77, "f32").cuda()
    yb = nvq.nv_qmm_batched(x, c, s, b, 64, 4, True)
    for i in range(3):
        assert torch.equal(yb[i], nvq.nv_qmm(x[i], c, s, b, 64, 4, True))
