"""The floating-point modes (MXFP4, MXFP8, NVFP4; "Docs / Quantization", section
"Floating-point formats") on the GPU against the oracle: quantizer and
dequantizer bit for bit, products within the tolerance, row exactness of the
matrix-vector route, and unit activations reading out every weight exactly."""
import pytest
import torch

import group_wise_affine_dequant_b200 as nvq
import oracle as O
from group_wise_affine_dequant_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16
MODES = ["mxfp4", "mxfp8", "nvfp4"]


def _weights(rows, cols, seed, dtype=BF16):
    """N(0, 1) rows scaled by 10^u, u in [-6, 3], with zero groups, signed
    zeros, values at a tie of the element grid and huge and tiny binades."""
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(rows, cols, generator=g) * (10.0 ** (torch.rand(rows, 1, generator=g) * 9 - 6))
    w[0, :32] = 0.0
    w[1, :32] = -0.0
    w[2, :16] = torch.tensor([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, -0.25, 7.0, 6.5, 0.1, -0.1, 3.0, 0.5])
    w[3, :32] = 2.0 ** 100
    w[4, :32] = 2.0 ** -100
    w[5, :32] = -(2.0 ** -130)
    return w.to(dtype)


@pytest.mark.parametrize("dtype", [BF16, torch.float32])
@pytest.mark.parametrize("mode", MODES)
def test_quantize_and_dequantize_bit_exact(mode, dtype):
    w = _weights(96, 512, 1, dtype)
    c0, s0 = O.quantize_fp(w, mode)
    c, s = nvq.nv_quantize_fp(w.cuda(), mode)
    torch.cuda.synchronize()
    assert torch.equal(s.cpu(), s0), f"{mode}: {int((s.cpu() != s0).sum())} scale codes differ"
    assert torch.equal(c.cpu(), c0), f"{mode}: {int((c.cpu() != c0).sum())} code words differ"
    wh = nvq.nv_dequantize_fp(c, s, mode)
    torch.cuda.synchronize()
    wh0 = O.dequantize_fp(c0, s0, mode)
    assert torch.equal(wh.cpu().view(torch.int16), wh0.view(torch.int16)), mode


@pytest.mark.parametrize("mode", ["mxfp4", "nvfp4"])
def test_quantize_decode_weight_bit_exact(mode):
    """The decode weight W [14336, 4096] ~N(0, 0.02) (bf16)."""
    w = W.normal((14336, 4096), 0.02, 0, "bf16")
    c0, s0 = O.quantize_fp(w, mode)
    c, s = nvq.nv_quantize_fp(w.cuda(), mode)
    torch.cuda.synchronize()
    assert torch.equal(s.cpu(), s0) and torch.equal(c.cpu(), c0), mode


def _product_case(mode, M, N, K, seed):
    w = W.normal((N, K), 0.02, seed, "bf16")
    c, s = O.quantize_fp(w, mode)
    x = W.normal((M, K), 1.0, seed + 1, "bf16")
    return x, c, s


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M", [1, 3, 8])
def test_matvec_products(mode, M):
    x, c, s = _product_case(mode, M, 1040, 2048, 3)
    y = nvq.nv_qmm_fp(x.cuda(), c.cuda(), s.cuda(), mode)
    torch.cuda.synchronize()
    yr, a = O.qmm_fp(x, c, s, mode)
    P.assert_within(y, yr, a, BF16, f"{mode} M={M}")


@pytest.mark.parametrize("mode", MODES)
def test_matvec_rows_are_exact(mode):
    """Every row of an 8-row product is bytewise equal to its one-row product."""
    x, c, s = _product_case(mode, 8, 520, 1024, 5)
    cd, sd = c.cuda(), s.cuda()
    y = nvq.nv_qmm_fp(x.cuda(), cd, sd, mode)
    for m in range(8):
        y1 = nvq.nv_qmm_fp(x[m:m + 1].cuda(), cd, sd, mode)
        assert torch.equal(y[m:m + 1].view(torch.int16), y1.view(torch.int16)), (mode, m)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M", [9, 300])
def test_tiled_products(mode, M):
    x, c, s = _product_case(mode, M, 704, 1024, 7)
    y = nvq.nv_qmm_fp(x.cuda(), c.cuda(), s.cuda(), mode)
    torch.cuda.synchronize()
    yr, a = O.qmm_fp(x, c, s, mode)
    P.assert_within(y, yr, a, BF16, f"{mode} M={M}")


@pytest.mark.parametrize("mode", MODES)
def test_split_k_shape(mode):
    """A small output with a long inner dimension (the split-K route)."""
    x, c, s = _product_case(mode, 64, 1024, 14336, 9)
    y = nvq.nv_qmm_fp(x.cuda(), c.cuda(), s.cuda(), mode)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(1)
    rows = torch.randint(0, 64, (4,), generator=g).tolist()
    for m in rows:
        yr, a = O.qmm_fp(x[m:m + 1], c, s, mode)
        P.assert_within(y[m:m + 1], yr, a, BF16, f"{mode} split-K row {m}")


@pytest.mark.parametrize("mode", MODES)
def test_prefill_sampled(mode):
    """x [2048, 4096] . W[14336, 4096]^T: whole rows against the oracle."""
    x, c, s = _product_case(mode, 2048, 14336, 4096, 0)
    y = nvq.nv_qmm_fp(x.cuda(), c.cuda(), s.cuda(), mode)
    torch.cuda.synchronize()
    for m in (0, 1337, 2047):
        yr, a = O.qmm_fp(x[m:m + 1], c, s, mode)
        P.assert_within(y[m:m + 1], yr, a, BF16, f"{mode} prefill row {m}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M", [4, 40])
def test_unit_activations_read_out_the_weights(mode, M):
    """Unit-vector rows of x give each dequantized weight back exactly (one
    exact product plus exact zeros), on both routes. Compared as values: a
    weight that is -0 comes back as +0, since (-0) + (+0) is +0 in any sum."""
    w = _weights(264, 1024, 21)
    c, s = O.quantize_fp(w, mode)
    wh = O.dequantize_fp(c, s, mode)
    ks = torch.randperm(1024, generator=torch.Generator().manual_seed(M))[:M]
    x = torch.zeros(M, 1024, dtype=BF16)
    x[torch.arange(M), ks] = 1.0
    y = nvq.nv_qmm_fp(x.cuda(), c.cuda(), s.cuda(), mode).cpu()
    want = wh[:, ks].t()
    bad = y.float() != want.float()
    assert (want.float() == 0).any() and (want.float() != 0).any()
    assert not bad.any(), f"{mode} M={M}: {int(bad.sum())} differ, first {bad.nonzero()[0].tolist()}"


def test_argument_errors():
    w = torch.zeros(4, 64, dtype=BF16, device="cuda")
    with pytest.raises(ValueError):
        nvq.nv_quantize_fp(w, "fp6")
    with pytest.raises(nvq.NvqError):
        nvq.nv_quantize_fp(torch.zeros(4, 48, dtype=BF16, device="cuda"), "mxfp4")  # cols % 32
    c, s = nvq.nv_quantize_fp(w, "mxfp4")
    with pytest.raises(nvq.NvqError):  # fp32 activations are not supported by the product
        nvq.nv_qmm_fp(torch.zeros(2, 64, device="cuda"), c, s, "mxfp4")
