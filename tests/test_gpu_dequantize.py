"""The dequantizer and the 1-bit width on the GPU against the oracle, through
the C ABI ("Docs / Quantization", section "Affine": w ~= scale * code + bias).

Dequantized weights are compared bit for bit with the oracle's stored value
(scale * code + bias rounded once to fp32, then to the dtype with ties to
even); 1-bit codes, scales and biases bit for bit with the oracle's quantizer.
Sizes: every width and group size with a word count that is not a multiple of
four (the kernel's tail), a 3-D stack of matrices, and the full decode weight.
"""
import pytest
import torch

import group_wise_affine_dequant_b200 as nvq
import oracle as O
from group_wise_affine_dequant_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

BF16, F32 = torch.bfloat16, torch.float32
WIDTHS = [(1, 32), (1, 64), (1, 128), (2, 32), (2, 128), (4, 32), (4, 64), (4, 128), (8, 32), (8, 64)]


def _bits_of(t):
    return t.view(torch.int16) if t.dtype == BF16 else t.view(torch.int32)


def _gpu_dequantize(c, s, b, gs, bits):
    dc, ds, db = P.to_dev(c, s, b)
    w = nvq.nv_dequantize_affine(dc, ds, db, gs, bits)
    torch.cuda.synchronize()
    return w.cpu()


@pytest.mark.parametrize("dt", [BF16, F32])
@pytest.mark.parametrize("bits,gs", WIDTHS)
def test_dequantize_bit_exact(bits, gs, dt):
    # 37 rows of 5 groups: 37 * 5 * gs * bits / 32 words, never a multiple of 4
    # at 1 bit and g32 (185 words), so the tail path runs too
    w = W.normal((37, 5 * gs), 0.02 if dt == BF16 else 1.0, 21 + bits, "bf16" if dt == BF16 else "f32")
    c, s, b = O.quantize_affine(w, gs, bits)
    got = _gpu_dequantize(c, s, b, gs, bits)
    ref = O.dequantize_stored(c, s, b, gs, bits)
    assert got.dtype == dt and got.shape == ref.shape
    assert torch.equal(_bits_of(got), _bits_of(ref)), f"{int((got != ref).sum())} values differ"


def test_dequantize_rounding_cases():
    """The oracle's rounding pins, run on the GPU: ties to even in the bf16
    store, one rounding of the exact scale * code + bias."""
    words = torch.tensor([[1 | (2 << 8) | (3 << 16)]], dtype=torch.int32).repeat(1, 8)
    s, b = torch.tensor([[2.0 ** -9]], dtype=BF16), torch.tensor([[1.0]], dtype=BF16)
    got = _gpu_dequantize(words, s, b, 32, 8)
    assert got[0, :4].to(torch.float64).tolist() == [1.0, 1.0, 1.0 + 2.0 ** -7, 1.0]
    assert torch.equal(_bits_of(got), _bits_of(O.dequantize_stored(words, s, b, 32, 8)))
    w3 = torch.full((1, 8), 3 | (3 << 8) | (3 << 16) | (3 << 24), dtype=torch.int32)
    s32, b32 = torch.tensor([[1.0 + 2.0 ** -23]]), torch.tensor([[-3.0]])
    got = _gpu_dequantize(w3, s32, b32, 32, 8)
    assert (got == 3 * 2.0 ** -23).all(), got
    # 37 * 7 = 259 is a bf16 tie; the exact 259 - 2^-20 (or - 2^-60) rounds once to 258
    w7 = torch.tensor([[7 | (7 << 8) | (7 << 16) | (7 << 24)]], dtype=torch.int32).repeat(1, 8)
    for e in (-20, -60):
        s37, bb = torch.tensor([[37.0]], dtype=BF16), torch.tensor([[-(2.0 ** e)]], dtype=BF16)
        got = _gpu_dequantize(w7, s37, bb, 32, 8)
        assert (got.float() == 258.0).all(), (e, got)
        assert torch.equal(_bits_of(got), _bits_of(O.dequantize_stored(w7, s37, bb, 32, 8)))
    # the same tie through 4-bit codes (exact bf16 codes by the 128 + c form)
    w4 = torch.full((1, 4), 0x77777777, dtype=torch.int32)
    s37, bb = torch.tensor([[37.0]], dtype=BF16), torch.tensor([[-(2.0 ** -20)]], dtype=BF16)
    got = _gpu_dequantize(w4, s37, bb, 32, 4)
    assert (got.float() == 258.0).all(), got


def test_dequantize_stack_of_matrices():
    """Leading axes are flattened into rows: [E, N, K] weights of a mixture of
    experts dequantize like one [E * N, K] matrix."""
    w = W.normal((6, 96, 256), 0.02, 5, "bf16")
    c, s, b = O.quantize_affine(w.reshape(-1, 256), 64, 4)
    c, s, b = c.reshape(6, 96, -1), s.reshape(6, 96, -1), b.reshape(6, 96, -1)
    got = _gpu_dequantize(c, s, b, 64, 4)
    assert got.shape == (6, 96, 256)
    ref = O.dequantize_stored(c.reshape(576, -1), s.reshape(576, -1), b.reshape(576, -1), 64, 4)
    assert torch.equal(_bits_of(got.reshape(576, 256)), _bits_of(ref))


def test_dequantize_full_decode_weight():
    """W [14336, 4096] bf16, 4-bit g64 (the decode weight), in full."""
    w = W.decode_weight()
    c, s, b = O.quantize_affine(w, 64, 4)
    got = _gpu_dequantize(c, s, b, 64, 4)
    ref = O.dequantize_stored(c, s, b, 64, 4)
    assert torch.equal(_bits_of(got), _bits_of(ref))


@pytest.mark.parametrize("dt", [BF16, F32])
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_quantizer_one_bit_bit_exact(gs, dt):
    w = W.normal((300, 8 * gs), 0.02 if dt == BF16 else 1.0, 31, "bf16" if dt == BF16 else "f32")
    c0, s0, b0 = O.quantize_affine(w, gs, 1)
    c1, s1, b1 = nvq.nv_quantize_affine(w.cuda(), gs, 1)
    torch.cuda.synchronize()
    assert torch.equal(c0, c1.cpu())
    assert torch.equal(_bits_of(s0), _bits_of(s1.cpu())) and torch.equal(_bits_of(b0), _bits_of(b1.cpu()))


def test_one_bit_round_trip_on_device():
    """Quantize and dequantize on the GPU at 1 bit: every value comes back as
    its group's minimum or maximum (scale = max - min, bias = min), up to the
    rounding of max - min and of scale + bias."""
    w = W.normal((64, 256), 1.0, 41, "f32").cuda()
    c, s, b = nvq.nv_quantize_affine(w, 32, 1)
    wh = nvq.nv_dequantize_affine(c, s, b, 32, 1)
    g = w.reshape(64, 8, 32)
    lo, hi = g.amin(-1, keepdim=True), g.amax(-1, keepdim=True)
    whg = wh.reshape(64, 8, 32)
    # (max - min) + min is max up to the two fp32 roundings
    near = torch.minimum((whg - lo).abs(), (whg - hi).abs())
    assert bool((near <= 2 ** -22 * g.abs().amax()).all())


def test_products_refuse_one_bit():
    x = torch.zeros(1, 64, dtype=BF16, device="cuda")
    c = torch.zeros(16, 2, dtype=torch.int32, device="cuda")
    s = torch.zeros(16, 2, dtype=BF16, device="cuda")
    with pytest.raises(nvq.NvqError):
        nvq.nv_qmm(x, c, s, s, 32, 1, True)
