"""The bench's output checks (plain torch on the timed outputs) against the
oracle, on the CPU: the torch unpacking of codes equals the oracle's
dequantization, and the tolerance ratio passes a correct product and fails a
wrong one."""
import torch

import bench
import oracle as O
from group_wise_affine_dequant_b200 import workloads as W


def test_unpack_equals_the_oracle_dequantization():
    for bits, gs in ((1, 32), (2, 64), (4, 64), (4, 128), (8, 32)):
        w = W.normal((40, 4 * gs), 0.02, bits, "bf16")
        c, s, b = O.quantize_affine(w, gs, bits)
        got = bench.unpack_dequant(c, s, b, gs, bits)
        assert torch.equal(got.double(), O.dequantize(c, s, b, gs, bits)), (bits, gs)
        assert torch.equal(got.to(torch.bfloat16), O.dequantize_stored(c, s, b, gs, bits)), (bits, gs)


def test_worst_ratio_passes_the_oracle_product_and_fails_a_wrong_one():
    w = W.normal((96, 256), 0.02, 1, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    x = W.normal((3, 256), 1.0, 2, "bf16")
    y, _ = O.qmm(x, c, s, b, 64, 4, True)
    wh = bench.unpack_dequant(c, s, b, 64, 4)
    assert bench.worst_ratio(y.to(torch.bfloat16), x, wh) <= 1.0
    bad = y.clone()
    bad[1, 7] += 0.5
    assert bench.worst_ratio(bad.to(torch.bfloat16), x, wh) > 1.0


def test_unpack_fp_equals_the_oracle_dequantization():
    """The bench's torch decode of the floating-point modes (table lookup of
    every code, times the scale) equals the oracle's dequantization."""
    g = torch.Generator().manual_seed(4)
    w = torch.randn(24, 256, generator=g) * (10.0 ** (torch.rand(24, 1, generator=g) * 6 - 4))
    for mode in ("mxfp4", "mxfp8", "nvfp4"):
        c, s = O.quantize_fp(w, mode)
        got = bench.unpack_fp(c, s, mode)
        assert torch.equal(got.to(torch.bfloat16), O.dequantize_fp(c, s, mode)), mode
