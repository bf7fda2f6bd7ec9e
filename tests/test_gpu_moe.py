"""The routed SwiGLU mixture-of-experts block over quantized experts
("Docs / Quantization", section "Mixture of experts"), nv_moe_swiglu through
the C ABI, against the oracle's fp64 block. Tolerance: the product tolerance
carried through silu(g) * u (the oracle's a), |y - y_ref| <= 4e-3 a + 1e-5."""
import pytest
import torch

import group_wise_affine_dequant_b200 as nvq
import oracle as O
from group_wise_affine_dequant_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


def _block(E, I, K, T, topk, gs, bits, seed):
    gate = O.quantize_affine(W.normal((E, I, K), 0.02, seed, "bf16"), gs, bits)
    up = O.quantize_affine(W.normal((E, I, K), 0.02, seed + 1, "bf16"), gs, bits)
    down = O.quantize_affine(W.normal((E, K, I), 0.02, seed + 2, "bf16"), gs, bits)
    x = W.normal((T, K), 1.0, seed + 3, "bf16")
    ids = W.expert_ids(T, E, topk, seed + 4)
    g = torch.Generator().manual_seed(seed + 5)
    rw = torch.rand(T, topk, generator=g)
    rw = (rw / rw.sum(1, keepdim=True)).to(torch.float32)
    return x, gate, up, down, ids, rw


def _gpu(x, gate, up, down, ids, rw, gs, bits, ws=None):
    dev = lambda q: tuple(t.cuda() for t in q)  # noqa: E731
    y = nvq.nv_moe_swiglu(x.cuda(), dev(gate), dev(up), dev(down), ids.to(torch.int32).cuda(),
                          rw.cuda(), gs, bits, workspace=ws)
    torch.cuda.synchronize()
    return y.cpu()


@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 64), (2, 128), (4, 32)])
def test_moe_swiglu_small(bits, gs):
    x, gate, up, down, ids, rw = _block(8, 1024, 1024, 24, 2, gs, bits, 80)
    y = _gpu(x, gate, up, down, ids, rw, gs, bits)
    yr, a = O.moe_swiglu(x, gate, up, down, ids, rw, gs, bits)
    assert tuple(y.shape) == (24, 1024)
    P.assert_within(y, yr, a, BF16, f"moe swiglu b{bits} g{gs}")


def test_moe_swiglu_expert_shapes():
    """The mixture-of-experts shapes (64 experts, gate/up [1536, 2048], down
    [2048, 1536], top-4, 4-bit g64) on 32 tokens, every output against the
    oracle."""
    x, gate, up, down, ids, rw = _block(64, 1536, 2048, 32, 4, 64, 4, 81)
    y = _gpu(x, gate, up, down, ids, rw, 64, 4)
    yr, a = O.moe_swiglu(x, gate, up, down, ids, rw, 64, 4)
    P.assert_within(y, yr, a, BF16, "moe swiglu expert shapes")


def test_moe_swiglu_deterministic_scaled_and_flagged():
    x, gate, up, down, ids, rw = _block(6, 512, 512, 20, 3, 64, 4, 82)
    ws = torch.empty(nvq.nv_moe_swiglu_workspace_size(20, 3, 6, 512, 512), dtype=torch.uint8,
                     device="cuda")
    y1 = _gpu(x, gate, up, down, ids, rw, 64, 4, ws)
    y2 = _gpu(x, gate, up, down, ids, rw, 64, 4, ws)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), "run to run"
    assert nvq.nv_gather_qmm_flags(ws) == 0
    y3 = _gpu(x, gate, up, down, ids, 2 * rw, 64, 4, ws)
    assert torch.equal(y3.view(torch.int16), (2 * y1.float()).to(BF16).view(torch.int16))
    # an expert id out of range adds nothing and raises the flag
    bad = ids.clone()
    bad[:, 2] = 6
    yb = _gpu(x, gate, up, down, bad, rw, 64, 4, ws)
    assert nvq.nv_gather_qmm_flags(ws) & nvq.binding.NV_FLAG_EXPERT_OUT_OF_RANGE
    yr, a = O.moe_swiglu(x, gate, up, down, bad, rw, 64, 4)
    P.assert_within(yb, yr, a, BF16, "out-of-range expert ids")
