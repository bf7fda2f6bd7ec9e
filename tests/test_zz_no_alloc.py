"""nv_gather_qmm_noalloc, the mixture-of-experts product for callers that
cannot allocate device memory (runtimes that own every byte and forbid
cudaMalloc on their hot path, allocator-less plugins, real-time loops).

It is called through the C ABI and must give what nv_gather_qmm (caller-given
workspace) gives, within the product tolerance, on two calls in a row: the
second call reuses the library's fixed scratch array that the first one left
behind. This file is collected last so that a failure here stops a
first-failure run only after every other test has run.
"""
import ctypes as C

import pytest
import torch

import group_wise_affine_dequant_b200 as nvq
import oracle as O
from group_wise_affine_dequant_b200 import binding as B
from group_wise_affine_dequant_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


def _noalloc(x, c, s, b, rhs, lhs, gs, bits, row_exact=False):
    R = rhs.numel()
    E, N = c.shape[0], c.shape[1]
    K = x.shape[-1]
    y = torch.empty(R, N, dtype=x.dtype, device=x.device)
    st = nvq.lib().nv_gather_qmm_noalloc(
        x.data_ptr(), B.NV_BF16, x.numel() // K, K, lhs.data_ptr(), rhs.data_ptr(), R, E, N,
        c.data_ptr(), s.data_ptr(), b.data_ptr(), gs, bits, 1, 0, int(row_exact), y.data_ptr(),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == B.NV_OK, nvq.nv_status_string(st)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("row_exact", [False, True])
def test_noalloc_matches_workspace_entry_point(row_exact):
    E, N, K, tokens, top_k = 16, 384, 512, 96, 4
    w = W.normal((E, N, K), 0.02, 0, "bf16")
    x = W.normal((tokens, K), 1.0, 1, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    lhs, rhs = W.flatten_pairs(W.expert_ids(tokens, E, top_k, 2))
    dx, dc, ds, db = P.to_dev(x, c, s, b)
    dl, dr = lhs.to(torch.int32).cuda(), rhs.to(torch.int32).cuda()
    y_ws = nvq.nv_gather_qmm(dx, dc, ds, db, dr, dl, 64, 4, True, False, row_exact).cpu()
    yr, a = O.gather_qmm(x, c, s, b, lhs, rhs, 64, 4)
    for call in range(2):
        y = _noalloc(dx, dc, ds, db, dr, dl, 64, 4, row_exact).cpu()
        # within the tolerance of the tests, against the workspace entry point's output
        ok = (y.double() - y_ws.double()).abs() <= O.TOL_REL[torch.bfloat16] * a + O.TOL_ABS
        assert bool(ok.all()), f"call {call}"
        # the same kernels on the same routing: the same bits
        assert torch.equal(y.view(torch.int16), y_ws.view(torch.int16)), f"call {call}"
        P.assert_within(y, yr, a, torch.bfloat16, f"noalloc call {call}")


def test_noalloc_at_its_capacity():
    """R = 32768 pairs over E = 256 experts, the largest request the fixed
    array holds: twice in a row, bitwise equal to the workspace entry point."""
    E, N, K, tokens, top_k = 256, 128, 512, 8192, 4
    w = W.normal((E, N, K), 0.02, 7, "bf16")
    c, s, b = P.to_dev(*O.quantize_affine(w, 64, 4))
    x = W.normal((tokens, K), 1.0, 8, "bf16").cuda()
    lhs, rhs = W.flatten_pairs(W.expert_ids(tokens, E, top_k, 9))
    assert rhs.numel() == 32768
    dl, dr = lhs.to(torch.int32).cuda(), rhs.to(torch.int32).cuda()
    y_ws = nvq.nv_gather_qmm(x, c, s, b, dr, dl, 64, 4, True, False, False)
    for call in range(2):
        y = _noalloc(x, c, s, b, dr, dl, 64, 4)
        assert torch.equal(y.view(torch.int16), y_ws.view(torch.int16)), f"call {call}"


def test_noalloc_rejects_requests_beyond_its_capacity():
    L = nvq.lib()
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    for R, E in ((32769, 8), (128, 257)):
        st = L.nv_gather_qmm_noalloc(p, B.NV_BF16, 1, 64, p, p, R, E, 64, p, p, p, 64, 4, 1, 0, 0,
                                     p, None)
        assert st == B.NV_ERR_WORKSPACE
