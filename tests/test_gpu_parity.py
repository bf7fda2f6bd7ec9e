"""The CUDA path against the oracle, element by element, through the C ABI.

Sizes: small cases span several tiles, slices and a ragged tail; the full
workloads (decode, transposed decode, few-row, mixture of experts) are checked
in full where the oracle takes seconds and on sampled outputs otherwise.
Tolerance: |y - y_ref| <= 4e-3 * sum_k |x_k w_k| + 1e-5 for bf16
activations, 1e-5 relative for fp32. Codes, scales and biases: bit-exact.
"""
import pytest
import torch

import group_wise_affine_dequant_b200 as nvq
import oracle as O
from group_wise_affine_dequant_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

QUANTS = [(4, 32), (4, 64), (4, 128), (8, 32), (8, 64), (8, 128), (2, 32), (2, 64), (2, 128)]
BF16, F32 = torch.bfloat16, torch.float32


def _gpu_quantize(w, gs, bits):
    c, s, b = nvq.nv_quantize_affine(w.cuda(), gs, bits)
    torch.cuda.synchronize()
    return c.cpu(), s.cpu(), b.cpu()


def _assert_same_quant(w, gs, bits, what):
    c0, s0, b0 = O.quantize_affine(w, gs, bits)
    c1, s1, b1 = _gpu_quantize(w, gs, bits)
    assert torch.equal(c0, c1), f"{what}: codes differ ({int((c0 != c1).sum())} words)"
    assert torch.equal(s0.view(torch.int16) if s0.dtype == BF16 else s0.view(torch.int32),
                       s1.view(torch.int16) if s1.dtype == BF16 else s1.view(torch.int32)), f"{what}: scales"
    assert torch.equal(b0.view(torch.int16) if b0.dtype == BF16 else b0.view(torch.int32),
                       b1.view(torch.int16) if b1.dtype == BF16 else b1.view(torch.int32)), f"{what}: biases"


# ---------------------------------------------------------------- quantizer
def test_quantizer_tiny_bit_exact():
    w, _ = W.tiny_inputs()
    _assert_same_quant(w, 64, 4, "tiny")


@pytest.mark.parametrize("bits,gs", QUANTS)
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_quantizer_random_bit_exact(bits, gs, dt):
    w = W.normal((300, 1024), 0.02, 11, dt)
    _assert_same_quant(w, gs, bits, f"{dt} b{bits} g{gs}")


def test_quantizer_handbuilt_groups_bit_exact():
    from tests import oracle_pins as pins
    for name, bits, gs, vals, *_ in pins.handbuilt_cases():
        if bits not in (2, 4, 8):  # the library quantizes to 2, 4 and 8 bits
            continue
        w = torch.tensor([pins._cycle(vals, gs), pins._cycle(vals[::-1], gs)], dtype=F32)
        _assert_same_quant(w, gs, bits, name)
        _assert_same_quant(w.to(BF16), gs, bits, name + " bf16")
    for vals in ([0.0, -0.0, 1.0], [-0.0, 0.0, 1.0], [1.0, 0.0, -0.0], [0.0, -0.0, -1.0]):
        w = torch.tensor([pins._cycle(vals, 64)], dtype=F32)
        _assert_same_quant(w, 64, 4, f"signed zeros {vals}")


@pytest.mark.parametrize("bits", [4, 8])
def test_quantizer_decode_weights_bit_exact(bits):
    w = W.decode_weight()
    _assert_same_quant(w, 64, bits, f"decode b{bits}")


def test_quantizer_moe_weights_bit_exact():
    w = W.normal((W.MOE["E"], W.MOE["N"], W.MOE["K"]), 0.02, 0, "bf16")
    _assert_same_quant(w, 64, 4, "moe")


# ---------------------------------------------------------------- products
def _run(x, c, s, b, gs, bits, transpose, row_exact=False):
    y = nvq.nv_qmm(x.cuda(), c.cuda(), s.cuda(), b.cuda(), gs, bits, transpose, row_exact)
    torch.cuda.synchronize()
    return y.cpu()


def _check_product(N, K, M, bits, gs, transpose, dt="bf16", seed=5):
    wshape = (N, K) if transpose else (K, N)
    w = W.normal(wshape, 0.02, seed, dt)
    x = W.normal((M, K), 1.0, seed + 1, dt)
    c, s, b = O.quantize_affine(w, gs, bits)
    y = _run(x, c, s, b, gs, bits, transpose)
    yr, a = O.qmm(x, c, s, b, gs, bits, transpose)
    P.assert_within(y, yr, a, x.dtype, f"N={N} K={K} M={M} b{bits} g{gs} t{transpose} {dt}")
    return x, c, s, b, y


def test_tiny_workload_fp32():
    w, x = W.tiny_inputs()
    c, s, b = O.quantize_affine(w, 64, 4)
    y = _run(x, c, s, b, 64, 4, True)
    yr, a = O.qmm(x, c, s, b, 64, 4, True)
    assert y.shape == (4, 256)
    P.assert_within(y, yr, a, F32, "tiny")


@pytest.mark.parametrize("bits,gs", QUANTS)
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8])
def test_qmm_transpose_small(bits, gs, M):
    # 1000 rows: several CTAs and a ragged last tile; K = 640: a partial last slice
    _check_product(1000, 640, M, bits, gs, True)


@pytest.mark.parametrize("bits,gs", QUANTS)
@pytest.mark.parametrize("M", [1, 2, 4, 7])
def test_qmm_no_transpose_small(bits, gs, M):
    _check_product(640, 1000, M, bits, gs, False)


@pytest.mark.parametrize("bits,gs", QUANTS)
@pytest.mark.parametrize("M", [9, 300])
def test_qmm_no_transpose_tiled(bits, gs, M):
    """Weights stored [K, N] grouped along N with more than 8 rows: the tiled
    tensor-core kernel with its transposing dequantizer (ragged rows, several
    column tiles; N is a multiple of the group size but not of 256)."""
    _check_product(704 if gs < 128 else 896, 1024, M, bits, gs, False)


@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 64), (2, 128)])
def test_qmm_no_transpose_tiled_2048_rows(bits, gs):
    """x [2048, 4096] . W with W stored [4096, 14336] (grouped along N):
    sampled outputs and whole rows against the oracle."""
    w = W.normal((4096, 14336), 0.02, 0, "bf16")
    x = W.activations(2048, 4096)
    c, s, b = O.quantize_affine(w, gs, bits)
    y = _run(x, c, s, b, gs, bits, False)
    g = torch.Generator().manual_seed(bits * 10 + gs)
    mi = torch.randint(0, 2048, (2000,), generator=g)
    ni = torch.randint(0, 14336, (2000,), generator=g)
    yr, a = O.qmm_sampled(x, c, s, b, gs, bits, False, mi, ni)
    P.assert_within(y[mi, ni], yr, a, BF16, f"transpose=0 2048 rows b{bits} g{gs} sampled")
    for m in (0, 2047):
        yr, a = O.qmm(x[m:m + 1], c, s, b, gs, bits, False)
        P.assert_within(y[m:m + 1], yr, a, BF16, f"transpose=0 2048 rows b{bits} g{gs} row {m}")


@pytest.mark.parametrize("transpose", [True, False])
@pytest.mark.parametrize("M", [1, 3, 8, 20])
def test_qmm_fp32_small(transpose, M):
    _check_product(256, 384, M, 4, 64, transpose, dt="f32")


@pytest.mark.parametrize("bits,gs", QUANTS)
@pytest.mark.parametrize("transpose", [True, False])
def test_integer_products_exact(bits, gs, transpose):
    """Scale 1, bias 0, integer x in [-2, 2]: every product is an exact integer
    (|y| <= 256 so bf16 holds it), so the GPU must equal the oracle exactly."""
    gen = torch.Generator().manual_seed(bits * 1000 + gs)
    N, K, M = 256, 256, 4
    wi = P.integer_weights(N, K, gs, bits, gen) if transpose else P.integer_weights(K, N, gs, bits, gen)
    hi = 2 ** bits - 1
    xi = torch.randint(-2, 3, (M, K), generator=gen)
    # keep |y| <= 256 for bf16: zero x beyond the first 256 // (2 * hi) columns
    keep = max(1, 256 // (2 * hi))
    xi[:, keep:] = 0
    for dt in (F32, BF16):
        c, s, b = O.quantize_affine(wi.to(dt), gs, bits)
        assert (s == 1).all() and (b == 0).all()
        y = _run(xi.to(dt), c, s, b, gs, bits, transpose)
        yr, _ = O.qmm(xi.to(dt), c, s, b, gs, bits, transpose)
        assert torch.equal(y.to(torch.float64), yr), (dt, bits, gs, transpose)


@pytest.mark.parametrize("bits,gs", QUANTS)
@pytest.mark.parametrize("transpose", [True, False])
def test_row_exact_bit_identity(bits, gs, transpose):
    """Each row of an M-row product equals its one-row product bit for bit
    (row_exact on and off give the same bits here: the few-row kernels keep
    every row's arithmetic independent of the others)."""
    N, K = (1000, 640) if transpose else (640, 1000)
    w = W.normal((N, K) if transpose else (K, N), 0.02, 3, "bf16")
    c, s, b = O.quantize_affine(w, gs, bits)
    dc, ds, db = P.to_dev(c, s, b)
    x = W.normal((8, K), 1.0, 4, "bf16").cuda()
    singles = [nvq.nv_qmm(x[m:m + 1], dc, ds, db, gs, bits, transpose, True) for m in range(8)]
    for M in (2, 3, 4, 5, 8):
        for row_exact in (True, False):
            yM = nvq.nv_qmm(x[:M], dc, ds, db, gs, bits, transpose, row_exact)
            for m in range(M):
                assert torch.equal(yM[m].view(torch.int16), singles[m][0].view(torch.int16)), \
                    (bits, gs, transpose, M, m, row_exact)


def test_deterministic_and_scaling_invariant():
    w = W.normal((1000, 1024), 0.02, 8, "bf16")
    c, s, b = P.to_dev(*O.quantize_affine(w, 64, 4))
    x = W.normal((3, 1024), 1.0, 9, "bf16").cuda()
    for transpose in (True,):
        y1 = nvq.nv_qmm(x, c, s, b, 64, 4, transpose)
        y2 = nvq.nv_qmm(x, c, s, b, 64, 4, transpose)
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
        y8 = nvq.nv_qmm(x * 8, c, s, b, 64, 4, transpose)
        assert torch.equal((y1.float() * 8).to(BF16).view(torch.int16), y8.view(torch.int16))


# ------------------------------------------------------- full-size workloads
@pytest.fixture(scope="module")
def decode_quant():
    w = W.decode_weight()
    return {bits: O.quantize_affine(w, 64, bits) for bits in (4, 8)}


@pytest.mark.parametrize("bits", [4, 8])
def test_decode_full(decode_quant, bits):
    c, s, b = decode_quant[bits]
    x = W.activations(1, 4096)
    y = _run(x, c, s, b, 64, bits, True)
    yr, a = O.qmm(x, c, s, b, 64, bits, True)
    P.assert_within(y, yr, a, BF16, f"decode b{bits}")


@pytest.mark.parametrize("bits", [4, 8])
def test_decode_transposed_full(bits):
    """W [4096, 14336] stored [K, N], grouped along N: y = x . w, [1, 14336]."""
    w = W.normal((4096, 14336), 0.02, 0, "bf16")
    c, s, b = O.quantize_affine(w, 64, bits)
    x = W.activations(1, 4096)
    y = _run(x, c, s, b, 64, bits, False)
    yr, a = O.qmm(x, c, s, b, 64, bits, False)
    P.assert_within(y, yr, a, BF16, f"decode transposed b{bits}")


def test_decode_long_k():
    """The other reading of the transposed case: x [1, 14336] times W [4096, 14336]^T."""
    w = W.normal((4096, 14336), 0.02, 0, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    x = W.activations(1, 14336)
    y = _run(x, c, s, b, 64, 4, True)
    yr, a = O.qmm(x, c, s, b, 64, 4, True)
    P.assert_within(y, yr, a, BF16, "x[1,14336] W[4096,14336]^T")


@pytest.mark.parametrize("N", [4096, 14336])
def test_few_row_full(decode_quant, N):
    if N == 14336:
        c, s, b = decode_quant[4]
    else:
        c, s, b = O.quantize_affine(W.decode_weight(N=4096), 64, 4)
    dc, ds, db = P.to_dev(c, s, b)
    x = W.activations(8, 4096)
    ones = [nvq.nv_qmm(x[m:m + 1].cuda(), dc, ds, db, 64, 4, True) for m in range(8)]
    for M in (2, 4, 8):
        for row_exact in (False, True):
            y = nvq.nv_qmm(x[:M].cuda(), dc, ds, db, 64, 4, True, row_exact).cpu()
            yr, a = O.qmm(x[:M], c, s, b, 64, 4, True)
            P.assert_within(y, yr, a, BF16, f"few-row N={N} M={M}")
            for m in range(M):
                assert torch.equal(y[m].view(torch.int16), ones[m][0].cpu().view(torch.int16))


# -------------------------------------------------------------------- gather
def _gather(x, c, s, b, rhs, lhs, gs, bits, transpose=True, sorted_=False, row_exact=False):
    ws = torch.empty(nvq.nv_gather_qmm_workspace_size(rhs.numel(), c.shape[0]), dtype=torch.uint8,
                     device="cuda")
    y = nvq.nv_gather_qmm(x.cuda(), c.cuda(), s.cuda(), b.cuda(),
                          rhs.to(torch.int32).cuda(),
                          None if lhs is None else lhs.to(torch.int32).cuda(), gs, bits, transpose,
                          sorted_, row_exact, workspace=ws)
    flags = nvq.nv_gather_qmm_flags(ws)
    return y.cpu(), flags


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_gather_page_example(dt):
    w = W.normal((8, 128, 256), 1.0, 0, dt)
    x = W.normal((4, 1, 256), 1.0, 1, dt)
    c, s, b = O.quantize_affine(w, 64, 4)
    ids = torch.tensor([0, 0, 3, 5])
    y, flags = _gather(x, c, s, b, ids, None, 64, 4, sorted_=True)
    assert flags == 0 and tuple(y.shape) == (4, 128)
    yr, a = O.gather_qmm(x, c, s, b, None, ids, 64, 4)
    P.assert_within(y, yr, a, x.dtype, "page example")


@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 32), (2, 128), (4, 128), (4, 32), (8, 128)])
@pytest.mark.parametrize("row_exact", [False, True])
def test_gather_ragged(bits, gs, row_exact):
    """37 pairs over 5 experts (one empty, one with 17 pairs), random token map:
    both routes within tolerance of the oracle; under row_exact every pair
    equals its one-row product with its expert's weights, bit for bit."""
    g = torch.Generator().manual_seed(41)
    E, N, K = 5, 200, 512
    w = W.normal((E, N, K), 0.02, 2, "bf16")
    x = W.normal((23, K), 1.0, 3, "bf16")
    c, s, b = O.quantize_affine(w, gs, bits)
    rhs = torch.tensor([0] * 9 + [2] * 17 + [3] * 4 + [4] * 7)[torch.randperm(37, generator=g)]
    lhs = torch.randint(0, 23, (37,), generator=g)
    y, flags = _gather(x, c, s, b, rhs, lhs, gs, bits, row_exact=row_exact)
    assert flags == 0
    yr, a = O.gather_qmm(x, c, s, b, lhs, rhs, gs, bits)
    P.assert_within(y, yr, a, BF16, f"ragged gather row_exact={row_exact}")
    if row_exact:
        for r in range(37):
            e, t = int(rhs[r]), int(lhs[r])
            one = _run(x[t:t + 1], c[e], s[e], b[e], gs, bits, True)
            assert torch.equal(one[0].view(torch.int16), y[r].view(torch.int16)), r


def test_gather_many_pairs_per_expert():
    """An expert with more pairs than one tensor-core pass holds (600 > 256)
    and an expert whose weight rows end mid-tile (N = 300)."""
    E, N, K = 3, 300, 256
    w = W.normal((E, N, K), 0.02, 4, "bf16")
    x = W.normal((700, K), 1.0, 5, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    g = torch.Generator().manual_seed(3)
    rhs = torch.cat([torch.full((600,), 1), torch.full((40,), 2), torch.full((5,), 0)])
    rhs = rhs[torch.randperm(645, generator=g)]
    lhs = torch.randint(0, 700, (645,), generator=g)
    y, flags = _gather(x, c, s, b, rhs, lhs, 64, 4)
    assert flags == 0
    yr, a = O.gather_qmm(x, c, s, b, lhs, rhs, 64, 4)
    P.assert_within(y, yr, a, BF16, "many pairs")


def test_gather_back_to_back_share_a_workspace():
    """Eight calls queued on one stream without synchronising, each with its
    own routing and output but one workspace: every call's routing kernel must
    wait for the previous grouped kernel (which still reads the tables) and
    every grouped kernel for its own routing (a programmatic dependent
    launch). Each output is checked against the oracle afterwards."""
    E, N, K, T = 6, 256, 512, 40
    w = W.normal((E, N, K), 0.02, 6, "bf16")
    x = W.normal((T, K), 1.0, 7, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    dc, ds, db, dx = c.cuda(), s.cuda(), b.cuda(), x.cuda()
    g = torch.Generator().manual_seed(11)
    R = 96
    ws = torch.empty(nvq.nv_gather_qmm_workspace_size(R, E), dtype=torch.uint8, device="cuda")
    calls = []
    for i in range(8):
        rhs = torch.randint(0, E if i % 2 else 2, (R,), generator=g)  # skewed, then spread
        lhs = torch.randint(0, T, (R,), generator=g)
        y = nvq.nv_gather_qmm(dx, dc, ds, db, rhs.to(torch.int32).cuda(), lhs.to(torch.int32).cuda(),
                              64, 4, True, False, False, workspace=ws)
        calls.append((rhs, lhs, y))
    torch.cuda.synchronize()
    for i, (rhs, lhs, y) in enumerate(calls):
        yr, a = O.gather_qmm(x, c, s, b, lhs, rhs, 64, 4)
        P.assert_within(y.cpu(), yr, a, BF16, f"back-to-back call {i}")


def test_gather_flags_and_invalid_ids():
    E, N, K = 4, 64, 128
    w = W.normal((E, N, K), 0.02, 2, "bf16")
    x = W.normal((6, K), 1.0, 3, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    rhs = torch.tensor([0, 1, 9, 2, 1])
    lhs = torch.tensor([0, 1, 2, 7, 5])
    y, flags = _gather(x, c, s, b, rhs, lhs, 64, 4, sorted_=True)
    assert flags & nvq.binding.NV_FLAG_EXPERT_OUT_OF_RANGE
    assert flags & nvq.binding.NV_FLAG_TOKEN_OUT_OF_RANGE
    assert flags & nvq.binding.NV_FLAG_NOT_SORTED
    assert (y[2] == 0).all() and (y[3] == 0).all()
    ok = torch.tensor([0, 1, 4])
    yr, a = O.gather_qmm(x, c, s, b, lhs[ok], rhs[ok], 64, 4)
    P.assert_within(y[ok], yr, a, BF16, "valid rows")
    # a sorted promise that holds raises no flag
    y2, flags2 = _gather(x, c, s, b, torch.tensor([0, 1, 1, 3]), torch.tensor([5, 4, 3, 2]), 64, 4,
                         sorted_=True)
    assert flags2 == 0


@pytest.fixture(scope="module")
def moe_case():
    m = W.MOE
    w = W.normal((m["E"], m["N"], m["K"]), 0.02, 0, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    x = W.normal((m["tokens"], 1, m["K"]), 1.0, 1, "bf16")
    ids = W.expert_ids(m["tokens"], m["E"], m["top_k"], 2)
    lhs, rhs = W.flatten_pairs(ids)
    return x, c, s, b, lhs, rhs


def test_moe_gather_sorted_and_unsorted(moe_case):
    x, c, s, b, lhs, rhs = moe_case
    lhs_s, rhs_s, order = W.stable_sort_pairs(lhs, rhs)
    y_u, f_u = _gather(x, c, s, b, rhs, lhs, 64, 4, sorted_=False)
    y_s, f_s = _gather(x, c, s, b, rhs_s, lhs_s, 64, 4, sorted_=True)
    assert f_u == 0 and f_s == 0
    assert tuple(y_u.shape) == (2048, 1536)
    # the same pair gives the same bits in either order
    assert torch.equal(y_s.view(torch.int16), y_u[order].view(torch.int16))
    # sampled outputs against the oracle
    g = torch.Generator().manual_seed(0)
    r_idx = torch.randint(0, 2048, (4096,), generator=g)
    n_idx = torch.randint(0, 1536, (4096,), generator=g)
    yr, a = O.gather_qmm_sampled(x, c, s, b, lhs, rhs, 64, 4, True, r_idx, n_idx)
    P.assert_within(y_u[r_idx, n_idx], yr, a, BF16, "moe sampled")
    # the row-exact route on the same workload
    y_x, f_x = _gather(x, c, s, b, rhs, lhs, 64, 4, row_exact=True)
    assert f_x == 0
    P.assert_within(y_x[r_idx, n_idx], yr, a, BF16, "moe sampled, row_exact")
    # whole rows for a few pairs
    rows = torch.tensor([0, 1, 777, 2047])
    yr, a = O.gather_qmm(x, c, s, b, lhs[rows], rhs[rows], 64, 4)
    P.assert_within(y_u[rows], yr, a, BF16, "moe rows")


# ------------------------------------------------------------------- prefill
@pytest.mark.parametrize("bits,gs", [(4, 64), (4, 32), (4, 128), (2, 64), (8, 64), (8, 32), (2, 128)])
@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (200, 480, 640), (9, 100, 128), (300, 1000, 512)])
def test_prefill_small(bits, gs, M, N, K):
    """Tensor-core tiles: ragged M (rows beyond a 128 tile), ragged N (beyond a
    column tile), several k-steps, every width and group size."""
    if K % gs:
        pytest.skip("K must be a multiple of the group size")
    _check_product(N, K, M, bits, gs, True)


def test_prefill_deterministic_and_integer_exact():
    w = W.normal((512, 512), 0.02, 8, "bf16")
    c, s, b = P.to_dev(*O.quantize_affine(w, 64, 4))
    x = W.normal((300, 512), 1.0, 9, "bf16").cuda()
    y1 = nvq.nv_qmm(x, c, s, b, 64, 4, True)
    y2 = nvq.nv_qmm(x, c, s, b, 64, 4, True)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    gen = torch.Generator().manual_seed(77)
    wi = P.integer_weights(256, 512, 64, 4, gen)
    xi = torch.randint(-2, 3, (200, 512), generator=gen)
    xi[:, 8:] = 0  # |y| <= 8 * 2 * 15 = 240: exact in bf16
    ci, si, bi = O.quantize_affine(wi.to(BF16), 64, 4)
    y = _run(xi.to(BF16), ci, si, bi, 64, 4, True)
    yr, _ = O.qmm(xi.to(BF16), ci, si, bi, 64, 4, True)
    assert torch.equal(y.to(torch.float64), yr)


@pytest.fixture(scope="module")
def prefill_inputs():
    w = W.normal((14336, 4096), 0.02, 0, "bf16")
    x = W.activations(2048, 4096)
    return w, x


@pytest.mark.parametrize("bits,gs", W.PREFILL_VARIANTS)
def test_prefill_full(prefill_inputs, bits, gs):
    """x [2048, 4096] . W[14336, 4096]^T at the five quantizations: sampled
    outputs and whole rows against the oracle."""
    w, x = prefill_inputs
    c, s, b = O.quantize_affine(w, gs, bits)
    y = _run(x, c, s, b, gs, bits, True)
    assert tuple(y.shape) == (2048, 14336)
    g = torch.Generator().manual_seed(bits * 100 + gs)
    mi = torch.randint(0, 2048, (3000,), generator=g)
    ni = torch.randint(0, 14336, (3000,), generator=g)
    yr, a = O.qmm_sampled(x, c, s, b, gs, bits, True, mi, ni)
    P.assert_within(y[mi, ni], yr, a, BF16, f"prefill b{bits} g{gs} sampled")
    for m in (0, 1337, 2047):
        yr, a = O.qmm(x[m:m + 1], c, s, b, gs, bits, True)
        P.assert_within(y[m:m + 1], yr, a, BF16, f"prefill b{bits} g{gs} row {m}")


def test_pipelines_never_timed_out():
    """No wait inside the TMA / tensor-core pipelines gave up during the tests
    above (the sticky error word is 0)."""
    assert nvq.nv_pipeline_error() == 0


def test_bounded_wait_gives_up_reports_and_leaves_the_next_call_correct():
    """A wait on a barrier that nothing completes gives up after its limit
    (here 50 ms, measured by CUDA events around it), records its code, and
    the kernel returns: the context stays usable and the next product is
    correct and reports no error."""
    import time
    assert nvq.nv_pipeline_error() == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    e0.record()
    nvq.nv_pipeline_selftest(50000)
    e1.record()
    assert nvq.nv_pipeline_error() == 0x5E
    assert time.time() - t0 < 10.0
    assert e0.elapsed_time(e1) >= 49.0, e0.elapsed_time(e1)
    assert nvq.nv_pipeline_error() == 0  # read and cleared
    nvq.nv_pipeline_selftest(1)
    assert nvq.nv_pipeline_error() == 0x5E
    # the next products run normally (the recorded code does not cut them short)
    nvq.nv_pipeline_selftest(1000)
    _check_product(1000, 640, 1, 4, 64, True)
    _check_product(300, 512, 40, 4, 64, True)
    assert nvq.nv_pipeline_error() == 0x5E  # the self-test's code, nothing else
    assert nvq.nv_pipeline_error() == 0
