"""Edge cases of the method on every product route, against the oracle.

Routes (a pure function of the call's shape, dtype and flags):
  * nv_qmm transpose=1, M <= 8, bf16   -> matrix-vector kernel (tensor cores, exact codes)
  * nv_qmm transpose=0, M <= 8, bf16   -> transposed matrix-vector kernel
  * nv_qmm transpose=1, M > 8, bf16    -> tcgen05 tiled kernel
  * nv_qmm transpose=0, M > 8, bf16    -> tcgen05 tiled kernel (transposing dequantizer)
  * nv_qmm fp32, either layout         -> plain per-output kernel
  * nv_gather_qmm transpose=1, bf16    -> grouped tensor-core kernel (row_exact: per-row kernel)
  * nv_gather_qmm transpose=0          -> plain per-output kernel

Cases ("Docs / Quantization", section "Affine": w ~ scale * code + bias for
any group, any activations):
  * constant groups (scale 0, every code 0, w_hat = bias) mixed with normal ones;
  * activation rows whose entries span many binades: large values (2^60, 2^110,
    near the bf16 maximum) where the dequantized weight is exactly 0, so that
    the result rests on the O(1) entries beside them;
  * rows of tiny activations (near the smallest normal bf16), and all-zero rows;
  * exact power-of-two scalings of the activations by 2^-100 .. 2^120, which
    must scale every output by the same power of two, bit for bit.
"""
import pytest
import torch

import group_wise_affine_dequant_b200 as nvq
import oracle as O
from group_wise_affine_dequant_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

BF16, F32 = torch.bfloat16, torch.float32
QUANTS = [(4, 64), (8, 32), (2, 128), (4, 128), (8, 64), (2, 32)]

# (name, transpose, M, dtype): one per nv_qmm route
QMM_ROUTES = [
    ("matvec", True, 3, BF16),
    ("matvec_m1", True, 1, BF16),
    ("matvec_t0", False, 3, BF16),
    ("matvec_t0_m1", False, 1, BF16),
    ("tiled", True, 40, BF16),
    ("tiled_t0", False, 20, BF16),
    ("simt_fp32_t1", True, 5, F32),
    ("simt_fp32_t0", False, 5, F32),
]


def _weights(rows, cols, gs, dtype, seed, const_frac=0.3, nonneg=False):
    """N(0, 0.02) weights [rows, cols] grouped along cols; a share of the
    (row, group) blocks set to one constant each (0, negative or positive)."""
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(rows, cols, generator=g) * 0.02
    if nonneg:
        w = w.abs()
    blocks = w.view(rows, cols // gs, gs)
    pick = torch.rand(rows, cols // gs, generator=g) < const_frac
    vals = torch.randn(rows, cols // gs, generator=g) * 0.03
    vals[torch.rand(rows, cols // gs, generator=g) < 0.2] = 0.0
    if nonneg:
        vals = vals.abs()
    blocks[pick] = vals[pick].unsqueeze(-1).expand(-1, gs).clone()
    return w.to(dtype)


def _run(x, c, s, b, gs, bits, t):
    y = nvq.nv_qmm(x.cuda(), c.cuda(), s.cuda(), b.cuda(), gs, bits, t)
    torch.cuda.synchronize()
    return y.cpu()


def _shape(t, M, gs):
    N, K = 264 if t else 384, 1024
    return N, K


@pytest.mark.parametrize("bits,gs", QUANTS)
@pytest.mark.parametrize("name,t,M,dt", QMM_ROUTES)
def test_constant_groups(name, t, M, dt, bits, gs):
    N, K = _shape(t, M, gs)
    w = _weights(N, K, gs, dt, 10 + bits) if t else _weights(K, N, gs, dt, 10 + bits)
    c, s, b = O.quantize_affine(w, gs, bits)
    assert (s == 0).any() and (s != 0).any(), "the case must mix constant and normal groups"
    x = W.normal((M, K), 1.0, 3, "bf16" if dt == BF16 else "f32")
    y = _run(x, c, s, b, gs, bits, t)
    yr, a = O.qmm(x, c, s, b, gs, bits, t)
    P.assert_within(y, yr, a, dt, f"{name} constant groups b{bits} g{gs}")


def _wide_case(t, M, gs, dt, big):
    """Nonnegative weights with the positions S (every 64th k) zeroed: for
    transpose=1 columns of [N, K] (each group's minimum is 0 there, so bias 0,
    code 0, w_hat exactly 0); for transpose=0 whole rows of [K, N] (constant
    groups of zeros). Activations: +-big at S, N(0, 1) elsewhere (row 0), a
    row of zeros, a row of values near the smallest normal bf16 (2^-126)."""
    N, K = _shape(t, M, gs)
    S = torch.arange(0, K, 64)
    if t:
        w = _weights(N, K, gs, F32, 20, const_frac=0.0, nonneg=True)
        w[:, S] = 0.0
    else:
        w = _weights(K, N, gs, F32, 20, const_frac=0.0, nonneg=True)
        w[S, :] = 0.0
    w = w.to(dt)
    g = torch.Generator().manual_seed(21)
    x = torch.randn(M, K, generator=g)
    sign = torch.where(torch.rand(len(S), generator=g) < 0.5, -1.0, 1.0)
    x[:, S] = big * sign
    if M > 1:
        x[1] = 0.0
    if M > 2:
        x[2] = torch.randn(K, generator=g) * 2.0 ** -126
    return w, x.to(dt)


@pytest.mark.parametrize("big", [2.0 ** 60, 2.0 ** 110, 1.5 * 2.0 ** 127])
@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 64), (2, 64), (4, 32)])
@pytest.mark.parametrize("name,t,M,dt", QMM_ROUTES)
def test_wide_activation_ranges(name, t, M, dt, bits, gs, big):
    if dt == F32 and big > 2.0 ** 100:
        big = 2.0 ** 100  # fp32 inputs: keep sum |x| finite in the fp64 reference too
    w, x = _wide_case(t, M, gs, dt, big)
    c, s, b = O.quantize_affine(w, gs, bits)
    wh = O.dequantize(c, s, b, gs, bits)
    S = torch.arange(0, 1024, 64)
    assert ((wh[:, S] if t else wh[S, :]) == 0).all(), "weights under the large values are 0"
    y = _run(x, c, s, b, gs, bits, t)
    yr, a = O.qmm(x, c, s, b, gs, bits, t)
    assert torch.isfinite(y).all(), f"{name}: non-finite output"
    assert (yr[0].abs() > 1e-3).sum() > 0.5 * yr.shape[1], "row 0 rests on its O(1) entries"
    P.assert_within(y, yr, a, dt, f"{name} wide range big={big} b{bits} g{gs}")
    if M > 1:
        assert (y[1] == 0).all(), f"{name}: an all-zero row gives zeros"


@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 64), (2, 128)])
@pytest.mark.parametrize("name,t,M,dt", [r for r in QMM_ROUTES if r[3] == BF16])
def test_power_of_two_scalings_are_exact(name, t, M, dt, bits, gs):
    """y(2^j x) == 2^j y(x) bit for bit from 2^-100 to 2^120: no step of any
    route rounds, flushes or overflows differently at other magnitudes."""
    N, K = _shape(t, M, gs)
    w = W.normal((N, K) if t else (K, N), 0.02, 30, "bf16")
    c, s, b = P.to_dev(*O.quantize_affine(w, gs, bits))
    x = W.normal((M, K), 1.0, 31, "bf16").cuda()
    y0 = nvq.nv_qmm(x, c, s, b, gs, bits, t)
    for j in (-100, -40, 40, 100, 120):
        yj = nvq.nv_qmm(x * 2.0 ** j, c, s, b, gs, bits, t)
        want = (y0.float() * 2.0 ** j).to(BF16)
        assert torch.equal(yj.view(torch.int16), want.view(torch.int16)), (name, j)


# ----------------------------------------------------------------- gather routes
def _gather(x, c, s, b, rhs, lhs, gs, bits, t, row_exact=False):
    y = nvq.nv_gather_qmm(x.cuda(), c.cuda(), s.cuda(), b.cuda(), rhs.to(torch.int32).cuda(),
                          lhs.to(torch.int32).cuda(), gs, bits, t, False, row_exact)
    torch.cuda.synchronize()
    return y.cpu()


GATHER_ROUTES = [("grouped", True, False, BF16), ("per_row", True, True, BF16),
                 ("grouped_t0_bf16", False, False, BF16), ("simt_t0_fp32", False, False, F32),
                 ("simt_t1_fp32", True, False, F32)]


@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 32), (2, 128)])
@pytest.mark.parametrize("name,t,rx,dt", GATHER_ROUTES)
def test_gather_constant_groups_and_wide_rows(name, t, rx, dt, bits, gs):
    """Constant groups in every expert, and token rows that hold large values
    (2^60) where all experts' weights are exactly 0 next to O(1) values."""
    E, N, K, T = 4, 256, 1024, 12
    S = torch.arange(0, K, 64)
    ws = []
    for e in range(E):
        if t:
            we = _weights(N, K, gs, F32, 40 + e, const_frac=0.25, nonneg=True)
            we[:, S] = 0.0
        else:
            we = _weights(K, N, gs, F32, 40 + e, const_frac=0.25, nonneg=True)
            we[S, :] = 0.0
        ws.append(we)
    w = torch.stack(ws).to(dt)
    c, s, b = O.quantize_affine(w, gs, bits)
    assert (s == 0).any()
    g = torch.Generator().manual_seed(42)
    x = torch.randn(T, K, generator=g)
    x[: T // 2, S] = 2.0 ** 60
    x[T - 1] = 0.0
    x = x.to(dt)
    R = 40
    rhs = torch.randint(0, E, (R,), generator=g)
    lhs = torch.randint(0, T, (R,), generator=g)
    y = _gather(x, c, s, b, rhs, lhs, gs, bits, t, rx)
    yr, a = O.gather_qmm(x, c, s, b, lhs, rhs, gs, bits, t)
    P.assert_within(y, yr, a, dt, f"gather {name} b{bits} g{gs}")


@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 128), (2, 32)])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_gather_transpose0(bits, gs, dt):
    """Experts stored [E, K, N] grouped along N (transpose = 0): ragged experts,
    a token map with repeats, against the oracle."""
    E, K, N, T = 5, 512, 384, 30
    w = W.normal((E, K, N), 0.02, 50, dt)
    x = W.normal((T, K), 1.0, 51, dt)
    c, s, b = O.quantize_affine(w, gs, bits)
    g = torch.Generator().manual_seed(52)
    rhs = torch.tensor([0] * 3 + [2] * 19 + [3] * 6 + [4] * 9)[torch.randperm(37, generator=g)]
    lhs = torch.randint(0, T, (37,), generator=g)
    y = _gather(x, c, s, b, rhs, lhs, gs, bits, False)
    yr, a = O.gather_qmm(x, c, s, b, lhs, rhs, gs, bits, False)
    P.assert_within(y, yr, a, x.dtype, f"gather transpose=0 b{bits} g{gs} {dt}")


def test_gather_with_more_than_2_32_activation_elements():
    """x with x_rows * K > 2^32 elements (8.6 GB of bf16): the grouped kernel's
    32-bit offsets into x count 16-byte units, so rows past element 2^32 are
    read correctly. Only the rows the pairs use hold data (the rest is zero)."""
    K = 4096
    x_rows = (1 << 32) // K + 64
    x = torch.zeros(x_rows, K, dtype=BF16, device="cuda")
    E, N = 3, 256
    w = W.normal((E, N, K), 0.02, 60, "bf16")
    c, s, b = O.quantize_affine(w, 64, 4)
    used = torch.tensor([0, 5, x_rows - 64, x_rows - 3, x_rows - 1, (1 << 20) + 7])
    xs = W.normal((len(used), K), 1.0, 61, "bf16")
    x[used.cuda()] = xs.cuda()
    g = torch.Generator().manual_seed(62)
    R = 48
    pick = torch.randint(0, len(used), (R,), generator=g)
    rhs = torch.randint(0, E, (R,), generator=g)
    y = nvq.nv_gather_qmm(x, c.cuda(), s.cuda(), b.cuda(), rhs.to(torch.int32).cuda(),
                          used[pick].to(torch.int32).cuda(), 64, 4, True, False, False).cpu()
    del x
    torch.cuda.empty_cache()
    yr, a = O.gather_qmm(xs, c, s, b, pick, rhs, 64, 4)
    P.assert_within(y, yr, a, BF16, "gather beyond 2^32 elements of x")


def _cancelling_case(t, M, bits, gs, big):
    """Integer weights in [-(2^bits - 1), 0] with both ends in every group, so
    scale 1 and bias -(2^bits - 1): code 2^bits - 1 dequantizes to exactly 0
    while scale * code and bias are each large. Activations +-big where the
    weight is 0, N(0, 1) elsewhere. A route that sums scale * code * x and
    bias * x separately cancels 2^60-sized terms and loses the rest."""
    N, K = _shape(t, M, gs)
    hi = 2 ** bits - 1
    g = torch.Generator().manual_seed(90 + bits)
    S = torch.arange(3, K, 64)  # never a group's first column
    if t:  # W [N, K] grouped along K: column k in S is 0 (the groups' maximum)
        w = -torch.randint(0, hi + 1, (N, K), generator=g).to(torch.float32)
        w[:, ::gs] = -hi
        w[:, 1::gs] = 0.0
        w[:, S] = 0.0
    else:  # W [K, N] grouped along N: rows k in S are 0 except one -max per group
        w = -torch.randint(0, hi + 1, (K, N), generator=g).to(torch.float32)
        w[:, ::gs] = -hi
        w[:, 1::gs] = 0.0
        w[S, :] = 0.0
        w[S.unsqueeze(1), torch.arange(0, N, gs).unsqueeze(0)] = -hi
    x = torch.randn(M, K, generator=g)
    x[:, S] = big * torch.where(torch.rand(len(S), generator=g) < 0.5, -1.0, 1.0)
    return w, x


@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 64), (2, 32), (4, 128)])
@pytest.mark.parametrize("name,t,M,dt", [r for r in QMM_ROUTES if r[3] == BF16])
def test_zero_weights_with_nonzero_bias_under_huge_activations(name, t, M, dt, bits, gs):
    w, x = _cancelling_case(t, M, bits, gs, 2.0 ** 60)
    w, x = w.to(dt), x.to(dt)
    c, s, b = O.quantize_affine(w, gs, bits)
    assert (s.float() == 1).all() and (b.float() == -(2 ** bits - 1)).all()
    y = _run(x, c, s, b, gs, bits, t)
    yr, a = O.qmm(x, c, s, b, gs, bits, t)
    assert torch.isfinite(y).all(), name
    P.assert_within(y, yr, a, dt, f"{name} cancelling bias b{bits} g{gs}")


def _wide_magnitude_weights(rows, cols, gs, dtype, seed):
    """Rows of N(0, 1) weights scaled by 10^u, u uniform in [-5, 2], plus a
    share of constant groups: group scales from ~1e-7 to ~1e1, on both sides
    of every power-of-two threshold a kernel might special-case."""
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(rows, cols, generator=g) * (10.0 ** (torch.rand(rows, 1, generator=g) * 7 - 5))
    blocks = w.view(rows, cols // gs, gs)
    pick = torch.rand(rows, cols // gs, generator=g) < 0.1
    blocks[pick] = blocks[pick][:, :1].expand(-1, gs).clone()
    return w.to(dtype)


@pytest.mark.parametrize("bits,gs", QUANTS)
@pytest.mark.parametrize("name,t,M,dt", QMM_ROUTES)
def test_unit_activations_read_out_the_weights(name, t, M, dt, bits, gs):
    """x rows that are unit vectors e_k: every output is one exact product
    1 * w_hat plus exact zeros, so y[m, n] must equal the dequantized weight
    (scale * code + bias rounded once to the scales' type) bit for bit, for
    groups of every magnitude."""
    N, K = _shape(t, M, gs)
    w = _wide_magnitude_weights(N, K, gs, dt, 50 + bits) if t else \
        _wide_magnitude_weights(K, N, gs, dt, 50 + bits)
    c, s, b = O.quantize_affine(w, gs, bits)
    assert (s.float() < 2.0 ** -5).any() and (s.float() >= 2.0 ** -5).any()
    wh = O.dequantize_stored(c, s, b, gs, bits)          # [N, K] or [K, N]
    ks = torch.randperm(K, generator=torch.Generator().manual_seed(bits + gs))[:M]
    x = torch.zeros(M, K, dtype=dt)
    x[torch.arange(M), ks] = 1.0
    y = _run(x, c, s, b, gs, bits, t)
    want = wh[:, ks].t() if t else wh[ks, :]
    bad = (y.view(torch.int16 if dt == BF16 else torch.int32) !=
           want.to(dt).view(torch.int16 if dt == BF16 else torch.int32))
    assert not bad.any(), (f"{name} b{bits} g{gs}: {int(bad.sum())} outputs differ from the "
                           f"dequantized weight, first at {bad.nonzero()[0].tolist()}")
