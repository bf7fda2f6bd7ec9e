"""Pins of the host oracle: facts fixed by the pages and by mathematics, not by
the oracle itself.

Each ``pin_*`` takes a loaded oracle library (ctypes handle) and raises
AssertionError when the oracle disagrees with the fact. test_oracle_pins.py runs
them on the real oracle; test_oracle_mutations.py runs them on copies of the
oracle with a planted mistake and expects at least one pin to fail each time.

Sources: "Docs / Quantization" (sections "Affine", "Mixture of experts") and
the nuvec crate docs ("Structs": Quantized).
"""
from __future__ import annotations

import math
import os

import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------------------
# golden fixture readers
# ---------------------------------------------------------------------------
def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [p.strip() for p in line.split("|")]


def pack_word_cases():
    for bits, codes, word in _rows("pack_words.txt"):
        yield int(bits), [int(c) for c in codes.split()], int(word, 16)


def handbuilt_cases():
    for name, bits, gs, vals, scale, bias, codes in _rows("handbuilt_groups.txt"):
        yield (name, int(bits), int(gs), [float(v) for v in vals.split()], float(scale),
               float(bias), [int(c) for c in codes.split()])


def _cycle(vals, n):
    return [vals[i % len(vals)] for i in range(n)]


def _u32(t):
    return t.to(torch.int64) & 0xFFFFFFFF


def _unpack_div_mod(words: torch.Tensor, bits: int) -> torch.Tensor:
    """Codes from packed words by integer division and remainder (no shifts, no
    masks): code j of word w is floor(w / 2^(j*bits)) mod 2^bits."""
    per = 32 // bits
    w = _u32(words).tolist()
    out = []
    for row in w:
        r = []
        for word in row:
            for j in range(per):
                r.append((word // (2 ** (j * bits))) % (2 ** bits))
        out.append(r)
    return torch.tensor(out, dtype=torch.int64)


def _groups_with_extremes(rows, cols, gs, bits, gen):
    """Integer weights in [0, 2^b-1] where every group along a row holds both 0
    and 2^b-1, so the quantizer must return scale 1, bias 0 and code = weight."""
    hi = 2 ** bits - 1
    w = torch.randint(0, hi + 1, (rows, cols), generator=gen)
    for g in range(cols // gs):
        pos = torch.randperm(gs, generator=gen)[:2] + g * gs
        w[:, pos[0]] = 0
        w[:, pos[1]] = hi
    return w


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------
def pin_pack_words(lib):
    """Hand-written words: a group holding the word's codes (plus 0 and the top
    code, so scale is 1 and bias 0) must pack into exactly that word."""
    for bits, codes, word in pack_word_cases():
        gs = 32 if bits >= 2 else 32
        per = 32 // bits
        hi = 2 ** bits - 1
        vals = list(codes) + [0, hi] * ((gs - per) // 2) if per < gs else list(codes)
        vals = vals[:gs] + [0] * (gs - len(vals))
        if per == gs:  # the word is the whole group: it must hold 0 and hi itself
            assert 0 in codes and hi in codes, "fixture needs 0 and the top code"
        w = torch.tensor([vals], dtype=torch.float32)
        c, s, b = O.quantize_affine(w, gs, bits, lib=lib)
        assert float(s[0, 0]) == 1.0 and float(b[0, 0]) == 0.0, (bits, codes)
        got = int(_u32(c)[0, 0])
        assert got == word, f"bits={bits} codes={codes}: {got:#010x} != {word:#010x}"


def pin_unpack_words(lib):
    """Dequantizing a hand-written word with scale 1 and bias 0 returns its codes."""
    for bits, codes, word in pack_word_cases():
        gs = 32
        words = torch.zeros(1, gs * bits // 32, dtype=torch.int32)
        words[0, 0] = word - 2 ** 32 if word >= 2 ** 31 else word
        ones = torch.ones(1, 1)
        zeros = torch.zeros(1, 1)
        wh = O.dequantize(words, ones, zeros, gs, bits, lib=lib)
        assert wh[0, :len(codes)].tolist() == [float(c) for c in codes], (bits, codes)


def pin_handbuilt_groups(lib):
    """Hand-built groups (golden/handbuilt_groups.txt): exact scale, bias, codes,
    for fp32 storage, and through bf16 storage where every number is bf16-exact."""
    for name, bits, gs, vals, scale, bias, codes in handbuilt_cases():
        for dt in (torch.float32, torch.bfloat16):
            w = torch.tensor([_cycle(vals, gs), _cycle(vals[::-1], gs)], dtype=torch.float32)
            assert torch.equal(w.to(dt).to(torch.float32), w), name
            c, s, b = O.quantize_affine(w.to(dt), gs, bits, lib=lib)
            got = _unpack_div_mod(c, bits)
            assert s.to(torch.float32).tolist() == [[scale], [scale]], (name, dt, s)
            assert b.to(torch.float32).tolist() == [[bias], [bias]], (name, dt, b)
            assert got[0].tolist() == _cycle(codes, gs), (name, dt)
            assert got[1].tolist() == _cycle(codes[::-1], gs), (name, dt)


def pin_dequantize_stored_rounding(lib):
    """The stored dequantized value is the exact scale * code + bias rounded
    once, to nearest with ties to even, to the dtype (the reading the
    dequantizer follows):
    * bf16, scale 2^-9, bias 1: codes 1, 2, 3 give 1 + 2^-9 (below half a bf16
      step: 1), 1 + 2^-8 (exactly half: the even neighbour 1), 1 + 3 * 2^-9
      (above half: 1 + 2^-7);
    * bf16, scale 37, code 7: 37 * 7 = 259 lies exactly halfway between the
      bf16 neighbours 258 and 260. With bias -2^-20 the exact value
      259 - 2^-20 is below the halfway point, so one rounding gives 258; an
      fp32 step first (fp32 spacing 2^-15 there) would land on 259 and the tie
      would go to the even 260. With bias -2^-60 even an fp64 step lands on 259
      (fp64 spacing 2^-44): the single rounding still gives 258;
    * fp32, scale 1 + 2^-23, bias -3, code 3: the exact value 3 * 2^-23 is an
      fp32 number, so one rounding keeps it (a product rounded first would give
      3 + 2^-21 and then 2^-21);
    * scale 1 and bias 0 return the codes, in both dtypes."""
    w7 = torch.tensor([[7]], dtype=torch.int32).repeat(1, 8)  # 8-bit codes 7, 0, 0, 0
    s37 = torch.tensor([[37.0]], dtype=torch.bfloat16)
    for b_exp in (-20, -60):
        bb = torch.tensor([[-(2.0 ** b_exp)]], dtype=torch.bfloat16)
        assert float(bb[0, 0]) == -(2.0 ** b_exp)
        got = O.dequantize_stored(w7, s37, bb, 32, 8, lib=lib)
        assert float(got[0, 0]) == 258.0, (b_exp, got[0, 0])
        assert float(got[0, 1]) == -(2.0 ** b_exp), got[0, 1]
    words = torch.tensor([[1 | (2 << 8) | (3 << 16)]], dtype=torch.int32)  # 8-bit codes 1, 2, 3, 0
    s = torch.tensor([[2.0 ** -9]], dtype=torch.bfloat16)
    b = torch.tensor([[1.0]], dtype=torch.bfloat16)
    got = O.dequantize_stored(torch.cat([words] * 8, 1), s, b, 32, 8, lib=lib)
    assert got.dtype == torch.bfloat16
    assert got[0, :4].to(torch.float64).tolist() == [1.0, 1.0, 1.0 + 2.0 ** -7, 1.0], got[0, :4]
    s32 = torch.tensor([[1.0 + 2.0 ** -23]], dtype=torch.float32)
    b32 = torch.tensor([[-3.0]], dtype=torch.float32)
    w3 = torch.full((1, 8), 3 | (3 << 8) | (3 << 16) | (3 << 24), dtype=torch.int32)
    got = O.dequantize_stored(w3, s32, b32, 32, 8, lib=lib)
    assert got.dtype == torch.float32 and (got == 3 * 2.0 ** -23).all(), got
    for bits, codes, word in pack_word_cases():
        gs = 32
        words = torch.zeros(1, gs * bits // 32, dtype=torch.int32)
        words[0, 0] = word - 2 ** 32 if word >= 2 ** 31 else word
        for dt in (torch.float32, torch.bfloat16):
            one, zero = torch.ones(1, 1, dtype=dt), torch.zeros(1, 1, dtype=dt)
            wh = O.dequantize_stored(words, one, zero, gs, bits, lib=lib)
            assert wh.dtype == dt and wh[0, :len(codes)].tolist() == [float(c) for c in codes]


def pin_signed_zero_extremes(lib):
    """A group whose smallest values are -0 and +0 (in either order) has bias -0;
    one whose largest are -0 and +0 has its range measured to +0."""
    for vals in ([0.0, -0.0, 1.0], [-0.0, 0.0, 1.0], [1.0, 0.0, -0.0]):
        w = torch.tensor([_cycle(vals, 32)], dtype=torch.float32)
        c, s, b = O.quantize_affine(w, 32, 4, lib=lib)
        assert b.view(torch.int32)[0, 0] == torch.tensor(-0.0).view(torch.int32), vals
        assert float(s[0, 0]) == 1.0 / 15.0 or float(s[0, 0]) == float(torch.tensor(1.0) / 15)
    for vals in ([0.0, -0.0, -1.0], [-0.0, 0.0, -1.0]):
        w = torch.tensor([_cycle(vals, 32)], dtype=torch.float32)
        c, s, b = O.quantize_affine(w, 32, 4, lib=lib)
        assert float(b[0, 0]) == -1.0 and float(s[0, 0]) == float(torch.tensor(1.0) / 15)
        assert set(_unpack_div_mod(c, 4)[0].tolist()) == {15, 0}


def pin_bf16_cast(lib):
    """The oracle's fp32 -> bf16 rounding equals torch's round-to-nearest-even
    cast (a library routine), including exact ties."""
    g = torch.Generator().manual_seed(7)
    x = torch.randn(4096, generator=g) * torch.logspace(-20, 20, 4096)
    ties = torch.tensor([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -100 * (1 + 2 ** -8),
                         3.0, 0.0, -0.0, 65504.0], dtype=torch.float32)
    x = torch.cat([x, ties])
    got = O.cast_bf16(x, lib=lib)
    ref = x.to(torch.bfloat16)
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    assert float(got[4096]) == 1.0 and float(got[4097]) == 1 + 2 ** -6


def pin_stored_scale_is_bf16_rounding(lib):
    """bf16 weights store scale = bf16(fp32((max-min)/(2^b-1))): range 1 at 4 bits
    gives 1/15 in fp32, stored rounded to bf16 (the weights' dtype)."""
    vals = [0.0, 1.0] + [0.5] * 62
    w = torch.tensor([vals]).to(torch.bfloat16)
    c, s, b = O.quantize_affine(w, 64, 4, lib=lib)
    want = (torch.tensor(1.0, dtype=torch.float32) / torch.tensor(15.0)).to(torch.bfloat16)
    assert s.dtype == torch.bfloat16 and s[0, 0].view(torch.int16) == want.view(torch.int16)
    assert float(b[0, 0]) == 0.0
    # the code of 0.5 is rne(0.5 / fp32(1/15)) = rne(7.4999998...) = 7
    assert _unpack_div_mod(c, 4)[0, 2] == 7


def pin_extremes_and_range(lib):
    """On random data every group's minimum gets code 0, its maximum the top code,
    and every code lies in [0, 2^b - 1]."""
    g = torch.Generator().manual_seed(3)
    for bits in (1, 2, 4, 8):
        for gs in (32, 64, 128):
            w = torch.randn(16, 256, generator=g)
            c, s, b = O.quantize_affine(w, gs, bits, lib=lib)
            q = _unpack_div_mod(c, bits).reshape(16, 256 // gs, gs)
            wg = w.reshape(16, 256 // gs, gs)
            amin = wg.argmin(-1, keepdim=True)
            amax = wg.argmax(-1, keepdim=True)
            assert (q.gather(-1, amin) == 0).all(), (bits, gs)
            assert (q.gather(-1, amax) == 2 ** bits - 1).all(), (bits, gs)
            assert q.min() >= 0 and q.max() <= 2 ** bits - 1
            # bias is the group minimum, scale the range over the step count
            assert torch.equal(b.reshape(16, -1), wg.min(-1).values)


def pin_round_trip_bound(lib):
    """|w_hat - w| <= scale/2 (+ fp32 rounding of the division and, for bf16
    storage, the cast of scale and bias) on random data at every width."""
    g = torch.Generator().manual_seed(5)
    for dt in (torch.float32, torch.bfloat16):
        for bits in (1, 2, 4, 8):
            for gs in (32, 64, 128):
                w = (torch.randn(32, 512, generator=g) * 0.02).to(dt)
                c, s, b = O.quantize_affine(w, gs, bits, lib=lib)
                wh = O.dequantize(c, s, b, gs, bits, lib=lib)
                w64 = w.to(torch.float64).reshape(32, -1, gs)
                wg = w.to(torch.float32).reshape(32, -1, gs)
                scale_f = ((wg.max(-1).values - wg.min(-1).values) / (2 ** bits - 1)).to(torch.float64)
                bound = 0.5 * scale_f * (1 + 2 ** -20) + 2 ** -23 * w64.abs().amax(-1)
                if dt == torch.bfloat16:
                    bias_abs = b.to(torch.float64).reshape(32, -1).abs()
                    bound = bound + 2 ** -8 * (bias_abs + (2 ** bits - 1) * scale_f)
                err = (wh.reshape(32, -1, gs) - w64).abs().amax(-1)
                assert (err <= bound).all(), (dt, bits, gs, float((err - bound).max()))


def pin_bits_per_weight(lib):
    """4-bit, groups of 64, 16-bit scale and bias: 4.5 bits per weight; with fp32
    scale and bias (the tiny workload) 5 bits per weight."""
    w = torch.randn(8, 1024)
    for dt, want in ((torch.bfloat16, 4.5), (torch.float32, 5.0)):
        c, s, b = O.quantize_affine(w.to(dt), 64, 4, lib=lib)
        total_bits = 8 * (c.numel() * 4 + s.numel() * s.element_size() + b.numel() * b.element_size())
        assert total_bits / w.numel() == want


def pin_integer_products(lib):
    """Integer-valued groups (scale 1, bias 0) and integer x: the quantized product
    is an integer matmul, computed exactly by torch int64 matmul; both layouts."""
    gen = torch.Generator().manual_seed(11)
    for bits in (1, 2, 4, 8):
        for gs in (32, 64, 128):
            N, K, M = 24, 256, 5
            wi = _groups_with_extremes(N, K, gs, bits, gen)
            xi = torch.randint(-2, 3, (M, K), generator=gen)
            for dt in (torch.float32, torch.bfloat16):
                c, s, b = O.quantize_affine(wi.to(dt), gs, bits, lib=lib)
                y, a = O.qmm(xi.to(dt), c, s, b, gs, bits, True, lib=lib)
                exact = xi @ wi.T
                assert torch.equal(y, exact.to(torch.float64)), (bits, gs, dt)
                assert torch.equal(a, (xi.abs() @ wi.T).to(torch.float64))
            # transpose = 0: weights stored [K, N], grouped along N
            wt = _groups_with_extremes(K, 256, gs, bits, gen)
            c, s, b = O.quantize_affine(wt.to(torch.float32), gs, bits, lib=lib)
            y, a = O.qmm(xi.to(torch.float32), c, s, b, gs, bits, False, lib=lib)
            assert torch.equal(y, (xi @ wt).to(torch.float64)), (bits, gs, "transpose=0")


def pin_affine_integer_products(lib):
    """w = 2*code - 5 per group: scale 2 and bias -5 are exact, so the product
    must equal x @ (2*c - 5)^T exactly (the bias term and its sign)."""
    gen = torch.Generator().manual_seed(13)
    N, K, M, gs, bits = 16, 128, 3, 32, 4
    ci = _groups_with_extremes(N, K, gs, bits, gen)
    w = (2 * ci - 5).to(torch.float32)
    c, s, b = O.quantize_affine(w, gs, bits, lib=lib)
    assert (s == 2).all() and (b == -5).all()
    xi = torch.randint(-3, 4, (M, K), generator=gen)
    y, _ = O.qmm(xi.to(torch.float32), c, s, b, gs, bits, True, lib=lib)
    assert torch.equal(y, (xi @ (2 * ci - 5).T).to(torch.float64))


def pin_brute_force_8x8(lib):
    """An 8x8 output (M = 8, N = 8, K = 2 groups) on random data against a
    brute-force sum: codes unpacked by division and remainder, scale and bias
    read back from storage, products summed exactly (math.fsum)."""
    g = torch.Generator().manual_seed(17)
    for dt in (torch.float32, torch.bfloat16):
        for bits, gs in ((4, 64), (2, 32), (8, 64), (4, 128)):
            K = 2 * gs
            w = torch.randn(8, K, generator=g).to(dt)
            x = torch.randn(8, K, generator=g).to(dt)
            c, s, b = O.quantize_affine(w, gs, bits, lib=lib)
            q = _unpack_div_mod(c, bits)
            sv = s.to(torch.float64).tolist()
            bv = b.to(torch.float64).tolist()
            xv = x.to(torch.float64).tolist()
            y, a = O.qmm(x, c, s, b, gs, bits, True, lib=lib)
            for m in range(8):
                for n in range(8):
                    terms = [xv[m][k] * (sv[n][k // gs] * int(q[n, k]) + bv[n][k // gs])
                             for k in range(K)]
                    exact = math.fsum(terms)
                    mag = math.fsum(abs(t) for t in terms)
                    assert abs(float(y[m, n]) - exact) <= 1e-13 * mag + 1e-300, (dt, bits, gs, m, n)
                    assert abs(float(a[m, n]) - mag) <= 1e-13 * mag


def pin_scaling_invariant(lib):
    """y(2^j x) == 2^j y(x) exactly (power-of-two scaling is exact in fp64)."""
    g = torch.Generator().manual_seed(19)
    w = torch.randn(32, 256, generator=g)
    x = torch.randn(3, 256, generator=g)
    c, s, b = O.quantize_affine(w, 64, 4, lib=lib)
    y1, _ = O.qmm(x, c, s, b, 64, 4, True, lib=lib)
    y8, _ = O.qmm(x * 8, c, s, b, 64, 4, True, lib=lib)
    assert torch.equal(y8, 8 * y1)


def pin_transpose_layouts_agree(lib):
    """The same integer weight matrix stored [N, K] (grouped along K) and stored
    transposed [K, N] (grouped along N) gives the same product x @ W^T. Values:
    0 where (n + k) % gs == 0, the top code where it is 1, random elsewhere, so
    every group of either grouping holds both extremes (scale 1, bias 0)."""
    gen = torch.Generator().manual_seed(23)
    gs, bits, n = 32, 4, 96
    W = torch.randint(0, 16, (n, n), generator=gen)
    diag = (torch.arange(n)[:, None] + torch.arange(n)[None, :]) % gs
    W[diag == 0] = 0
    W[diag == 1] = 15
    x = torch.randint(-2, 3, (4, n), generator=gen)
    c1, s1, b1 = O.quantize_affine(W.to(torch.float32), gs, bits, lib=lib)
    c2, s2, b2 = O.quantize_affine(W.T.contiguous().to(torch.float32), gs, bits, lib=lib)
    y1, _ = O.qmm(x.float(), c1, s1, b1, gs, bits, True, lib=lib)
    y2, _ = O.qmm(x.float(), c2, s2, b2, gs, bits, False, lib=lib)
    assert torch.equal(y1, (x @ W.T).double()) and torch.equal(y2, y1)


def pin_gather(lib):
    """gather_qmm on the page's example shapes (q from [8,128,256], x [4,1,256],
    experts [0,0,3,5] -> y [4,128]) equals each row times its expert's
    dequantized weights; lhs selects the x row; out-of-range ids are refused."""
    g = torch.Generator().manual_seed(29)
    for dt in (torch.float32, torch.bfloat16):
        w = torch.randn(8, 128, 256, generator=g).to(dt)
        x = torch.randn(4, 1, 256, generator=g).to(dt)
        c, s, b = O.quantize_affine(w, 64, 4, lib=lib)
        ids = torch.tensor([0, 0, 3, 5])
        y, a = O.gather_qmm(x, c, s, b, None, ids, 64, 4, True, lib=lib)
        assert tuple(y.shape) == (4, 128)
        wh = O.dequantize(c, s, b, 64, 4, lib=lib)  # [8, 128, 256] fp64
        x2 = x.reshape(4, 256).to(torch.float64)
        for r in range(4):
            ref = wh[int(ids[r])] @ x2[r]
            mag = wh[int(ids[r])].abs() @ x2[r].abs()
            assert ((y[r] - ref).abs() <= 1e-12 * mag).all(), (dt, r)
        # lhs picks rows of x; pairs (token, expert)
        lhs = torch.tensor([3, 1, 1, 0, 2])
        rhs = torch.tensor([7, 2, 6, 6, 0])
        y2, _ = O.gather_qmm(x, c, s, b, lhs, rhs, 64, 4, True, lib=lib)
        for r in range(5):
            ref = wh[int(rhs[r])] @ x2[int(lhs[r])]
            assert ((y2[r] - ref).abs() <= 1e-12 * (wh[int(rhs[r])].abs() @ x2[int(lhs[r])].abs())).all()
        # all rows on expert 5: the gather is a plain quantized product with expert 5
        y3, _ = O.gather_qmm(x, c, s, b, None, torch.full((4,), 5), 64, 4, True, lib=lib)
        y4, _ = O.qmm(x.reshape(4, 256), c[5], s[5], b[5], 64, 4, True, lib=lib)
        assert torch.equal(y3, y4)
    try:
        O.gather_qmm(x, c, s, b, None, torch.tensor([0, 8, 1, 1]), 64, 4, True, lib=lib)
    except ValueError:
        pass
    else:
        raise AssertionError("expert id 8 of 8 experts accepted")


def pin_gather_mm(lib):
    """gather_mm with full-precision experts: integer x and weights give exact
    integer rows equal to an int64 brute force per pair; scaled-identity
    experts return (e + 1) times the selected x row, with sum |x w| the same
    multiple of |x|; out-of-range ids are refused."""
    g = torch.Generator().manual_seed(37)
    E, N, K, T = 5, 24, 128, 9
    for dt in (torch.float32, torch.bfloat16):
        wi = torch.randint(-8, 9, (E, N, K), generator=g)
        xi = torch.randint(-2, 3, (T, K), generator=g)
        lhs = torch.randint(0, T, (17,), generator=g)
        rhs = torch.randint(0, E, (17,), generator=g)
        y, a = O.gather_mm(xi.to(dt), wi.to(dt), lhs, rhs, lib=lib)
        for r in range(17):
            t, e = int(lhs[r]), int(rhs[r])
            ref = (wi[e] * xi[t]).sum(-1)          # int64, exact
            assert torch.equal(y[r], ref.to(torch.float64)), (dt, r)
            assert torch.equal(a[r], (wi[e] * xi[t]).abs().sum(-1).to(torch.float64)), (dt, r)
    eye = torch.stack([torch.eye(K) * (e + 1) for e in range(E)])  # [E, K, K]
    x = torch.randn(T, K, generator=g).to(torch.bfloat16)
    rhs = torch.tensor([0, 4, 2, 2, 1])
    y, a = O.gather_mm(x[:5], eye.to(torch.bfloat16), None, rhs, lib=lib)
    for r in range(5):
        mult = float(rhs[r]) + 1.0
        assert torch.equal(y[r], x[r].double() * mult), r
        assert torch.equal(a[r], x[r].double().abs() * mult), r
    try:
        O.gather_mm(x, eye, None, torch.tensor([0, 5]), lib=lib)
    except ValueError:
        pass
    else:
        raise AssertionError("expert id 5 of 5 experts accepted")


def _pack_codes(codes: torch.Tensor, bits: int) -> torch.Tensor:
    """Pack integer codes [..., cols] into int32 words, code j at bits [j*bits, (j+1)*bits)."""
    per = 32 // bits
    c = codes.to(torch.int64).reshape(*codes.shape[:-1], -1, per)
    word = (c << (torch.arange(per, dtype=torch.int64) * bits)).sum(-1)
    return torch.where(word >= 2 ** 31, word - 2 ** 32, word).to(torch.int32)


def pin_moe_swiglu(lib):
    """The MoE SwiGLU block against closed forms, with integer data (scale
    +-1, bias 0): silu(z) - silu(-z) = z and silu(z) + silu(-z) = z tanh(z/2),
    so y(G) - y(-G) is the exact integer routed sum of (x G^T) * (x U^T) times
    D^T (int64 brute force) and y(G) + y(-G) the same with g tanh(g/2) for g;
    a zero gate gives zero; doubling the routing weights doubles y; the top-k
    order does not matter; an out-of-range expert id is refused."""
    g = torch.Generator().manual_seed(53)
    E, I, K, T, top, gs, bits = 3, 64, 64, 5, 2, 32, 4
    Gc = torch.randint(0, 4, (E, I, K), generator=g)
    Uc = torch.randint(0, 4, (E, I, K), generator=g)
    Dc = torch.randint(0, 16, (E, K, I), generator=g)
    x = torch.randint(-2, 3, (T, K), generator=g).to(torch.bfloat16)
    ids = torch.stack([torch.randperm(E, generator=g)[:top] for _ in range(T)])
    rw = torch.randint(-2, 3, (T, top), generator=g).to(torch.float32)
    one = lambda shape, v: torch.full(shape, float(v), dtype=torch.bfloat16)  # noqa: E731
    q = lambda c, sign: (_pack_codes(c, bits), one((*c.shape[:-1], c.shape[-1] // gs), sign),  # noqa: E731
                         one((*c.shape[:-1], c.shape[-1] // gs), 0))
    G, Gn, U, D = q(Gc, 1), q(Gc, -1), q(Uc, 1), q(Dc, 1)
    yp, a = O.moe_swiglu(x, G, U, D, ids, rw, gs, bits, lib=lib)
    ym, _ = O.moe_swiglu(x, Gn, U, D, ids, rw, gs, bits, lib=lib)
    xi = x.to(torch.int64)
    odd = torch.zeros(T, K, dtype=torch.int64)
    even = torch.zeros(T, K, dtype=torch.float64)
    for t in range(T):
        for j in range(top):
            e, w = int(ids[t, j]), int(rw[t, j])
            gv = Gc[e] @ xi[t]                      # [I], exact
            uv = Uc[e] @ xi[t]
            odd[t] += w * (Dc[e] @ (gv * uv))
            gf = gv.to(torch.float64)
            th = torch.tensor([math.tanh(v / 2) for v in gf.tolist()], dtype=torch.float64)
            even[t] += w * (Dc[e].to(torch.float64) @ (gf * th * uv.to(torch.float64)))
    tol = 1e-12 * (a + 1)
    assert ((yp - ym) - odd.to(torch.float64)).abs().le(tol).all(), "odd part"
    assert ((yp + ym) - even).abs().le(tol).all(), "even part"
    Z = q(torch.zeros_like(Gc), 1)
    y0, _ = O.moe_swiglu(x, Z, U, D, ids, rw, gs, bits, lib=lib)
    assert (y0 == 0).all(), "zero gate"
    y2, _ = O.moe_swiglu(x, G, U, D, ids, 2 * rw, gs, bits, lib=lib)
    assert torch.equal(y2, 2 * yp), "routing weights scale the output"
    ys, _ = O.moe_swiglu(x, G, U, D, ids.flip(1), rw.flip(1), gs, bits, lib=lib)
    assert (ys - yp).abs().le(tol).all(), "top-k order"
    # an expert id out of range contributes nothing (as a zero routing weight)
    bad = ids.clone()
    bad[:, 1] = E
    rw0 = rw.clone()
    rw0[:, 1] = 0
    yb, _ = O.moe_swiglu(x, G, U, D, bad, rw, gs, bits, lib=lib)
    y0w, _ = O.moe_swiglu(x, G, U, D, ids, rw0, gs, bits, lib=lib)
    assert (yb - y0w).abs().le(tol).all(), "out-of-range expert"


def pin_moe_swiglu_tolerance_scale(lib):
    """The block's tolerance scale carries each product's sum |x w_hat| through
    h = silu(g) * u: a = sum_j |rw| sum_i |wd| 2 (|h| + |silu'(g) u| a_g +
    |silu(g)| a_u). Two cases where h = 0 exactly but the products do not
    vanish term by term (x = (1, 1, 0, ...); weights +1 and -1 as codes 2 and 0
    with scale 1, bias -1):
    * gate rows (1, -1, ...): g = 0, a_g = 2, silu'(0) = 1/2, so
      a[n] = 2 |rw| sum_i |wd_ni| |u_i| (an exact integer) and y = 0;
    * up rows (1, -1, ...) and gate rows (2, 0, ...) (codes 3, 1 with bias -1):
      u = 0, a_u = 2, g = 2, so a[n] = 2 |rw| sum_i |wd_ni| silu(2) 2 with
      silu(2) = 2 / (1 + e^-2)."""
    g = torch.Generator().manual_seed(54)
    E, I, K, T, top, gs, bits = 2, 32, 32, 1, 1, 32, 4
    x = torch.zeros(T, K, dtype=torch.bfloat16)
    x[0, 0] = 1.0
    x[0, 1] = 1.0
    pm = torch.zeros(E, I, K, dtype=torch.int64)
    pm[:, :, 0], pm[:, :, 1] = 2, 0                 # w_hat = code - 1: +1, -1, then -1 ...
    Uc = torch.randint(1, 16, (E, I, K), generator=g)
    Dc = torch.randint(0, 16, (E, K, I), generator=g)
    ids = torch.tensor([[1]])
    rw = torch.tensor([[-3.0]])
    one = lambda shape, v: torch.full(shape, float(v), dtype=torch.bfloat16)  # noqa: E731
    q = lambda c, b: (_pack_codes(c, bits), one((*c.shape[:-1], c.shape[-1] // gs), 1),  # noqa: E731
                      one((*c.shape[:-1], c.shape[-1] // gs), b))
    y, a = O.moe_swiglu(x, q(pm, -1), q(Uc, 0), q(Dc, 0), ids, rw, gs, bits, lib=lib)
    u = Uc[1, :, 0] + Uc[1, :, 1]                    # x . w_up, exact integers
    want = 2 * 3 * (Dc[1] @ u)
    assert (y == 0).all(), "zero gate gives zero"
    assert torch.equal(a[0], want.to(torch.float64)), (a[0], want)
    gc = pm.clone()
    gc[:, :, 0], gc[:, :, 1] = 3, 1                  # w_hat = code - 1: 2, 0, so g = 2
    y2, a2 = O.moe_swiglu(x, q(gc, -1), q(pm, -1), q(Dc, 0), ids, rw, gs, bits, lib=lib)
    silu2 = 2.0 / (1.0 + math.exp(-2.0))
    want2 = 2 * 3 * Dc[1].sum(1).to(torch.float64) * silu2 * 2
    assert (y2 == 0).all(), "zero up gives zero"
    assert (a2[0] - want2).abs().le(1e-12 * want2).all(), (a2[0], want2)
    # g = 2 and u = 2 (up weights +1, +1): every term counts, the slope
    # silu'(2) = s(2) (1 + 2 (1 - s(2))) with s(2) = 1 / (1 + e^-2)
    uc = torch.zeros(E, I, K, dtype=torch.int64)
    uc[:, :, 0], uc[:, :, 1] = 1, 1
    y3, a3 = O.moe_swiglu(x, q(gc, -1), q(uc, 0), q(Dc, 0), ids, rw, gs, bits, lib=lib)
    s2 = 1.0 / (1.0 + math.exp(-2.0))
    slope2 = s2 * (1.0 + 2.0 * (1.0 - s2))
    h = silu2 * 2.0
    want3 = 2 * 3 * Dc[1].sum(1).to(torch.float64) * (h + slope2 * 2.0 * 2.0 + silu2 * 2.0)
    assert (y3[0] - (-3.0) * Dc[1].sum(1).to(torch.float64) * h).abs().le(1e-9).all()
    assert (a3[0] - want3).abs().le(1e-12 * want3).all(), (a3[0], want3)


def pin_sampled_match_full(lib):
    """The sampled product entry points agree with the full ones."""
    g = torch.Generator().manual_seed(31)
    w = torch.randn(40, 256, generator=g).to(torch.bfloat16)
    x = torch.randn(6, 256, generator=g).to(torch.bfloat16)
    c, s, b = O.quantize_affine(w, 64, 4, lib=lib)
    y, a = O.qmm(x, c, s, b, 64, 4, True, lib=lib)
    mi = torch.tensor([0, 5, 3, 3])
    ni = torch.tensor([0, 39, 17, 18])
    ys, as_ = O.qmm_sampled(x, c, s, b, 64, 4, True, mi, ni, lib=lib)
    assert torch.equal(ys, y[mi, ni]) and torch.equal(as_, a[mi, ni])
    we = torch.randn(3, 40, 256, generator=g).to(torch.bfloat16)
    c, s, b = O.quantize_affine(we, 64, 4, lib=lib)
    lhs, rhs = torch.tensor([0, 1, 5, 5]), torch.tensor([2, 0, 1, 2])
    y, a = O.gather_qmm(x, c, s, b, lhs, rhs, 64, 4, True, lib=lib)
    ri, ni = torch.tensor([3, 0, 2]), torch.tensor([1, 39, 20])
    ys, as_ = O.gather_qmm_sampled(x, c, s, b, lhs, rhs, 64, 4, True, ri, ni, lib=lib)
    assert torch.equal(ys, y[ri, ni]) and torch.equal(as_, a[ri, ni])


# ---- floating-point modes ("Docs / Quantization", section "Floating-point
# formats"; the formats are the published definitions of MXFP4 / MXFP8 / NVFP4)

# E2M1 magnitudes listed in the microscaling format definition, codes 0..7.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def pin_fp_element_and_scale_values(lib):
    """Codes -> values from the format definitions: the E2M1 list with its
    sign bit, E4M3 (bias 7, no infinities, S.1111.111 NaN) and E8M0 (2^(s-127),
    255 NaN) at their edges."""
    for c in range(16):
        want = E2M1_TABLE[c & 7] * (-1.0 if c & 8 else 1.0)
        got = O.fp_value("e2m1", c, lib=lib)
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), (c, got)
    e4m3 = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
            0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0, 0xB8: -1.0}
    for c, want in e4m3.items():
        assert O.fp_value("e4m3", c, lib=lib) == want, (hex(c), want)
    assert math.isnan(O.fp_value("e4m3", 0x7F, lib=lib)) and math.isnan(O.fp_value("e4m3", 0xFF, lib=lib))
    assert O.fp_value("e4m3", 0x77, lib=lib) == 240.0  # 2^7 * (1 + 7/8)
    for c, want in {127: 1.0, 0: 2.0 ** -127, 254: 2.0 ** 127, 128: 2.0, 120: 2.0 ** -7}.items():
        assert O.fp_value("e8m0", c, lib=lib) == want, (c, want)
    assert math.isnan(O.fp_value("e8m0", 255, lib=lib))


def pin_fp_nearest_ties_and_saturation(lib):
    """Round to nearest, ties to the even mantissa field, saturate at the
    largest finite value (E2M1 6, E4M3 448); the sign follows the value."""
    e2m1 = {0.25: 0.0, 0.26: 0.5, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0,
            5.01: 6.0, 6.0: 6.0, 7.0: 6.0, 1e30: 6.0, -2.5: -2.0, -0.2: -0.0, -5.5: -6.0}
    for v, want in e2m1.items():
        got = O.fp_value("e2m1", O.fp_nearest("e2m1", v, lib=lib), lib=lib)
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), (v, got, want)
    e4m3 = {1.0 + 1 / 16: 1.0, 1.0 + 3 / 16: 1.25, 2.0 ** -10: 0.0, 3 * 2.0 ** -10: 2.0 ** -8,
            464.0: 448.0, 1e9: 448.0, -(1.0 + 1 / 16): -1.0, 240.0: 240.0, 248.0: 256.0}
    for v, want in e4m3.items():
        assert O.fp_value("e4m3", O.fp_nearest("e4m3", v, lib=lib), lib=lib) == want, (v, want)


def _fp_group_row(vals, gs):
    return torch.tensor([(vals * ((gs + len(vals) - 1) // len(vals)))[:gs]], dtype=torch.float32)


def pin_fp_mx_scale_rule(lib):
    """MXFP4 / MXFP8: X = 2^(floor(log2 amax) - emax), emax 2 (E2M1) or 8 (E4M3):
    amax in [4, 8) * 2^k gives scale code 127 + k at 4 bits, amax in [256, 512)
    * 2^k gives 127 + k at 8 bits; a zero group gets scale code 0 and zero codes."""
    for k in (-20, -3, 0, 5, 40):
        for amax, want in ((4.0, 127), (6.0, 127), (7.99, 127), (8.0, 128), (3.99, 126)):
            w = _fp_group_row([0.5, -1.0, amax * 2.0 ** k / 2 ** k], 32) * 2.0 ** k
            w[0, 0] = amax * 2.0 ** k
            _, s = O.quantize_fp(w, "mxfp4", lib=lib)
            assert int(s[0, 0]) == want + k, (k, amax, int(s[0, 0]))
        for amax, want in ((256.0, 127), (448.0, 127), (511.0, 127), (512.0, 128)):
            w = torch.zeros(1, 32)
            w[0, 5] = amax * 2.0 ** k
            w[0, 6] = -1.0 * 2.0 ** k
            _, s = O.quantize_fp(w, "mxfp8", lib=lib)
            assert int(s[0, 0]) == want + k, (k, amax, int(s[0, 0]))
    c, s = O.quantize_fp(torch.zeros(2, 64), "mxfp4", lib=lib)
    assert (s == 0).all() and (c == 0).all()
    # the saturating step: a 7.5 * 2^k value in a group whose scale is 2^k
    w = torch.tensor([[7.5, 1.0] + [0.0] * 30])
    c, s = O.quantize_fp(w, "mxfp4", lib=lib)
    wh = O.dequantize_fp(c, s, "mxfp4", lib=lib).float()
    assert int(s[0, 0]) == 127 and wh[0, 0] == 6.0 and wh[0, 1] == 1.0


def pin_fp_grid_round_trip(lib):
    """Values already on a mode's grid come back exactly: E2M1 values (both
    signs) times 2^k for MXFP4, E4M3 values for MXFP8, E2M1 values times an
    E4M3 scale S = amax / 6 for NVFP4; dequantized to bf16 exactly."""
    g = torch.Generator().manual_seed(7)
    for k in (-9, 0, 3):
        vals = torch.tensor(E2M1_TABLE + [-v for v in E2M1_TABLE[1:]] + [6.0] * 17)[:32] * 2.0 ** k
        vals = vals[torch.randperm(32, generator=g)].view(1, 32)
        c, s = O.quantize_fp(vals, "mxfp4", lib=lib)
        assert int(s[0, 0]) == 127 + k
        assert torch.equal(O.dequantize_fp(c, s, "mxfp4", lib=lib).float(), vals)
    e4m3_vals = torch.tensor([O.fp_value("e4m3", c, lib=lib) for c in range(0, 127, 4)])
    vals = e4m3_vals.clone()
    vals[0] = 448.0  # amax 448: scale 2^0
    vals = vals.view(1, 32)
    c, s = O.quantize_fp(vals, "mxfp8", lib=lib)
    assert int(s[0, 0]) == 127
    assert torch.equal(O.dequantize_fp(c, s, "mxfp8", lib=lib).float(), vals)
    for S in (1.0, 1.25, 0.09375, 3.5):  # E4M3 numbers
        base = torch.tensor(E2M1_TABLE + [-v for v in E2M1_TABLE])[:16]
        base[3] = 6.0
        vals = (base * S).view(1, 16)
        c, s = O.quantize_fp(vals, "nvfp4", lib=lib)
        assert O.fp_value("e4m3", int(s[0, 0]), lib=lib) == S, (S, int(s[0, 0]))
        assert torch.equal(O.dequantize_fp(c, s, "nvfp4", lib=lib).float(), vals), S


def pin_fp_round_trip_bound(lib):
    """Random groups: every MXFP4 value is within half the E2M1 grid step of
    w / X (times X), or saturated at 6X; NVFP4 the same with the stored scale;
    the codes pack 8 to a word and unpack by division and remainder."""
    g = torch.Generator().manual_seed(11)
    w = torch.randn(8, 256, generator=g) * (10.0 ** (torch.rand(8, 1, generator=g) * 4 - 2))
    for mode, gs in (("mxfp4", 32), ("nvfp4", 16)):
        c, s = O.quantize_fp(w, mode, lib=lib)
        codes = _unpack_div_mod(c, 4)
        kind = "e8m0" if mode == "mxfp4" else "e4m3"
        X = torch.tensor([[O.fp_value(kind, int(v), lib=lib) for v in row] for row in s.tolist()],
                         dtype=torch.float64).repeat_interleave(gs, dim=1)
        elem = torch.tensor([[E2M1_TABLE[q & 7] * (-1.0 if q & 8 else 1.0) for q in row]
                             for row in codes.tolist()], dtype=torch.float64)
        t = w.double() / X
        step = torch.where(t.abs() < 2, 0.5, torch.where(t.abs() < 4, 1.0, 2.0))
        ok = ((elem - t).abs() <= step / 2 + 1e-6) | ((t.abs() >= 6) & (elem.abs() == 6))
        assert ok.all(), (mode, int((~ok).sum()))
        wh = O.dequantize_fp(c, s, mode, lib=lib).double()
        assert torch.equal(wh, (elem * X).to(torch.bfloat16).double())


def pin_fp_products(lib):
    """qmm_fp against a brute force over unpacked codes: on-grid weights with
    scale 1 and integer x give exact results (8 x 8 outputs), and a random case
    agrees with fp64 sums of the dequantized weights."""
    g = torch.Generator().manual_seed(13)
    idx = torch.randint(0, 16, (8, 64), generator=g)
    w = torch.tensor([[E2M1_TABLE[q & 7] * (-1.0 if q & 8 else 1.0) for q in row] for row in idx.tolist()])
    w[:, 0] = 6.0
    w[:, 32] = -6.0
    x = torch.randint(-2, 3, (8, 64), generator=g).float()
    c, s = O.quantize_fp(w, "mxfp4", lib=lib)
    y, a = O.qmm_fp(x, c, s, "mxfp4", lib=lib)
    brute = [[sum(x[m, k].item() * w[n, k].item() for k in range(64)) for n in range(8)] for m in range(8)]
    assert torch.equal(y, torch.tensor(brute, dtype=torch.float64))
    assert torch.equal(a, (x.double().abs() @ w.double().abs().t()))
    w = torch.randn(16, 96, generator=g)
    x = torch.randn(3, 96, generator=g).to(torch.bfloat16)
    for mode in ("mxfp4", "mxfp8", "nvfp4"):
        c, s = O.quantize_fp(w, mode, lib=lib)
        wh = O.dequantize_fp(c, s, mode, lib=lib).double()
        y, a = O.qmm_fp(x, c, s, mode, lib=lib)
        ref = x.double() @ wh.t()
        assert torch.allclose(y, ref, rtol=0, atol=1e-12), mode


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
