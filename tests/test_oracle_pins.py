"""Pins for the CPU oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own formula: each compares it with an
independent construction (Sylvester recursion, exact rational arithmetic,
pure-Python brute force), a closed form, or an invariant.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a) -> np.ndarray:
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return O.bf16_bits(t)


def _is_bf16(v: Fraction) -> bool:
    f = np.float32(float(v))
    if Fraction(float(f)) != v:
        return False
    return O.bf16_bits_to_f32(_bf16([f]))[0] == f


# ------------------------------------------------------------ Hadamard matrix


@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_definition_matches_sylvester_and_is_orthogonal(b):
    H = O.hadamard(b)
    S = np.array(O.hadamard_sylvester(b), dtype=np.int64)
    assert (H == S).all()
    assert (H == H.T).all()
    assert (H[0] == 1).all() and (H[:, 0] == 1).all()
    assert (H @ H.T == b * np.eye(b, dtype=np.int64)).all()


@pytest.mark.parametrize("b", [4, 16, 64, 256])
def test_regular_hadamard_definition_matches_kronecker_power_and_is_regular(b):
    # The pages' regular matrix: H_256 = H_4 (x) H_4 (x) H_4 (x) H_4, orthogonal
    # and "DC-balanced": every row has the same sum, so a constant block stays
    # constant.  Read with H_4 = J - 2I (row sum +2).
    H = O.hadamard(b, regular=True)
    K = O.hadamard_regular_kron(b)
    assert (H == K).all()
    assert (H == H.T).all()
    assert (H @ H.T == b * np.eye(b, dtype=np.int64)).all()
    r = int(round(b ** 0.5))
    assert (H.sum(axis=1) == r).all() and (H.sum(axis=0) == r).all()
    # a regular Hadamard matrix is not a Sylvester one: H_b 1 is constant,
    # while Sylvester sends 1 to (b, 0, ..., 0)
    S = np.array(O.hadamard_sylvester(b), dtype=np.int64)
    assert (S @ np.ones(b, dtype=np.int64) == np.eye(b, dtype=np.int64)[0] * b).all()
    assert (H @ np.ones(b, dtype=np.int64) == r).all()


# ------------------------------------------------------------ rotation


@pytest.mark.parametrize("b", [2, 4, 16, 128, 256])
def test_fwht_equals_explicit_matrix_on_integers(b):
    rng = np.random.default_rng(b)
    x = rng.integers(-1000, 1000, size=3 * b).astype(np.float32)  # every fp32 op exact
    z = O.fwht(x, b)
    exact = O.py_fwht_exact([int(v) for v in x], b)
    assert [Fraction(float(v)) for v in z] == exact


@pytest.mark.parametrize("b", [4, 128])
def test_fwht_is_involution_up_to_b(b):
    # the pages: the Hadamard rotation can be undone exactly
    rng = np.random.default_rng(7)
    x = rng.integers(-500, 500, size=4 * b).astype(np.float32)
    zz = O.fwht(O.fwht(x, b), b)
    assert (zz == b * x).all()


def test_fwht_f32_within_summation_error_bound():
    # general bf16 inputs: fp32 butterflies vs the exact product; a depth-7
    # tree of roundings is bounded by 7 * 2^-24 * sum|x| (first order)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    x[:, 5] *= 20
    x = O.bf16_bits_to_f32(_bf16(x)).reshape(8, 256)
    z = np.stack([O.fwht(r, 128) for r in x])
    exact = O.rotate_explicit_f64(x, 128)
    absx = np.abs(x).reshape(8, 2, 128).sum(-1)
    bound = 7 * 2.0 ** -24 * np.repeat(absx, 128, axis=1) * 1.0001
    assert (np.abs(z - exact) <= bound).all()
    assert np.abs(z - exact).max() > 0  # the bound is exercised, not vacuous


def test_rotation_of_constant_block_is_dc_spike():
    b, c = 128, 0.75
    x = np.full((1, 2 * b), c, dtype=np.float32)
    q, s = O.quantize_act(_bf16(x), b)
    expect = np.zeros(2 * b, dtype=np.int8)
    expect[0] = expect[b] = 127
    assert (q[0] == expect).all()
    assert s[0] == np.float32(b * c) / np.float32(127)


@pytest.mark.parametrize("i", [0, 1, 77, 127])
def test_rotation_of_spike_gives_hadamard_column_signs(i):
    b, c = 128, -3.0
    x = np.zeros((1, b), dtype=np.float32)
    x[0, i] = c
    q, s = O.quantize_act(_bf16(x), b)
    H = np.array(O.hadamard_sylvester(b))
    assert (q[0] == (-127 * H[:, i])).all()
    assert s[0] == np.float32(3.0) / np.float32(127)


# ------------------------------------------------------------ quantiser


def _load_ties():
    rows = []
    with open(os.path.join(GOLDEN, "quant_ties.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, codes, scale = [p.strip() for p in line.split("|")]
            path, block, z = head.split()
            rows.append((path, int(block), [int(v) for v in z.split(",")],
                         [int(v) for v in codes.split(",")], Fraction(scale)))
    return rows


@pytest.mark.parametrize("case", _load_ties(), ids=lambda c: f"{c[0]}-b{c[1]}")
def test_quantiser_ties_round_half_to_even(case):
    path, b, zlead, codes_lead, scale = case
    K = max(b, len(zlead))
    z = zlead + [0] * (K - len(zlead))
    bb = max(b, 1)
    H = O.hadamard_sylvester(bb) if bb > 1 else [[1]]
    x = [Fraction(sum(H[i][j] * z[o + j] for j in range(bb)), bb) for o in range(0, K, bb) for i in range(bb)]
    expect = codes_lead + [0] * (K - len(codes_lead))
    if path == "act":
        assert all(_is_bf16(v) for v in x)
        q, s = O.quantize_act(_bf16([[float(v) for v in x]]), b)
    else:
        assert all(Fraction(float(np.float32(float(v)))) == v for v in x)
        q, s = O.pack_weight(np.array([[float(v) for v in x]], dtype=np.float32), b)
    assert q[0].tolist() == expect
    assert Fraction(float(s[0])) == scale


def test_quantiser_matches_exact_rational_arbiter():
    rng = np.random.default_rng(11)
    z = (rng.standard_normal((40, 96)) * rng.uniform(0.01, 100, (40, 1))).astype(np.float32)
    z[3] = 0.0
    z[5, 7] = 1e4
    q, s = O.quantize_rows(z)
    for m in range(z.shape[0]):
        codes, sc = O.py_quantize_row_exact([Fraction(float(v)) for v in z[m]])
        assert q[m].tolist() == codes
        assert Fraction(float(s[m])) == sc


def test_quantiser_invariances():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((16, 256)) * 3).astype(np.float32)
    xb = _bf16(x)
    q, s = O.quantize_act(xb, 128)
    qn, sn = O.quantize_act(_bf16(-O.bf16_bits_to_f32(xb)), 128)
    assert (qn == -q).all() and (sn == s).all()
    for k in (-6, -1, 3, 9):
        q2, s2 = O.quantize_act(_bf16(O.bf16_bits_to_f32(xb) * np.float32(2.0 ** k)), 128)
        assert (q2 == q).all()
        assert (s2 == s * np.float32(2.0 ** k)).all()
    assert (np.abs(q).max(axis=1) == 127).all()


def test_zero_row_gives_zero_scale_and_codes():
    x = np.zeros((3, 256), dtype=np.float32)
    x[1, 9] = 1.0
    q, s = O.quantize_act(_bf16(x), 128)
    assert s[0] == 0 and s[2] == 0 and not q[0].any() and not q[2].any()
    assert s[1] > 0


def test_block_one_is_plain_rowwise_absmax():
    rng = np.random.default_rng(2)
    x = O.bf16_bits_to_f32(_bf16(rng.standard_normal((6, 64)))).reshape(6, 64)
    q1, s1 = O.quantize_act(_bf16(x), 1)
    q0, s0 = O.quantize_act(_bf16(x), 0)
    for m in range(6):
        codes, sc = O.py_quantize_row_exact([Fraction(float(v)) for v in x[m]])
        assert q1[m].tolist() == codes and q0[m].tolist() == codes
        assert Fraction(float(s1[m])) == sc == Fraction(float(s0[m]))


def test_weight_scales_are_per_output_channel():
    rng = np.random.default_rng(8)
    w = (rng.standard_normal((5, 256)) * 0.02).astype(np.float32)
    w[2] *= 100
    q, s = O.pack_weight(w, 128)
    for n in range(5):
        zr = O.fwht(w[n], 128)
        codes, sc = O.py_quantize_row_exact([Fraction(float(v)) for v in zr])
        assert q[n].tolist() == codes and Fraction(float(s[n])) == sc


# ------------------------------------------------------------ GEMM and epilogue


@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 5, 7), (8, 4, 32), (2, 3, 300)])
def test_igemm_equals_bruteforce(shape):
    M, N, K = shape
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    qa = rng.integers(-127, 128, (M, K)).astype(np.int8)
    qb = rng.integers(-127, 128, (N, K)).astype(np.int8)
    qa[0, 0] = -127
    qb[-1, -1] = 127
    assert O.igemm(qa, qb).tolist() == O.py_igemm(qa.tolist(), qb.tolist())
    mi = np.array([0, M - 1, M // 2], dtype=np.int64)
    ni = np.array([N - 1, 0, N // 2], dtype=np.int64)
    full = O.py_igemm(qa.tolist(), qb.tolist())
    assert O.igemm_pairs(qa, qb, mi, ni).tolist() == [full[m][n] for m, n in zip(mi, ni)]


def test_igemm_extreme_accumulator_fits_int32_at_largest_k():
    K = 21504
    qa = np.full((1, K), -127, dtype=np.int8)
    qb = np.full((2, K), 127, dtype=np.int8)
    qb[1] = -127
    acc = O.igemm(qa, qb)
    assert acc[0, 0] == -127 * 127 * K and acc[0, 1] == 127 * 127 * K
    assert abs(acc).max() < 2 ** 31


def test_dequant_exact_rational():
    rng = np.random.default_rng(4)
    acc = rng.integers(-10 ** 6, 10 ** 6, (3, 4))
    sa = rng.uniform(0.01, 1, 3).astype(np.float32)
    sb = rng.uniform(0.001, 0.1, 4).astype(np.float32)
    bias = rng.standard_normal(4).astype(np.float32)
    y = O.dequant(acc, sa, sb, bias, 128)
    for m in range(3):
        for n in range(4):
            ex = Fraction(int(acc[m, n])) * Fraction(float(sa[m])) * Fraction(float(sb[n])) / 128 + Fraction(float(bias[n]))
            assert abs(Fraction(y[m, n]) - ex) <= abs(ex) * Fraction(1, 2 ** 50)
    y0 = O.dequant(acc, sa, sb, None, 0)
    assert np.allclose(y0, acc * sa[:, None].astype(np.float64) * sb[None, :].astype(np.float64), rtol=1e-15)


def test_gelu_closed_forms():
    acc = np.array([[0, 10 ** 6, -10 ** 6]], dtype=np.int64)
    y = O.dequant(acc, np.array([1e-3], np.float32), np.array([1.0, 1.0, 1.0], np.float32), None, 0, gelu=True)
    assert y[0, 0] == 0.0
    x1 = float(np.float32(1e-3)) * 1e6
    assert abs(y[0, 1] - x1) < 1e-12 * x1  # gelu(x) -> x for large x
    assert abs(y[0, 2]) < 1e-12           # gelu(x) -> 0 for large negative x


# ------------------------------------------------------------ the whole linear


def _tiny():
    from w8a8_int8_quantized_block_b200 import workloads as W
    x, w, bias = W.linear_inputs(W.TINY)
    return x, w.numpy(), bias.numpy()


def test_linear_close_to_unquantised_product():
    # The pages accept a block when its cosine to the reference is >= 0.995
    # ("HyperFlow H3 Flash MLX", "How they were checked"); one quantised linear
    # must sit well inside that.
    x, w, bias = _tiny()
    xb = O.bf16_bits(x)
    y, *_ = O.linear(xb, w, bias, 128)
    ref = O.bf16_bits_to_f32(xb).astype(np.float64) @ w.T.astype(np.float64) + bias
    cos = (y * ref).sum() / np.sqrt((y * y).sum() * (ref * ref).sum())
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert cos > 0.999 and rel < 0.03


def test_rotation_reduces_error_with_outlier_channels():
    x, w, bias = _tiny()
    xb = O.bf16_bits(x)
    ref = O.bf16_bits_to_f32(xb).astype(np.float64) @ w.T.astype(np.float64) + bias
    err = {}
    for b in (0, 128):
        y, *_ = O.linear(xb, w, bias, b)
        err[b] = np.linalg.norm(y - ref)
    assert err[128] < 0.8 * err[0]


def test_rotated_linear_equals_unrotated_math_on_exact_inputs():
    # With integer inputs every step before rounding is exact, and
    # (H x) . (H w) / b = x . w: the rotation cancels in the product.
    rng = np.random.default_rng(12)
    b = 128
    xz = rng.integers(-3, 4, (2, b)).astype(np.float32)
    wz = rng.integers(-3, 4, (3, b)).astype(np.float32)
    zx = np.stack([O.fwht(r, b) for r in xz]).astype(np.int64)
    zw = np.stack([O.fwht(r, b) for r in wz]).astype(np.int64)
    assert ((zx @ zw.T) == b * (xz.astype(np.int64) @ wz.astype(np.int64).T)).all()


@pytest.mark.parametrize("block", [128, 0])
def test_quantiser_rounds_the_f32_product_before_the_integer(block):
    # Rows where f32(z * inv) is exactly 63.5 but z * inv is a little below:
    # rounding twice gives 64 (ties to even), rounding the exact product once
    # would give 63.  Every such element must come out as +-64.
    from near_ties import plain_rows, rotated_rows
    x = rotated_rows() if block == 128 else plain_rows()
    q, s = O.quantize_act(_bf16(x), block)
    half = np.abs(x) > 0
    assert (np.abs(q) == 64).sum() >= x.shape[0]
    assert not (np.abs(q) == 63).any()
    if block == 0:
        # the a/2 entries are exactly the near-tie elements
        assert ((np.abs(q) == 64) == (half & (np.abs(x) < x.max(axis=1, keepdims=True)))).all()



# ------------------------------------------------------------ regular rotation H_4^(x)k


@pytest.mark.parametrize("b", [16, 64, 256])
def test_regular_rotation_equals_explicit_matrix_on_integers(b):
    rng = np.random.default_rng(b + 1)
    x = rng.integers(-1000, 1000, size=3 * b).astype(np.float32)  # every fp32 op exact
    z = O.fwht(x, b, regular=True)
    exact = O.py_fwht_exact([int(v) for v in x], b, regular=True)
    assert [Fraction(float(v)) for v in z] == exact


@pytest.mark.parametrize("b", [16, 64, 256])
def test_regular_rotation_is_involution_up_to_b(b):
    rng = np.random.default_rng(b + 2)
    x = rng.integers(-500, 500, size=2 * b).astype(np.float32)
    assert (O.fwht(O.fwht(x, b, regular=True), b, regular=True) == b * x).all()


@pytest.mark.parametrize("b", [16, 64, 256])
def test_regular_rotation_f32_within_error_bound(b):
    # k = log4(b) radix-4 stages; each output of a stage is t - 2x with
    # t = (x0 + x1) + (x2 + x3): three roundings per stage, each bounded by
    # 2^-24 times the sum of the magnitudes feeding it, so the error stays
    # within 3k * 2^-24 * sum|x| of the block (first order).
    # f32 inputs (the weight path), so that the sums do round.
    k = {16: 2, 64: 3, 256: 4}[b]
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 2 * b)).astype(np.float32)
    x[:, 3] *= 30
    z = np.stack([O.fwht(r, b, regular=True) for r in x])
    exact = O.rotate_explicit_f64(x, b, regular=True)
    absx = np.abs(x).reshape(6, 2, b).sum(-1)
    bound = 3 * k * 2.0 ** -24 * np.repeat(absx, b, axis=1) * 1.0001
    assert (np.abs(z - exact) <= bound).all()
    assert np.abs(z - exact).max() > 0


@pytest.mark.parametrize("b", [16, 64, 256])
def test_regular_rotation_of_constant_block_stays_constant(b):
    # DC-balanced: x = c 1 gives z = sqrt(b) c 1, so every code is 127
    c = 0.75
    x = np.full((1, 2 * b), c, dtype=np.float32)
    q, s = O.quantize_act(_bf16(x), b, regular=True)
    assert (q[0] == 127).all()
    assert s[0] == np.float32(b ** 0.5 * c) / np.float32(127)
    qw, sw = O.pack_weight(x, b, regular=True)
    assert (qw[0] == 127).all() and sw[0] == s[0]


@pytest.mark.parametrize("b,i", [(16, 0), (16, 11), (64, 37), (256, 200)])
def test_regular_rotation_of_spike_gives_column_signs(b, i):
    c = -3.0
    x = np.zeros((1, b), dtype=np.float32)
    x[0, i] = c
    q, s = O.quantize_act(_bf16(x), b, regular=True)
    H = O.hadamard_regular_kron(b)
    assert (q[0] == (-127 * H[:, i])).all()
    assert s[0] == np.float32(3.0) / np.float32(127)


@pytest.mark.parametrize("b,regular", [(64, False), (256, False), (16, True), (64, True), (256, True)])
def test_linear_with_other_blocks_matches_unquantised_product(b, regular):
    # H_b H_b^T = b I for both kinds, so the rotated codes dequantised with
    # alpha = 1/b approximate x W^T + bias; quantisation error bounds the gap
    rng = np.random.default_rng(b + regular)
    M, K, N = 24, 512, 40
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, 9] *= 25
    xb = _bf16(x)
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.01).astype(np.float32)
    y, *_ = O.linear(xb, w, bias, b, regular=regular)
    ref = O.bf16_bits_to_f32(xb).astype(np.float64) @ w.T.astype(np.float64) + bias
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 0.02
    # rotating spreads the outlier channel: the error is well below no rotation
    y0, *_ = O.linear(xb, w, bias, 0)
    assert rel < np.linalg.norm(y0 - ref) / np.linalg.norm(ref)


# ------------------------------------------------------------ activation prologue (down projection)

# Standard normal CDF from printed tables: Phi(0.5), Phi(1), Phi(2), Phi(3);
# Phi(-x) = 1 - Phi(x); Phi(-10) = 7.619853024160527e-24.
_PHI = {0.5: 0.6914624612740131, 1.0: 0.8413447460685429, 2.0: 0.9772498680518208, 3.0: 0.9986501019683699}


def test_gelu_is_h_times_the_normal_cdf():
    h, expect = [0.0], [0.0]
    for x, p in _PHI.items():
        h += [x, -x]
        expect += [x * p, -x * (1.0 - p)]
    h += [10.0, -10.0]
    expect += [10.0, -10.0 * 7.619853024160527e-24]
    a = O.act_f32(_bf16([h]), O.ACT_GELU)[0]
    assert (a == np.array(expect, dtype=np.float32)).all(), (a, np.array(expect, dtype=np.float32))


def test_gelu_odd_part_is_the_identity():
    # gelu(x) - gelu(-x) = x Phi(x) + x Phi(-x) = x: each side is rounded
    # once to f32, so the identity holds to one ulp of x
    rng = np.random.default_rng(21)
    x = O.bf16_bits_to_f32(_bf16(rng.standard_normal(4096) * 3))
    a = O.act_f32(_bf16([x]), O.ACT_GELU)[0].astype(np.float64)
    b = O.act_f32(_bf16([-x]), O.ACT_GELU)[0].astype(np.float64)
    assert (np.abs(a - b - x) <= np.spacing(np.abs(x).astype(np.float32)).astype(np.float64) + 1e-45).all()


def test_silu_and_swiglu_closed_forms_gate_first():
    # silu(g) = g / (1 + e^-g): silu(2) = 2/(1 + e^-2), silu(-2), silu(1)
    s2, sm2, s1 = 1.7615941559557646, -0.2384058440442351, 0.7310585786300049
    g = [2.0, -2.0, 1.0, 0.0, 20.0]
    u = [3.0, 0.5, -4.0, 7.0, 1.0]
    a = O.act_f32(_bf16([g + u]), O.ACT_SWIGLU)[0]
    expect = np.array([3 * s2, 0.5 * sm2, -4 * s1, 0.0, 20.0], dtype=np.float32)
    assert (a == expect).all(), (a, expect)


def test_silu_odd_part_is_the_identity():
    # silu(x) - silu(-x) = x (sigmoid(x) + sigmoid(-x) = 1), with u = 1
    rng = np.random.default_rng(22)
    x = O.bf16_bits_to_f32(_bf16(rng.standard_normal(2048) * 4))
    one = np.ones_like(x)
    a = O.act_f32(_bf16([np.concatenate([x, one])]), O.ACT_SWIGLU)[0].astype(np.float64)
    b = O.act_f32(_bf16([np.concatenate([-x, one])]), O.ACT_SWIGLU)[0].astype(np.float64)
    assert (np.abs(a - b - x) <= np.spacing(np.abs(x).astype(np.float32)).astype(np.float64) + 1e-45).all()


@pytest.mark.parametrize("b,regular", [(0, False), (64, False), (128, False), (64, True)])
def test_act_none_prologue_is_the_plain_quantiser(b, regular):
    rng = np.random.default_rng(23)
    h = _bf16(rng.standard_normal((9, 256)) * 2)
    q1, s1 = O.act_quantize(h, O.ACT_NONE, b, regular)
    q2, s2 = O.quantize_act(h, b, regular)
    assert (q1 == q2).all() and (s1.view(np.uint32) == s2.view(np.uint32)).all()


@pytest.mark.parametrize("act", [1, 2])
def test_down_projection_with_prologue_matches_unquantised_product(act):
    # the prologue's codes times the packed down weights approximate
    # act(h) W^T, with act from the library's erf / exp in fp64
    import math
    rng = np.random.default_rng(24 + act)
    M, K, N = 20, 512, 48
    h = rng.standard_normal((M, 2 * K if act == 2 else K)) * 1.5
    hb = _bf16(h)
    hf = O.bf16_bits_to_f32(hb).astype(np.float64)
    if act == 1:
        x = hf * 0.5 * np.vectorize(math.erfc)(-hf / math.sqrt(2.0))
    else:
        g, u = hf[:, :K], hf[:, K:]
        x = g / (1.0 + np.exp(-g)) * u
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    for b in (64, 128):
        qx, sx = O.act_quantize(hb, act, b)
        qw, sw = O.pack_weight(w, b)
        y = O.dequant(O.igemm(qx, qw), sx, sw, None, b)
        ref = x @ w.T.astype(np.float64)
        assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.02


# ------------------------------------------------------------ int8 attention (f3)


def _qkv(H, Lq, Lk, d, seed, qs=1.0):
    rng = np.random.default_rng(seed)
    q = _bf16(rng.standard_normal((H * Lq, d)) * qs).reshape(H, Lq, d)
    k = _bf16(rng.standard_normal((H * Lk, d))).reshape(H, Lk, d)
    v = _bf16(rng.standard_normal((H * Lk, d))).reshape(H, Lk, d)
    return q, k, v


def test_attention_matches_plain_python_loops():
    q, k, v = _qkv(1, 5, 7, 8, 31)
    att, (qx, sq, kx, sk) = O.attention(q, k, v)
    ref = O.py_attention_exact_scores(qx[0].astype(int).tolist(), sq[0].astype(float).tolist(),
                                      kx[0].astype(int).tolist(), sk[0].astype(float).tolist(),
                                      O.bf16_bits_to_f32(v[0]).astype(float).tolist(), 1.0 / np.sqrt(8))
    assert np.allclose(att[0], np.array(ref), rtol=1e-12, atol=1e-12)


def test_attention_of_constant_values_is_that_constant():
    # softmax rows sum to one: V = c everywhere gives O = c
    q, k, _ = _qkv(2, 16, 24, 32, 32)
    v = _bf16(np.full((2 * 24, 32), 0.625)).reshape(2, 24, 32)
    att, _ = O.attention(q, k, v)
    assert np.allclose(att, 0.625, rtol=0, atol=1e-14)


def test_attention_of_zero_queries_is_the_mean_of_values():
    # a zero query row has s_q = 0: every score is 0, P is uniform
    q, k, v = _qkv(1, 4, 20, 16, 33)
    q[:] = 0
    att, _ = O.attention(q, k, v)
    assert np.allclose(att[0], O.bf16_bits_to_f32(v[0]).astype(np.float64).mean(axis=0), atol=1e-14)


def test_attention_is_invariant_to_a_joint_permutation_of_keys_and_values():
    q, k, v = _qkv(1, 8, 40, 16, 34)
    perm = np.random.default_rng(0).permutation(40)
    a1, _ = O.attention(q, k, v)
    a2, _ = O.attention(q, k[:, perm], v[:, perm])
    assert np.allclose(a1, a2, rtol=1e-12, atol=1e-14)


def test_attention_picks_out_a_dominant_key():
    # query and one key along the same axis with a large scale: the softmax
    # puts almost all weight on that key
    d = 16
    q = np.zeros((1, 2, d)); q[0, :, 0] = 16.0
    k = np.random.default_rng(35).standard_normal((1, 10, d)) * 0.1
    k[0, 6, :] = 0.0; k[0, 6, 0] = 16.0  # score 16 * 16 / sqrt(16) = 64 against ~0.3
    v = np.random.default_rng(36).standard_normal((1, 10, d))
    att, _ = O.attention(_bf16(q.reshape(2, d)).reshape(1, 2, d), _bf16(k.reshape(10, d)).reshape(1, 10, d),
                       _bf16(v.reshape(10, d)).reshape(1, 10, d))
    v6 = O.bf16_bits_to_f32(_bf16(v[0, 6:7]))[0]
    assert np.abs(att[0] - v6).max() < 1e-12


def test_attention_scores_are_the_dequantised_qk_product():
    # S is the config-5 skinny-K GEMM's output (before bf16) times the scale
    q, k, v = _qkv(1, 6, 9, 128, 37)
    a1, (qx, sq, kx, sk) = O.attention(q, k, v, scale=0.5)
    S = O.dequant(O.igemm(qx[0], kx[0]), sq[0], sk[0], None, 0) * 0.5
    P = np.exp(S - S.max(1, keepdims=True)); P /= P.sum(1, keepdims=True)
    assert np.allclose(a1[0], P @ O.bf16_bits_to_f32(v[0]).astype(np.float64), rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ inputs outside the contract

@pytest.mark.parametrize("bad", [0x7F80, 0xFF80, 0x7FC0, 0x7F81])  # +inf, -inf, quiet and signalling NaN
def test_oracle_refuses_non_finite_bf16_inputs(bad):
    x = np.full((3, 256), 0x3F80, dtype=np.uint16)  # 1.0
    x[1, 77] = bad
    with pytest.raises(ValueError):
        O.quantize_act(x, 128)
    with pytest.raises(ValueError):
        O.act_quantize(x, O.ACT_GELU, 128)
    # the largest finite bf16 magnitudes are inside the contract
    x[1, 77] = 0x7F7F
    q, s = O.quantize_act(x, 128)
    assert np.isfinite(s).all() and np.abs(q).max() == 127


@pytest.mark.parametrize("bad", [np.inf, -np.inf, np.nan])
def test_oracle_refuses_non_finite_weights(bad):
    w = np.ones((4, 128), dtype=np.float32)
    w[2, 5] = bad
    with pytest.raises(ValueError):
        O.pack_weight(w, 128)
