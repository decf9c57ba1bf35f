"""Pins for the CPU oracle, independent of the oracle's own formulas.

Each check comes from something other than the oracle itself: the
mathematics of the definitions (closed forms, invariants, special cases),
library routines that implement the same definition (torch CPU float64),
high-precision brute force (mpmath), or exhaustive enumeration (bf16).
They are chosen so that a plausible slip in the oracle -- a dropped cubic
term, a wrong constant, a sign error, a missing max subtraction, a wrong
axis, a bad rounding rule -- fails at least one of them.

Definitions:
  GELU (tanh form): lecture-6 notes (kyc001.github.io), section 4.2.
  Row softmax: lecture 6 (cs336.sjfarmltd.com), section 7.2; lecture-6
  notes, section 5.2.
"""
import math

import mpmath
import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(12345)


# ====================================================================== GELU

def test_gelu_zero_and_signed_zero():
    assert oracle.gelu_tanh(0.0) == 0.0
    assert oracle.gelu_tanh(-0.0) == 0.0


def test_gelu_odd_part_identity():
    # tanh is odd, so 0.5x(1+t) - (0.5(-x)(1-t)) = x exactly in real
    # arithmetic: GELU(x) - GELU(-x) = x.
    x = np.concatenate([np.linspace(-20, 20, 40001), RNG.standard_normal(10000) * 5])
    d = oracle.gelu_tanh_f64(x) - oracle.gelu_tanh_f64(-x)
    assert np.all(np.abs(d - x) <= 4e-16 * np.maximum(np.abs(x), 1e-300) + 1e-300)


def test_gelu_large_arguments_tend_to_identity_and_zero():
    big = np.linspace(10, 1e4, 5001)
    y = oracle.gelu_tanh_f64(big)
    # tanh(u) == 1 in double once u > ~19; the fp32 rounding is then x itself
    assert np.array_equal(oracle.round_to_f32(y), big.astype(np.float32))
    neg = -big
    yn = oracle.gelu_tanh_f64(neg)
    assert np.all(np.abs(yn) < 1e-30)


def test_gelu_special_values():
    assert oracle.gelu_tanh(math.inf) == math.inf
    r = oracle.gelu_tanh(-math.inf)
    assert r == 0.0 and math.copysign(1.0, r) == -1.0
    assert math.isnan(oracle.gelu_tanh(math.nan))
    # cubic overflow to +-inf inside the tanh argument still gives the limits
    assert oracle.gelu_tanh(1e200) == 1e200
    assert oracle.gelu_tanh(-1e200) == 0.0


def test_gelu_matches_torch_tanh_gelu_float64():
    # torch.nn.functional.gelu(approximate='tanh') implements the same
    # definition independently.
    x = np.concatenate([np.linspace(-20, 20, 100001), RNG.standard_normal(100000) * 3])
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    y = oracle.gelu_tanh_f64(x)
    assert np.max(np.abs(y - ref)) <= 1e-14


def test_gelu_is_within_tanh_approximation_error_of_exact_gelu():
    # x * Phi(x) with Phi from erf is the exact GELU; the tanh form is known to
    # differ from it by at most ~4.7e-4 (largest near x = -2.7).  Dropping the
    # cubic term pushes the gap above 1e-2; a different inner constant moves
    # both the size and the place of the largest gap.
    x = np.linspace(-10, 10, 200001)
    exact = np.array([v * 0.5 * (1.0 + math.erf(v / math.sqrt(2.0))) for v in x])
    gap = np.abs(oracle.gelu_tanh_f64(x) - exact)
    assert 4.6e-4 < gap.max() < 4.8e-4
    assert -2.75 < x[gap.argmax()] < -2.65


def test_gelu_sigmoid_form():
    # 0.5 x (1 + tanh(u)) = x / (1 + exp(-2u)) -- a second closed form
    x = np.linspace(-12, 12, 24001)
    u = math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)
    alt = x / (1.0 + np.exp(-2.0 * u))
    y = oracle.gelu_tanh_f64(x)
    assert np.max(np.abs(y - alt)) <= 1e-15 * 12


def test_gelu_brute_force_mpmath():
    mpmath.mp.dps = 50
    xs = np.concatenate([np.linspace(-20, 20, 1201), RNG.standard_normal(800) * 4])
    c = mpmath.sqrt(2 / mpmath.pi)
    for x in xs:
        xm = mpmath.mpf(float(x))
        exact = mpmath.mpf("0.5") * xm * (1 + mpmath.tanh(c * (xm + mpmath.mpf("0.044715") * xm ** 3)))
        got = oracle.gelu_tanh(float(x))
        # double evaluation: a few roundings of relative size 2^-53 in the
        # inputs of tanh and of the final product; bounded in absolute terms
        assert abs(mpmath.mpf(got) - exact) <= 8e-16 * max(abs(float(x)), 1.0), x


def test_gelu_negative_tail_relative_accuracy_mpmath():
    # For x < 0 GELU is tiny (GELU(-8) ~ -3e-21; GELU(-10.2) ~ -1e-39, a bf16
    # subnormal), and a bf16 comparison needs it to relative accuracy, not
    # merely within 1e-16 absolute.  mpmath evaluates the defining formula
    # with enough digits that 1 + tanh(u) keeps ~40 significant ones.
    xs = np.concatenate([-np.linspace(0.01, 21.5, 2150), -np.abs(RNG.standard_normal(300)) * 8])
    for x in xs:
        xm = mpmath.mpf(float(x))
        with mpmath.workdps(40):
            u0 = float(mpmath.sqrt(2 / mpmath.pi) * (xm + mpmath.mpf("0.044715") * xm ** 3))
        with mpmath.workdps(40 + int(2 * abs(u0) / 2.302585) + 1):
            c = mpmath.sqrt(2 / mpmath.pi)
            u = c * (xm + mpmath.mpf("0.044715") * xm ** 3)
            exact = mpmath.mpf("0.5") * xm * (1 + mpmath.tanh(u))
            got = oracle.gelu_tanh(float(x))
            # u carries up to ~6 roundings (sqrt(2/pi), the cube, the sum, the
            # products), relative 6 * 2^-53 in all, so e^(2u) is off by up to
            # 2|u| * 6 * 2^-53 = 6|u| * 2^-52 relative, plus a few roundings
            # after it.  Once e^(2u) is a double subnormal (x < ~-20.5) it holds
            # only to its spacing 2^-1074, which the product with x scales by |x|.
            tol = (6 * abs(u0) + 6) * 2.3e-16 * abs(exact) + (abs(float(x)) + 1) * mpmath.mpf(2) ** -1074
            assert abs(mpmath.mpf(got) - exact) <= tol, (x, got, exact)


def test_gelu_f32_wrapper_rounds_the_double_result_once():
    x = (RNG.standard_normal(100000) * 6).astype(np.float32)
    via64 = oracle.round_to_f32(oracle.gelu_tanh_f64(x.astype(np.float64)))
    assert np.array_equal(oracle.gelu_tanh_f32(x).view(np.uint32), via64.view(np.uint32))


def test_gelu_thread_count_invariance():
    x = RNG.standard_normal(100003) * 4
    a = oracle.gelu_tanh_f64(x, nthreads=1)
    b = oracle.gelu_tanh_f64(x, nthreads=7)
    assert np.array_equal(a, b)


# =============================================================== exact GELU

def test_gelu_erf_textbook_quantiles():
    # Phi(1.959963985) = 0.975 and Phi(1.644853627) = 0.95 (standard normal
    # table), Phi(0) = 1/2, Phi(-x) = 1 - Phi(x)
    for z, p in ((1.959963984540054, 0.975), (1.6448536269514722, 0.95), (0.0, 0.5)):
        if z != 0.0:
            assert abs(oracle.gelu_erf(z) / z - p) <= 1e-15
            assert abs(oracle.gelu_erf(-z) / -z - (1 - p)) <= 1e-15
    assert oracle.gelu_erf(0.0) == 0.0


def test_gelu_erf_odd_part_identity_and_limits():
    x = np.concatenate([np.linspace(-30, 30, 60001), RNG.standard_normal(10000) * 5])
    d = oracle.gelu_erf_f64(x) - oracle.gelu_erf_f64(-x)
    assert np.all(np.abs(d - x) <= 4e-16 * np.maximum(np.abs(x), 1e-300) + 1e-300)
    assert oracle.gelu_erf(math.inf) == math.inf
    r = oracle.gelu_erf(-math.inf)
    assert r == 0.0 and math.copysign(1.0, r) == -1.0
    assert math.isnan(oracle.gelu_erf(math.nan))
    assert np.all(np.abs(oracle.gelu_erf_f64(-np.linspace(40, 100, 61))) < 1e-300)


def test_gelu_erf_matches_torch_exact_gelu_float64():
    x = np.concatenate([np.linspace(-20, 20, 100001), RNG.standard_normal(100000) * 3])
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="none").numpy()
    assert np.max(np.abs(oracle.gelu_erf_f64(x) - ref)) <= 1e-14


def test_gelu_erf_brute_force_mpmath_in_the_tail():
    # relative accuracy also deep in the negative tail, where 1 + erf loses it
    mpmath.mp.dps = 50
    for v in list(np.linspace(-38, 8, 461)):
        xm = mpmath.mpf(float(v))
        exact = xm * mpmath.ncdf(xm)
        got = oracle.gelu_erf(float(v))
        # error bound of the double evaluation: d ln erfc(z)/dz ~ -(2z + 1/z)
        # in the tail, so a relative error d in z = -x/sqrt(2) moves the result
        # by (2 z^2 + 1) d = (x^2 + 1) d; z carries two roundings (sqrt(2), the
        # division), d <= 2 * 2^-53; erfc itself adds a few ulp; and an
        # absolute 1e-300 where the double result nears underflow (far below
        # the smallest fp32/bf16 output, 1.4e-45)
        tol = (float(v) ** 2 + 5.0) * 2.3e-16 * abs(exact) + 1e-300
        assert abs(mpmath.mpf(got) - exact) <= tol, v


# =================================================================== softmax

@pytest.mark.parametrize("cols", [1, 2, 3, 1000, 4096, 131072])
def test_softmax_rows_sum_to_one(cols):
    rows = max(1, 2 ** 18 // cols)
    x = RNG.standard_normal((rows, cols)) * 4
    y = oracle.softmax_rows_f64(x)
    s = y.sum(axis=1, dtype=np.float64)
    assert np.max(np.abs(s - 1.0)) <= 1e-12


def test_softmax_sums_along_rows_not_columns():
    x = RNG.standard_normal((3, 7)) * 2
    y = oracle.softmax_rows_f64(x)
    assert np.allclose(y.sum(axis=1), 1.0, atol=1e-14)
    assert not np.allclose(y.sum(axis=0), 1.0, atol=1e-3)


def test_softmax_shift_invariance_bit_exact():
    # multiples of 2^-10 in [-64, 64] plus an integer shift stay exact in
    # double, so x_j - max(x) is the same number and the outputs are equal.
    x = np.round(RNG.uniform(-64, 64, (64, 777)) * 1024) / 1024
    for c in (1.0, -37.0, 1024.0):
        assert np.array_equal(oracle.softmax_rows_f64(x), oracle.softmax_rows_f64(x + c))


@pytest.mark.parametrize("n", [1, 1000, 4096, 131072])
def test_softmax_constant_row_gives_one_over_n(n):
    x = np.full((2, n), 3.25)
    y = oracle.softmax_rows_f64(x)
    assert np.all(y == 1.0 / n)


def test_softmax_one_huge_entry_is_one_hot():
    x = RNG.standard_normal((5, 300)) * 3
    k = RNG.integers(0, 300, 5)
    x[np.arange(5), k] += 1000.0
    y = oracle.softmax_rows_f64(x)
    expect = np.zeros_like(y)
    expect[np.arange(5), k] = 1.0
    assert np.array_equal(y, expect)


def test_softmax_two_element_closed_form():
    a = RNG.standard_normal(2000) * 10
    b = RNG.standard_normal(2000) * 10
    y = oracle.softmax_rows_f64(np.stack([a, b], axis=1))
    sig = lambda d: 1.0 / (1.0 + np.exp(-d))  # noqa: E731
    assert np.max(np.abs(y[:, 0] - sig(a - b))) <= 2e-16
    assert np.max(np.abs(y[:, 1] - sig(b - a))) <= 2e-16


def test_softmax_ratio_of_outputs_is_exp_of_difference():
    x = RNG.standard_normal((10, 50)) * 3
    y = oracle.softmax_rows_f64(x)
    r = y[:, 1:] / y[:, :1]
    assert np.allclose(r, np.exp(x[:, 1:] - x[:, :1]), rtol=1e-14, atol=0)


def test_softmax_permutation_equivariance():
    x = RNG.standard_normal((8, 513)) * 5
    p = RNG.permutation(513)
    assert np.allclose(oracle.softmax_rows_f64(x[:, p]), oracle.softmax_rows_f64(x)[:, p],
                       rtol=0, atol=1e-16)


def test_softmax_neg_inf_entries_are_exact_zeros_and_causal_row():
    x = RNG.standard_normal((4, 64)) * 4
    x[:, ::3] = -np.inf
    y = oracle.softmax_rows_f64(x)
    assert np.all(y[:, ::3] == 0.0)
    assert np.allclose(y.sum(axis=1), 1.0, atol=1e-14)
    # causal mask, query 0: only key 0 is visible -> exactly [1, 0, ..., 0]
    t = 16
    s = RNG.standard_normal((t, t)) * 8
    s[np.triu_indices(t, 1)] = -np.inf
    ys = oracle.softmax_rows_f64(s)
    assert ys[0, 0] == 1.0 and np.all(ys[0, 1:] == 0.0)
    assert np.all(ys[np.triu_indices(t, 1)] == 0.0)


def test_softmax_degenerate_rows_are_nan():
    x = np.zeros((3, 5))
    x[0, :] = -np.inf         # all -inf: 0/0
    x[1, 2] = np.nan          # any NaN
    x[2, 4] = np.inf          # a +inf: inf - inf
    y = oracle.softmax_rows_f64(x)
    assert np.all(np.isnan(y))


def test_softmax_matches_torch_float64():
    for cols in (1, 7, 1000, 4096):
        x = RNG.standard_normal((64, cols)) * 6
        x[:, ::5] = -np.inf if cols > 1 else x[:, ::5]
        ref = torch.softmax(torch.from_numpy(x), dim=-1).numpy()
        # torch's vectorised exp and summation order differ from libm's by a
        # few double ulps; outputs are <= 1, so 1e-14 is ~50 ulps of 1.0
        assert np.max(np.abs(oracle.softmax_rows_f64(x) - ref)) <= 1e-14


def test_softmax_brute_force_mpmath():
    mpmath.mp.dps = 50
    for n in (1, 2, 5, 17, 100):
        for _ in range(4):
            x = RNG.standard_normal(n) * 6
            xm = [mpmath.mpf(float(v)) for v in x]
            den = mpmath.fsum(mpmath.exp(v) for v in xm)
            exact = [mpmath.exp(v) / den for v in xm]
            y = oracle.softmax_rows_f64(x.reshape(1, n))[0]
            m = float(np.max(x))
            for got, ex, xj in zip(y, exact, x):
                # error bound of the double evaluation: rounding x_j - m costs
                # |x_j - m| * 2^-53 in the exponent; exp, the compensated sum
                # and the division add a few units of 2^-53 relative
                tol = (abs(xj - m) * 1.2e-16 + 8e-16) * ex
                assert abs(mpmath.mpf(float(got)) - ex) <= tol + 1e-300


def test_softmax_online_recurrence_gives_the_same_normaliser():
    # The running (max, sum) recurrence of lecture 6, section 7.2, applied
    # block by block, must reach the same max and normaliser as the two-pass
    # definition; it is a different algorithm for the same quantity.
    x = RNG.standard_normal(5000) * 7
    x[::11] = -np.inf
    m_prev, l_prev = -math.inf, 0.0
    for blk in np.array_split(x, 37):
        m_cur = max(m_prev, float(np.max(blk)))
        corr = math.exp(m_prev - m_cur) if m_prev != -math.inf else 0.0
        l_prev = corr * l_prev + float(np.sum(np.exp(blk - m_cur)))
        m_prev = m_cur
    y_online = np.exp(x - m_prev) / l_prev
    y = oracle.softmax_rows_f64(x.reshape(1, -1))[0]
    assert np.max(np.abs(y - y_online)) <= 1e-16 * 50


def test_softmax_f32_and_bf16_wrappers_round_once():
    x = (RNG.standard_normal((33, 1001)) * 4).astype(np.float32)
    x[:, ::7] = -np.inf
    ref = oracle.round_to_f32(oracle.softmax_rows_f64(x.astype(np.float64)))
    assert np.array_equal(oracle.softmax_rows_f32(x).view(np.uint32), ref.view(np.uint32))
    xb = oracle.round_to_bf16((RNG.standard_normal((17, 2048)) * 8))
    xb[:, 1000:] = 0xFF80  # -inf
    refb = oracle.round_to_bf16(oracle.softmax_rows_f64(oracle.bf16_to_f64(xb)))
    assert np.array_equal(oracle.softmax_rows_bf16(xb), refb)


def test_softmax_thread_count_invariance():
    x = RNG.standard_normal((101, 333)) * 3
    assert np.array_equal(oracle.softmax_rows_f64(x, nthreads=1), oracle.softmax_rows_f64(x, nthreads=5))


# ======================================================= causal softmax
# Scaled, causally masked softmax (lecture 6, "GPU Kernels and Triton",
# section 8): row r keeps columns j <= (r mod period) + offset, scores
# scale * x_j, -inf for the rest, then softmax.


def _torch_causal(x, scale, period, offset):
    """Independent construction: a boolean mask from torch.triu over each
    [period, cols] block (True strictly above the diagonal shifted by offset),
    masked_fill with -inf, then torch.softmax, all in float64."""
    t = torch.from_numpy(x) * scale
    rows, cols = x.shape
    if period:
        block = torch.triu(torch.ones(period, cols, dtype=torch.bool), diagonal=offset + 1)
        mask = block.repeat(-(-rows // period), 1)[:rows]
        t = t.masked_fill(mask, float("-inf"))
    return torch.softmax(t, dim=-1).numpy()


@pytest.mark.parametrize("rows,cols,scale,period,offset", [
    (64, 64, 0.125, 64, 0), (96, 48, 1.0, 32, 0), (50, 80, 0.3, 50, 30), (40, 33, 2.5, 7, 3),
    (17, 17, 1.0, 0, 0), (30, 20, 0.7, 100, 0), (12, 9, 1.3, 4, 50)])
def test_causal_softmax_matches_torch_masked_fill(rows, cols, scale, period, offset):
    x = RNG.standard_normal((rows, cols)) * 4
    y = oracle.softmax_rows_causal(x, scale, period, offset)
    ref = _torch_causal(x, scale, period, offset)
    assert np.max(np.abs(y - ref)) <= 1e-14
    assert np.array_equal(y == 0.0, ref == 0.0)


def test_causal_softmax_first_rows_closed_form():
    # row 0 of a block keeps offset + 1 columns; with offset 0 it is one-hot on
    # column 0, and row 1 is the two-element softmax 1 / (1 + e^(s(x0 - x1)))
    x = RNG.standard_normal((8, 6)) * 3
    s = 0.4
    y = oracle.softmax_rows_causal(x, s, period=4)
    assert list(y[0]) == [1.0, 0, 0, 0, 0, 0] and list(y[4]) == [1.0, 0, 0, 0, 0, 0]
    p0 = 1.0 / (1.0 + math.exp(s * (x[1, 1] - x[1, 0])))
    assert abs(y[1, 0] - p0) <= 2e-16 and abs(y[1, 1] - (1 - p0)) <= 2e-16
    assert np.all(y[1, 2:] == 0.0)
    # with offset 2 the first row keeps 3 columns
    y2 = oracle.softmax_rows_causal(x, s, period=4, offset=2)
    assert np.all(y2[0, 3:] == 0.0) and np.all(y2[0, :3] > 0.0)


def test_causal_softmax_invariants():
    x = RNG.standard_normal((120, 70)) * 5
    y = oracle.softmax_rows_causal(x, 0.25, period=40, offset=10)
    q = (np.arange(120) % 40) + 10
    kept = np.arange(70)[None, :] <= q[:, None]
    assert np.all(y[~kept] == 0.0)            # masked: exactly 0
    assert np.all(y[kept] > 0.0)
    assert np.max(np.abs(y.sum(axis=1) - 1.0)) <= 1e-14
    # the scale multiplies the scores: scaling x instead gives the same result
    z = oracle.softmax_rows_causal(x * 0.25, 1.0, period=40, offset=10)
    assert np.max(np.abs(y - z)) <= 1e-15
    # a constant added to a row changes nothing (up to the rounding of x + c)
    w = oracle.softmax_rows_causal(x + 3.0, 0.25, period=40, offset=10)
    assert np.max(np.abs(y - w)) <= 1e-14


def test_causal_softmax_never_reads_masked_entries():
    x = RNG.standard_normal((32, 32))
    q = np.arange(32)
    x_bad = x.copy()
    x_bad[np.arange(32)[None, :] > q[:, None]] = np.nan
    a = oracle.softmax_rows_causal(x, 0.5, period=32)
    b = oracle.softmax_rows_causal(x_bad, 0.5, period=32)
    assert np.array_equal(a, b)


def test_causal_softmax_without_mask_and_unit_scale_is_plain_softmax():
    x = RNG.standard_normal((33, 257)) * 4
    assert np.array_equal(oracle.softmax_rows_causal(x, 1.0, period=0), oracle.softmax_rows_f64(x))


def test_causal_softmax_brute_force_mpmath():
    mpmath.mp.dps = 50
    x = RNG.standard_normal((7, 9)) * 3
    scale, period, offset = 0.37, 5, 2
    y = oracle.softmax_rows_causal(x, scale, period, offset)
    for r in range(7):
        q = r % period + offset
        s = [mpmath.mpf(scale) * mpmath.mpf(float(v)) for v in x[r, :q + 1]]
        m = max(s)
        e = [mpmath.exp(v - m) for v in s]
        tot = mpmath.fsum(e)
        for j in range(9):
            exact = e[j] / tot if j <= q else mpmath.mpf(0)
            assert abs(mpmath.mpf(float(y[r, j])) - exact) <= 4e-16


def test_causal_softmax_f32_and_bf16_round_the_double_result_once():
    x = (RNG.standard_normal((40, 50)) * 4).astype(np.float32)
    via64 = oracle.round_to_f32(oracle.softmax_rows_causal(x.astype(np.float64), 0.6, 16, 3))
    assert np.array_equal(oracle.softmax_rows_causal(x, 0.6, 16, 3).view(np.uint32), via64.view(np.uint32))
    b = oracle.round_to_bf16(x.astype(np.float64))
    via64b = oracle.round_to_bf16(oracle.softmax_rows_causal(oracle.bf16_to_f64(b), 0.6, 16, 3))
    assert np.array_equal(oracle.softmax_rows_causal(b, 0.6, 16, 3), via64b)


# ============================================================ LayerNorm
# LayerNorm over rows (lecture 6, "GPU Kernels and Triton", sections 6.1-6.2:
# F.layer_norm(x, x.shape[-1:])), optional affine, optional GELU.


@pytest.mark.parametrize("rows,cols,eps,affine,gelu", [
    (16, 7, 1e-5, False, None), (64, 4096, 1e-5, True, None), (33, 1000, 1e-6, True, "tanh"),
    (9, 131, 1e-3, False, "erf"), (5, 1, 1e-5, True, None), (3, 65537, 1e-5, True, "erf")])
def test_layernorm_matches_torch_float64(rows, cols, eps, affine, gelu):
    x = RNG.standard_normal((rows, cols)) * RNG.uniform(0.1, 5, (rows, 1)) + RNG.uniform(-3, 3, (rows, 1))
    g = RNG.standard_normal(cols) * 0.3 + 1 if affine else None
    b = RNG.standard_normal(cols) * 0.3 if affine else None
    y = oracle.layernorm_rows(x, eps, g, b, gelu)
    t = torch.nn.functional.layer_norm(torch.from_numpy(x), (cols,),
                                       None if g is None else torch.from_numpy(g),
                                       None if b is None else torch.from_numpy(b), eps)
    if gelu:
        t = torch.nn.functional.gelu(t, approximate="tanh" if gelu == "tanh" else "none")
    assert np.max(np.abs(y - t.numpy())) <= 1e-13


def test_layernorm_moments_and_constant_rows():
    # without affine and with eps = 0 each row has mean 0 and mean square 1;
    # with eps the mean square is var / (var + eps); a constant row is 0
    x = RNG.standard_normal((50, 300)) * 2.5 + 7.0
    y = oracle.layernorm_rows(x, 0.0)
    assert np.max(np.abs(y.mean(axis=1))) <= 1e-15 * 50
    assert np.max(np.abs((y * y).mean(axis=1) - 1.0)) <= 1e-14
    eps = 0.3
    ye = oracle.layernorm_rows(x, eps)
    var = x.var(axis=1)
    assert np.max(np.abs((ye * ye).mean(axis=1) - var / (var + eps))) <= 1e-14
    c = np.full((2, 10), 4.25)
    assert np.all(oracle.layernorm_rows(c) == 0.0)
    beta = np.arange(10.0)
    assert np.array_equal(oracle.layernorm_rows(c, 1e-5, np.full(10, 3.0), beta), np.tile(beta, (2, 1)))


def test_layernorm_two_element_closed_form():
    # [a, b]: mean (a + b)/2, var ((a - b)/2)^2, y = +-d / sqrt(d^2 + eps), d = |a - b| / 2
    for a, b, eps in ((1.0, 3.0, 1e-5), (-2.5, 4.0, 0.5), (10.0, 10.5, 1e-5)):
        d = abs(a - b) / 2
        v = d / math.sqrt(d * d + eps)
        y = oracle.layernorm_rows(np.array([[a, b]]), eps)[0]
        assert abs(y[0] - (-v if a < b else v)) <= 4e-16 and abs(y[1] - (v if a < b else -v)) <= 4e-16


def test_layernorm_shift_and_scale_invariance():
    x = RNG.standard_normal((40, 257))
    y = oracle.layernorm_rows(x, 0.0)
    assert np.max(np.abs(oracle.layernorm_rows(x + 1000.0, 0.0) - y)) <= 1e-11
    assert np.max(np.abs(oracle.layernorm_rows(x * 37.0, 0.0) - y)) <= 1e-14
    # with eps, scaling by a moves the result as sqrt(var / (var + eps / a^2))
    ya = oracle.layernorm_rows(x * 4.0, 1e-2)
    assert np.max(np.abs(ya - oracle.layernorm_rows(x, 1e-2 / 16.0))) <= 1e-14


def test_layernorm_affine_and_gelu_are_applied_after_normalising():
    x = RNG.standard_normal((8, 64)) * 3
    g, b = RNG.standard_normal(64), RNG.standard_normal(64)
    base = oracle.layernorm_rows(x, 1e-5)
    assert np.max(np.abs(oracle.layernorm_rows(x, 1e-5, g, b) - (base * g + b))) <= 1e-15 * 8
    z = base * g + b
    assert np.max(np.abs(oracle.layernorm_rows(x, 1e-5, g, b, "erf") - oracle.gelu_erf_f64(z))) <= 1e-14
    assert np.max(np.abs(oracle.layernorm_rows(x, 1e-5, g, b, "tanh") - oracle.gelu_tanh_f64(z))) <= 1e-14


def test_layernorm_brute_force_mpmath():
    mpmath.mp.dps = 50
    x = RNG.standard_normal((4, 13)) * 3 + 5
    eps = 1e-5
    y = oracle.layernorm_rows(x, eps)
    for r in range(4):
        v = [mpmath.mpf(float(t)) for t in x[r]]
        m = mpmath.fsum(v) / len(v)
        var = mpmath.fsum([(t - m) ** 2 for t in v]) / len(v)
        rs = 1 / mpmath.sqrt(var + mpmath.mpf(eps))
        for j in range(13):
            assert abs(mpmath.mpf(float(y[r, j])) - (v[j] - m) * rs) <= 2e-15


def test_layernorm_f32_and_bf16_round_the_double_result_once():
    x = (RNG.standard_normal((30, 200)) * 3).astype(np.float32)
    g, b = RNG.standard_normal(200), RNG.standard_normal(200)
    via = oracle.round_to_f32(oracle.layernorm_rows(x.astype(np.float64), 1e-5, g, b, "tanh"))
    assert np.array_equal(oracle.layernorm_rows(x, 1e-5, g, b, "tanh").view(np.uint32), via.view(np.uint32))
    xb = oracle.round_to_bf16(x.astype(np.float64))
    viab = oracle.round_to_bf16(oracle.layernorm_rows(oracle.bf16_to_f64(xb), 1e-5, g, b))
    assert np.array_equal(oracle.layernorm_rows(xb, 1e-5, g, b), viab)


# ============================================================ attention
# Attention forward (lecture 6, "GPU Kernels and Triton", sections 7.3 and 8):
# softmax(scale Q K^T with the causal mask) V per (batch, head) slice.


def _torch_attention(q, k, v, scale, causal):
    s = torch.from_numpy(q) @ torch.from_numpy(k).transpose(1, 2) * scale
    if causal:
        tq, tk = q.shape[1], k.shape[1]
        s = s.masked_fill(torch.ones(tq, tk, dtype=torch.bool).triu(1 + tk - tq), float("-inf"))
    return (torch.softmax(s, dim=-1) @ torch.from_numpy(v)).numpy()


@pytest.mark.parametrize("bh,tq,tk,d,causal", [(3, 16, 16, 8, True), (2, 9, 23, 16, True), (2, 17, 17, 64, False),
                                                (1, 40, 40, 128, True), (2, 5, 31, 32, False)])
def test_attention_matches_torch_float64(bh, tq, tk, d, causal):
    q, k, v = (RNG.standard_normal((bh, t, d)) for t in (tq, tk, tk))
    scale = 1.0 / math.sqrt(d)
    o = oracle.attention(q, k, v, scale, causal)
    assert np.max(np.abs(o - _torch_attention(q, k, v, scale, causal))) <= 1e-13


def test_attention_closed_forms():
    # constant value rows: every output row is that row (the weights sum to 1)
    bh, t, d = 2, 12, 8
    q, k = RNG.standard_normal((bh, t, d)), RNG.standard_normal((bh, t, d))
    v = np.tile(RNG.standard_normal((bh, 1, d)), (1, t, 1))
    o = oracle.attention(q, k, v, 0.7, True)
    assert np.max(np.abs(o - v)) <= 1e-14
    # causal: query 0 sees key 0 only; identical keys give the mean of the visible values
    v = RNG.standard_normal((bh, t, d))
    o = oracle.attention(q, k, v, 0.7, True)
    assert np.max(np.abs(o[:, 0] - v[:, 0])) <= 1e-15
    kk = np.tile(RNG.standard_normal((bh, 1, d)), (1, t, 1))
    o = oracle.attention(q, kk, v, 0.7, True)
    means = np.cumsum(v, axis=1) / np.arange(1, t + 1)[None, :, None]
    assert np.max(np.abs(o - means)) <= 1e-14
    o = oracle.attention(q, kk, v, 0.7, False)
    assert np.max(np.abs(o - v.mean(axis=1, keepdims=True))) <= 1e-14
    # one key far ahead of the others: the output is its value row
    k2 = RNG.standard_normal((1, t, d)) * 0.01
    k2[0, 5] = q[0, 3] * 1000.0
    o = oracle.attention(q[:1], k2, v[:1], 1.0, False)
    assert np.max(np.abs(o[0, 3] - v[0, 5])) <= 1e-12


def test_attention_brute_force_mpmath():
    mpmath.mp.dps = 40
    q, k, v = (RNG.standard_normal((1, 4, 3)) for _ in range(3))
    o = oracle.attention(q, k, v, 0.5, True)
    for i in range(4):
        s = [mpmath.mpf(0.5) * mpmath.fsum(mpmath.mpf(float(a)) * mpmath.mpf(float(b)) for a, b in zip(q[0, i], k[0, j]))
             for j in range(i + 1)]
        m = max(s)
        e = [mpmath.exp(x - m) for x in s]
        tot = mpmath.fsum(e)
        for t in range(3):
            exact = mpmath.fsum(e[j] * mpmath.mpf(float(v[0, j, t])) for j in range(i + 1)) / tot
            assert abs(mpmath.mpf(float(o[0, i, t])) - exact) <= 1e-15


def test_attention_bf16_rounds_the_double_result_once():
    q, k, v = (oracle.round_to_bf16(RNG.standard_normal((2, 10, 16))) for _ in range(3))
    via = oracle.round_to_bf16(oracle.attention(*(oracle.bf16_to_f64(a) for a in (q, k, v)), 0.25, True))
    assert np.array_equal(oracle.attention(q, k, v, 0.25, True), via)


# ================================================================= rounding

def _all_finite_bf16():
    bits = np.arange(0, 0x7F80, dtype=np.uint32)          # +0 .. max finite
    vals = (bits << 16).view(np.float32).astype(np.float64)
    return bits.astype(np.uint16), vals


def _nearest_even_bf16(v: float, bits, vals) -> int:
    """Brute force: nearest finite bf16 magnitude, ties to the even pattern,
    overflow to infinity past the halfway point above the largest finite."""
    a = abs(v)
    sign = 0x8000 if math.copysign(1.0, v) < 0 else 0
    top = vals[-1]
    ulp_top = vals[-1] - vals[-2]
    if a >= top + ulp_top / 2:
        return sign | 0x7F80
    i = int(np.searchsorted(vals, a))
    cands = [j for j in (i - 1, i) if 0 <= j < len(vals)]
    best = min(cands, key=lambda j: (abs(vals[j] - a), int(bits[j]) & 1))
    return sign | int(bits[best])


def test_bf16_rounding_brute_force():
    bits, vals = _all_finite_bf16()
    samples = list(RNG.standard_normal(3000) * 10.0 ** RNG.integers(-40, 39, 3000))
    samples += list(RNG.standard_normal(500) * 1e-39)        # subnormal range
    # exact ties between neighbours, both parities
    for k in RNG.integers(1, 0x7F7F, 500):
        samples.append((vals[k] + vals[k + 1]) / 2)
        samples.append(-(vals[k] + vals[k + 1]) / 2)
    samples += [2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 2.0 ** -126, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]
    got = oracle.round_to_bf16(np.array(samples))
    for v, g in zip(samples, got):
        assert int(g) == _nearest_even_bf16(float(v), bits, vals), v


def test_bf16_rounding_special_values():
    top = float((np.uint32(0x7F7F) << 16).view(np.float32))
    half_ulp = 2.0 ** (127 - 8)
    r = oracle.round_to_bf16(np.array([np.inf, -np.inf, 0.0, -0.0, top, top + half_ulp,
                                       top + half_ulp * 0.999]))
    assert list(r) == [0x7F80, 0xFF80, 0x0000, 0x8000, 0x7F7F, 0x7F80, 0x7F7F]
    n = oracle.round_to_bf16(np.array([np.nan]))[0]
    assert (n & 0x7F80) == 0x7F80 and (n & 0x007F) != 0


def test_bf16_widening_is_exact_for_every_pattern():
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    got = oracle.bf16_to_f64(b)
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert np.all(same)


def test_f32_rounding_matches_numpy_cast():
    v = np.concatenate([RNG.standard_normal(100000) * 10.0 ** RNG.integers(-45, 39, 100000),
                        [np.inf, -np.inf, 0.0, -0.0, 3.4028235677973366e38]])
    assert np.array_equal(oracle.round_to_f32(v).view(np.uint32), v.astype(np.float32).view(np.uint32))
