"""Pin of the gate's quantized keys (the per-head gate kernel, rows with top_k <= 5 and more
than 64 candidate blocks; see the header of csrc/gate_tc.cu).

The kernel turns a score s (fp32) of column x of a 32-column group into
    t   = fl32(s * scl + 48)        one fused multiply-add, rounded once
    k1  = fl32(t - 46.5)
    key = fl32(k1 + (31 - x) * 2^-23)
and ranks keys as floats.  The claims checked here, on the exact fp32 operation sequence
(the fused multiply-add evaluated in rational arithmetic and rounded once to fp32, ties to
even): for |s * scl| <= 0.49 every key lies in [1, 2); its low five mantissa bits are 31 - x;
k1 is s * scl rounded to the grid 2^-18 (error at most 2^-19) plus 1.5; and key order equals
the order of (grid value, then lower column).
"""
from fractions import Fraction

import numpy as np

GRID = 2.0 ** -18


def f32(x: float) -> np.float32:
    return np.float32(x)


def fma32(a: np.float32, b: np.float32, c: np.float32) -> np.float32:
    """fp32 a * b + c with one rounding (round to nearest, ties to even)."""
    exact = Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c))
    lo = np.float32(float(exact))          # nearest double, then nearest float: may double-round
    # fix the double rounding by comparing against the neighbours of the candidate
    best = lo
    for cand in (np.nextafter(lo, np.float32(-np.inf)), lo, np.nextafter(lo, np.float32(np.inf))):
        if abs(Fraction(float(cand)) - exact) < abs(Fraction(float(best)) - exact):
            best = cand
        elif abs(Fraction(float(cand)) - exact) == abs(Fraction(float(best)) - exact) and cand != best:
            # tie: even mantissa wins
            if (int(np.float32(cand).view(np.uint32)) & 1) == 0:
                best = cand
    return np.float32(best)


def key(s: np.float32, scl: np.float32, x: int) -> np.float32:
    t = fma32(s, scl, f32(48.0))
    k1 = np.float32(t - f32(46.5))
    return np.float32(k1 + f32((31 - x) * 2.0 ** -23))


def test_fma32_rounds_once():
    # 1 + 2^-24 is a tie between 1 and 1 + 2^-23 in fp32; a product just above it must round up
    a, b = f32(1.0 + 2.0 ** -23), f32(1.0 + 2.0 ** -23)
    # exact a*b = 1 + 2^-22 + 2^-46, plus c = -2^-23 -> 1 + 2^-23 + 2^-46: nearest fp32 is 1 + 2^-23
    assert fma32(a, b, f32(-(2.0 ** -23))) == f32(1.0 + 2.0 ** -23)


def test_keys_lie_in_one_binade_with_the_column_code_in_the_low_bits():
    rng = np.random.default_rng(5)
    scl = f32(0.49 / 7.3)
    for _ in range(2000):
        s = f32(rng.uniform(-7.3, 7.3))
        x = int(rng.integers(0, 32))
        k = key(s, scl, x)
        assert f32(1.0) <= k < f32(2.0)
        bits = int(k.view(np.uint32))
        assert bits & 31 == 31 - x


def test_grid_value_is_the_scaled_score_rounded_to_two_to_the_minus_18():
    rng = np.random.default_rng(6)
    scl = f32(0.49 / 3.1)
    for _ in range(2000):
        s = f32(rng.uniform(-3.1, 3.1))
        k = key(s, scl, int(rng.integers(0, 32)))
        grid = float(np.uint32(int(k.view(np.uint32)) & ~31).view(np.float32)) - 1.5
        exact = float(Fraction(float(s)) * Fraction(float(scl)))
        assert abs(grid - exact) <= GRID / 2
        assert (grid / GRID) == round(grid / GRID)


def test_key_order_is_grid_value_then_lower_column():
    rng = np.random.default_rng(7)
    scl = f32(0.49 / 5.0)
    for _ in range(3000):
        s1, s2 = f32(rng.uniform(-5, 5)), f32(rng.uniform(-5, 5))
        if rng.random() < 0.3:          # near ties: same or adjacent grid points
            s2 = np.float32(s1 + f32(rng.integers(-2, 3) * GRID / float(scl) * 0.5))
        x1, x2 = int(rng.integers(0, 32)), int(rng.integers(0, 32))
        if x1 == x2:
            continue
        k1, k2 = key(s1, scl, x1), key(s2, scl, x2)
        g1 = int(k1.view(np.uint32)) & ~31
        g2 = int(k2.view(np.uint32)) & ~31
        want_first = g1 > g2 or (g1 == g2 and x1 < x2)
        assert (k1 > k2) == want_first


def test_equal_scores_rank_by_column_and_zero_scale_keeps_column_order():
    s = f32(0.7)
    scl = f32(0.49 / 2.0)
    ks = [key(s, scl, x) for x in range(32)]
    assert all(ks[x] > ks[x + 1] for x in range(31))
    # a zero scale (B = 0 or not finite) makes every score a tie: lower columns first
    ks0 = [key(f32(123.0), f32(0.0), x) for x in range(32)]
    assert all(ks0[x] > ks0[x + 1] for x in range(31))
    assert ks0[0] == f32(1.5 + 31 * 2.0 ** -23)
