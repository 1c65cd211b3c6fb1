"""Pin of the attention kernels' FMA-pipe exp2 (``exp2_poly2`` in csrc/attn_common.cuh).

The kernel's exact fp32 operation sequence is replayed on the CPU with the constants read
from the kernel source:
  clamp x to >= -126; t = x + 1.5*2^23 (round to nearest: t - 1.5*2^23 = rint(x));
  f = fma(rint(x), -1, x); p = ((c3 f + c2) f + c1) f + c0 by three fused multiply-adds;
  2^rint(x) added into the exponent field of p (integer add of rint(x) << 23).
Every fp32 fused multiply-add is emulated exactly (product and sum kept exact, one rounding
to fp32, ties to even).  Checked against the mathematical 2^x (fp64) over a dense set of
fp32 inputs in the range the softmax can produce, [-126, 8] (its running maximum lags the
true maximum by at most 2^8), and at the clamp (masked logits are -inf).
"""
from __future__ import annotations

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = os.path.join(ROOT, "block_sparse_attention_gate_b200", "csrc", "attn_common.cuh")
REL_BOUND = 7.5e-5   # the bound the kernel's comment states


def kernel_constants():
    src = open(KERNEL).read()
    body = src[src.index("void exp2_poly2"):]
    body = body[:body.index("\n}\n")]
    fmas = re.findall(r"fma2\(q0, q1, ([^;]*)\);", body)
    assert len(fmas) == 3, fmas
    lits = [re.findall(r"(-?\d+\.\d+(?:e-?\d+)?)f", x) for x in fmas]
    c3, c2 = float(lits[0][0]), float(lits[0][2])
    c1, c0 = float(lits[1][0]), float(lits[2][0])
    rnd = float(re.search(r"kRound = ([0-9.]+)f", body).group(1))
    clamp = float(re.search(r"fmaxf\(x0, (-[0-9.]+)f\)", body).group(1))
    return np.float32([c0, c1, c2, c3]), np.float32(rnd), np.float32(clamp)


def fma32(a, b, c):
    """Correctly rounded fp32 a*b + c for fp32 arrays."""
    a64, b64, c64 = (np.asarray(x, dtype=np.float32).astype(np.float64) for x in (a, b, c))
    p = a64 * b64                     # exact: 24 + 24 significant bits
    s = p + c64
    bp = s - c64
    e = (p - bp) + (c64 - (s - bp))   # two-sum: s + e == p + c exactly
    r = s.astype(np.float32)
    r64 = r.astype(np.float64)
    other = np.nextafter(r, np.where(s > r64, np.float32(np.inf), np.float32(-np.inf)))
    d = other.astype(np.float64) - r64
    tie = (s != r64) & (2.0 * (s - r64) == d)
    fix = tie & (e != 0) & (np.sign(e) == np.sign(d))
    return np.where(fix, other, r).astype(np.float32)


def exp2_poly(x):
    (c0, c1, c2, c3), rnd, clamp = kernel_constants()
    x = np.maximum(np.asarray(x, dtype=np.float32), clamp)
    t = (x.astype(np.float64) + np.float64(rnd)).astype(np.float32)
    r = (t.astype(np.float64) - np.float64(rnd)).astype(np.float32)
    f = fma32(r, np.float32(-1.0), x)
    q = fma32(f, c3, c2)
    q = fma32(q, f, c1)
    q = fma32(q, f, c0)
    bits = (q.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def inputs():
    rng = np.random.default_rng(0)
    xs = [np.linspace(-125.0, 8.0, 2_000_001)]
    # every fraction finely, at several integer offsets
    f = np.linspace(-0.5, 0.5, 400_001)
    for j in (0, -1, -2, -7, -60, -124, 7):
        xs.append(f + j)
    # random fp32 bit patterns: negative values down to -125 and positive ones up to 8
    neg_lo, neg_hi = np.float32(-1e-30).view(np.uint32), np.float32(-125.0).view(np.uint32)
    pos_lo, pos_hi = np.float32(1e-30).view(np.uint32), np.float32(8.0).view(np.uint32)
    xs.append(rng.integers(neg_lo, neg_hi, 1_000_000, dtype=np.uint32).view(np.float32))
    xs.append(rng.integers(pos_lo, pos_hi, 200_000, dtype=np.uint32).view(np.float32))
    x = np.concatenate([np.asarray(a, dtype=np.float32) for a in xs])
    return x[(x >= -125.0) & (x <= 8.0)]


def test_relative_error_within_stated_bound():
    x = inputs()
    y = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert np.all(np.isfinite(y))
    assert rel.max() <= REL_BOUND, (rel.max(), x[np.argmax(rel)])
    # the bound is not loose: the cubic equioscillates close to it
    assert rel.max() > 0.9 * REL_BOUND


def test_masked_and_clamped_inputs_are_negligible():
    x = np.float32([-np.inf, -1e30, -1000.0, -200.0, -126.0, -125.75, -125.5, -125.25])
    y = exp2_poly(x).astype(np.float64)
    assert np.all(np.isfinite(y)) and np.all(y >= 0.0)
    # next to a row sum >= 1 (the row maximum contributes 2^0, or at least 2^-8), these
    # vanish in fp32
    assert np.all(y <= 2.0 ** -124)
    # everything at or below the clamp gives the clamp's value
    assert np.all(y[:5] == y[4])


def test_integer_inputs_are_nearly_exact_powers():
    j = np.arange(-125, 9, dtype=np.float32)
    y = exp2_poly(j).astype(np.float64)
    # p(0) = c0 is within the bound of 1, and the exponent add is exact
    assert np.all(np.abs(y / np.exp2(j.astype(np.float64)) - 1.0) <= REL_BOUND)


def test_fit_tool_reproduces_kernel_coefficients():
    from block_sparse_attention_gate_b200 import exp2_fit
    c, err = exp2_fit.fit(3)
    kc, _, _ = kernel_constants()
    assert err <= REL_BOUND
    np.testing.assert_allclose(c.astype(np.float32), kc, rtol=2e-6, atol=0)


def test_fma_emulation_rounds_ties_by_the_exact_sum():
    # a*b = 2^-24 (1 - 2^-36) exactly; c = 1 + 2^-23.  The exact sum 1 + 3*2^-24 - 2^-60 lies
    # just below the midpoint of 1 + 2^-23 and 1 + 2^-22, so the fused result is 1 + 2^-23;
    # the sum rounded to fp64 first is the midpoint itself, which ties to even (1 + 2^-22).
    a = np.float32(2.0 ** -24 * (1 + 2.0 ** -18))
    b = np.float32(1 - 2.0 ** -18)
    c = np.float32(1 + 2.0 ** -23)
    want = np.float32(1 + 2.0 ** -23)
    assert fma32(a, b, c) == want
    assert np.float32(np.float64(a) * np.float64(b) + np.float64(c)) == np.float32(1 + 2.0 ** -22)
    # an exact sum needs no correction
    assert fma32(np.float32(1.5), np.float32(2.0), np.float32(0.25)) == np.float32(3.25)
