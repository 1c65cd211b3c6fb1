"""The FMA-pipe 2^x used for part of the softmax exponentials: its coefficients (read from
the CUDA header) evaluated with fp32 fused multiply-adds stay within the stated relative
error bound of the true 2^x over the whole range the softmax feeds it."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    txt = open(os.path.join(ROOT, "block_sparse_attention_gate_b200", "csrc", "sm100.cuh")).read()
    m = re.search(r"kEx2P0 = ([0-9.eE+-]+)f, kEx2P1 = ([0-9.eE+-]+)f, kEx2P2 = ([0-9.eE+-]+)f, "
                  r"kEx2P3 = ([0-9.eE+-]+)f", txt)
    return [np.float32(float(v)) for v in m.groups()]


def _fma32(a, b, c):
    # a*b is exact in fp64 for fp32 a, b; one rounding of the sum to fp32 (double rounding
    # through fp64 can differ from a true fused op in the last bit only)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_poly_model(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_relative_error_bound_over_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32) + np.float32(0.5)])
    got = ex2_poly_model(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.0e-4, rel.max()


def test_underflow_side_is_tiny_and_nonnegative():
    x = np.array([-126.0, -200.0, -np.inf, -1e30], dtype=np.float32)
    got = ex2_poly_model(x)
    assert np.all(got >= 0) and np.all(got < 2.0 ** -124)
