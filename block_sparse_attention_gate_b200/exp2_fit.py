"""Fit of the polynomial behind the attention kernels' FMA-pipe exp2 (``exp2_poly2`` in
``csrc/attn_tc.cu``).

The kernels evaluate 2^x for a share of the softmax exponentials on the FMA pipe:
x = j + f with j = rint(x) and f in [-0.5, 0.5], 2^f from a cubic p(f) and 2^j added into
the exponent field.  The cubic minimises the maximum RELATIVE error |p(f) / 2^f - 1| on
[-0.5, 0.5].  It is found by Lawson's algorithm: iteratively reweighted least squares whose
weights grow where the error is largest, which converges to the minimax (equioscillating)
solution.  Run as a script, this prints the coefficients (lowest degree first) and the
achieved maximum relative error, with the coefficients in fp64 and then rounded to fp32 and
evaluated by Horner's rule in fp32.
"""
from __future__ import annotations

import numpy as np


def fit(degree: int = 3, points: int = 20001, iterations: int = 200) -> tuple[np.ndarray, float]:
    """Coefficients c[0..degree] of the near-minimax relative-error fit of 2^f on
    [-0.5, 0.5], and its maximum relative error on the fitting grid."""
    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.full(points, 1.0 / points)
    c = np.zeros(degree + 1)
    for _ in range(iterations):
        sw = np.sqrt(w)
        # relative residual p(f)/y - 1, weighted
        c, *_ = np.linalg.lstsq(V / y[:, None] * sw[:, None], sw, rcond=None)
        err = np.abs(V @ c / y - 1.0)
        w = w * err
        w /= w.sum()
    return c, float(np.max(np.abs(V @ c / y - 1.0)))


def horner_f32(c: np.ndarray, f: np.ndarray) -> np.ndarray:
    """p(f) with fp32 coefficients, evaluated by Horner's rule in fp32 (separate roundings)."""
    cf = np.asarray(c, dtype=np.float32)
    ff = np.asarray(f, dtype=np.float32)
    p = np.full_like(ff, cf[-1])
    for k in range(len(cf) - 2, -1, -1):
        p = (p * ff + cf[k]).astype(np.float32)
    return p


if __name__ == "__main__":
    for deg in (3, 4, 5):
        c, e64 = fit(deg)
        f = np.linspace(-0.5, 0.5, 20001)
        e32 = float(np.max(np.abs(horner_f32(c, f).astype(np.float64) / np.exp2(f) - 1.0)))
        print("degree %d: max rel err %.3e (fp64 coefficients), %.3e (fp32 Horner); coefficients %s"
              % (deg, e64, e32, [float(x) for x in c.astype(np.float32)]))
