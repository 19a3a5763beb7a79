"""The FMA-pipe exp2 used for a quarter of the attention softmax's
exponentials (exp2_poly2): for x <= 8, xh = x - 1/2 is clamped at -125.5 and
split as xh = n + u with n the nearest integer (adding and subtracting
1.5 * 2^23 in float32) and u in [-1/2, 1/2]; 2^(u + 1/2) is a cubic
minimax polynomial q(u) and 2^n is added into q's exponent field (the clamp at
-125.5 keeps every result a normal float).  The
coefficients are read from the kernel source and the evaluation is replayed
in float32; the relative error against exp2 must stay below 1e-4 (the bf16
probabilities it feeds are rounded to 2^-9 anyway), and a Remez fit done here
must land on the same coefficients."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "learned_token_pruning_b200",
                   "csrc", "attn_tc.cuh")
MAGIC = np.float32(12582912.0)   # 1.5 * 2^23


def _coeffs():
    body = open(SRC).read()
    c = [float(re.search(rf"constexpr float kExp2C{i} = ([0-9.e+-]+)f;", body).group(1)) for i in range(4)]
    return [np.float32(v) for v in c]


def _fma32(a, b, c):
    # a * b + c with one rounding to float32 (the product of two float32
    # values is exact in float64)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly2(x):
    c0, c1, c2, c3 = _coeffs()
    xh = np.maximum((x.astype(np.float32) - np.float32(0.5)).astype(np.float32), np.float32(-125.5))
    t = (xh + MAGIC).astype(np.float32)
    n = (t - MAGIC).astype(np.float32)
    u = _fma32(n, np.full_like(n, -1.0), xh)
    q = _fma32(np.full_like(u, c3), u, np.full_like(u, c2))
    q = _fma32(q, u, np.full_like(u, c1))
    q = _fma32(q, u, np.full_like(u, c0))
    bits = q.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_exp2_poly_relative_error_bound():
    x = np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = _exp2_poly2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got - want) / want) < 1e-4


def test_exp2_poly_special_values():
    x = np.array([0.0, 1.0, -1.0, 8.0, -125.0, -200.0, 7.25], np.float32)
    got = _exp2_poly2(x).astype(np.float64)
    want = np.exp2(np.array([0.0, 1.0, -1.0, 8.0, -125.0, -125.0, 7.25]))
    assert np.all(np.abs(got / want - 1.0) < 1e-4)
    assert np.all(got > 0)          # clamped far below the maximum, never garbage


def remez_exp2_cubic(iters: int = 40):
    """Minimax (Remez exchange) fit of 2^(u + 1/2) on [-1/2, 1/2] by
    q(u) = c0 + c1 u + c2 u^2 + c3 u^3 for RELATIVE error.  Four free
    coefficients: at the optimum the relative error q(u)/2^(u+1/2) - 1 takes
    its maximum magnitude E with alternating signs at five points.  Each step
    solves q(x_i)/2^(x_i+1/2) - 1 = (-1)^i E on the current reference points,
    then moves them to the extremum of each sign run of the error on a fine
    grid.  Returns (c0, c1, c2, c3, max relative error)."""
    xs = np.linspace(-0.5, 0.5, 400001)
    ref = np.linspace(-0.5, 0.5, 5)
    for _ in range(iters):
        a = np.stack([np.ones(5), ref, ref ** 2, ref ** 3, -((-1.0) ** np.arange(5)) * 2.0 ** (ref + 0.5)], 1)
        c0, c1, c2, c3, _ = np.linalg.solve(a, 2.0 ** (ref + 0.5))
        err = (c0 + c1 * xs + c2 * xs ** 2 + c3 * xs ** 3) / 2.0 ** (xs + 0.5) - 1.0
        runs = np.split(np.arange(xs.size), np.flatnonzero(np.diff(np.sign(err))) + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) > 5:
            ext = sorted(ext, key=lambda i: -abs(err[i]))[:5]
        if len(ext) == 5:
            ref = np.sort(xs[ext])
    return c0, c1, c2, c3, float(np.max(np.abs(err)))


def test_exp2_poly_coefficients_are_the_remez_minimax_fit():
    # the kernel's constants re-derived: a Remez fit must land on them (to the
    # float32 digits they were printed with) and its error bound must hold
    *fit, e = remez_exp2_cubic()
    for c, k in zip(fit, _coeffs()):
        assert abs(c - k) < 2e-6
    assert 7.0e-5 < e < 8.0e-5
