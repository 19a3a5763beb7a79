"""The FMA-pipe exp2 used for part of the attention softmax: Cody-Waite split
x = n + f (n = floor(x), f in [0, 1)) and a cubic minimax polynomial for 2^f.
The coefficients are read from the kernel source and the evaluation is
replayed in float32; the relative error against exp2 must stay below 1e-4
(the bf16 probabilities it feeds are rounded to 2^-9 anyway)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "learned_token_pruning_b200",
                   "csrc", "attn_tc.cuh")


def _coeffs():
    body = open(SRC).read()
    body = body[body.index("float exp2_poly(float x)"):]
    body = body[:body.index("}")]
    nums = [float(x) for x in re.findall(r"([0-9]+\.[0-9]+)f", body)]
    # fmaf(f, c3, c2); fmaf(q, f, c1); fmaf(q, f, 1.0f), after the -127 clamp
    assert nums[0] == 127.0
    c3, c2, c1, one = nums[1], nums[2], nums[3], nums[4]
    assert one == 1.0
    return np.float32(c1), np.float32(c2), np.float32(c3)


def _exp2_poly(x):
    c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    n = np.floor(x)
    f = (x - n).astype(np.float32)
    q = (f * c3 + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + np.float32(1.0)).astype(np.float32)
    bits = q.view(np.int32) + (n.astype(np.int32) << 23)
    return bits.view(np.float32)


def test_exp2_poly_relative_error_bound():
    x = np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = _exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got - want) / want) < 1e-4


def test_exp2_poly_special_values():
    x = np.array([0.0, 1.0, -1.0, 8.0, -126.0, -np.inf, -200.0], np.float32)
    got = _exp2_poly(x)
    assert got[0] == 1.0 and got[1] == 2.0 and got[2] == 0.5 and got[3] == 256.0
    assert got[5] == 0.0 and got[6] == 0.0
    assert abs(got[4] / 2.0 ** -126 - 1.0) < 1e-4


def remez_exp2_cubic(iters: int = 30):
    """Minimax (Remez exchange) fit of 2^f on [0, 1] by p(f) = 1 + c1 f + c2 f^2
    + c3 f^3 for RELATIVE error, with p(0) = 1 fixed so that exact powers of
    two stay exact.  Three free coefficients: at the optimum the relative error
    p(f)/2^f - 1 takes its maximum magnitude E with alternating signs at four
    points of (0, 1].  Each step solves p(x_i)/2^x_i - 1 = (-1)^i E on the
    current reference points, then moves them to the extremum of each sign run
    of the error on a fine grid.  Returns (c1, c2, c3, max relative error)."""
    xs = np.linspace(0.0, 1.0, 200001)[1:]
    ref = np.array([0.1, 0.4, 0.75, 1.0])
    for _ in range(iters):
        a = np.stack([ref, ref ** 2, ref ** 3, -((-1.0) ** np.arange(4)) * 2.0 ** ref], 1)
        c1, c2, c3, _ = np.linalg.solve(a, 2.0 ** ref - 1.0)
        err = (1.0 + c1 * xs + c2 * xs ** 2 + c3 * xs ** 3) / 2.0 ** xs - 1.0
        runs = np.split(np.arange(xs.size), np.flatnonzero(np.diff(np.sign(err))) + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) > 4:
            ext = sorted(ext, key=lambda i: -abs(err[i]))[:4]
        if len(ext) == 4:
            ref = np.sort(xs[ext])
    return c1, c2, c3, float(np.max(np.abs(err)))


def test_exp2_poly_coefficients_are_the_remez_minimax_fit():
    # the kernel's constants re-derived: a Remez fit must land on them (to the
    # few float32 ulps the fit was printed with) and its error bound must hold
    c1, c2, c3, e = remez_exp2_cubic()
    k1, k2, k3 = _coeffs()
    assert abs(c1 - k1) < 5e-6 and abs(c2 - k2) < 5e-6 and abs(c3 - k3) < 5e-6
    assert 8.0e-5 < e < 8.7e-5
