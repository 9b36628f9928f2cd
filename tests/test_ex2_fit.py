"""The coefficients of the spatial kernel's FMA-pipe 2^x polynomial (CPU).

The softmax evaluates 2^f for f in [-1/2, 1/2] as p(f) = P0 + P1 f + P2 f^2 +
P3 f^3.  The coefficients were fitted by a Remez exchange that minimises the
maximum relative error |p(f) / 2^f - 1| over [-1/2, 1/2] for degree 3.  A
minimax fit of degree n equioscillates: its relative error reaches the same
magnitude E, with alternating signs, at n + 2 = 5 points including both ends.
These tests read the coefficients out of the kernel source and check, in
float64, that (a) the error bound stated in the source and the C header
(7.48e-5) holds, (b) the error equioscillates at five alternating extrema of
equal size (so the fit is the minimax one, not an arbitrary polynomial), and
(c) p is close to the Taylor series of 2^f (a transposed or mistyped
coefficient breaks both).
"""
import math
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "sequence_parallelism_st_b200", "csrc", "attn_spatial_sm100.cu")


def coefficients():
    text = open(SRC).read()
    vals = {}
    for m in re.finditer(r"kP([0-3])\s*=\s*([0-9.eE+-]+)f", text):
        vals[int(m.group(1))] = float(np.float32(float(m.group(2))))
    assert sorted(vals) == [0, 1, 2, 3]
    return [vals[i] for i in range(4)]


def rel_error(f):
    P = coefficients()
    p = ((P[3] * f + P[2]) * f + P[1]) * f + P[0]
    return p / np.exp2(f) - 1.0


def test_max_relative_error_matches_the_stated_bound():
    f = np.linspace(-0.5, 0.5, 2_000_001)
    e = np.abs(rel_error(f)).max()
    assert 7.4e-5 <= e <= 7.5e-5, e


def test_error_equioscillates_at_five_points():
    f = np.linspace(-0.5, 0.5, 2_000_001)
    e = rel_error(f)
    ext = [0] + [k for k in range(1, f.size - 1) if (e[k] - e[k - 1]) * (e[k + 1] - e[k]) <= 0] + [f.size - 1]
    vals = e[ext]
    assert len(vals) == 5, vals
    assert all(np.sign(vals[i]) == -np.sign(vals[i + 1]) for i in range(4))
    mags = np.abs(vals)
    assert (mags.max() - mags.min()) / mags.max() < 1e-3, mags


def test_close_to_the_taylor_series():
    P = coefficients()
    ln2 = math.log(2.0)
    taylor = [1.0, ln2, ln2 ** 2 / 2, ln2 ** 3 / 6]
    for c, t in zip(P, taylor):
        assert abs(c - t) / t < 0.02, (P, taylor)
    assert P[0] == float(np.float32(P[0]))        # exactly representable fp32 values
