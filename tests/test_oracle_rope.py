"""Pins of the oracle's rotary position embedding against closed forms and
invariants that a wrong sign, pair layout, frequency or position would break
(the pages print no example, so none is pinned from the text)."""
import math

import numpy as np
import pytest

import oracle


def test_rope_is_complex_multiplication():
    """Pair 0 turns by the position itself (theta^0 = 1): (1, 0) at m = pi/2 -> (0, 1)."""
    x = np.array([[1.0, 0.0, 0.0, 1.0]])
    y = oracle.rope_heads(x, [math.pi / 2], 4, theta=10000.0)
    assert np.allclose(y[0, :2], [0.0, 1.0], atol=1e-15)
    # pair 1 turns by m * theta^(-1/2) = (pi/2) / 100 at D = 4
    a = (math.pi / 2) / 100.0
    assert np.allclose(y[0, 2:], [-math.sin(a), math.cos(a)], atol=1e-15)
    z = oracle.rope_heads(np.array([[3.0, 4.0]]), [1.0], 2)
    w = complex(3.0, 4.0) * complex(math.cos(1.0), math.sin(1.0))
    assert np.allclose(z[0], [w.real, w.imag], atol=1e-14)


def test_rope_frequencies_and_position_zero():
    D, theta = 72, 10000.0
    unit = np.tile([1.0, 0.0], D // 2).reshape(1, D)
    assert np.array_equal(oracle.rope_heads(unit, [0], D, theta), unit)      # position 0: identity
    y = oracle.rope_heads(unit, [1], D, theta).reshape(D // 2, 2)
    got = np.arctan2(y[:, 1], y[:, 0])
    want = theta ** (-2.0 * np.arange(D // 2) / D)
    assert np.allclose(got, want, atol=1e-14)


def test_rope_norm_and_relative_position():
    """Rotations keep every pair's length, and <R(m) q, R(n) k> depends only on m - n."""
    rng = np.random.default_rng(3)
    D = 64
    q, k = rng.normal(size=(1, D)), rng.normal(size=(1, D))
    for m in (0, 5, 117, 1199):
        r = oracle.rope_heads(q, [m], D)
        assert np.allclose(np.hypot(r[0, 0::2], r[0, 1::2]), np.hypot(q[0, 0::2], q[0, 1::2]), atol=1e-12)
    for m, n in ((7, 3), (300, 296), (1000, 996)):              # the same offset 4
        dot = float((oracle.rope_heads(q, [m], D) @ oracle.rope_heads(k, [n], D).T)[0, 0])
        ref = float((oracle.rope_heads(q, [m - n], D) @ k.T)[0, 0])
        assert dot == pytest.approx(ref, rel=1e-9, abs=1e-9)


def test_rope_table_matches_angles():
    t = oracle.rope_table(5, 8, 100.0)
    a = oracle.rope_angles(np.arange(5), 8, 100.0)
    assert t.shape == (5, 4, 2)
    assert np.allclose(t[..., 0], np.cos(a)) and np.allclose(t[..., 1], np.sin(a))
    assert np.allclose(a[3], 3 * 100.0 ** (-2.0 * np.arange(4) / 8))


def test_relayout_rope_positions():
    """The fused relayout rotates each moved head by its token's place s in the frame (S2T)
    or its sequence index n (SEQ2HEAD), after the RMSNorm."""
    rng = np.random.default_rng(5)
    P, B, T, S, H, D = 2, 1, 4, 8, 2, 4
    C = H * D
    x = rng.normal(size=(B * T * S * C,))
    gamma = rng.normal(1.0, 0.1, size=D)
    y = oracle.st_relayout("S2T", x, P, B, T, S, C, 2, 2, rms=(gamma, D, 1e-6), rope=(D, 50.0))
    y0 = oracle.st_relayout("S2T", x, P, B, T, S, C, 2, 2, rms=(gamma, D, 1e-6))
    y_log, _, _ = oracle.st_y_rows(P, B, T, S, 2, 2)
    want = oracle.rope_heads(y0.reshape(-1, C), y_log % S, D, 50.0)
    assert np.allclose(y.reshape(-1, C), want, atol=1e-12)
    N = 8
    z = rng.normal(size=(B * N * H * D,))
    h = oracle.seq_head_relayout("SEQ2HEAD", z, P, B, N, H, D, rope=(D, 50.0))
    h0 = oracle.seq_head_relayout("SEQ2HEAD", z, P, B, N, H, D)
    # head-sharded rows (q, b, h1, n): the sequence index is the fastest
    n_of_row = np.tile(np.arange(N), P * B * (H // P))
    assert np.allclose(h.reshape(-1, D), oracle.rope_heads(h0.reshape(-1, D), n_of_row, D, 50.0), atol=1e-12)
    with pytest.raises(ValueError):
        oracle.st_relayout("T2S", x, P, B, T, S, C, rope=(D, 50.0))
