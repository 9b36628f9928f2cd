"""Rotary position embedding on Q and K (CoCoDiff article, "V-First" section).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The article says Q and K receive, besides the RMSNorm, a rotary position
encoding (RoPE) that carries relative positions, and V does not; it prints no
formula, base or channel layout.  The reading taken is the rotary embedding
as introduced for transformers: the D channels of one head form D/2
interleaved pairs (x[2i], x[2i+1]), and pair i of the token at position m is
turned by the angle a = m * theta^(-2i/D) (theta = 10000 unless stated):

    y[2i]   = x[2i] cos a - x[2i+1] sin a
    y[2i+1] = x[2i] sin a + x[2i+1] cos a

i.e. the pair, read as the complex number x[2i] + i x[2i+1], is multiplied by
exp(i a).  The position of a token is its index in the sequence the
attention runs over: the token index s inside its frame for the spatial
layer, the sequence index n for image attention.  When both are applied the
RMSNorm comes first (the article lists the RMSNorm, then RoPE).
"""
from __future__ import annotations

import numpy as np


def rope_angles(pos, head_dim, theta=10000.0):
    """Angles a[m, i] = pos[m] * theta^(-2i/D), fp64 [len(pos), D/2]."""
    if head_dim % 2:
        raise ValueError("RoPE needs an even head dim")
    i = np.arange(head_dim // 2, dtype=np.float64)
    freq = np.power(float(theta), -2.0 * i / head_dim)
    return np.asarray(pos, dtype=np.float64).reshape(-1, 1) * freq.reshape(1, -1)


def rope_table(n_pos, head_dim, theta=10000.0):
    """(cos, sin) of every angle: fp64 [n_pos, D/2, 2]."""
    a = rope_angles(np.arange(n_pos), head_dim, theta)
    return np.stack([np.cos(a), np.sin(a)], axis=-1)


def rope_heads(rows, pos, head_dim, theta=10000.0):
    """Rotate every head_dim-wide segment of row r by the angles of position pos[r] (fp64)."""
    from .attention import _f64
    x = _f64(rows)
    n = x.shape[0]
    seg = x.reshape(n, -1, head_dim // 2, 2)             # [row, head, pair, (even, odd)]
    a = rope_angles(pos, head_dim, theta).reshape(n, 1, head_dim // 2)
    c, s = np.cos(a), np.sin(a)
    y0 = seg[..., 0] * c - seg[..., 1] * s
    y1 = seg[..., 0] * s + seg[..., 1] * c
    return np.stack([y0, y1], axis=-1).reshape(x.shape)
