"""Per-head RMSNorm on Q and K (CoCoDiff article, "V-First" section).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The article says Q and K receive an RMSNorm (and RoPE) that V does not; it
prints no formula, epsilon or gain.  The reading taken is the standard
root-mean-square normalisation over the D channels of one head of one token:

    r   = sqrt( (1/D) * sum_d x_d^2 + eps )
    y_d = x_d / r * gamma_d

with one gain vector gamma[D] shared by all heads.
"""
from __future__ import annotations

import numpy as np


def rmsnorm_heads(rows, gamma, head_dim, eps):
    """Apply the RMSNorm to every head_dim-wide segment of each row (fp64)."""
    from .attention import _f64
    x = _f64(rows)
    shape = x.shape
    seg = x.reshape(-1, head_dim)
    g = _f64(gamma).reshape(1, head_dim)
    r = np.sqrt((seg * seg).mean(axis=1, keepdims=True) + eps)
    return (seg / r * g).reshape(shape)
