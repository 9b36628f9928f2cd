"""V-Major selective communication: change mask, compaction, cache update.

TEST INFRASTRUCTURE ONLY (see the package docstring).

CoCoDiff article, "V-Major" section: at every denoising step the freshly
computed V of each token is compared with the previous step's V by L1
distance; only tokens whose change exceeds a threshold are marked active and
have their Q/K/V sent; the others read cached data.  Every tenth step sends
everything.  The readings taken (the article prints no formula):

    L1_n   = sum_c |v_cur[n, c] - v_prev[n, c]|     over all C = H*D channels
    mask_n = (L1_n > tau) or force_all              strict comparison
    idx    = the active n in ascending order,  count = |idx|
    cache[n] <- cur[n] for every active n

computed from the stored (bf16 or fp32) values, exactly, in float64.
"""
from __future__ import annotations

import numpy as np


def l1_change(v_cur, v_prev):
    """Per-token L1 distance, [N, C] x [N, C] -> [N] (float64)."""
    from .attention import _f64
    a, b = _f64(v_cur), _f64(v_prev)
    a = a.reshape(a.shape[0], -1)
    b = b.reshape(b.shape[0], -1)
    return np.abs(a - b).sum(axis=1)


def change_mask(l1, tau, force_all=False):
    """uint8 mask: 1 where the token is active."""
    l1 = np.asarray(l1, dtype=np.float64)
    if force_all:
        return np.ones(l1.shape, dtype=np.uint8)
    return (l1 > float(tau)).astype(np.uint8)


def compact(mask):
    """Ascending list of active token indices (int32) and its length."""
    idx = []
    for n, m in enumerate(np.asarray(mask).tolist()):
        if m:
            idx.append(n)
    return np.asarray(idx, dtype=np.int32), len(idx)


def scatter_rows(idx, count, src, cache):
    """Return a copy of ``cache`` with rows idx[:count] replaced from ``src``."""
    from .attention import _f64
    out = _f64(cache).copy()
    s = _f64(src)
    for i in range(count):
        out[idx[i]] = s[idx[i]]
    return out


def pack_rows(idx, count, src):
    """The active rows of ``src`` in idx order: the message a rank would send."""
    from .attention import _f64
    s = _f64(src)
    return np.stack([s[idx[i]] for i in range(count)]) if count else s[:0]


def tau_for_fraction(l1, f):
    """Threshold that leaves a fraction ``f`` of tokens active.

    tau is the midpoint of the two sorted L1 values that straddle the
    (1 - f) quantile, so round(N * f) tokens are strictly above it.  Returns
    (tau, margin) with margin = min_n |L1_n - tau| / tau.
    """
    v = np.sort(np.asarray(l1, dtype=np.float64))
    n = v.size
    k = n - int(round(n * f))                   # tokens at or below tau
    k = min(max(k, 1), n - 1)
    tau = 0.5 * (v[k - 1] + v[k])
    margin = float(np.min(np.abs(v - tau)) / tau) if tau > 0 else 0.0
    return float(tau), margin
