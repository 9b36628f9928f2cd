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


def tau_for_fraction(l1, f, window=0.01):
    """Threshold that leaves about a fraction ``f`` of tokens active.

    Sort the L1 values; among the consecutive pairs whose rank lies within
    ``window * N`` of N * (1 - f), take the pair with the widest relative gap
    and put tau at its midpoint.  The widest gap keeps every L1 far from tau
    compared with the rounding of an fp32 sum, so the mask does not depend on
    the precision or order of the summation.  Returns (tau, margin,
    active_fraction) with margin = min_n |L1_n - tau| / tau.
    """
    v = np.sort(np.asarray(l1, dtype=np.float64))
    n = v.size
    k0 = n - int(round(n * f))                  # tokens at or below tau
    w = int(round(window * n))
    k0 = min(max(k0, 1), n - 1)
    lo, hi = max(1, k0 - w), min(n - 1, k0 + w)
    best, best_k = -1.0, k0
    for k in range(lo, hi + 1):
        mid = 0.5 * (v[k - 1] + v[k])
        gap = (v[k] - v[k - 1]) / mid if mid > 0 else 0.0
        if gap > best:
            best, best_k = gap, k
    tau = 0.5 * (v[best_k - 1] + v[best_k])
    margin = float(np.min(np.abs(v - tau)) / tau) if tau > 0 else 0.0
    return float(tau), margin, float((v > tau).sum()) / n
