"""The all-to-all relayouts, written out as index maps on a virtual partition.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"Virtual P": the P shards of a distributed tensor are stacked as the outermost
axis of one buffer, so an all-to-all becomes a permutation of rows inside one
array.  A row is the unit both sides keep contiguous: C = H*D channels of one
token for the spatial/temporal exchange, D channels of one (token, head) for
the Ulysses sequence<->head exchange.

Spatial-temporal exchange (ScaleFusion review, "三、技术架构": the layer table,
the distributed execution flow, and "四、核心创新": the intra-layer algorithm
and the pseudo-code that rearranges x to [B,N_T,N_S,T/N_T,S/N_S/P,C] and y to
[B,N_T,N_S,T/N_T/P,S/N_S,C]):

  x, spatially sharded; shard p has layout [B, N_T, N_S, T/N_T, S/(N_S*P), C].
     Row (p, b, i, j, t1, s1) holds token s of frame t of batch b with
         t = i*T/N_T + t1,      s = j*S/N_S + p*S/(N_S*P) + s1.
  y, temporally sharded; shard q has layout [B, N_T, N_S, T/(N_T*P), S/N_S, C].
     Row (q, b, i, j, t2, s2) holds
         t = i*T/N_T + q*T/(N_T*P) + t2,   s = j*S/N_S + s2.

  S2T writes every y row from the x row that holds the same (b, t, s); T2S is
  the inverse.  With N_T = N_S = 1 these are the plain layouts [B,T,S/P,C] and
  [B,T/P,S,C] of the layer table.  Which shard owns which block is not stated
  on the pages; contiguous ownership inside each slice is the reading taken.
  A block range (i0, i1, j0, j1) writes only the destination rows of blocks
  i0 <= i < i1, j0 <= j < j1 (the partitions the inter-layer schedule hoists).

Ulysses sequence<->head exchange (CoCoDiff article, Ulysses section; DeepSpeed
Ulysses row of the ScaleFusion related-work table):

  in,  sequence sharded; shard p has layout [B, N/P, H, D]:
       row (p, b, n1, h) holds token n = p*N/P + n1, head h.
  out, head sharded;     shard q has layout [B, H/P, N, D]:
       row (q, b, h1, n) holds token n, head h = q*H/P + h1.

An optional per-head RMSNorm (CoCoDiff "V-First" section: RMSNorm is applied
to Q and K before their exchange) may be applied to every D-channel head
segment of the rows that are moved.
"""
from __future__ import annotations

import numpy as np

from .rmsnorm import rmsnorm_heads
from .rope import rope_heads


def _f64(x):
    from .attention import _f64 as f
    return f(x)


def st_x_rows(P, B, T, S, n_t=1, n_s=1):
    """Logical row (b*T + t)*S + s held by each x row, and its block (i, j)."""
    Tb, Sb = T // n_t, S // (n_s * P)
    p, b, i, j, t1, s1 = np.meshgrid(np.arange(P), np.arange(B), np.arange(n_t),
                                     np.arange(n_s), np.arange(Tb), np.arange(Sb),
                                     indexing="ij")
    t = i * (T // n_t) + t1
    s = j * (S // n_s) + p * Sb + s1
    return ((b * T + t) * S + s).reshape(-1), i.reshape(-1), j.reshape(-1)


def st_y_rows(P, B, T, S, n_t=1, n_s=1):
    """Logical row (b*T + t)*S + s held by each y row, and its block (i, j)."""
    Tb, Sb = T // (n_t * P), S // n_s
    q, b, i, j, t2, s2 = np.meshgrid(np.arange(P), np.arange(B), np.arange(n_t),
                                     np.arange(n_s), np.arange(Tb), np.arange(Sb),
                                     indexing="ij")
    t = i * (T // n_t) + q * Tb + t2
    s = j * (S // n_s) + s2
    return ((b * T + t) * S + s).reshape(-1), i.reshape(-1), j.reshape(-1)


def _check_st(P, T, S, n_t, n_s):
    if T % (n_t * P) or S % (n_s * P):
        raise ValueError("N_T*P must divide T and N_S*P must divide S")


def _move_rows(src, dst, src_log, dst_log, sel, row_len, rms, rope=None, position=None):
    pos = np.empty(src_log.size, dtype=np.int64)
    pos[src_log] = np.arange(src_log.size)              # logical -> source row
    rows = src.reshape(-1, row_len)[pos[dst_log[sel]]]
    if rms is not None:
        gamma, head_dim, eps = rms
        rows = rmsnorm_heads(rows, gamma, head_dim, eps)
    if rope is not None:                                # after the RMSNorm
        head_dim, theta = rope
        rows = rope_heads(rows, position(dst_log[sel]), head_dim, theta)
    dst.reshape(-1, row_len)[sel] = rows
    return dst


def st_relayout(mode, buf, P, B, T, S, C, n_t=1, n_s=1, blocks=None, out=None, rms=None, rope=None):
    """S2T (x -> y) or T2S (y -> x) on a flat buffer of B*T*S*C elements.

    blocks = (i0, i1, j0, j1) limits the destination rows written; rows
    outside the range keep the values of ``out`` (NaN when ``out`` is None).
    rms = (gamma[D], D, eps) applies the per-head RMSNorm to moved rows;
    rope = (D, theta) then rotates them by their token's index s in its frame
    (S2T only: the spatial layer's positions).
    """
    if rope is not None and mode != "S2T":
        raise ValueError("RoPE applies on the way to the spatial layer (S2T)")
    _check_st(P, T, S, n_t, n_s)
    x_log, xi, xj = st_x_rows(P, B, T, S, n_t, n_s)
    y_log, yi, yj = st_y_rows(P, B, T, S, n_t, n_s)
    if mode == "S2T":
        src_log, dst_log, di, dj = x_log, y_log, yi, yj
    elif mode == "T2S":
        src_log, dst_log, di, dj = y_log, x_log, xi, xj
    else:
        raise ValueError(mode)
    i0, i1, j0, j1 = blocks if blocks is not None else (0, n_t, 0, n_s)
    sel = np.flatnonzero((di >= i0) & (di < i1) & (dj >= j0) & (dj < j1))
    src = _f64(buf).reshape(-1)
    dst = np.full(src.size, np.nan) if out is None else _f64(out).reshape(-1).copy()
    return _move_rows(src, dst, src_log, dst_log, sel, C, rms, rope, lambda logical: logical % S)


def st_row_pairs(mode, P, B, T, S, n_t=1, n_s=1, blocks=None):
    """(dst_rows, src_rows): destination row r of the relayout holds source row src.

    The same definition as st_relayout, returned as index arrays so that a
    full-size result can be checked with one gather.
    """
    _check_st(P, T, S, n_t, n_s)
    x_log, xi, xj = st_x_rows(P, B, T, S, n_t, n_s)
    y_log, yi, yj = st_y_rows(P, B, T, S, n_t, n_s)
    src_log, dst_log, di, dj = (x_log, y_log, yi, yj) if mode == "S2T" else (y_log, x_log, xi, xj)
    i0, i1, j0, j1 = blocks if blocks is not None else (0, n_t, 0, n_s)
    sel = np.flatnonzero((di >= i0) & (di < i1) & (dj >= j0) & (dj < j1))
    pos = np.empty(src_log.size, dtype=np.int64)
    pos[src_log] = np.arange(src_log.size)
    return sel, pos[dst_log[sel]]


def seq_head_row_pairs(mode, P, B, N, H):
    """(dst_rows, src_rows) of the sequence<->head exchange (rows of D)."""
    seq_log, head_log = _seq_rows(P, B, N, H), _head_rows(P, B, N, H)
    src_log, dst_log = (seq_log, head_log) if mode == "SEQ2HEAD" else (head_log, seq_log)
    pos = np.empty(src_log.size, dtype=np.int64)
    pos[src_log] = np.arange(src_log.size)
    return np.arange(dst_log.size), pos[dst_log]


def st_logical_from_x(buf, P, B, T, S, C, n_t=1, n_s=1):
    """[B, T, S, C] logical tensor held by an x buffer."""
    x_log, _, _ = st_x_rows(P, B, T, S, n_t, n_s)
    out = np.empty((B * T * S, C))
    out[x_log] = _f64(buf).reshape(-1, C)
    return out.reshape(B, T, S, C)


def st_logical_from_y(buf, P, B, T, S, C, n_t=1, n_s=1):
    """[B, T, S, C] logical tensor held by a y buffer."""
    y_log, _, _ = st_y_rows(P, B, T, S, n_t, n_s)
    out = np.empty((B * T * S, C))
    out[y_log] = _f64(buf).reshape(-1, C)
    return out.reshape(B, T, S, C)


def _seq_rows(P, B, N, H):
    n1_len = N // P
    p, b, n1, h = np.meshgrid(np.arange(P), np.arange(B), np.arange(n1_len),
                              np.arange(H), indexing="ij")
    n = p * n1_len + n1
    return ((b * N + n) * H + h).reshape(-1)


def _head_rows(P, B, N, H):
    h1_len = H // P
    q, b, h1, n = np.meshgrid(np.arange(P), np.arange(B), np.arange(h1_len),
                              np.arange(N), indexing="ij")
    h = q * h1_len + h1
    return ((b * N + n) * H + h).reshape(-1)


def seq_head_relayout(mode, buf, P, B, N, H, D, rms=None, rope=None):
    """SEQ2HEAD ([P,B,N/P,H,D] -> [P,B,H/P,N,D]) or HEAD2SEQ (its inverse).

    rope = (D, theta) rotates moved heads by their token's sequence index n
    after the RMSNorm (SEQ2HEAD only)."""
    if rope is not None and mode != "SEQ2HEAD":
        raise ValueError("RoPE applies on the way to the attention (SEQ2HEAD)")
    if N % P or H % P:
        raise ValueError("P must divide N and H")
    seq_log, head_log = _seq_rows(P, B, N, H), _head_rows(P, B, N, H)
    if mode == "SEQ2HEAD":
        src_log, dst_log = seq_log, head_log
    elif mode == "HEAD2SEQ":
        src_log, dst_log = head_log, seq_log
    else:
        raise ValueError(mode)
    src = _f64(buf).reshape(-1)
    dst = np.full(src.size, np.nan)
    return _move_rows(src, dst, src_log, dst_log, np.arange(dst_log.size), D, rms, rope,
                      lambda logical: (logical // H) % N)
