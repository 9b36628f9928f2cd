"""fp64 softmax attention, spatial/temporal units and the KV-chunk merge.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Definitions (none of the pages prints a formula for attention, the softmax or
the merge; these are the textbook definitions the pages build on):

    s_ij  = (q_i . k_j) * scale,          scale = 1/sqrt(D) unless given
    m_i   = max_j s_ij
    l_i   = sum_j exp(s_ij - m_i)
    o_i   = sum_j exp(s_ij - m_i) v_j / l_i
    lse_i = m_i + ln l_i                   (natural log)

computed in two passes in float64 with no online rescaling.  A unit with no
keys gives o = 0 and lse = -inf, the identity of the merge below.

Spatial units are (b, t, head) and attend over the S tokens of frame t; the
temporal units are (b, s, head) and attend over the T frames of token s
(ScaleFusion review, section "三、技术架构": the layer table pairs the spatial
layer with dimension S and the temporal layer with dimension T).  An image
DiT's full attention is the spatial layer with T = 1 (xDiT summary, section 3).

Merge of R partial results over disjoint key ranges (ring attention and the
chunked all-to-all of SwiftFusion's Torus attention, Methodology 2):

    M   = max_c lse_c
    lse = M + ln sum_c exp(lse_c - M)
    o   = sum_c exp(lse_c - lse) o_c
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):                       # torch tensor
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def attention(q, k, v, scale=None):
    """softmax(q k^T * scale) v over the last-but-one axis of k/v.

    q: [..., M, D], k: [..., N, D], v: [..., N, Dv]  ->  o [..., M, Dv],
    lse [..., M].  Leading axes broadcast like ``np.matmul``.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    D = q.shape[-1]
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    if k.shape[-2] == 0:
        lead = np.broadcast_shapes(q.shape[:-2], k.shape[:-2])
        o = np.zeros(lead + (q.shape[-2], v.shape[-1]))
        lse = np.full(lead + (q.shape[-2],), -np.inf)
        return o, lse
    s = np.matmul(q, np.swapaxes(k, -1, -2)) * scale          # pass 1: scores
    m = s.max(axis=-1, keepdims=True)                         # row max
    e = np.exp(s - m)                                         # pass 2: weights
    l = e.sum(axis=-1, keepdims=True)
    o = np.matmul(e, v) / l
    lse = m[..., 0] + np.log(l[..., 0])
    return o, lse


def spatial(q, k, v, scale=None, kv=None, rows=None, frames=None):
    """Spatial layer: per (b, t, head) attention over the S tokens of frame t.

    q, k, v: logical [B, T, S, H, D] (torch or numpy, any float dtype).
    kv:      optional (begin, end) key range; the partial result of one chunk.
    rows:    optional query token indices (sampled parity); default all S.
    frames:  optional frame indices t to compute; default all T.
    Returns o [B, len(frames), len(rows), H, D] and lse [B, len(frames), H, len(rows)].
    """
    B, T, S, H, D = q.shape
    frames = list(range(T)) if frames is None else list(frames)
    rows = np.arange(S) if rows is None else np.asarray(rows)
    kb, ke = (0, S) if kv is None or kv == (0, 0) else kv
    o = np.empty((B, len(frames), len(rows), H, D))
    lse = np.empty((B, len(frames), H, len(rows)))
    for b in range(B):
        for fi, t in enumerate(frames):
            qf = _f64(q[b, t][rows]).transpose(1, 0, 2)        # [H, R, D]
            kf = _f64(k[b, t][kb:ke]).transpose(1, 0, 2)       # [H, n, D]
            vf = _f64(v[b, t][kb:ke]).transpose(1, 0, 2)
            of, lf = attention(qf, kf, vf, scale)
            o[b, fi] = of.transpose(1, 0, 2)
            lse[b, fi] = lf
    return o, lse


def temporal(q, k, v, scale=None, tokens=None, chunk=256):
    """Temporal layer: per (b, s, head) attention over the T frames of token s.

    q, k, v: logical [B, T, S, H, D].  tokens: optional token indices.
    Returns o [B, T, len(tokens), H, D] and lse [B, len(tokens), H, T].
    """
    B, T, S, H, D = q.shape
    tokens = np.arange(S) if tokens is None else np.asarray(tokens)
    o = np.empty((B, T, len(tokens), H, D))
    lse = np.empty((B, len(tokens), H, T))
    for b in range(B):
        for c0 in range(0, len(tokens), chunk):
            sel = tokens[c0:c0 + chunk]
            # [T, n, H, D] -> [n, H, T, D]: one unit per (token, head)
            qs = _f64(q[b][:, sel]).transpose(1, 2, 0, 3)
            ks = _f64(k[b][:, sel]).transpose(1, 2, 0, 3)
            vs = _f64(v[b][:, sel]).transpose(1, 2, 0, 3)
            ou, lu = attention(qs, ks, vs, scale)
            o[b, :, c0:c0 + len(sel)] = ou.transpose(2, 0, 1, 3)
            lse[b, c0:c0 + len(sel)] = lu
    return o, lse


def merge_chunks(o_parts, lse_parts):
    """Log-sum-exp merge of partials over disjoint key ranges.

    o_parts:   list of [..., D] arrays (normalised partial outputs)
    lse_parts: list of [...] arrays (their natural-log LSE)
    Returns (o [..., D], lse [...]).  Chunks with lse = -inf contribute 0.
    """
    lse_c = np.stack([_f64(x) for x in lse_parts])            # [R, ...]
    o_c = np.stack([_f64(x) for x in o_parts])                # [R, ..., D]
    M = lse_c.max(axis=0)
    Ms = np.where(np.isfinite(M), M, 0.0)
    with np.errstate(divide="ignore"):                        # rows with no keys: ln 0 = -inf
        lse = Ms + np.log(np.exp(lse_c - Ms).sum(axis=0))
    lse = np.where(np.isfinite(M), lse, -np.inf)
    w = np.where(np.isfinite(lse), np.exp(lse_c - np.where(np.isfinite(lse), lse, 0.0)), 0.0)
    o = (w[..., None] * o_c).sum(axis=0)
    return o, lse


def frames_view(buf, B, T, S, H, D, stride_b=0, stride_t=0, stride_s=0,
                t_block=0, stride_tb=0, s_block=0, stride_sb=0):
    """Logical [B,T,S,H,D] array of a strided buffer, as the attention calls read it.

    Element (b, t, s, h, d) lives at flat offset
        b*stride_b + (t // t_block)*stride_tb + (t % t_block)*stride_t
                   + (s // s_block)*stride_sb + (s % s_block)*stride_s + h*D + d
    with t_block = T (s_block = S) when given as 0; zero strides mean the
    dense layout [B, T, S, H*D].
    """
    C = H * D
    stride_s = stride_s or C
    stride_t = stride_t or S * stride_s
    stride_b = stride_b or T * stride_t
    tb = t_block or T
    sb = s_block or S
    stride_tb = stride_tb if t_block else tb * stride_t
    stride_sb = stride_sb if s_block else sb * stride_s
    flat = _f64(buf).reshape(-1)
    t = np.arange(T)
    s = np.arange(S)
    off = (np.arange(B)[:, None, None, None] * stride_b
           + ((t // tb) * stride_tb + (t % tb) * stride_t)[None, :, None, None]
           + ((s // sb) * stride_sb + (s % sb) * stride_s)[None, None, :, None]
           + np.arange(C)[None, None, None, :])
    return flat[off].reshape(B, T, S, H, D)
