"""Pins of the fp64 attention oracle and the chunk merge (CPU only).

Every check here compares the oracle with something other than itself:
closed forms worked by hand, a pure-Python brute force written separately,
invariants of softmax attention, and the merge identity (R chunks merged by
log-sum-exp equal attention over all keys).
"""
import json
import math
import os
import random

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def brute_force(q, k, v, scale):
    """Pure-Python loops, one query at a time, exp via math.exp."""
    out, lses = [], []
    for qi in q:
        scores = [scale * sum(a * b for a, b in zip(qi, kj)) for kj in k]
        top = max(scores)
        w = [math.exp(s - top) for s in scores]
        tot = sum(w)
        out.append([sum(w[j] * v[j][d] for j in range(len(k))) / tot for d in range(len(v[0]))])
        lses.append(top + math.log(tot))
    return np.array(out), np.array(lses)


def test_golden_closed_forms():
    cases = json.load(open(os.path.join(GOLDEN, "attention_closed_forms.json")))["cases"]
    for c in cases:
        o, lse = oracle.attention(np.array(c["q"]), np.array(c["k"]), np.array(c["v"]), c["scale"])
        np.testing.assert_allclose(o, c["o"], rtol=0, atol=1e-12, err_msg=c["name"])
        np.testing.assert_allclose(lse, c["lse"], rtol=0, atol=1e-12, err_msg=c["name"])


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_tiny(seed):
    rng = random.Random(seed)
    M, N, D = rng.randint(1, 6), rng.randint(1, 16), rng.randint(1, 8)
    r = np.random.default_rng(seed)
    q, k, v = r.normal(size=(M, D)) * 2, r.normal(size=(N, D)) * 2, r.normal(size=(N, D))
    o, lse = oracle.attention(q, k, v)
    ob, lb = brute_force(q.tolist(), k.tolist(), v.tolist(), 1.0 / math.sqrt(D))
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


def test_tiny_workload_against_brute_force():
    """Config-1 shapes: every spatial and temporal unit against the brute force."""
    w = synth.BY_NAME["tiny"]
    q, k, v = (x.double().numpy() for x in synth.qkv(w))
    o, lse = oracle.spatial(q, k, v)
    sc = 1.0 / math.sqrt(w.D)
    for t in range(w.T):
        for h in range(w.H):
            ob, lb = brute_force(q[0, t, :, h].tolist(), k[0, t, :, h].tolist(), v[0, t, :, h].tolist(), sc)
            np.testing.assert_allclose(o[0, t, :, h], ob, atol=1e-12)
            np.testing.assert_allclose(lse[0, t, h], lb, atol=1e-12)
    ot, lt = oracle.temporal(q, k, v)
    for s in range(0, w.S, 7):
        for h in range(w.H):
            ob, lb = brute_force(q[0, :, s, h].tolist(), k[0, :, s, h].tolist(), v[0, :, s, h].tolist(), sc)
            np.testing.assert_allclose(ot[0, :, s, h], ob, atol=1e-12)
            np.testing.assert_allclose(lt[0, s, h], lb, atol=1e-12)


def test_single_frame_temporal_is_v():
    """T = 1: the only key is the token itself, so o = v and lse = the score."""
    r = np.random.default_rng(1)
    q, k, v = (r.normal(size=(1, 1, 9, 3, 8)) for _ in range(3))
    o, lse = oracle.temporal(q, k, v)
    np.testing.assert_array_equal(o, v)
    score = (q * k).sum(-1) / math.sqrt(8)                     # [1,1,9,3]
    np.testing.assert_allclose(lse[0, :, :, 0], score[0, 0], atol=1e-14)


def test_equal_keys_and_zero_query_give_mean():
    r = np.random.default_rng(2)
    v = r.normal(size=(10, 16))
    k = np.repeat(r.normal(size=(1, 16)), 10, axis=0)
    q = r.normal(size=(4, 16))
    o, _ = oracle.attention(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(0), o.shape), atol=1e-13)
    o0, l0 = oracle.attention(np.zeros((3, 16)), r.normal(size=(10, 16)), v)
    np.testing.assert_allclose(o0, np.broadcast_to(v.mean(0), o0.shape), atol=1e-13)
    np.testing.assert_allclose(l0, math.log(10), atol=1e-14)


def test_dominant_key():
    """A score ahead of every other by more than 800 selects that value row."""
    D = 4
    q = np.array([[1.0, 0, 0, 0]])
    k = np.zeros((5, D))
    k[3, 0] = 2000.0                                            # score 1000 at scale 1/2
    v = np.arange(5 * D, dtype=float).reshape(5, D)
    o, lse = oracle.attention(q, k, v)
    np.testing.assert_array_equal(o[0], v[3])
    assert lse[0] == pytest.approx(1000.0, abs=1e-12)


def test_permutation_equivariance_and_scale():
    r = np.random.default_rng(3)
    q, k, v = r.normal(size=(7, 12)), r.normal(size=(11, 12)), r.normal(size=(11, 5))
    o, lse = oracle.attention(q, k, v)
    perm = r.permutation(11)
    o2, l2 = oracle.attention(q, k[perm], v[perm])
    np.testing.assert_allclose(o2, o, atol=1e-13)
    np.testing.assert_allclose(l2, lse, atol=1e-13)
    qp = r.permutation(7)
    o3, _ = oracle.attention(q[qp], k, v)
    np.testing.assert_allclose(o3, o[qp], atol=1e-13)
    o4, _ = oracle.attention(q, k, v, scale=1 / math.sqrt(12))
    np.testing.assert_array_equal(o4, o)
    o5, _ = oracle.attention(q * 2, k, v, scale=0.5 / math.sqrt(12))
    np.testing.assert_allclose(o5, o, atol=1e-13)


def test_spatial_is_per_frame_and_temporal_is_per_token():
    """Spatial attention mixes tokens within one frame only; temporal mixes frames only."""
    r = np.random.default_rng(4)
    q, k, v = (r.normal(size=(1, 3, 5, 2, 4)) for _ in range(3))
    o, _ = oracle.spatial(q, k, v)
    k2, v2 = k.copy(), v.copy()
    k2[0, 1] += 1.0
    v2[0, 1] -= 2.0                                             # perturb frame 1 only
    o2, _ = oracle.spatial(q, k2, v2)
    np.testing.assert_array_equal(o2[0, [0, 2]], o[0, [0, 2]])
    assert not np.allclose(o2[0, 1], o[0, 1])
    ot, _ = oracle.temporal(q, k, v)
    k3 = k.copy()
    k3[0, :, 2] += 1.0                                           # perturb token 2 only
    ot3, _ = oracle.temporal(q, k3, v)
    np.testing.assert_array_equal(ot3[:, :, [0, 1, 3, 4]], ot[:, :, [0, 1, 3, 4]])


def test_st_independence_identity():
    """Slicing the spatial layer along T (temporal along S) changes nothing.

    ScaleFusion review, section "三、技术架构", core formulas.
    """
    w = synth.BY_NAME["tiny"]
    q, k, v = (x.double().numpy() for x in synth.qkv(w))
    o, lse = oracle.spatial(q, k, v)
    parts = [oracle.spatial(q[:, i:i + 2], k[:, i:i + 2], v[:, i:i + 2]) for i in (0, 2)]
    np.testing.assert_array_equal(np.concatenate([p[0] for p in parts], axis=1), o)
    np.testing.assert_array_equal(np.concatenate([p[1] for p in parts], axis=1), lse)
    ot, lt = oracle.temporal(q, k, v)
    tp = [oracle.temporal(q[:, :, j:j + 32], k[:, :, j:j + 32], v[:, :, j:j + 32]) for j in (0, 32)]
    np.testing.assert_array_equal(np.concatenate([p[0] for p in tp], axis=2), ot)
    np.testing.assert_array_equal(np.concatenate([p[1] for p in tp], axis=1), lt)


@pytest.mark.parametrize("R", range(1, 9))
def test_merge_of_chunks_equals_full(R):
    r = np.random.default_rng(10 + R)
    N = 37
    q, k, v = r.normal(size=(2, 6, 8)), r.normal(size=(2, N, 8)) * 1.5, r.normal(size=(2, N, 8))
    o, lse = oracle.attention(q, k, v)
    cuts = np.sort(r.choice(np.arange(1, N), size=R - 1, replace=False)) if R > 1 else []
    edges = [0, *cuts, N]
    parts = [oracle.attention(q, k[:, a:b], v[:, a:b]) for a, b in zip(edges[:-1], edges[1:])]
    om, lm = oracle.merge_chunks([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(om, o, atol=1e-12)
    np.testing.assert_allclose(lm, lse, atol=1e-12)
    # any chunk order merges to the same result
    order = r.permutation(len(parts))
    om2, lm2 = oracle.merge_chunks([parts[i][0] for i in order], [parts[i][1] for i in order])
    np.testing.assert_allclose(om2, om, atol=1e-13)
    np.testing.assert_allclose(lm2, lm, atol=1e-13)


def test_merge_special_cases():
    r = np.random.default_rng(5)
    o, lse = r.normal(size=(4, 3, 8)), r.normal(size=(4, 3))
    o1, l1 = oracle.merge_chunks([o], [lse])
    np.testing.assert_allclose(o1, o, atol=1e-15)
    np.testing.assert_allclose(l1, lse, atol=1e-15)
    o2, l2 = oracle.merge_chunks([o, o], [lse, lse])              # a chunk merged with itself
    np.testing.assert_allclose(o2, o, atol=1e-14)
    np.testing.assert_allclose(l2, lse + math.log(2), atol=1e-14)
    # an empty key range is the identity of the merge
    q = r.normal(size=(5, 8))
    k, v = r.normal(size=(9, 8)), r.normal(size=(9, 8))
    oe, le = oracle.attention(q, k[:0], v[:0])
    assert np.all(le == -np.inf) and np.all(oe == 0)
    of, lf = oracle.attention(q, k, v)
    om, lm = oracle.merge_chunks([of, oe], [lf, le])
    np.testing.assert_allclose(om, of, atol=1e-15)
    np.testing.assert_allclose(lm, lf, atol=1e-15)


def test_spatial_kv_range_and_rows():
    r = np.random.default_rng(6)
    q, k, v = (r.normal(size=(1, 2, 20, 2, 8)) for _ in range(3))
    o, lse = oracle.spatial(q, k, v)
    parts = [oracle.spatial(q, k, v, kv=(a, b)) for a, b in ((0, 7), (7, 20))]
    om, lm = oracle.merge_chunks([p[0] for p in parts],
                                 [p[1].transpose(0, 1, 3, 2) for p in parts])
    np.testing.assert_allclose(om, o, atol=1e-12)
    np.testing.assert_allclose(lm.transpose(0, 1, 3, 2), lse, atol=1e-12)
    rows = [3, 0, 19]
    osub, lsub = oracle.spatial(q, k, v, rows=rows, frames=[1])
    np.testing.assert_array_equal(osub[0, 0], o[0, 1, rows])
    np.testing.assert_array_equal(lsub[0, 0], lse[0, 1][:, rows])


def test_frames_view_two_level_strides():
    """The strided view reads the two-level slice layout back to logical order."""
    B, T, S, H, D = 2, 4, 6, 1, 2
    logical = np.arange(B * T * S * H * D, dtype=float).reshape(B, T, S, H, D)
    # store frames in blocks of 2 and tokens in blocks of 3 with the block axes outermost
    buf = logical.reshape(B, 2, 2, 2, 3, H * D).transpose(0, 1, 3, 2, 4, 5).copy()
    C = H * D
    view = oracle.frames_view(buf, B, T, S, H, D, stride_b=T * S * C, stride_t=3 * C,
                              stride_s=C, t_block=2, stride_tb=2 * 2 * 3 * C,
                              s_block=3, stride_sb=2 * 3 * C)
    np.testing.assert_array_equal(view, logical)
