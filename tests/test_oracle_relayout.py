"""Pins of the relayout, RMSNorm and V-Major oracles (CPU only).

The relayout oracle is pinned against an independent derivation with
np.reshape / np.transpose, against index-tagged inputs (every destination
element comes from exactly one source element), round trips and P = 1.
"""
import math

import numpy as np
import pytest

import oracle
import synth


def logical_to_x_by_transpose(X, P, n_t, n_s):
    """[B,T,S,C] -> stacked x shards, by reshapes only (independent of the oracle)."""
    B, T, S, C = X.shape
    # s = j*S/n_s + p*S/(n_s P) + s1 ; t = i*T/n_t + t1
    a = X.reshape(B, n_t, T // n_t, n_s, P, S // (n_s * P), C)   # b i t1 j p s1 c
    return a.transpose(4, 0, 1, 3, 2, 5, 6).copy()               # p b i j t1 s1 c


def logical_to_y_by_transpose(X, P, n_t, n_s):
    B, T, S, C = X.shape
    # t = i*T/n_t + q*T/(n_t P) + t2 ; s = j*S/n_s + s2
    a = X.reshape(B, n_t, P, T // (n_t * P), n_s, S // n_s, C)   # b i q t2 j s2 c
    return a.transpose(2, 0, 1, 4, 3, 5, 6).copy()               # q b i j t2 s2 c


ST_CASES = [(2, 1, 4, 8, 3, 1, 1), (2, 1, 4, 64, 5, 2, 2), (4, 2, 8, 24, 2, 2, 3),
            (1, 1, 3, 5, 2, 1, 1), (3, 1, 6, 9, 1, 2, 3), (2, 1, 8, 16, 4, 4, 2)]


@pytest.mark.parametrize("P,B,T,S,C,n_t,n_s", ST_CASES)
def test_st_matches_transpose_derivation(P, B, T, S, C, n_t, n_s):
    X = np.random.default_rng(P * 100 + T).normal(size=(B, T, S, C))
    x = logical_to_x_by_transpose(X, P, n_t, n_s)
    y = logical_to_y_by_transpose(X, P, n_t, n_s)
    y_o = oracle.st_relayout("S2T", x, P, B, T, S, C, n_t, n_s)
    np.testing.assert_array_equal(y_o, y.reshape(-1))
    x_o = oracle.st_relayout("T2S", y, P, B, T, S, C, n_t, n_s)
    np.testing.assert_array_equal(x_o, x.reshape(-1))
    np.testing.assert_array_equal(oracle.st_logical_from_x(x, P, B, T, S, C, n_t, n_s), X)
    np.testing.assert_array_equal(oracle.st_logical_from_y(y, P, B, T, S, C, n_t, n_s), X)


def test_plain_layouts_match_layer_table():
    """N_T = N_S = 1: x is [P][B,T,S/P,C] and y is [P][B,T/P,S,C]."""
    P, B, T, S, C = 4, 1, 8, 12, 3
    X = np.arange(B * T * S * C, dtype=float).reshape(B, T, S, C)
    x = np.stack([X[:, :, p * S // P:(p + 1) * S // P] for p in range(P)])
    y = np.stack([X[:, q * T // P:(q + 1) * T // P] for q in range(P)])
    np.testing.assert_array_equal(oracle.st_relayout("S2T", x, P, B, T, S, C), y.reshape(-1))
    np.testing.assert_array_equal(oracle.st_relayout("T2S", y, P, B, T, S, C), x.reshape(-1))


def test_index_tagged_bijection():
    P, B, T, S, C, n_t, n_s = 4, 1, 16, 48, 6, 2, 3
    tagged = synth.index_tagged(P * B * (T // P) * S, C).double().numpy()
    y = oracle.st_relayout("S2T", tagged, P, B, T, S, C, n_t, n_s)
    assert not np.isnan(y).any()
    np.testing.assert_array_equal(np.sort(y), np.arange(y.size, dtype=float))
    # every element keeps its channel: column = value mod C
    np.testing.assert_array_equal(y.reshape(-1, C) % C, np.broadcast_to(np.arange(C), (y.size // C, C)))


def test_p1_is_identity_and_round_trip():
    r = np.random.default_rng(7)
    B, T, S, C = 1, 4, 6, 5
    x = r.normal(size=B * T * S * C)
    np.testing.assert_array_equal(oracle.st_relayout("S2T", x, 1, B, T, S, C), x)
    for (P, n_t, n_s) in [(2, 2, 3), (4, 1, 1), (2, 1, 3)]:
        T2, S2 = 8, 12
        x = r.normal(size=B * T2 * S2 * C)
        y = oracle.st_relayout("S2T", x, P, B, T2, S2, C, n_t, n_s)
        np.testing.assert_array_equal(oracle.st_relayout("T2S", y, P, B, T2, S2, C, n_t, n_s), x)


def test_block_ranges_compose_to_full():
    """Any partition of the (i, j) blocks, in any order, gives the full relayout."""
    P, B, T, S, C, n_t, n_s = 2, 1, 8, 12, 2, 4, 3
    r = np.random.default_rng(8)
    x = r.normal(size=P * B * (T) * (S // P) * C)
    full = oracle.st_relayout("S2T", x, P, B, T, S, C, n_t, n_s)
    out = np.full(full.size, np.nan)
    blocks = [(i, i + 1, j, j + 1) for i in range(n_t) for j in range(n_s)]
    for bi in r.permutation(len(blocks)):
        out = oracle.st_relayout("S2T", x, P, B, T, S, C, n_t, n_s, blocks=blocks[bi], out=out)
    np.testing.assert_array_equal(out, full)
    part = oracle.st_relayout("S2T", x, P, B, T, S, C, n_t, n_s, blocks=(0, 1, 0, n_s))
    assert np.isnan(part).sum() == full.size * (n_t - 1) // n_t


@pytest.mark.parametrize("P,B,N,H,D", [(2, 1, 6, 4, 3), (4, 2, 8, 8, 2), (1, 1, 5, 3, 2), (8, 1, 16, 24, 4)])
def test_seq_head_matches_transpose(P, B, N, H, D):
    X = np.random.default_rng(N).normal(size=(B, N, H, D))
    inp = X.reshape(B, P, N // P, H, D).transpose(1, 0, 2, 3, 4)            # p b n1 h d
    out = X.reshape(B, N, P, H // P, D).transpose(2, 0, 3, 1, 4)            # q b h1 n d
    np.testing.assert_array_equal(oracle.seq_head_relayout("SEQ2HEAD", inp, P, B, N, H, D), out.reshape(-1))
    np.testing.assert_array_equal(oracle.seq_head_relayout("HEAD2SEQ", out, P, B, N, H, D), inp.reshape(-1))


def test_rmsnorm_pins():
    r = np.random.default_rng(9)
    D = 16
    x = r.normal(size=(10, 4 * D)) * 3
    y = oracle.rmsnorm_heads(x, np.ones(D), D, 0.0)
    seg = y.reshape(-1, D)
    np.testing.assert_allclose(np.sqrt((seg ** 2).mean(1)), 1.0, atol=1e-14)     # unit RMS
    np.testing.assert_allclose(oracle.rmsnorm_heads(x * 7.5, np.ones(D), D, 0.0), y, atol=1e-13)
    c = np.full((1, D), 0.5)                                                     # constant vector
    g = r.normal(size=D)
    np.testing.assert_allclose(oracle.rmsnorm_heads(c, g, D, 1e-6), 0.5 / math.sqrt(0.25 + 1e-6) * g[None], atol=1e-15)
    # commutes with the sequence->head exchange (D stays contiguous)
    P, B, N, H = 2, 1, 4, 4
    X = r.normal(size=(P * B * (N // P) * H * D))
    a = oracle.seq_head_relayout("SEQ2HEAD", X, P, B, N, H, D, rms=(g, D, 1e-6))
    b = oracle.seq_head_relayout("SEQ2HEAD", oracle.rmsnorm_heads(X.reshape(-1, D), g, D, 1e-6), P, B, N, H, D)
    np.testing.assert_allclose(a, b, atol=1e-14)


def test_vmajor_pins():
    r = np.random.default_rng(11)
    prev = r.normal(size=(50, 12))
    cur = prev.copy()
    cur[[3, 17, 40]] += 0.5
    l1 = oracle.l1_change(cur, prev)
    np.testing.assert_allclose(l1[[3, 17, 40]], 6.0, atol=1e-12)                  # 12 channels * 0.5
    assert np.count_nonzero(l1) == 3
    m = oracle.change_mask(l1, 1.0)
    idx, cnt = oracle.compact(m)
    np.testing.assert_array_equal(idx, [3, 17, 40])
    assert cnt == 3
    assert oracle.change_mask(l1, -1.0).all()                                     # tau < 0: all active
    assert not oracle.change_mask(oracle.l1_change(prev, prev), 0.0).any()        # no change: none
    assert oracle.change_mask(l1, 6.0).sum() == 0                                 # strict comparison
    assert oracle.change_mask(l1, 1e9, force_all=True).all()                      # full refresh step
    mm = (r.random(1000) < 0.3).astype(np.uint8)
    i2, c2 = oracle.compact(mm)
    np.testing.assert_array_equal(i2, np.flatnonzero(mm))
    assert c2 == mm.sum()
    cache = r.normal(size=(50, 12))
    new = oracle.scatter_rows(idx, cnt, cur, cache)
    np.testing.assert_array_equal(new[[3, 17, 40]], cur[[3, 17, 40]])
    keep = np.setdiff1d(np.arange(50), [3, 17, 40])
    np.testing.assert_array_equal(new[keep], cache[keep])
    np.testing.assert_array_equal(oracle.pack_rows(idx, cnt, cur), cur[[3, 17, 40]])


def test_tau_for_fraction():
    l1 = np.random.default_rng(12).lognormal(size=1000)
    for f in (0.1, 0.5, 0.9):
        tau, margin, frac = oracle.tau_for_fraction(l1, f, window=0.0)
        assert (l1 > tau).sum() == round(1000 * f) and frac == (l1 > tau).mean()
        assert margin > 0
        tau2, margin2, frac2 = oracle.tau_for_fraction(l1, f, window=0.02)
        assert abs(frac2 - f) <= 0.021 and margin2 >= margin


def test_vmajor_recipe_small_sigma_rounds_back():
    """bf16 storage: a perturbation well below half an ulp leaves the stored value unchanged."""
    w = synth.BY_NAME["vmajor_2304px"]
    cur, prev = synth.vmajor_pair(w, 512, 64)
    sig = synth.token_sigma(w, 512)
    l1 = oracle.l1_change(cur, prev)
    assert l1[sig < 2e-4].mean() < l1[sig > 5e-2].mean() / 50


def test_row_pairs_agree_with_relayout():
    r = np.random.default_rng(13)
    P, B, T, S, C, n_t, n_s = 2, 1, 8, 12, 3, 2, 3
    x = r.normal(size=P * B * T * (S // P) * C)
    dst, src = oracle.st_row_pairs("S2T", P, B, T, S, n_t, n_s, blocks=(1, 2, 0, 2))
    full = oracle.st_relayout("S2T", x, P, B, T, S, C, n_t, n_s, blocks=(1, 2, 0, 2))
    np.testing.assert_array_equal(full.reshape(-1, C)[dst], x.reshape(-1, C)[src])
    P, N, H, D = 4, 8, 8, 2
    y = r.normal(size=B * N * H * D)
    dst, src = oracle.seq_head_row_pairs("HEAD2SEQ", P, B, N, H)
    np.testing.assert_array_equal(oracle.seq_head_relayout("HEAD2SEQ", y, P, B, N, H, D).reshape(-1, D)[dst],
                                  y.reshape(-1, D)[src])
