"""Pieces of the intra-GPU chunk-and-overlap schedule, through the C ABI:
the relayout restricted to a range of temporally sharded shards (each range
writes exactly its rows, bit for bit as the oracle; any partition of the
shards in any order equals one full call, with and without the fused
RMSNorm), and the SM budget (grids sized for fewer SMs give identical
results in every kernel the bench step launches)."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import sequence_parallelism_st_b200 as st
    return st


def bits(t):
    t = t.detach().to("cpu").contiguous()
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


@pytest.mark.parametrize("name", ["tiny", "opensora_low", "video_1080p"])
@pytest.mark.parametrize("mode", ["S2T", "T2S"])
def test_st_relayout_shard_range_rows(st, name, mode):
    w = synth.BY_NAME[name]
    rows = w.B * w.T * w.S
    per = rows // w.P                                   # rows of one shard
    x = synth.randn(w, "q", (rows, w.C))
    dst, src = oracle.st_row_pairs(mode, w.P, w.B, w.T, w.S, w.n_t, w.n_s)
    y_row = dst if mode == "S2T" else src               # the y (temporally sharded) side of each pair
    q0, q1 = (1, w.P - 1) if w.P > 2 else (1, 2)
    fill = torch.full((rows, w.C), float("nan"), dtype=x.dtype)
    out = fill.to(DEV)
    st.ulysses_relayout_range(mode, x.to(DEV), out, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s, shards=(q0, q1))
    torch.cuda.synchronize()
    sel = (y_row // per >= q0) & (y_row // per < q1)
    assert sel.sum() == rows * (q1 - q0) // w.P
    got, xb = bits(out), bits(x)
    assert torch.equal(got[torch.from_numpy(dst[sel])], xb[torch.from_numpy(src[sel])])
    assert torch.equal(got[torch.from_numpy(dst[~sel])], bits(fill)[torch.from_numpy(dst[~sel])])


@pytest.mark.parametrize("name", ["opensora_low", "video_1080p"])
def test_st_relayout_shard_partitions_equal_full(st, name):
    w = synth.BY_NAME[name]
    rows = w.B * w.T * w.S
    x = synth.randn(w, "k", (rows, w.C)).to(DEV)
    rng = np.random.default_rng(5)
    for mode in ("S2T", "T2S"):
        full = torch.empty_like(x)
        st.ulysses_relayout(mode, x, full, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s)
        cuts = sorted(rng.choice(np.arange(1, w.P), size=min(2, w.P - 1), replace=False).tolist())
        edges = [0] + cuts + [w.P]
        ranges = list(zip(edges[:-1], edges[1:]))
        out = torch.zeros_like(x)
        for r in rng.permutation(len(ranges)):
            st.ulysses_relayout_range(mode, x, out, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s, shards=ranges[r])
        assert torch.equal(bits(out), bits(full)), (mode, ranges)
    # shard ranges combine with the (i, j) block ranges of the inter-layer schedule
    full = torch.empty_like(x)
    st.ulysses_relayout("S2T", x, full, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s)
    out = torch.zeros_like(x)
    for q in range(w.P):
        for i in range(w.n_t):
            st.ulysses_relayout_range("S2T", x, out, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s,
                                      blocks=(i, i + 1, 0, w.n_s), shards=(q, q + 1))
    assert torch.equal(bits(out), bits(full))


def test_st_relayout_rms_shard_ranges(st):
    """The fused RMSNorm path over shard ranges equals one full call bit for bit."""
    w = synth.BY_NAME["opensora_low"]
    rows = w.B * w.T * w.S
    x = synth.randn(w, "q", (rows, w.C)).to(DEV)
    gamma = synth.rms_gamma(w).to(DEV)
    kw = dict(rms_gamma=gamma, rms_head_dim=w.D, rms_eps=w.rms_eps)
    full = torch.empty_like(x)
    st.ulysses_relayout("S2T", x, full, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s, **kw)
    out = torch.zeros_like(x)
    for r in [(2, 4), (0, 1), (1, 2)]:
        st.ulysses_relayout_range("S2T", x, out, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s, shards=r, **kw)
    assert torch.equal(bits(out), bits(full))


def test_sm_budget_does_not_change_results(st):
    """Every kernel of the bench step gives the same bits with its grid sized for 20 SMs."""
    w = synth.BY_NAME["opensora_low"]
    B, T, S, H, D, C = w.B, w.T, w.S, w.H, w.D, w.C
    n = B * T * S
    q, k, v = (t.to(DEV) for t in synth.qkv(w))
    gamma = synth.rms_gamma(w).to(DEV)
    cur, prev = (t.to(DEV) for t in synth.vmajor_pair(w, n, C))
    tau = float(oracle.tau_for_fraction(oracle.l1_change(*synth.vmajor_pair(w, n, C)), 0.5)[0])
    ws = torch.empty(max(16, st.vmajor_workspace_bytes(n)), dtype=torch.uint8, device=DEV)

    def run():
        res = []
        y = torch.empty(n * C, dtype=torch.bfloat16, device=DEV)
        st.ulysses_relayout("S2T", q, y, w.P, B, T, S, C, w.n_t, w.n_s, rms_gamma=gamma, rms_head_dim=D,
                            rms_eps=w.rms_eps)
        res.append(y)
        y2 = torch.empty_like(y)
        st.ulysses_relayout("T2S", y, y2, w.P, B, T, S, C, w.n_t, w.n_s)
        res.append(y2)
        parts, lses = [], []
        for c in range(2):
            o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
            L = torch.empty((B, T, H, S), dtype=torch.float32, device=DEV)
            st.st_attn_spatial(q, k, v, o, L, o_fp32=1, kv_begin=c * S // 2, kv_end=(c + 1) * S // 2)
            parts.append(o)
            lses.append(L)
        res += parts + lses
        om = torch.empty(q.shape, dtype=torch.bfloat16, device=DEV)
        st.attn_chunk_merge(parts, lses, B * T, S, H, D, om)
        res.append(om)
        ot = torch.empty_like(q)
        st.st_attn_temporal(q, k, v, ot, None)
        res.append(ot)
        mask = torch.empty(n, dtype=torch.uint8, device=DEV)
        idx = torch.full((n,), -1, dtype=torch.int32, device=DEV)
        cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
        st.vmajor_mask_compact(cur.view(n, C), prev.view(n, C), tau, mask, idx, cnt, ws)
        kc, vc = prev.clone().view(n, C), prev.clone().view(n, C)
        st.vmajor_scatter_rows(idx, cnt, [cur.view(n, C), cur.view(n, C)], [kc, vc])
        res += [mask, idx, cnt, kc, vc]
        torch.cuda.synchronize()
        return res

    ref = run()
    try:
        st.st_set_sm_budget(20)
        assert st.st_get_sm_budget() == 20
        got = run()
    finally:
        st.st_set_sm_budget(0)
    assert st.st_get_sm_budget() == 0
    for i, (a, b) in enumerate(zip(got, ref)):
        assert torch.equal(a, b), f"output {i} differs under an SM budget"
    assert st.st_check_device_status() == st.ST_OK
