"""GPU parity of the relayout, V-Major, chunk-merge and temporal kernels
against the fp64 oracle, through the C ABI (via the ctypes binding)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, assert_lse_close, f64

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


# ------------------------------------------------------------------ relayout
ST_CASES = [("tiny", 1, 1), ("tiny", None, None), ("opensora_low", None, None), ("opensora_low", 1, 1),
            ("video_1080p", None, None)]


@pytest.mark.parametrize("name,n_t,n_s", ST_CASES)
@pytest.mark.parametrize("mode", ["S2T", "T2S"])
def test_st_relayout_bit_exact(st, name, n_t, n_s, mode):
    w = synth.BY_NAME[name]
    n_t = w.n_t if n_t is None else n_t
    n_s = w.n_s if n_s is None else n_s
    rows = w.B * w.T * w.S
    x = synth.randn(w, "q", (rows, w.C))
    out = torch.full((rows, w.C), float("nan"), dtype=x.dtype, device=DEV)
    st.ulysses_relayout(mode, x.to(DEV), out, w.P, w.B, w.T, w.S, w.C, n_t, n_s)
    torch.cuda.synchronize()
    dst, src = oracle.st_row_pairs(mode, w.P, w.B, w.T, w.S, n_t, n_s)
    assert len(dst) == rows
    got = bits(out)
    assert torch.equal(got[torch.from_numpy(dst)], bits(x)[torch.from_numpy(src)])


def test_st_relayout_round_trip_and_blocks(st):
    """T2S(S2T(x)) == x; L_S/L_T block partitions in any order == full relayout."""
    w = synth.BY_NAME["video_1080p"]
    rows = w.B * w.T * w.S
    x = synth.randn(w, "k", (rows, w.C)).to(DEV)
    y = torch.empty_like(x)
    st.ulysses_relayout("S2T", x, y, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s)
    back = torch.empty_like(x)
    st.ulysses_relayout("T2S", y, back, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s)
    assert torch.equal(bits(back), bits(x))
    # the inter-layer schedule hoists partitions: L_S of the N_T row blocks first, then the rest
    y2 = torch.zeros_like(x)
    parts = [(0, w.L_S, 0, w.n_s), (w.L_S, w.n_t, 0, w.n_s)]
    for blk in reversed(parts):
        st.ulysses_relayout("S2T", x, y2, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s, blocks=blk)
    assert torch.equal(bits(y2), bits(y))
    y3 = torch.zeros_like(x)
    rng = np.random.default_rng(0)
    blocks = [(i, i + 1, j, j + 1) for i in range(w.n_t) for j in range(w.n_s)]
    for b in rng.permutation(len(blocks)):
        st.ulysses_relayout("S2T", x, y3, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s, blocks=blocks[b])
    assert torch.equal(bits(y3), bits(y))


@pytest.mark.parametrize("mode", ["SEQ2HEAD", "HEAD2SEQ"])
def test_seq_head_bit_exact(st, mode):
    w = synth.BY_NAME["image_4096px"]
    N, H, D = w.S, w.H, w.D
    x = synth.randn(w, "v", (N * H, D))
    out = torch.empty((N * H, D), dtype=x.dtype, device=DEV)
    st.ulysses_relayout(mode, x.to(DEV), out, w.P, w.B, N, H, D)
    torch.cuda.synchronize()
    dst, src = oracle.seq_head_row_pairs(mode, w.P, w.B, N, H)
    assert torch.equal(bits(out)[torch.from_numpy(dst)], bits(x)[torch.from_numpy(src)])


def test_relayout_odd_widths(st):
    """Rows that are not 16-byte multiples take narrower vectors; uint8 and fp64 rows."""
    rng = np.random.default_rng(1)
    for dtype, C in ((torch.uint8, 6), (torch.float64, 5), (torch.bfloat16, 36), (torch.float32, 3)):
        P, B, T, S = 2, 1, 4, 10
        if dtype == torch.uint8:
            x = torch.from_numpy(rng.integers(0, 255, size=(B * T * S, C), dtype=np.uint8))
        else:
            x = torch.from_numpy(rng.normal(size=(B * T * S, C))).to(dtype)
        out = torch.zeros_like(x, device=DEV)
        st.ulysses_relayout("S2T", x.to(DEV), out, P, B, T, S, C, 2, 1)
        dst, src = oracle.st_row_pairs("S2T", P, B, T, S, 2, 1)
        o = out.cpu()
        assert torch.equal(o[torch.from_numpy(dst)], x[torch.from_numpy(src)]), dtype


@pytest.mark.parametrize("name", ["tiny", "opensora_low"])
def test_st_relayout_fused_rmsnorm(st, name):
    w = synth.BY_NAME[name]
    rows = w.B * w.T * w.S
    x = synth.randn(w, "q", (rows, w.C))
    gamma = synth.rms_gamma(w)
    out = torch.empty((rows, w.C), dtype=x.dtype, device=DEV)
    st.ulysses_relayout("S2T", x.to(DEV), out, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s,
                        rms_gamma=gamma.to(DEV), rms_head_dim=w.D, rms_eps=w.rms_eps)
    ref = oracle.st_relayout("S2T", x, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s, rms=(gamma, w.D, w.rms_eps))
    assert_close(out.reshape(-1), ref, w.dtype, f"rms {name}")


def test_seq2head_fused_rmsnorm_sampled(st):
    w = synth.BY_NAME["image_4096px"]
    N, H, D = w.S, w.H, w.D
    x = synth.randn(w, "q", (N * H, D))
    gamma = synth.rms_gamma(w)
    out = torch.empty((N * H, D), dtype=x.dtype, device=DEV)
    st.ulysses_relayout("SEQ2HEAD", x.to(DEV), out, w.P, w.B, N, H, D, rms_gamma=gamma.to(DEV),
                        rms_head_dim=D, rms_eps=w.rms_eps)
    dst, src = oracle.seq_head_row_pairs("SEQ2HEAD", w.P, w.B, N, H)
    pick = np.random.default_rng(2).choice(len(dst), 8192, replace=False)
    ref = oracle.rmsnorm_heads(f64(x)[src[pick]], gamma, D, w.rms_eps)
    assert_close(out.cpu()[torch.from_numpy(dst[pick])], ref, "bf16", "seq2head rms")


# ------------------------------------------------------------------ V-Major
def taus():
    path = os.path.join(os.path.dirname(__file__), "golden", "vmajor_tau.json")
    return json.load(open(path))["workloads"]


VM_CASES = [("vmajor_2304px", 0.5), ("vmajor_2304px", 0.1), ("vmajor_2304px", 0.9), ("opensora_low", 0.5),
            ("video_1080p", 0.5), ("tiny", 0.5)]


def l1_sliced(cur, prev, rows=32768):
    """oracle.l1_change over slices of tokens (bounds the fp64 copies on the host)."""
    return np.concatenate([oracle.l1_change(cur[a:a + rows], prev[a:a + rows]) for a in range(0, cur.shape[0], rows)])


@pytest.mark.parametrize("name,f", VM_CASES)
def test_vmajor_mask_compact_bit_exact(st, name, f):
    w = synth.BY_NAME[name]
    n, C = w.B * w.T * w.S, w.C
    cur, prev = synth.vmajor_pair(w, n, C)
    l1 = l1_sliced(cur, prev)
    tau, margin, _ = oracle.tau_for_fraction(l1, f)
    assert tau == pytest.approx(taus()[name][str(f)]["tau"], rel=1e-12)
    # decision is precision independent: margin above the fp32 summation bound
    assert margin > (C - 1) * 2.0 ** -24 * 1.5
    mask_ref = oracle.change_mask(l1, tau)
    idx_ref, cnt_ref = oracle.compact(mask_ref)
    mask = torch.full((n,), 7, dtype=torch.uint8, device=DEV)
    idx = torch.full((n,), -1, dtype=torch.int32, device=DEV)
    count = torch.zeros(1, dtype=torch.int32, device=DEV)
    l1_out = torch.zeros(n, dtype=torch.float32, device=DEV)
    ws = torch.zeros(st.vmajor_workspace_bytes(n), dtype=torch.uint8, device=DEV)
    st.vmajor_mask_compact(cur.to(DEV), prev.to(DEV), tau, mask, idx, count, ws, l1_out=l1_out)
    torch.cuda.synchronize()
    assert count.item() == cnt_ref
    assert np.array_equal(mask.cpu().numpy(), mask_ref)
    assert np.array_equal(idx.cpu().numpy()[:cnt_ref], idx_ref)
    assert np.all(idx.cpu().numpy()[cnt_ref:] == -1)
    np.testing.assert_allclose(l1_out.cpu().numpy(), l1, rtol=2e-5, atol=1e-6)


def test_vmajor_special_cases(st):
    w = synth.BY_NAME["vmajor_2304px"]
    n, C = 3000, w.C
    cur, prev = synth.vmajor_pair(w, n, C)
    cd, pd = cur.to(DEV), prev.to(DEV)
    mask = torch.empty(n, dtype=torch.uint8, device=DEV)
    idx = torch.empty(n, dtype=torch.int32, device=DEV)
    count = torch.empty(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(st.vmajor_workspace_bytes(n), dtype=torch.uint8, device=DEV)
    st.vmajor_mask_compact(cd, pd, 1e30, mask, idx, count, ws, force_all=True)   # full refresh
    assert count.item() == n and torch.equal(idx.cpu(), torch.arange(n, dtype=torch.int32))
    st.vmajor_mask_compact(cd, pd, -1.0, mask, idx, count, ws)                   # tau < 0
    assert count.item() == n and bool(mask.all())
    st.vmajor_mask_compact(pd, pd, 0.0, mask, idx, count, ws)                    # no change
    assert count.item() == 0 and not bool(mask.any())
    for m in (1, 31, 33, 2047, 2049):                                            # ragged tails
        st.vmajor_mask_compact(cd[:m], pd[:m], -1.0, mask, idx, count, ws)
        assert count.item() == m and torch.equal(idx[:m].cpu(), torch.arange(m, dtype=torch.int32))


def test_vmajor_scatter_rows(st):
    w = synth.BY_NAME["vmajor_2304px"]
    n, C = w.S, w.C
    cur_v, prev_v = synth.vmajor_pair(w, n, C)
    cur_k, prev_k = synth.vmajor_pair(w, n, C, prev="kprev", noise="knoise")
    tau = taus()[w.name]["0.5"]["tau"]
    l1 = oracle.l1_change(cur_v, prev_v)
    idx_ref, cnt_ref = oracle.compact(oracle.change_mask(l1, tau))
    mask = torch.empty(n, dtype=torch.uint8, device=DEV)
    idx = torch.empty(n, dtype=torch.int32, device=DEV)
    count = torch.empty(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(st.vmajor_workspace_bytes(n), dtype=torch.uint8, device=DEV)
    cv, ck = cur_v.to(DEV), cur_k.to(DEV)
    st.vmajor_mask_compact(cv, prev_v.to(DEV), tau, mask, idx, count, ws)
    kc, vc = prev_k.to(DEV), prev_v.to(DEV)                 # caches hold the previous step
    pk = torch.zeros_like(kc)
    pv = torch.zeros_like(vc)
    st.vmajor_scatter_rows(idx, count, [ck, cv], [kc, vc], packed=[pk, pv])
    torch.cuda.synchronize()
    for cache, cur, prev, packed in ((kc, cur_k, prev_k, pk), (vc, cur_v, prev_v, pv)):
        ref = oracle.scatter_rows(idx_ref, cnt_ref, cur, prev)
        assert np.array_equal(f64(cache), ref)
        assert np.array_equal(f64(packed[:cnt_ref]), oracle.pack_rows(idx_ref, cnt_ref, cur))


@pytest.mark.parametrize("name,f,keep", [("vmajor_2304px", 0.5, True), ("vmajor_2304px", 0.1, True),
                                         ("vmajor_2304px", 0.9, False), ("opensora_low", 0.5, True),
                                         ("opensora_low", 0.5, False), ("tiny", 0.5, True), ("tiny", 0.5, False)])
def test_vmajor_mask_compact_scatter_fused(st, name, f, keep):
    """The fused call gives the mask, indices, count and caches of the oracle,
    and the same bits as vmajor_mask_compact + vmajor_scatter_rows.  keep: V's
    cache takes rows of the very tensor the mask is taken on (the kernel then
    writes them from the registers that hold them); otherwise from a copy."""
    w = synth.BY_NAME[name]
    n, C = w.B * w.T * w.S, w.C
    cur_v, prev_v = synth.vmajor_pair(w, n, C)
    cur_k, prev_k = synth.vmajor_pair(w, n, C, prev="kprev", noise="knoise")
    tau = taus()[name][str(f)]["tau"]
    mask_ref = oracle.change_mask(oracle.l1_change(cur_v, prev_v), tau)
    idx_ref, cnt_ref = oracle.compact(mask_ref)
    cv, pvd, ck = cur_v.to(DEV), prev_v.to(DEV), cur_k.to(DEV)
    ws = torch.zeros(st.vmajor_workspace_bytes(n), dtype=torch.uint8, device=DEV)
    outs = []
    for fused in (True, False):
        mask = torch.full((n,), 7, dtype=torch.uint8, device=DEV)
        idx = torch.full((n,), -1, dtype=torch.int32, device=DEV)
        count = torch.zeros(1, dtype=torch.int32, device=DEV)
        kc, vc = prev_k.to(DEV), prev_v.to(DEV)
        if fused:
            st.vmajor_mask_compact_scatter(cv, pvd, tau, mask, idx, count, ws, [ck, cv if keep else cv.clone()],
                                           [kc, vc])
        else:
            st.vmajor_mask_compact(cv, pvd, tau, mask, idx, count, ws)
            st.vmajor_scatter_rows(idx, count, [ck, cv], [kc, vc])
        torch.cuda.synchronize()
        outs.append((mask.cpu(), idx.cpu(), count.cpu(), kc.cpu(), vc.cpu()))
    mask, idx, count, kc, vc = outs[0]
    assert count.item() == cnt_ref
    assert np.array_equal(mask.numpy(), mask_ref)
    assert np.array_equal(idx.numpy()[:cnt_ref], idx_ref)
    assert np.array_equal(f64(kc), oracle.scatter_rows(idx_ref, cnt_ref, cur_k, prev_k))
    assert np.array_equal(f64(vc), oracle.scatter_rows(idx_ref, cnt_ref, cur_v, prev_v))
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)


# ------------------------------------------------------------------ merge
@pytest.mark.parametrize("R,out_dtype", [(1, torch.float32), (2, torch.bfloat16), (3, torch.float32),
                                         (8, torch.bfloat16), (16, torch.float32)])
def test_chunk_merge(st, R, out_dtype):
    rng = np.random.default_rng(R)
    U, S, H, D = 3, 77, 5, 72
    o = [torch.from_numpy(rng.normal(size=(U, S, H, D))).float() for _ in range(R)]
    lse = [torch.from_numpy(rng.normal(size=(U, H, S)) * 3).float() for _ in range(R)]
    lse[0][0, 0, :5] = -math.inf                          # empty chunk rows contribute nothing
    if R == 1:
        lse[0][1, 2, 7] = -math.inf                       # a row with no keys at all
    out = torch.empty((U, S, H, D), dtype=out_dtype, device=DEV)
    lse_out = torch.empty((U, H, S), dtype=torch.float32, device=DEV)
    st.attn_chunk_merge([x.to(DEV) for x in o], [x.to(DEV) for x in lse], U, S, H, D, out, lse_out)
    torch.cuda.synchronize()
    ro, rl = oracle.merge_chunks(o, [x.permute(0, 2, 1) for x in lse])      # align lse to [U,S,H]
    ro = np.nan_to_num(ro)
    assert_close(out.cpu(), ro, "bf16" if out_dtype == torch.bfloat16 else "f32", f"merge R={R}")
    assert_lse_close(lse_out.cpu().permute(0, 2, 1), rl, "merge lse")


# ------------------------------------------------------------------ temporal
def run_temporal(st, w, q, k, v, lse=True, **kw):
    o = torch.empty(q.shape, dtype=q.dtype if not kw.get("o_fp32") else torch.float32, device=DEV)
    L = torch.empty((w.B, w.S, w.H, w.T), dtype=torch.float32, device=DEV) if lse else None
    st.st_attn_temporal(q.to(DEV), k.to(DEV), v.to(DEV), o, L, **kw)
    torch.cuda.synchronize()
    return o, L


@pytest.mark.parametrize("name", ["tiny", "opensora_low"])
def test_temporal_full(st, name):
    w = synth.BY_NAME[name]
    q, k, v = synth.qkv(w)
    o, L = run_temporal(st, w, q, k, v)
    ro, rl = oracle.temporal(q, k, v)
    assert_close(o.cpu(), ro, w.dtype, f"temporal {name}")
    assert_lse_close(L.cpu(), rl, "temporal lse")


def test_temporal_video_sampled_and_slices(st):
    w = synth.BY_NAME["video_1080p"]
    q, k, v = synth.qkv(w)
    o, L = run_temporal(st, w, q, k, v)
    tok = np.sort(np.random.default_rng(3).choice(w.S, 384, replace=False))
    ro, rl = oracle.temporal(q, k, v, tokens=tok)
    assert_close(o.cpu()[:, :, torch.from_numpy(tok)], ro, "bf16", "temporal video")
    assert_lse_close(L.cpu()[:, torch.from_numpy(tok)], rl, "temporal video lse")
    # ST independence: slicing the temporal layer along S gives bit-identical results
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o2 = torch.zeros_like(qd)
    for j in range(w.n_s):
        st.st_attn_temporal(qd, kd, vd, o2, None, n_slices=w.n_s, slice=j)
    torch.cuda.synchronize()
    assert torch.equal(bits(o2), bits(o))


@pytest.mark.parametrize("T,D,H", [(1, 72, 4), (7, 64, 6), (16, 32, 8), (33, 128, 3), (64, 80, 4), (24, 96, 5),
                                   (48, 72, 2), (12, 72, 11), (16, 80, 9), (16, 128, 5)])
def test_temporal_shapes(st, T, D, H):
    w = synth.Workload("t", 9, B=2, T=T, S=37, H=H, D=D, dtype="bf16")
    q, k, v = synth.qkv(w)
    o, L = run_temporal(st, w, q, k, v)
    ro, rl = oracle.temporal(q, k, v)
    assert_close(o.cpu(), ro, "bf16", f"temporal T={T} D={D}")
    assert_lse_close(L.cpu(), rl, "lse")
    of, _ = run_temporal(st, w, q, k, v, lse=False, o_fp32=1)
    assert_close(of.cpu(), ro, "bf16", "fp32 out")


def test_temporal_on_sliced_x_layout(st):
    """The temporal layer reads the [P,B,N_T,N_S,T/N_T,S/(N_S P),C] layout in place."""
    w = synth.BY_NAME["opensora_low"]
    q, k, v = synth.qkv(w)
    P, n_t, n_s = w.P, w.n_t, w.n_s
    Tb, Sb = w.T // n_t, w.S // (n_s * P)

    def to_x(t):
        X = t.reshape(w.B, w.T, w.S, w.C)
        return X.reshape(w.B, n_t, Tb, n_s, P, Sb, w.C).permute(4, 0, 1, 3, 2, 5, 6).contiguous()

    qx, kx, vx = to_x(q), to_x(k), to_x(v)
    C = w.C
    desc = st.make_desc(P * w.B, w.T, w.S // P, w.H, w.D, st.ST_BF16,
                        stride_b=n_t * n_s * Tb * Sb * C, stride_t=Sb * C, stride_s=C,
                        t_block=Tb, stride_tb=n_s * Tb * Sb * C, s_block=Sb, stride_sb=Tb * Sb * C)
    o = torch.empty_like(qx, device=DEV)
    st.st_attn_temporal(qx.to(DEV), kx.to(DEV), vx.to(DEV), o, None, desc=desc)
    ref_o, _ = run_temporal(st, w, q, k, v, lse=False)
    ref_x = to_x(ref_o.cpu())
    assert torch.equal(bits(o), bits(ref_x))


def test_f32_spatial_tiny(st):
    w = synth.BY_NAME["tiny"]
    q, k, v = synth.qkv(w)
    o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    L = torch.empty((w.B, w.T, w.H, w.S), dtype=torch.float32, device=DEV)
    st.st_attn_spatial(q.to(DEV), k.to(DEV), v.to(DEV), o, L)
    torch.cuda.synchronize()
    ro, rl = oracle.spatial(q, k, v)
    assert_close(o.cpu(), ro, "f32", "f32 spatial")
    assert_lse_close(L.cpu(), rl, "f32 lse")
    # KV chunks R=2 merged by LSE == full
    parts = []
    for c in range(w.R):
        kb, ke = c * w.S // w.R, (c + 1) * w.S // w.R
        oc = torch.empty_like(o)
        lc = torch.empty_like(L)
        st.st_attn_spatial(q.to(DEV), k.to(DEV), v.to(DEV), oc, lc, kv_begin=kb, kv_end=ke, o_fp32=1)
        parts.append((oc, lc))
    om = torch.empty_like(o)
    st.attn_chunk_merge([p[0] for p in parts], [p[1] for p in parts], w.B * w.T, w.S, w.H, w.D, om)
    torch.cuda.synchronize()
    assert_close(om.cpu(), ro, "f32", "f32 chunk merge")


def test_failure_detection_timeout(st):
    """A bounded wait that runs out is reported as ST_ERR_TIMEOUT, and the context stays usable."""
    assert st.st_check_device_status() == st.ST_OK
    assert st.st_selftest_wait_timeout() == st.ST_OK
    assert st.st_check_device_status() == st.ST_ERR_TIMEOUT
    assert st.st_check_device_status() == st.ST_OK            # the word was cleared
    x = torch.ones(4, device=DEV)
    assert float((x * 2).sum().item()) == 8.0
