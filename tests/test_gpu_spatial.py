"""GPU parity of the tcgen05 spatial / full attention kernel against the fp64
oracle, through the C ABI: small multi-tile cases with ragged tails, KV-chunk
partials + LSE merge, slices, strided layouts, and the full-size workloads
(sampled rows where the oracle would be too slow)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import sequence_parallelism_st_b200 as st
    return st


def bits(t):
    return t.detach().to("cpu").contiguous().view(torch.int16)


def run(st, q, k, v, o_fp32=0, lse=True, **kw):
    B, T, S, H, D = q.shape
    o = torch.empty(q.shape, dtype=torch.float32 if o_fp32 else q.dtype, device=DEV)
    L = torch.empty((B, T, H, S), dtype=torch.float32, device=DEV) if lse else None
    st.st_attn_spatial(q, k, v, o, L, o_fp32=o_fp32, **kw)
    torch.cuda.synchronize()
    assert st.st_check_device_status() == st.ST_OK
    return o, L


SMALL = [(1, 2, 128, 2, 64), (1, 2, 200, 2, 72), (1, 1, 256, 3, 128), (2, 1, 300, 2, 128), (1, 1, 513, 1, 72),
         (1, 3, 77, 2, 32), (1, 1, 260, 2, 80), (1, 1, 390, 2, 96), (1, 1, 1030, 1, 128),
         # 24 or more 64-key steps per item: head dims 72 and 80 keep Q in TMEM (last query block: one tile)
         (1, 2, 1600, 2, 72), (2, 1, 1540, 1, 80), (1, 1, 1537, 3, 72)]


@pytest.mark.parametrize("B,T,S,H,D", SMALL)
def test_spatial_small(st, B, T, S, H, D):
    w = synth.Workload("s", 11, B=B, T=T, S=S, H=H, D=D, dtype="bf16")
    q, k, v = synth.qkv(w)
    o, L = run(st, q.to(DEV), k.to(DEV), v.to(DEV))
    ro, rl = oracle.spatial(q, k, v)
    assert_close(o.cpu(), ro, "bf16", f"spatial {B,T,S,H,D}")
    assert_lse_close(L.cpu(), rl, "spatial lse")


def test_spatial_large_logits_rescale(st):
    """Scores spread over a wide range force the running-max rescale of O in TMEM."""
    w = synth.Workload("s", 12, B=1, T=1, S=1500, H=2, D=128, dtype="bf16")
    q, k, v = synth.qkv(w)
    ramp = torch.linspace(0.2, 3.0, w.S).reshape(1, 1, w.S, 1, 1)
    k = (k.float() * ramp).to(torch.bfloat16)                 # later keys score higher
    q = (q.float() * 2.0).to(torch.bfloat16)
    o, L = run(st, q.to(DEV), k.to(DEV), v.to(DEV))
    ro, rl = oracle.spatial(q, k, v)
    assert_close(o.cpu(), ro, "bf16", "rescale")
    assert_lse_close(L.cpu(), rl, "rescale lse")


@pytest.mark.parametrize("D", [72, 128])
def test_spatial_kv_chunks_merge(st, D):
    w = synth.Workload("s", 13, B=1, T=2, S=700, H=2, D=D, dtype="bf16")
    q, k, v = synth.qkv(w)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    edges = [0, 128, 300, 301, 700]                           # uneven, one single-key chunk
    parts = []
    for a, b in zip(edges[:-1], edges[1:]):
        o, L = run(st, qd, kd, vd, o_fp32=1, kv_begin=a, kv_end=b)
        ro, rl = oracle.spatial(q, k, v, kv=(a, b))
        assert_close(o.cpu(), ro, "bf16", f"partial {a}:{b}")
        assert_lse_close(L.cpu(), rl, f"partial lse {a}:{b}")
        parts.append((o, L))
    om = torch.empty(q.shape, dtype=torch.bfloat16, device=DEV)
    lm = torch.empty((1, 2, w.H, w.S), dtype=torch.float32, device=DEV)
    st.attn_chunk_merge([p[0] for p in parts], [p[1] for p in parts], w.B * w.T, w.S, w.H, w.D, om, lm)
    torch.cuda.synchronize()
    ro, rl = oracle.spatial(q, k, v)
    assert_close(om.cpu(), ro, "bf16", "merged")
    assert_lse_close(lm.cpu(), rl, "merged lse")


def test_spatial_empty_range(st):
    w = synth.Workload("s", 14, B=1, T=1, S=64, H=1, D=64, dtype="bf16")
    q, k, v = (x.to(DEV) for x in synth.qkv(w))
    o, L = run(st, q, k, v, o_fp32=1, kv_begin=10, kv_end=10)
    assert torch.all(o == 0) and torch.all(torch.isinf(L)) and torch.all(L < 0)


def test_spatial_slices_bit_identical(st):
    """ST independence: the spatial layer sliced along T is bit-identical."""
    w = synth.BY_NAME["opensora_low"]
    q, k, v = (x.to(DEV) for x in synth.qkv(w))
    o, _ = run(st, q, k, v, lse=False)
    o2 = torch.zeros_like(o)
    for i in reversed(range(w.n_t)):
        st.st_attn_spatial(q, k, v, o2, None, n_slices=w.n_t, slice=i)
    torch.cuda.synchronize()
    assert torch.equal(bits(o2), bits(o))


def test_spatial_full_opensora(st):
    w = synth.BY_NAME["opensora_low"]
    q, k, v = synth.qkv(w)
    o, L = run(st, q.to(DEV), k.to(DEV), v.to(DEV))
    ro, rl = oracle.spatial(q, k, v)
    assert_close(o.cpu(), ro, "bf16", "opensora spatial")
    assert_lse_close(L.cpu(), rl, "opensora lse")


def test_spatial_on_sliced_y_layout(st):
    """The spatial layer reads the [P,B,N_T,N_S,T/(N_T P),S/N_S,C] layout in place."""
    w = synth.BY_NAME["opensora_low"]
    q, k, v = synth.qkv(w)
    P, n_t, n_s = w.P, w.n_t, w.n_s
    Tq, Ss = w.T // (n_t * P), w.S // n_s

    def to_y(t):
        X = t.reshape(w.B, w.T, w.S, w.C)
        return X.reshape(w.B, n_t, P, Tq, n_s, Ss, w.C).permute(2, 0, 1, 4, 3, 5, 6).contiguous()

    qy, ky, vy = (to_y(x).to(DEV) for x in (q, k, v))
    C = w.C
    # frames (q, b, i, t2) as two levels: t2 inside a block, (q, b, i) blocks of n_s*Tq*Ss rows
    desc = st.make_desc(1, P * w.B * n_t * Tq, w.S, w.H, w.D, st.ST_BF16, stride_t=Ss * C, stride_s=C,
                        t_block=Tq, stride_tb=n_s * Tq * Ss * C, s_block=Ss, stride_sb=Tq * Ss * C)
    o = torch.empty_like(qy)
    st.st_attn_spatial(qy, ky, vy, o, None, desc=desc)
    ref, _ = run(st, q.to(DEV), k.to(DEV), v.to(DEV), lse=False)
    torch.cuda.synchronize()
    assert torch.equal(bits(o), bits(to_y(ref.cpu())))


def test_spatial_video_sampled(st):
    w = synth.BY_NAME["video_1080p"]
    q, k, v = synth.qkv(w)
    o, L = run(st, q.to(DEV), k.to(DEV), v.to(DEV))
    rng = np.random.default_rng(5)
    frames = sorted(rng.choice(w.T, 4, replace=False).tolist())
    rows = np.sort(rng.choice(w.S, 256, replace=False))
    ro, rl = oracle.spatial(q, k, v, rows=rows, frames=frames)
    sel = o.cpu()[:, frames][:, :, torch.from_numpy(rows)]
    assert_close(sel, ro, "bf16", "video spatial")
    assert_lse_close(L.cpu()[:, frames][:, :, :, torch.from_numpy(rows)], rl, "video lse")


def test_full_attention_image_chunks(st):
    """Image-DiT full attention (T = 1, S = N) as R ring chunks merged by LSE."""
    w = synth.BY_NAME["image_4096px"]
    q, k, v = synth.qkv(w)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o_full, L_full = run(st, qd, kd, vd)
    R, N = w.R, w.S
    parts = []
    for c in range(R):
        o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
        L = torch.empty((1, 1, w.H, N), dtype=torch.float32, device=DEV)
        st.st_attn_spatial(qd, kd, vd, o, L, kv_begin=c * N // R, kv_end=(c + 1) * N // R, o_fp32=1)
        parts.append((o, L))
    om = torch.empty_like(qd)
    st.attn_chunk_merge([p[0] for p in parts], [p[1] for p in parts], 1, N, w.H, w.D, om)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(6).choice(N, 192, replace=False))
    ro, rl = oracle.spatial(q, k, v, rows=rows)
    r = torch.from_numpy(rows)
    assert_close(o_full.cpu()[:, :, r], ro, "bf16", "image full")
    assert_lse_close(L_full.cpu()[:, :, :, r], rl, "image lse")
    assert_close(om.cpu()[:, :, r], ro, "bf16", "image merged")
    del parts


def test_cached_kv_attention_vmajor(st):
    """Attention of fresh Q against K/V caches updated for the active tokens."""
    w = synth.BY_NAME["vmajor_2304px"]
    n, C = w.S, w.C
    cur_v, prev_v = synth.vmajor_pair(w, n, C)
    cur_k, prev_k = synth.vmajor_pair(w, n, C, prev="kprev", noise="knoise")
    q = synth.randn(w, "q", (1, 1, n, w.H, w.D))
    l1 = oracle.l1_change(cur_v, prev_v)
    tau, _, _ = oracle.tau_for_fraction(l1, 0.5)
    idx_ref, cnt = oracle.compact(oracle.change_mask(l1, tau))
    mask = torch.empty(n, dtype=torch.uint8, device=DEV)
    idx = torch.empty(n, dtype=torch.int32, device=DEV)
    count = torch.empty(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(st.vmajor_workspace_bytes(n), dtype=torch.uint8, device=DEV)
    st.vmajor_mask_compact(cur_v.to(DEV), prev_v.to(DEV), tau, mask, idx, count, ws)
    kc, vc = prev_k.to(DEV), prev_v.to(DEV)
    st.vmajor_scatter_rows(idx, count, [cur_k.to(DEV), cur_v.to(DEV)], [kc, vc])
    o, L = run(st, q.to(DEV), kc.reshape(q.shape), vc.reshape(q.shape))
    k_ref = oracle.scatter_rows(idx_ref, cnt, cur_k, prev_k).reshape(q.shape)
    v_ref = oracle.scatter_rows(idx_ref, cnt, cur_v, prev_v).reshape(q.shape)
    rows = np.sort(np.random.default_rng(7).choice(n, 256, replace=False))
    ro, rl = oracle.spatial(q, k_ref, v_ref, rows=rows)
    r = torch.from_numpy(rows)
    assert_close(o.cpu()[:, :, r], ro, "bf16", "cached-kv attention")
    assert_lse_close(L.cpu()[:, :, :, r], rl, "cached-kv lse")
