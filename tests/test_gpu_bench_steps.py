"""The benchmark's timed steps, run once through the C ABI, against the oracle
composition of the same steps on the same seeded inputs: every buffer the
step hands from one call to the next (relayout outputs, masks, index lists,
caches, attention outputs) is compared, so a mix-up of the arguments between
calls (a stride, a cache layout, a chunk edge) fails here even when every
kernel passes its own parity test.  Full-size workloads; the attention is
compared on sampled frames, tokens and rows."""
import os
import sys

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import sequence_parallelism_st_b200 as st
    return st


def bench_mod():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


@pytest.mark.parametrize("attn", ["ring", "chunks"])
def test_image_step_against_oracle(st, attn):
    """SEQ2HEAD (+RMSNorm of Q and K) -> R-chunk attention -> HEAD2SEQ at N = 65536."""
    bench = bench_mod()
    w = synth.BY_NAME["image_4096px"]
    stp = bench.ImageStep(st, w, "cuda", attn=attn)
    stp.run()
    torch.cuda.synchronize()
    assert st.st_check_device_status() == st.ST_OK
    N, H, D, C, P = w.S, w.H, w.D, w.C, w.P
    q, k, v = synth.qkv(w)
    g = synth.rms_gamma(w)
    # V moves bit-exactly: head-sharded row (q, b, h1, n) holds token n, head q*H/P + h1
    dst, src = oracle.seq_head_row_pairs("SEQ2HEAD", P, w.B, N, H)
    vy = stp.vy.view(-1, D).cpu()
    assert torch.equal(vy.view(torch.int16), v.reshape(-1, D)[torch.from_numpy(src)].view(torch.int16))
    # Q and K: normalised rows at their head-sharded places (sampled rows)
    rng = np.random.default_rng(41)
    pick = rng.choice(dst.size, 4096, replace=False)
    for name, x in (("q", q), ("k", k)):
        got = stp.qy if name == "q" else stp.ky
        ref = oracle.rmsnorm_heads(x.reshape(-1, D)[torch.from_numpy(src[pick])], g, D, w.rms_eps)
        assert_close(got.view(-1, D)[torch.from_numpy(dst[pick])].cpu(), ref, "bf16", f"{name} SEQ2HEAD + RMSNorm")
    # the output, back in the sequence-sharded layout, on sampled query tokens
    rows = np.sort(rng.choice(N, 64, replace=False))
    qn = oracle.rmsnorm_heads(q.reshape(N, C)[torch.from_numpy(rows)], g, D, w.rms_eps).reshape(1, 1, -1, H, D)
    kn = oracle.rmsnorm_heads(k.reshape(N, C), g, D, w.rms_eps).reshape(1, 1, N, H, D)
    ro, rl = oracle.spatial(qn, kn, v, kv=(0, N))              # the sampled rows against all N keys
    ox = stp.ox.view(1, 1, N, H, D).cpu()
    assert_close(ox[:, :, torch.from_numpy(rows)], ro, "bf16", f"image step output ({attn})")
    # the merged LSE of the last launch: head-sharded frames (one per head) of N rows
    lse = stp.lse[0 if attn == "ring" else 1].view(H, N).cpu()
    assert_lse_close(lse[:, torch.from_numpy(rows)].unsqueeze(0).unsqueeze(0), rl, "image step lse")


def test_vmajor_step_against_oracle(st):
    """Mask, compaction, cache update and cached-K/V attention at N = 20736, f = 0.5."""
    bench = bench_mod()
    w = synth.BY_NAME["vmajor_2304px"]
    stp = bench.VMajorStep(st, w, "cuda", frac=0.5)
    stp.reset_caches()
    stp.run()
    torch.cuda.synchronize()
    assert st.st_check_device_status() == st.ST_OK
    N, H, D, C = w.S, w.H, w.D, w.C
    q = synth.randn(w, "q", (1, 1, N, H, D))
    cur_v, prev_v = synth.vmajor_pair(w, N, C)
    cur_k, prev_k = synth.vmajor_pair(w, N, C, prev="kprev", noise="knoise")
    mask = oracle.change_mask(oracle.l1_change(cur_v, prev_v), stp.tau)
    idx, cnt = oracle.compact(mask)
    assert np.array_equal(stp.mask.cpu().numpy(), mask.astype(np.uint8))
    assert int(stp.count.item()) == cnt
    assert np.array_equal(stp.idx.cpu().numpy()[:cnt], idx)
    kc = oracle.scatter_rows(idx, cnt, cur_k, prev_k)
    vc = oracle.scatter_rows(idx, cnt, cur_v, prev_v)
    assert np.array_equal(f64(stp.kc.view(N, C)), kc)
    assert np.array_equal(f64(stp.vc.view(N, C)), vc)
    rows = np.sort(np.random.default_rng(42).choice(N, 128, replace=False))
    ro, _ = oracle.spatial(q, kc.reshape(1, 1, N, H, D), vc.reshape(1, 1, N, H, D), rows=rows)
    o = stp.o.view(1, 1, N, H, D).cpu()
    assert_close(o[:, :, torch.from_numpy(rows)], ro, "bf16", "vmajor step output")


def ibits(t):
    """The raw bits of a bf16 or fp32 tensor, for exact comparisons."""
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


@pytest.mark.parametrize("name,ring", [("tiny", False), ("tiny", True), ("opensora_low", False),
                                       ("opensora_low", True), ("video_1080p", False), ("video_1080p", True)])
def test_st_step_against_oracle(st, name, ring):
    """Sender-side V-Major -> S->T of Q (+RMSNorm) -> two KV chunks (one ring
    launch, or the chain with the fused merge) -> T->S -> temporal attention,
    against the oracle composition
    (mask, indices, count and the V cache bit-exact; the K cache's moved rows,
    the spatial output and the temporal output at the float bar)."""
    bench = bench_mod()
    w = synth.BY_NAME[name]
    stp = bench.Step(st, w, "cuda")
    stp.ring = ring                                            # R chunks in one launch, or the chunk chain
    stp.reset_caches()
    stp.run()
    torch.cuda.synchronize()
    assert st.st_check_device_status() == st.ST_OK
    P, B, T, S, H, D, C = w.P, w.B, w.T, w.S, w.H, w.D, w.C
    n = B * T * S
    bar = w.dtype                                              # float bar: "bf16" or "f32"
    q, k, _ = synth.qkv(w)
    vcur, vprev = synth.vmajor_pair(w, n, C)                   # logical token order (b, t, s)
    v = vcur.reshape(B, T, S, H, D)
    kprev = synth.randn(w, "kprev", (B, T, S, H, D)).reshape(n, C)
    g = synth.rms_gamma(w)
    # the oracle's mask per logical token (L1 in slices of tokens to bound host memory)
    l1 = np.concatenate([oracle.l1_change(vcur[a:a + 32768], vprev[a:a + 32768]) for a in range(0, n, 32768)])
    mask_log = oracle.change_mask(l1, stp.tau)
    # y row r holds logical token y_log[r]: mask, indices and count in y numbering
    y_log, _, _ = oracle.st_y_rows(P, B, T, S, w.n_t, w.n_s)
    mask_y = mask_log[y_log]
    idx_y, cnt = oracle.compact(mask_y)
    assert np.array_equal(stp.mask.cpu().numpy(), mask_y)
    assert int(stp.count.item()) == cnt
    assert np.array_equal(stp.idx.cpu().numpy()[:cnt], idx_y)
    # V cache (y layout): this step's V on active rows, the previous V elsewhere
    yl = torch.from_numpy(y_log)
    my = torch.from_numpy(mask_y).bool()[:, None]
    vc_ref = torch.where(my, vcur[yl], vprev[yl])
    assert torch.equal(ibits(stp.vc.view(n, C).cpu()), ibits(vc_ref))
    # K cache: inactive rows untouched, active rows normalised (sampled)
    kc = stp.kc.view(n, C).cpu()
    assert torch.equal(ibits(torch.where(my, kprev[yl], kc)), ibits(kprev[yl]))
    act = idx_y[np.random.default_rng(44).choice(cnt, min(cnt, 4096), replace=False)]
    ref = oracle.rmsnorm_heads(k.reshape(n, C)[torch.from_numpy(y_log[act])], g, D, w.rms_eps)
    assert_close(kc[torch.from_numpy(act)], ref, bar, "K cache active rows")
    # spatial output (T->S moves it to x; read back in logical order) on sampled frames
    rng = np.random.default_rng(43)
    frames = sorted(rng.choice(T, 2, replace=False).tolist())
    rows = np.sort(rng.choice(S, min(S, 128), replace=False))
    fr = lambda x: x.reshape(B, T, S, C)[:, frames].reshape(-1, C)           # the sampled frames' tokens
    mk = mask_log.reshape(B, T, S)[:, frames].reshape(-1, 1) == 1
    qn = oracle.rmsnorm_heads(fr(q), g, D, w.rms_eps)
    kc_log = np.where(mk, oracle.rmsnorm_heads(fr(k), g, D, w.rms_eps), fr(kprev).double().numpy())
    vc_log = np.where(mk, fr(vcur).double().numpy(), fr(vprev).double().numpy())
    shp = (B, len(frames), S, H, D)
    ro, _ = oracle.spatial(qn.reshape(shp), kc_log.reshape(shp), vc_log.reshape(shp), rows=rows)
    x_log, _, _ = oracle.st_x_rows(P, B, T, S, w.n_t, w.n_s)
    pos = np.empty(n, dtype=np.int64)
    pos[x_log] = np.arange(n)                                  # logical token -> x row
    want = np.array([(b * T + t) * S + s for b in range(B) for t in frames for s in rows])
    ox = stp.ox.view(n, C)[torch.from_numpy(pos[want]).to("cuda")].cpu().reshape(B, len(frames), len(rows), H, D)
    assert_close(ox, ro, bar, f"{name} spatial output")
    # temporal attention of the raw Q, K and this step's V on sampled tokens
    toks = np.sort(rng.choice(S, min(S, 96), replace=False))
    rt, _ = oracle.temporal(q[:, :, toks], k[:, :, toks], v[:, :, toks])
    want = np.array([(b * T + t) * S + s for b in range(B) for t in range(T) for s in toks])
    ot = stp.ot.view(n, C)[torch.from_numpy(pos[want]).to("cuda")].cpu().reshape(B, T, len(toks), H, D)
    assert_close(ot, rt, bar, f"{name} temporal output")
