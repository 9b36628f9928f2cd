"""Sender-side V-Major through the C ABI against the oracle: the L1 change is
measured on the spatially sharded layout x, the rows of active tokens move
S->T into the cache in the temporally sharded layout y and nothing else is
written; mask, compaction and count in y numbering are bit-exact; the masked
K move with the per-head RMSNorm writes exactly the bytes of the full
relayout on the active rows."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close

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


def tau_of(name, f, l1):
    """The committed threshold where one exists, else the oracle's for that active fraction."""
    path = os.path.join(os.path.dirname(__file__), "golden", "vmajor_tau.json")
    got = json.load(open(path))["workloads"].get(name, {}).get(str(f))
    return got["tau"] if got else float(oracle.tau_for_fraction(l1, f)[0])


CASES = [("opensora_low", 0.5, None, None), ("opensora_low", 0.9, None, None), ("opensora_low", 0.1, 1, 1),
         ("video_1080p", 0.5, None, None), ("tiny", 0.5, None, None)]


@pytest.mark.parametrize("name,f,n_t,n_s", CASES)
def test_vmajor_relayout_mask(st, name, f, n_t, n_s):
    w = synth.BY_NAME[name]
    n_t = w.n_t if n_t is None else n_t
    n_s = w.n_s if n_s is None else n_s
    n, C = w.B * w.T * w.S, w.C
    cur, prev = synth.vmajor_pair(w, n, C)             # taken as x-layout buffers (rows = sender rows)
    l1 = np.concatenate([oracle.l1_change(cur[a:a + 32768], prev[a:a + 32768])    # per x row, in slices of
                         for a in range(0, n, 32768)])                                # rows (host memory)
    tau = tau_of(name, f, l1)
    dst, src = oracle.st_row_pairs("S2T", w.P, w.B, w.T, w.S, n_t, n_s)
    mask_ref = np.zeros(n, dtype=np.uint8)
    mask_ref[dst] = oracle.change_mask(l1, tau)[src]
    idx_ref, cnt_ref = oracle.compact(mask_ref)
    cache0 = synth.randn(w, "kprev", (n, C))
    cache = cache0.to(DEV)
    mask = torch.full((n,), 7, dtype=torch.uint8, device=DEV)
    idx = torch.full((n,), -1, dtype=torch.int32, device=DEV)
    count = torch.zeros(1, dtype=torch.int32, device=DEV)
    l1_out = torch.zeros(n, dtype=torch.float32, device=DEV)
    ws = torch.zeros(st.vmajor_workspace_bytes(n), dtype=torch.uint8, device=DEV)
    st.vmajor_relayout_mask(cur.to(DEV), prev.to(DEV), cache, w.P, w.B, w.T, w.S, C, n_t, n_s, tau, mask, idx, count,
                            ws, l1_out=l1_out)
    torch.cuda.synchronize()
    assert count.item() == cnt_ref
    assert np.array_equal(mask.cpu().numpy(), mask_ref)
    assert np.array_equal(idx.cpu().numpy()[:cnt_ref], idx_ref)
    l1_y = np.zeros(n)
    l1_y[dst] = l1[src]
    np.testing.assert_allclose(l1_out.cpu().numpy(), l1_y, rtol=2e-5, atol=1e-6)
    got, cb, c0 = bits(cache), bits(cur), bits(cache0)
    act = mask_ref[dst] == 1
    assert torch.equal(got[torch.from_numpy(dst[act])], cb[torch.from_numpy(src[act])])
    assert torch.equal(got[torch.from_numpy(dst[~act])], c0[torch.from_numpy(dst[~act])])
    assert st.st_check_device_status() == st.ST_OK


def test_vmajor_relayout_mask_force_all_and_unchanged(st):
    w = synth.BY_NAME["opensora_low"]
    n, C = w.B * w.T * w.S, w.C
    cur, _ = synth.vmajor_pair(w, n, C)
    cd = cur.to(DEV)
    ws = torch.zeros(st.vmajor_workspace_bytes(n), dtype=torch.uint8, device=DEV)
    full = torch.empty_like(cd)
    st.ulysses_relayout("S2T", cd, full, w.P, w.B, w.T, w.S, C, w.n_t, w.n_s)
    for force, expect in ((True, n), (False, 0)):       # refresh step / v_cur == v_prev
        cache = torch.zeros_like(cd)
        mask = torch.empty(n, dtype=torch.uint8, device=DEV)
        idx = torch.full((n,), -1, dtype=torch.int32, device=DEV)
        count = torch.zeros(1, dtype=torch.int32, device=DEV)
        st.vmajor_relayout_mask(cd, cd, cache, w.P, w.B, w.T, w.S, C, w.n_t, w.n_s, 0.0, mask, idx, count, ws,
                                force_all=force)
        torch.cuda.synchronize()
        assert count.item() == expect
        if force:
            assert torch.equal(bits(cache), bits(full))      # every row moved: the full relayout
            assert torch.equal(idx.cpu(), torch.arange(n, dtype=torch.int32))
        else:
            assert not cache.any().item()


@pytest.mark.parametrize("name,rms", [("opensora_low", True), ("opensora_low", False), ("tiny", True),
                                      ("tiny", False)])
def test_vmajor_relayout_rows(st, name, rms):
    """Listed rows equal the full relayout's (with RMSNorm: the same bytes), the others stay."""
    w = synth.BY_NAME[name]
    n, C = w.B * w.T * w.S, w.C
    x = synth.randn(w, "k", (n, C)).to(DEV)
    gamma = synth.rms_gamma(w).to(DEV) if rms else None
    kw = dict(rms_gamma=gamma, rms_head_dim=w.D, rms_eps=w.rms_eps) if rms else {}
    full = torch.empty_like(x)
    st.ulysses_relayout("S2T", x, full, w.P, w.B, w.T, w.S, C, w.n_t, w.n_s, **kw)
    rng = np.random.default_rng(11)
    mask_np = (rng.random(n) < 0.5).astype(np.uint8)
    old = synth.randn(w, "kprev", (n, C))
    out = old.to(DEV)
    idx_np = np.flatnonzero(mask_np).astype(np.int32)
    idx = torch.full((n,), -1, dtype=torch.int32)
    idx[:idx_np.size] = torch.from_numpy(idx_np)
    count = torch.tensor([idx_np.size], dtype=torch.int32)
    st.vmajor_relayout_rows(x, out, idx.to(DEV), count.to(DEV), w.P, w.B, w.T, w.S, C, w.n_t, w.n_s, **kw)
    torch.cuda.synchronize()
    on = torch.from_numpy(np.flatnonzero(mask_np))
    off = torch.from_numpy(np.flatnonzero(mask_np == 0))
    assert torch.equal(bits(out)[on], bits(full)[on])
    assert torch.equal(bits(out)[off], bits(old)[off])
    if rms:                                             # and against the oracle, on the written rows
        ref = oracle.st_relayout("S2T", x.cpu(), w.P, w.B, w.T, w.S, C, w.n_t, w.n_s,
                                 rms=(gamma.cpu(), w.D, w.rms_eps)).reshape(n, C)
        assert_close(out.cpu()[on], ref[on.numpy()], w.dtype, f"masked rms {name}")
