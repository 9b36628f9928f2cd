"""Rotary position embedding of Q and K (after the per-head RMSNorm) through
the C ABI against the oracle: the (cos, sin) table, the S->T relayout of the
spatial layer and the sequence->head relayout of image attention with the
RMSNorm and RoPE fused, and the listed-rows move of the sender-side V-Major
(the same bytes as the full relayout on the moved rows)."""
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


@pytest.mark.parametrize("n_pos,D,theta", [(1200, 72, 10000.0), (8160, 72, 10000.0), (65536, 128, 10000.0),
                                           (64, 32, 500.0)])
def test_rope_table(st, n_pos, D, theta):
    t = st.st_rope_table(n_pos, D, theta)
    torch.cuda.synchronize()
    ref = oracle.rope_table(n_pos, D, theta)
    err = np.max(np.abs(t.cpu().double().numpy() - ref))
    assert err <= 1e-6, err                      # fp32 rounding of double-precision cos / sin


@pytest.mark.parametrize("name,n_t,n_s", [("opensora_low", None, None), ("opensora_low", 1, 1), ("tiny", None, None)])
def test_st_relayout_rms_rope(st, name, n_t, n_s):
    w = synth.BY_NAME[name]
    n_t = w.n_t if n_t is None else n_t
    n_s = w.n_s if n_s is None else n_s
    rows = w.B * w.T * w.S
    x = synth.randn(w, "q", (rows, w.C))
    gamma = synth.rms_gamma(w)
    table = st.st_rope_table(w.S, w.D)
    out = torch.empty((rows, w.C), dtype=x.dtype, device=DEV)
    st.ulysses_relayout_rope("S2T", x.to(DEV), out, w.P, w.B, w.T, w.S, w.C, n_t, n_s, rms_gamma=gamma.to(DEV),
                             rms_head_dim=w.D, rms_eps=w.rms_eps, rope_table=table)
    torch.cuda.synchronize()
    ref = oracle.st_relayout("S2T", x, w.P, w.B, w.T, w.S, w.C, n_t, n_s, rms=(gamma, w.D, w.rms_eps),
                             rope=(w.D, 10000.0))
    assert_close(out.reshape(-1), ref, w.dtype, f"rms+rope {name}")


def test_seq2head_rms_rope(st):
    w = synth.Workload("img", 31, B=1, T=1, S=4096, H=8, D=128, dtype="bf16", P=4)
    N, H, D = w.S, w.H, w.D
    x = synth.randn(w, "k", (N * H, D))
    gamma = synth.rms_gamma(w)
    table = st.st_rope_table(N, D)
    out = torch.empty((N * H, D), dtype=x.dtype, device=DEV)
    st.ulysses_relayout_rope("SEQ2HEAD", x.to(DEV), out, w.P, w.B, N, H, D, rms_gamma=gamma.to(DEV), rms_head_dim=D,
                             rms_eps=1e-6, rope_table=table)
    torch.cuda.synchronize()
    ref = oracle.seq_head_relayout("SEQ2HEAD", x, w.P, w.B, N, H, D, rms=(gamma, D, 1e-6), rope=(D, 10000.0))
    assert_close(out.reshape(-1), ref, "bf16", "seq2head rms+rope")


@pytest.mark.parametrize("name", ["opensora_low", "tiny"])
def test_listed_rows_rms_rope_equal_full_relayout(st, name):
    w = synth.BY_NAME[name]
    n, C = w.B * w.T * w.S, w.C
    x = synth.randn(w, "k", (n, C)).to(DEV)
    gamma = synth.rms_gamma(w).to(DEV)
    table = st.st_rope_table(w.S, w.D)
    kw = dict(rms_gamma=gamma, rms_head_dim=w.D, rms_eps=w.rms_eps, rope_table=table)
    full = torch.empty_like(x)
    st.ulysses_relayout_rope("S2T", x, full, w.P, w.B, w.T, w.S, C, w.n_t, w.n_s, **kw)
    rng = np.random.default_rng(17)
    idx_np = np.flatnonzero(rng.random(n) < 0.4).astype(np.int32)
    idx = torch.full((n,), -1, dtype=torch.int32)
    idx[:idx_np.size] = torch.from_numpy(idx_np)
    count = torch.tensor([idx_np.size], dtype=torch.int32)
    old = synth.randn(w, "kprev", (n, C))
    out = old.to(DEV)
    st.vmajor_relayout_rows(x, out, idx.to(DEV), count.to(DEV), w.P, w.B, w.T, w.S, C, w.n_t, w.n_s, **kw)
    torch.cuda.synchronize()
    on = torch.from_numpy(idx_np.astype(np.int64))
    off = torch.from_numpy(np.setdiff1d(np.arange(n), idx_np))
    assert torch.equal(bits(out)[on], bits(full)[on])
    assert torch.equal(bits(out)[off], bits(old)[off])
    assert st.st_check_device_status() == st.ST_OK
