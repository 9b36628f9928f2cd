"""The bench step's kernels launched back to back (each may start while the
previous one finishes, through programmatic dependent launch) must give the
same bits as the same step with a device synchronisation after every call.
Catches reads that run ahead of a producer kernel; the per-kernel parity tests
synchronise after each call and cannot see them."""
import os
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import sequence_parallelism_st_b200 as st
    return st


class _Synced:
    """The binding with a device synchronisation after every call."""

    def __init__(self, mod):
        self._m = mod

    def __getattr__(self, name):
        f = getattr(self._m, name)
        if not callable(f) or name in ("make_desc", "vmajor_workspace_bytes"):
            return f

        def call(*a, **k):
            r = f(*a, **k)
            torch.cuda.synchronize()
            return r
        return call


def outputs(stp):
    return [t.detach().clone() for t in (stp.ox, stp.ot, stp.kc, stp.vc, stp.mask, stp.idx, stp.count, stp.oy)]


@pytest.mark.parametrize("name", ["opensora_low"])
def test_step_chain_matches_synchronised(st, name):
    sys.path.insert(0, ROOT)
    import bench
    import synth
    w = synth.BY_NAME[name]
    stp = bench.Step(st, w, "cuda")
    stp.reset_caches()
    stp.st = _Synced(st)
    stp.run()
    torch.cuda.synchronize()
    ref = outputs(stp)
    stp.st = st
    for rep in range(10):
        stp.reset_caches()
        stp.run()
        torch.cuda.synchronize()
        got = outputs(stp)
        for i, (a, b) in enumerate(zip(got, ref)):
            assert torch.equal(a, b), f"{name}: output {i} differs from the synchronised step (repeat {rep})"
    assert st.st_check_device_status() == st.ST_OK


@pytest.mark.parametrize("n_slices,att_sms", [(2, 148), (4, 120)])
def test_overlap_schedule_matches_serial(st, n_slices, att_sms):
    """The chunk-and-overlap schedule (shard ranges on two streams, attention on
    part of the SMs) gives the serial step's bits; per-range compactions
    concatenate to the serial compaction."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    w = synth.BY_NAME["opensora_low"]
    stp = bench.Step(st, w, "cuda")
    stp.reset_caches()
    stp.run()
    torch.cuda.synchronize()
    ref = outputs(stp)
    cnt_ref = int(stp.count.item())
    idx_ref = stp.idx[:cnt_ref].clone()
    stp.setup_overlap(n_slices, att_sms)
    for rep in range(3):
        stp.reset_caches()
        stp.idx.fill_(-1)
        stp.run_overlap()
        torch.cuda.synchronize()
        got = outputs(stp)
        for i in (0, 1, 2, 3, 4, 7):            # ox, ot, kc, vc, mask, oy (idx and count differ in layout)
            assert torch.equal(got[i], ref[i]), f"overlap: output {i} differs (repeat {rep})"
        per = stp.n // n_slices
        parts = [stp.idx[s * per: s * per + int(c)] + s * per for s, c in enumerate(stp.counts.tolist())]
        assert torch.equal(torch.cat(parts), idx_ref)
    assert st.st_get_sm_budget() == 0
    assert st.st_check_device_status() == st.ST_OK


def test_fused_merge_step_matches_separate(st):
    """The bench step with the merge fused into the attention kernel agrees with
    the step that writes both partials and merges them with attn_chunk_merge
    (bf16 tolerance on the spatial output; every other output bit for bit)."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    w = synth.BY_NAME["opensora_low"]
    stp = bench.Step(st, w, "cuda")
    res = {}
    for fused in (False, True):
        stp.fused_merge = fused
        stp.reset_caches()
        stp.run()
        torch.cuda.synchronize()
        res[fused] = outputs(stp)
    for i in (1, 2, 3, 4, 5, 6):                 # ot, kc, vc, mask, idx, count
        assert torch.equal(res[True][i], res[False][i]), f"output {i} differs"
    for i in (0, 7):                             # ox, oy: the spatial result, two merge orders
        a, b = res[True][i].float(), res[False][i].float()
        assert (a - b).abs().max().item() <= 2e-2
        assert ((a - b).norm() / b.norm()).item() <= 5e-3
    assert st.st_check_device_status() == st.ST_OK


def test_sender_vmajor_step_matches_receiver(st):
    """Sender-side V-Major (mask on x, only active K/V rows moved into the
    caches) gives the receiver-side step's bits: mask, compaction, caches,
    and every attention output."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    w = synth.BY_NAME["opensora_low"]
    stp = bench.Step(st, w, "cuda")
    res = {}
    for sender in (False, True):
        stp.sender_vmajor = sender
        stp.reset_caches()
        stp.idx.fill_(-1)
        stp.run()
        torch.cuda.synchronize()
        res[sender] = outputs(stp) + [stp.qy.clone()]
    for i, (a, b) in enumerate(zip(res[True], res[False])):
        assert torch.equal(a, b), f"output {i} differs between sender and receiver V-Major"
    assert st.st_check_device_status() == st.ST_OK


def test_rope_step_sender_matches_receiver(st):
    """With the rotary embedding on Q and K, the sender-side and receiver-side
    V-Major steps still give the same bits for every output."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    w = synth.BY_NAME["opensora_low"]
    stp = bench.Step(st, w, "cuda")
    stp.rope_table = st.st_rope_table(w.S, w.D, 10000.0)
    res = {}
    for sender in (False, True):
        stp.sender_vmajor = sender
        stp.reset_caches()
        stp.idx.fill_(-1)
        stp.run()
        torch.cuda.synchronize()
        res[sender] = outputs(stp) + [stp.qy.clone()]
    for i, (a, b) in enumerate(zip(res[True], res[False])):
        assert torch.equal(a, b), f"output {i} differs between sender and receiver V-Major with RoPE"
    assert st.st_check_device_status() == st.ST_OK
