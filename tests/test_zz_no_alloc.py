"""The allocation-free V-Major entry point agrees with the workspace one.

vmajor_mask_compact_noalloc exists for callers that may not allocate device
memory while they run (a serving loop bound to a fixed memory pool, or code
that cannot risk cudaMalloc stalling or failing in the middle of a step).  It
keeps its scratch in the library's own static device array, so this test
calls it three times in a row, on inputs of different sizes (smaller, larger,
smaller), through the C ABI, and
checks mask, indices, count and per-token L1 against vmajor_mask_compact with a
caller workspace.  The file sorts last so that a failure here stops a -x run
only after every other test has run.
"""
import ctypes
import json
import os

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import sequence_parallelism_st_b200 as st
    return st


def workload_inputs(name, f):
    w = synth.BY_NAME[name]
    n = w.B * w.T * w.S
    cur, prev = synth.vmajor_pair(w, n, w.C)
    taus = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "vmajor_tau.json")))["workloads"]
    return cur.to(DEV), prev.to(DEV), taus[name][str(f)]["tau"]


def outputs(n):
    return (torch.full((n,), 9, dtype=torch.uint8, device=DEV), torch.full((n,), -1, dtype=torch.int32, device=DEV),
            torch.full((1,), -1, dtype=torch.int32, device=DEV), torch.zeros(n, dtype=torch.float32, device=DEV))


def test_noalloc_matches_workspace_entry_point_twice(st):
    fn = st._c["vmajor_mask_compact_noalloc"]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # smaller, larger, smaller: every call finds in the shared array what a
    # call of another size left there, and its results must not depend on it
    for name, f in (("opensora_low", 0.5), ("vmajor_2304px", 0.5), ("opensora_low", 0.5)):
        cur, prev, tau = workload_inputs(name, f)
        n, C = cur.shape
        mask_a, idx_a, cnt_a, l1_a = outputs(n)
        ws = torch.empty(st.vmajor_workspace_bytes(n), dtype=torch.uint8, device=DEV)
        st.vmajor_mask_compact(cur, prev, tau, mask_a, idx_a, cnt_a, ws, l1_out=l1_a)
        mask_b, idx_b, cnt_b, l1_b = outputs(n)
        r = fn(ctypes.c_void_p(cur.data_ptr()), ctypes.c_void_p(prev.data_ptr()), n, C, st.ST_BF16, float(tau), 0,
               ctypes.c_void_p(mask_b.data_ptr()), ctypes.c_void_p(idx_b.data_ptr()),
               ctypes.c_void_p(cnt_b.data_ptr()), ctypes.c_void_p(l1_b.data_ptr()), stream)
        assert r == st.ST_OK
        torch.cuda.synchronize()
        assert cnt_b.item() == cnt_a.item() > 0
        k = cnt_a.item()
        assert torch.equal(mask_b, mask_a)
        assert torch.equal(idx_b[:k], idx_a[:k])
        assert torch.equal(l1_b, l1_a)          # same kernels, same order: identical fp32 sums


def test_noalloc_rejects_sizes_beyond_its_scratch(st):
    fn = st._c["vmajor_mask_compact_noalloc"]
    fake = ctypes.c_void_p(0x100000)
    r = fn(fake, fake, (1 << 22) + 1, 64, st.ST_BF16, 1.0, 0, fake, fake, fake, None, None)
    assert r == st.ST_ERR_SHAPE
