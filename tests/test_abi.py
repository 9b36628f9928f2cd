"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before launching anything (CPU only: no call here
reaches the GPU)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def st():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "stattn_build", os.path.join(ROOT, "sequence_parallelism_st_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import sequence_parallelism_st_b200 as st
    return st


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?(?:st_status|int|size_t|char|void)\s*\*?\s*(\w+)\s*\(",
                             text, flags=re.M):
            names.append(m.group(1))
    return names


def test_every_declared_symbol_is_exported(st):
    names = declared_functions()
    assert {"st_attn_spatial", "st_attn_temporal", "attn_chunk_merge", "ulysses_relayout",
            "vmajor_mask_compact", "vmajor_scatter_rows", "st_check_device_status"} <= set(names)
    raw = ctypes.CDLL(st.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in include/ but not exported"
    assert set(names) <= set(st.EXPORTED)


def test_status_strings_and_version(st):
    assert st.st_status_string(0) == "ST_OK"
    for code in range(-8, 0):
        assert st.st_status_string(code).startswith("ST_ERR_")
    assert st._c["st_abi_version"]() == 1
    assert st.vmajor_workspace_bytes(20736) >= 4 * (20736 // 32)
    assert st.vmajor_workspace_bytes(0) == 0


FAKE_IN, FAKE_OUT = ctypes.c_void_p(0x100000), ctypes.c_void_p(0x90000000)


def relayout(st, mode, elem=2, P=2, B=1, T=8, S=16, C=64, n_t=1, n_s=1, blk=None, inp=FAKE_IN, out=FAKE_OUT,
             gamma=None, hd=0):
    i0, i1, j0, j1 = blk if blk else (0, n_t, 0, n_s)
    return st._c["ulysses_relayout"](mode, inp, out, elem, P, B, T, S, C, n_t, n_s, i0, i1, j0, j1, gamma, hd,
                                     1e-6, None)


def test_relayout_rejects(st):
    assert relayout(st, st.ST_S2T, inp=None) == st.ST_ERR_NULL
    assert relayout(st, st.ST_S2T, elem=3) == st.ST_ERR_DTYPE
    assert relayout(st, st.ST_S2T, T=6, P=4) == st.ST_ERR_DIVISIBILITY
    assert relayout(st, st.ST_S2T, n_t=2, T=6, P=2) == st.ST_ERR_DIVISIBILITY
    assert relayout(st, st.ST_S2T, n_t=2, blk=(0, 3, 0, 1)) == st.ST_ERR_SHAPE
    assert relayout(st, st.ST_S2T, n_t=2, blk=(1, 1, 0, 1)) == st.ST_ERR_SHAPE
    assert relayout(st, st.ST_SEQ2HEAD, n_t=2) == st.ST_ERR_SHAPE
    assert relayout(st, st.ST_SEQ2HEAD, S=3) == st.ST_ERR_DIVISIBILITY
    assert relayout(st, 7) == st.ST_ERR_UNSUPPORTED
    assert relayout(st, st.ST_S2T, P=0) == st.ST_ERR_SHAPE
    assert relayout(st, st.ST_S2T, gamma=FAKE_IN, hd=48) == st.ST_ERR_SHAPE
    assert relayout(st, st.ST_S2T, out=ctypes.c_void_p(0x100000 + 64)) == st.ST_ERR_SHAPE   # overlap


def relayout_range(st, mode, q0, q1, P=2, n_t=1, n_s=1):
    return st._c["ulysses_relayout_range"](mode, FAKE_IN, FAKE_OUT, 2, P, 1, 8, 16, 64, n_t, n_s, 0, n_t, 0, n_s,
                                           q0, q1, None, 0, 1e-6, None)


def test_relayout_range_rejects(st):
    """Shard ranges are validated before any launch: empty, reversed or out of range."""
    for q0, q1 in ((0, 0), (1, 0), (-1, 1), (0, 3), (2, 2)):
        assert relayout_range(st, st.ST_S2T, q0, q1) == st.ST_ERR_SHAPE, (q0, q1)
        assert relayout_range(st, st.ST_T2S, q0, q1) == st.ST_ERR_SHAPE, (q0, q1)
    # the sequence/head exchange has no shard range
    assert relayout_range(st, st.ST_SEQ2HEAD, 0, 1) == st.ST_ERR_SHAPE


def test_sm_budget_setting(st):
    assert st.st_get_sm_budget() == 0
    assert st._c["st_set_sm_budget"](-1) == st.ST_ERR_SHAPE
    st.st_set_sm_budget(32)
    try:
        assert st.st_get_sm_budget() == 32
    finally:
        st.st_set_sm_budget(0)
    assert st.st_get_sm_budget() == 0


def spatial(st, fn="st_attn_spatial", q=FAKE_IN, **kw):
    d = dict(B=1, T=2, S=64, H=2, D=72, dtype=st.ST_BF16)
    d.update(kw)
    desc = st.make_desc(**d)
    return st._c[fn](ctypes.byref(desc), q, FAKE_IN, FAKE_IN, FAKE_OUT, None, None)


def test_attention_rejects(st):
    assert st._c["st_attn_spatial"](None, FAKE_IN, FAKE_IN, FAKE_IN, FAKE_OUT, None, None) == st.ST_ERR_NULL
    assert spatial(st, q=None) == st.ST_ERR_NULL
    bad = st.make_desc(1, 2, 64, 2, 72)
    bad.size = 12
    assert st._c["st_attn_spatial"](ctypes.byref(bad), FAKE_IN, FAKE_IN, FAKE_IN, FAKE_OUT, None, None) == st.ST_ERR_SHAPE
    assert spatial(st, B=0) == st.ST_ERR_SHAPE
    assert spatial(st, dtype=5) == st.ST_ERR_DTYPE
    assert spatial(st, D=48) == st.ST_ERR_UNSUPPORTED
    assert spatial(st, q=ctypes.c_void_p(0x100008)) == st.ST_ERR_ALIGN
    assert spatial(st, stride_s=148) == st.ST_ERR_ALIGN
    assert spatial(st, kv_begin=10, kv_end=5) == st.ST_ERR_SHAPE
    assert spatial(st, kv_begin=0, kv_end=65) == st.ST_ERR_SHAPE
    assert spatial(st, n_slices=3, slice=0) == st.ST_ERR_DIVISIBILITY
    assert spatial(st, n_slices=2, slice=2) == st.ST_ERR_SHAPE
    assert spatial(st, t_block=3) == st.ST_ERR_DIVISIBILITY
    assert spatial(st, "st_attn_temporal", T=65) == st.ST_ERR_UNSUPPORTED
    assert spatial(st, "st_attn_temporal", kv_begin=1, kv_end=3) == st.ST_ERR_SHAPE
    assert spatial(st, "st_attn_temporal", D=40) == st.ST_ERR_UNSUPPORTED


def ring(st, n_chunks, q=FAKE_IN, **kw):
    d = dict(B=1, T=2, S=64, H=2, D=128, dtype=st.ST_BF16)
    d.update(kw)
    desc = st.make_desc(**d)
    return st._c["st_attn_ring"](ctypes.byref(desc), q, FAKE_IN, FAKE_IN, FAKE_OUT, None, n_chunks, None)


def test_ring_attention_rejects(st):
    """The ring-chunk call validates its chunk count and key range before any launch."""
    assert st._c["st_attn_ring"](None, FAKE_IN, FAKE_IN, FAKE_IN, FAKE_OUT, None, 2, None) == st.ST_ERR_NULL
    assert ring(st, 2, q=None) == st.ST_ERR_NULL
    assert ring(st, 0) == st.ST_ERR_SHAPE
    assert ring(st, -3) == st.ST_ERR_SHAPE
    assert ring(st, 65) == st.ST_ERR_SHAPE                       # at most 64 chunks
    assert ring(st, 9, S=8) == st.ST_ERR_SHAPE                   # more chunks than keys
    assert ring(st, 2, kv_begin=0, kv_end=32) == st.ST_ERR_SHAPE  # the chunks partition the whole frame
    assert ring(st, 2, kv_begin=8, kv_end=64) == st.ST_ERR_SHAPE
    assert ring(st, 2, D=48) == st.ST_ERR_UNSUPPORTED
    assert ring(st, 2, q=ctypes.c_void_p(0x100008)) == st.ST_ERR_ALIGN


def test_merge_and_vmajor_reject(st):
    VP = ctypes.c_void_p
    arr = (VP * 2)(0x100000, 0x200000)
    f = st._c["attn_chunk_merge"]
    assert f(0, arr, arr, 1, 8, 2, 64, FAKE_OUT, st.ST_BF16, None, None) == st.ST_ERR_SHAPE
    assert f(17, arr, arr, 1, 8, 2, 64, FAKE_OUT, st.ST_BF16, None, None) == st.ST_ERR_SHAPE
    assert f(2, arr, arr, 1, 8, 2, 66, FAKE_OUT, st.ST_BF16, None, None) == st.ST_ERR_ALIGN
    assert f(2, arr, arr, 1, 8, 2, 64, None, st.ST_BF16, None, None) == st.ST_ERR_NULL
    assert f(2, arr, arr, 1, 8, 2, 64, FAKE_OUT, 9, None, None) == st.ST_ERR_DTYPE
    # outputs overlapping a part (in place, or an LSE over an LSE part) are refused
    lse = (VP * 2)(0x300000, 0x400000)
    assert f(2, arr, lse, 1, 8, 2, 64, VP(0x200000), st.ST_F32, None, None) == st.ST_ERR_SHAPE
    assert f(2, arr, lse, 1, 8, 2, 64, VP(0x100000 + 512), st.ST_BF16, None, None) == st.ST_ERR_SHAPE
    assert f(2, arr, lse, 1, 8, 2, 64, FAKE_OUT, st.ST_BF16, VP(0x400000), None) == st.ST_ERR_SHAPE
    assert f(2, arr, lse, 1, 8, 2, 64, FAKE_OUT, st.ST_BF16, VP(0x200000 + 64), None) == st.ST_ERR_SHAPE
    assert f(2, arr, lse, 1, 8, 2, 64, FAKE_OUT, st.ST_BF16, VP(0x90000000 + 64), None) == st.ST_ERR_SHAPE
    g = st._c["vmajor_mask_compact"]
    ws = st.vmajor_workspace_bytes(100)
    assert g(None, FAKE_IN, 100, 64, st.ST_BF16, 1.0, 0, FAKE_OUT, FAKE_OUT, FAKE_OUT, None, FAKE_OUT, ws, None) == st.ST_ERR_NULL
    assert g(FAKE_IN, FAKE_IN, 100, 64, st.ST_BF16, 1.0, 0, FAKE_OUT, FAKE_OUT, FAKE_OUT, None, FAKE_OUT, ws - 4, None) == st.ST_ERR_SHAPE
    assert g(FAKE_IN, FAKE_IN, 100, 60, st.ST_BF16, 1.0, 0, FAKE_OUT, FAKE_OUT, FAKE_OUT, None, FAKE_OUT, ws, None) == st.ST_ERR_ALIGN
    assert g(FAKE_IN, FAKE_IN, 0, 64, st.ST_BF16, 1.0, 0, FAKE_OUT, FAKE_OUT, FAKE_OUT, None, FAKE_OUT, ws, None) == st.ST_ERR_SHAPE
    h = st._c["vmajor_scatter_rows"]
    assert h(FAKE_IN, FAKE_IN, 100, 64, 2, arr, arr, 0, None, None) == st.ST_ERR_SHAPE
    assert h(FAKE_IN, FAKE_IN, 100, 64, 2, arr, arr, 9, None, None) == st.ST_ERR_SHAPE
    assert h(FAKE_IN, FAKE_IN, 100, 64, 3, arr, arr, 2, None, None) == st.ST_ERR_DTYPE


def test_sender_vmajor_rejects(st):
    """vmajor_relayout_mask / vmajor_relayout_rows validate before any launch."""
    VP = ctypes.c_void_p
    ws = VP(0x300000)
    m = st._c["vmajor_relayout_mask"]

    def mask_call(P=2, T=8, S=16, C=64, n_t=1, n_s=1, dtype=st.ST_BF16, cur=FAKE_IN, cache=FAKE_OUT, wsb=1 << 20):
        return m(cur, VP(0x200000), cache, P, 1, T, S, C, n_t, n_s, dtype, 1.0, 0, VP(0x400000), VP(0x500000),
                 VP(0x600000), None, ws, wsb, None)
    assert mask_call(cur=None) == st.ST_ERR_NULL
    assert mask_call(dtype=7) == st.ST_ERR_DTYPE
    assert mask_call(T=6, P=4) == st.ST_ERR_DIVISIBILITY
    assert mask_call(S=16, P=2, n_s=3) == st.ST_ERR_DIVISIBILITY
    assert mask_call(C=3) == st.ST_ERR_ALIGN
    assert mask_call(cur=VP(0x100008)) == st.ST_ERR_ALIGN
    assert mask_call(wsb=0) == st.ST_ERR_SHAPE
    assert mask_call(cache=VP(0x100000 + 64)) == st.ST_ERR_SHAPE        # overlaps the input
    r = st._c["vmajor_relayout_rows"]

    def rows_call(gamma=None, hd=0, C=64, out=FAKE_OUT, idx=VP(0x400000), rope=None, n_pos=0):
        return r(FAKE_IN, out, idx, VP(0x500000), 2, 1, 8, 16, C, 1, 1, st.ST_BF16, gamma, hd, 1e-6, rope, n_pos, None)
    assert rows_call(idx=None) == st.ST_ERR_NULL
    assert rows_call(gamma=FAKE_IN, hd=48) == st.ST_ERR_SHAPE
    assert rows_call(gamma=FAKE_IN, hd=4) == st.ST_ERR_SHAPE            # 8-byte heads: not 16-byte rows
    assert rows_call(out=VP(0x100000 + 32)) == st.ST_ERR_SHAPE
    assert rows_call(rope=VP(0x700000), n_pos=16) == st.ST_ERR_NULL             # RoPE rides on the RMSNorm
    assert rows_call(gamma=FAKE_IN, hd=32, rope=VP(0x700000), n_pos=15) == st.ST_ERR_SHAPE   # table too short
    assert rows_call(gamma=FAKE_IN, hd=32, rope=VP(0x700008), n_pos=16) == st.ST_ERR_ALIGN   # table read 16 B at a time


def test_rope_rejects(st):
    VP = ctypes.c_void_p
    t = st._c["st_rope_table"]
    assert t(16, 64, 10000.0, None, None) == st.ST_ERR_NULL
    assert t(16, 63, 10000.0, VP(0x700000), None) == st.ST_ERR_SHAPE
    assert t(0, 64, 10000.0, VP(0x700000), None) == st.ST_ERR_SHAPE
    assert t(16, 64, 0.0, VP(0x700000), None) == st.ST_ERR_SHAPE
    rr = st._c["ulysses_relayout_rope"]

    def call(mode=st.ST_S2T, gamma=FAKE_IN, rope=VP(0x700000), n_pos=16, hd=32):
        return rr(mode, FAKE_IN, FAKE_OUT, 2, 2, 1, 8, 16, 64, 1, 1, gamma, hd, 1e-6, rope, n_pos, None)
    assert call(gamma=None) == st.ST_ERR_NULL
    assert call(rope=None) == st.ST_ERR_NULL
    assert call(mode=st.ST_T2S) == st.ST_ERR_UNSUPPORTED
    assert call(n_pos=15) == st.ST_ERR_SHAPE
    assert call(rope=VP(0x700008)) == st.ST_ERR_ALIGN
