"""Python binding of libstattn.so, the sm_100a spatial-temporal attention hot path.

Argument marshalling only: every step runs in the CUDA library.  Tensors are
torch CUDA tensors (PyTorch provides device memory and streams); the calls are
asynchronous on ``torch.cuda.current_stream()`` unless a stream is given.
Importing this module fails loudly when the library has not been built.

Entry points (same names as the C ABI in include/stattn.h):
    st_attn_spatial, st_attn_ring, st_attn_spatial_merge, st_attn_temporal, attn_chunk_merge, ulysses_relayout,
    ulysses_relayout_range, vmajor_mask_compact, vmajor_mask_compact_noalloc, vmajor_mask_compact_scatter,
    vmajor_scatter_rows, vmajor_workspace_bytes, vmajor_relayout_mask, vmajor_relayout_rows,
    st_rope_table, ulysses_relayout_rope,
    st_check_device_status, st_status_string, st_set_sm_budget, st_get_sm_budget
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libstattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m sequence_parallelism_st_b200.build` "
        "(there is no CPU fallback)")

lib = ctypes.CDLL(LIB_PATH)

# ---------------------------------------------------------------- C types
ST_OK, ST_ERR_NULL, ST_ERR_SHAPE, ST_ERR_DIVISIBILITY, ST_ERR_DTYPE = 0, -1, -2, -3, -4
ST_ERR_ALIGN, ST_ERR_UNSUPPORTED, ST_ERR_CUDA, ST_ERR_TIMEOUT = -5, -6, -7, -8
ST_F32, ST_BF16 = 0, 1
ST_S2T, ST_T2S, ST_SEQ2HEAD, ST_HEAD2SEQ = 0, 1, 2, 3
MODES = {"S2T": ST_S2T, "T2S": ST_T2S, "SEQ2HEAD": ST_SEQ2HEAD, "HEAD2SEQ": ST_HEAD2SEQ}

c_int, c_ll, c_float, c_void_p, c_size_t = (ctypes.c_int, ctypes.c_longlong, ctypes.c_float,
                                             ctypes.c_void_p, ctypes.c_size_t)


class st_attn_desc(ctypes.Structure):
    _fields_ = [("size", c_int), ("B", c_int), ("T", c_int), ("S", c_int), ("H", c_int), ("D", c_int),
                ("dtype", c_int), ("scale", c_float),
                ("stride_b", c_ll), ("stride_t", c_ll), ("stride_s", c_ll),
                ("t_block", c_int), ("stride_tb", c_ll), ("s_block", c_int), ("stride_sb", c_ll),
                ("n_slices", c_int), ("slice", c_int), ("kv_begin", c_int), ("kv_end", c_int),
                ("o_fp32", c_int)]


def _proto(name, res, *args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_VP = c_void_p
_c = {
    "st_status_string": _proto("st_status_string", ctypes.c_char_p, c_int),
    "st_abi_version": _proto("st_abi_version", c_int),
    "st_attn_spatial": _proto("st_attn_spatial", c_int, ctypes.POINTER(st_attn_desc), _VP, _VP, _VP, _VP, _VP, _VP),
    "st_attn_temporal": _proto("st_attn_temporal", c_int, ctypes.POINTER(st_attn_desc), _VP, _VP, _VP, _VP, _VP, _VP),
    "st_attn_ring": _proto("st_attn_ring", c_int, ctypes.POINTER(st_attn_desc), _VP, _VP, _VP, _VP, _VP, c_int, _VP),
    "st_attn_spatial_merge": _proto("st_attn_spatial_merge", c_int, ctypes.POINTER(st_attn_desc), _VP, _VP, _VP,
                                    _VP, _VP, _VP, _VP, _VP),
    "attn_chunk_merge": _proto("attn_chunk_merge", c_int, c_int, ctypes.POINTER(_VP), ctypes.POINTER(_VP), c_ll,
                               c_int, c_int, c_int, _VP, c_int, _VP, _VP),
    "ulysses_relayout": _proto("ulysses_relayout", c_int, c_int, _VP, _VP, c_int, c_int, c_int, c_int, c_int,
                               c_int, c_int, c_int, c_int, c_int, c_int, c_int, _VP, c_int, c_float, _VP),
    "ulysses_relayout_range": _proto("ulysses_relayout_range", c_int, c_int, _VP, _VP, c_int, c_int, c_int, c_int,
                                     c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, _VP,
                                     c_int, c_float, _VP),
    "vmajor_workspace_bytes": _proto("vmajor_workspace_bytes", c_size_t, c_ll),
    "vmajor_mask_compact": _proto("vmajor_mask_compact", c_int, _VP, _VP, c_ll, c_int, c_int, c_float, c_int,
                                  _VP, _VP, _VP, _VP, _VP, c_size_t, _VP),
    "vmajor_mask_compact_noalloc": _proto("vmajor_mask_compact_noalloc", c_int, _VP, _VP, c_ll, c_int, c_int,
                                          c_float, c_int, _VP, _VP, _VP, _VP, _VP),
    "vmajor_mask_compact_scatter": _proto("vmajor_mask_compact_scatter", c_int, _VP, _VP, c_ll, c_int, c_int,
                                          c_float, c_int, _VP, _VP, _VP, _VP, _VP, c_size_t,
                                          ctypes.POINTER(_VP), ctypes.POINTER(_VP), c_int, _VP),
    "vmajor_scatter_rows": _proto("vmajor_scatter_rows", c_int, _VP, _VP, c_ll, c_int, c_int,
                                  ctypes.POINTER(_VP), ctypes.POINTER(_VP), c_int, ctypes.POINTER(_VP), _VP),
    "st_check_device_status": _proto("st_check_device_status", c_int, _VP),
    "st_selftest_wait_timeout": _proto("st_selftest_wait_timeout", c_int, _VP),
    "st_selftest_ex2": _proto("st_selftest_ex2", c_int, _VP, _VP, _VP, c_int, _VP),
    "st_set_sm_budget": _proto("st_set_sm_budget", c_int, c_int),
    "vmajor_relayout_mask": _proto("vmajor_relayout_mask", c_int, _VP, _VP, _VP, c_int, c_int, c_int, c_int, c_int,
                                   c_int, c_int, c_int, c_float, c_int, _VP, _VP, _VP, _VP, _VP, c_size_t, _VP),
    "vmajor_relayout_rows": _proto("vmajor_relayout_rows", c_int, _VP, _VP, _VP, _VP, c_int, c_int, c_int, c_int,
                                   c_int, c_int, c_int, c_int, _VP, c_int, c_float, _VP, c_int, _VP),
    "st_rope_table": _proto("st_rope_table", c_int, c_int, c_int, c_float, _VP, _VP),
    "ulysses_relayout_rope": _proto("ulysses_relayout_rope", c_int, c_int, _VP, _VP, c_int, c_int, c_int, c_int,
                                    c_int, c_int, c_int, c_int, _VP, c_int, c_float, _VP, c_int, _VP),
    "st_get_sm_budget": _proto("st_get_sm_budget", c_int),
}

EXPORTED = ["st_status_string", "st_abi_version", "st_attn_spatial", "st_attn_ring", "st_attn_spatial_merge",
            "st_attn_temporal",
            "attn_chunk_merge",
            "ulysses_relayout", "vmajor_workspace_bytes", "vmajor_mask_compact", "vmajor_mask_compact_noalloc",
            "vmajor_scatter_rows", "vmajor_mask_compact_scatter",
            "st_check_device_status", "st_selftest_wait_timeout", "ulysses_relayout_range", "st_set_sm_budget",
            "st_get_sm_budget", "vmajor_relayout_mask", "vmajor_relayout_rows", "st_rope_table",
            "ulysses_relayout_rope", "st_selftest_ex2"]


class StattnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {st_status_string(code)} ({code})")


def st_status_string(code: int) -> str:
    return _c["st_status_string"](int(code)).decode()


def _check(code: int, where: str) -> int:
    if code != ST_OK:
        raise StattnError(code, where)
    return code


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return ST_F32
    if t.dtype == torch.bfloat16:
        return ST_BF16
    raise StattnError(ST_ERR_DTYPE, f"dtype {t.dtype}")


def make_desc(B, T, S, H, D, dtype=ST_BF16, scale=0.0, stride_b=0, stride_t=0, stride_s=0, t_block=0,
              stride_tb=0, s_block=0, stride_sb=0, n_slices=1, slice=-1, kv_begin=0, kv_end=0,
              o_fp32=0) -> st_attn_desc:
    return st_attn_desc(ctypes.sizeof(st_attn_desc), B, T, S, H, D, dtype, scale, stride_b, stride_t,
                        stride_s, t_block, stride_tb, s_block, stride_sb, n_slices, slice, kv_begin, kv_end,
                        o_fp32)


# ---------------------------------------------------------------- attention
def st_attn_spatial(q, k, v, o, lse=None, *, desc: st_attn_desc | None = None, stream=None, raw=False, **kw):
    """Spatial attention per (b, t, head) over the S tokens of each frame.

    q, k, v, o: CUDA tensors; with no ``desc`` they are [B, T, S, H, D]
    contiguous and the descriptor is derived from their shape (keyword
    arguments override its fields).  Returns the status code when ``raw``.
    """
    if desc is None:
        B, T, S, H, D = q.shape
        desc = make_desc(B, T, S, H, D, _dtype_code(q), **kw)
    r = _c["st_attn_spatial"](ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _stream(stream))
    return r if raw else _check(r, "st_attn_spatial")


def st_attn_ring(q, k, v, o, lse=None, n_chunks=1, *, desc: st_attn_desc | None = None, stream=None, raw=False,
                 **kw):
    """Full attention over ``n_chunks`` KV ring chunks in one launch: each query
    block starts at the chunk holding its first row and carries its running
    statistics across the chunks (include/stattn.h)."""
    if desc is None:
        B, T, S, H, D = q.shape
        desc = make_desc(B, T, S, H, D, _dtype_code(q), **kw)
    r = _c["st_attn_ring"](ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(n_chunks),
                           _stream(stream))
    return r if raw else _check(r, "st_attn_ring")


def st_attn_spatial_merge(q, k, v, o_acc, lse_acc, o, lse=None, *, desc: st_attn_desc | None = None, stream=None,
                          raw=False, **kw):
    """Spatial attention over one KV chunk merged into the accumulated fp32
    partial ``o_acc`` and its LSE ``lse_acc``; ``o`` may be ``o_acc`` when the
    result is fp32 (``o_fp32=1``)."""
    if desc is None:
        B, T, S, H, D = q.shape
        desc = make_desc(B, T, S, H, D, _dtype_code(q), **kw)
    r = _c["st_attn_spatial_merge"](ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o_acc), _ptr(lse_acc),
                                    _ptr(o), _ptr(lse), _stream(stream))
    return r if raw else _check(r, "st_attn_spatial_merge")


def st_attn_temporal(q, k, v, o, lse=None, *, desc: st_attn_desc | None = None, stream=None, raw=False, **kw):
    """Temporal attention per (b, s, head) over the T frames of each token."""
    if desc is None:
        B, T, S, H, D = q.shape
        desc = make_desc(B, T, S, H, D, _dtype_code(q), **kw)
    r = _c["st_attn_temporal"](ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _stream(stream))
    return r if raw else _check(r, "st_attn_temporal")


def attn_chunk_merge(o_parts, lse_parts, n_units, S, H, D, o_out, lse_out=None, *, stream=None, raw=False):
    """Log-sum-exp merge of fp32 KV-chunk partials into o_out (bf16 or fp32)."""
    n = len(o_parts)
    op = (c_void_p * n)(*[t.data_ptr() for t in o_parts])
    lp = (c_void_p * n)(*[t.data_ptr() for t in lse_parts])
    r = _c["attn_chunk_merge"](n, op, lp, int(n_units), int(S), int(H), int(D), _ptr(o_out), _dtype_code(o_out),
                               _ptr(lse_out), _stream(stream))
    return r if raw else _check(r, "attn_chunk_merge")


# ---------------------------------------------------------------- relayout
def ulysses_relayout(mode, inp, out, P, B, T_or_N, S_or_H, C_or_D, n_t=1, n_s=1, blocks=None, rms_gamma=None,
                     rms_head_dim=0, rms_eps=1e-6, *, stream=None, raw=False):
    """All-to-all on a virtual partition of P shards (see include/stattn.h)."""
    m = MODES[mode] if isinstance(mode, str) else int(mode)
    i0, i1, j0, j1 = blocks if blocks is not None else (0, n_t, 0, n_s)
    r = _c["ulysses_relayout"](m, _ptr(inp), _ptr(out), inp.element_size(), P, B, T_or_N, S_or_H, C_or_D,
                               n_t, n_s, i0, i1, j0, j1, _ptr(rms_gamma), int(rms_head_dim), float(rms_eps),
                               _stream(stream))
    return r if raw else _check(r, "ulysses_relayout")


def ulysses_relayout_range(mode, inp, out, P, B, T_or_N, S_or_H, C_or_D, n_t=1, n_s=1, blocks=None, shards=None,
                           rms_gamma=None, rms_head_dim=0, rms_eps=1e-6, *, stream=None, raw=False):
    """ulysses_relayout restricted to the temporally sharded shards ``shards`` = (q0, q1)."""
    m = MODES[mode] if isinstance(mode, str) else int(mode)
    i0, i1, j0, j1 = blocks if blocks is not None else (0, n_t, 0, n_s)
    q0, q1 = shards if shards is not None else (0, P)
    r = _c["ulysses_relayout_range"](m, _ptr(inp), _ptr(out), inp.element_size(), P, B, T_or_N, S_or_H, C_or_D,
                                     n_t, n_s, i0, i1, j0, j1, q0, q1, _ptr(rms_gamma), int(rms_head_dim),
                                     float(rms_eps), _stream(stream))
    return r if raw else _check(r, "ulysses_relayout_range")


# ---------------------------------------------------------------- V-Major
def vmajor_workspace_bytes(n_tokens: int) -> int:
    return int(_c["vmajor_workspace_bytes"](int(n_tokens)))


def vmajor_mask_compact(v_cur, v_prev, tau, mask, idx, count, workspace, force_all=False, l1_out=None, *,
                        stream=None, raw=False):
    """Per-token L1 change mask and ascending compaction of active tokens."""
    n, C = v_cur.shape[0], v_cur[0].numel()
    r = _c["vmajor_mask_compact"](_ptr(v_cur), _ptr(v_prev), n, C, _dtype_code(v_cur), float(tau),
                                  1 if force_all else 0, _ptr(mask), _ptr(idx), _ptr(count), _ptr(l1_out),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    return r if raw else _check(r, "vmajor_mask_compact")


def vmajor_mask_compact_noalloc(v_cur, v_prev, tau, mask, idx, count, force_all=False, l1_out=None, *,
                                stream=None, raw=False):
    """vmajor_mask_compact with the library's own static scratch (no workspace, no allocation)."""
    n, C = v_cur.shape[0], v_cur[0].numel()
    r = _c["vmajor_mask_compact_noalloc"](_ptr(v_cur), _ptr(v_prev), n, C, _dtype_code(v_cur), float(tau),
                                          1 if force_all else 0, _ptr(mask), _ptr(idx), _ptr(count),
                                          _ptr(l1_out), _stream(stream))
    return r if raw else _check(r, "vmajor_mask_compact_noalloc")


def vmajor_mask_compact_scatter(v_cur, v_prev, tau, mask, idx, count, workspace, src, dst_cache, force_all=False,
                                l1_out=None, *, stream=None, raw=False):
    """vmajor_mask_compact and the cache update of the active tokens' rows in one call."""
    n, C = v_cur.shape[0], v_cur[0].numel()
    nt = len(src)
    sp = (c_void_p * nt)(*[t.data_ptr() for t in src])
    dp = (c_void_p * nt)(*[t.data_ptr() for t in dst_cache])
    r = _c["vmajor_mask_compact_scatter"](_ptr(v_cur), _ptr(v_prev), n, C, _dtype_code(v_cur), float(tau),
                                          1 if force_all else 0, _ptr(mask), _ptr(idx), _ptr(count), _ptr(l1_out),
                                          _ptr(workspace), workspace.numel() * workspace.element_size(), sp, dp, nt,
                                          _stream(stream))
    return r if raw else _check(r, "vmajor_mask_compact_scatter")


def vmajor_scatter_rows(idx, count, src, dst_cache, packed=None, *, stream=None, raw=False):
    """cache[idx[i]] <- src[idx[i]] for i < count (and the packed message)."""
    n = len(src)
    n_tok, C = src[0].shape[0], src[0][0].numel()
    sp = (c_void_p * n)(*[t.data_ptr() for t in src])
    dp = (c_void_p * n)(*[t.data_ptr() for t in dst_cache])
    pp = (c_void_p * n)(*[t.data_ptr() for t in packed]) if packed is not None else None
    r = _c["vmajor_scatter_rows"](_ptr(idx), _ptr(count), n_tok, C, src[0].element_size(), sp, dp, n, pp,
                                  _stream(stream))
    return r if raw else _check(r, "vmajor_scatter_rows")


def vmajor_relayout_mask(v_cur_x, v_prev_x, v_cache_y, P, B, T, S, C, n_t, n_s, tau, mask, idx, count, workspace,
                         force_all=False, l1_out=None, *, stream=None, raw=False):
    """Sender-side V-Major: mask of the L1 change of V on the x layout, rows of active
    tokens moved S->T into the V cache; mask/idx/count in y numbering."""
    r = _c["vmajor_relayout_mask"](_ptr(v_cur_x), _ptr(v_prev_x), _ptr(v_cache_y), P, B, T, S, C, n_t, n_s,
                                   _dtype_code(v_cur_x), float(tau), 1 if force_all else 0, _ptr(mask), _ptr(idx),
                                   _ptr(count), _ptr(l1_out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    return r if raw else _check(r, "vmajor_relayout_mask")


def vmajor_relayout_rows(in_x, out_y, idx, count, P, B, T, S, C, n_t, n_s, rms_gamma=None, rms_head_dim=0,
                         rms_eps=1e-6, rope_table=None, *, stream=None, raw=False):
    """S->T move of the destination rows idx[:count] (device), with the optional per-head RMSNorm
    and rotary embedding (rope_table from st_rope_table)."""
    n_pos = rope_table.shape[0] if rope_table is not None else 0
    r = _c["vmajor_relayout_rows"](_ptr(in_x), _ptr(out_y), _ptr(idx), _ptr(count), P, B, T, S, C, n_t, n_s,
                                   _dtype_code(in_x), _ptr(rms_gamma), int(rms_head_dim), float(rms_eps),
                                   _ptr(rope_table), n_pos, _stream(stream))
    return r if raw else _check(r, "vmajor_relayout_rows")


def st_rope_table(n_pos, head_dim, theta=10000.0, *, device="cuda", stream=None):
    """Rotary (cos, sin) table, fp32 [n_pos, head_dim // 2, 2], computed on the device."""
    import torch
    t = torch.empty((n_pos, head_dim // 2, 2), dtype=torch.float32, device=device)
    _check(_c["st_rope_table"](int(n_pos), int(head_dim), float(theta), _ptr(t), _stream(stream)), "st_rope_table")
    return t


def ulysses_relayout_rope(mode, inp, out, P, B, T_or_N, S_or_H, C_or_D, n_t=1, n_s=1, rms_gamma=None,
                          rms_head_dim=0, rms_eps=1e-6, rope_table=None, *, stream=None, raw=False):
    """ulysses_relayout (S2T / SEQ2HEAD) with the per-head RMSNorm and the rotary embedding."""
    m = MODES[mode] if isinstance(mode, str) else int(mode)
    n_pos = rope_table.shape[0] if rope_table is not None else 0
    r = _c["ulysses_relayout_rope"](m, _ptr(inp), _ptr(out), inp.element_size(), P, B, T_or_N, S_or_H, C_or_D, n_t,
                                    n_s, _ptr(rms_gamma), int(rms_head_dim), float(rms_eps), _ptr(rope_table), n_pos,
                                    _stream(stream))
    return r if raw else _check(r, "ulysses_relayout_rope")


def st_check_device_status(stream=None) -> int:
    return int(_c["st_check_device_status"](_stream(stream)))


def st_set_sm_budget(sms: int) -> None:
    """Size the grids of this thread's later launches for at most ``sms`` SMs (0: all)."""
    _check(_c["st_set_sm_budget"](int(sms)), "st_set_sm_budget")


def st_get_sm_budget() -> int:
    return int(_c["st_get_sm_budget"]())


def st_selftest_wait_timeout(stream=None) -> int:
    return int(_c["st_selftest_wait_timeout"](_stream(stream)))


def st_selftest_ex2(x, y_poly, y_mufu, *, stream=None, raw=False):
    """The softmax's two exp2 implementations evaluated on the fp32 device tensor x."""
    r = _c["st_selftest_ex2"](_ptr(x), _ptr(y_poly), _ptr(y_mufu), int(x.numel()), _stream(stream))
    return r if raw else _check(r, "st_selftest_ex2")
