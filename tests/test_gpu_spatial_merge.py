"""GPU parity of st_attn_spatial_merge (KV-chunk attention with the log-sum-exp
merge fused into the kernel) against the fp64 oracle, through the C ABI:
uneven chains with a single-key chunk, in-place fp32 accumulation, the bf16
final output, an empty chunk, an empty accumulator (its values are never
read), the fp32 FMA path, and the full opensora_low shape on sampled frames."""
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


def chain(st, q, k, v, edges, out_dtype):
    """Chunk 0 into an fp32 accumulator, middle chunks merged in place, the
    last chunk merged into a fresh output of out_dtype."""
    B, T, S, H, D = q.shape
    acc = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    lacc = torch.empty((B, T, H, S), dtype=torch.float32, device=DEV)
    st.st_attn_spatial(q, k, v, acc, lacc, o_fp32=1, kv_begin=edges[0], kv_end=edges[1])
    for a, b in zip(edges[1:-2], edges[2:-1]):
        st.st_attn_spatial_merge(q, k, v, acc, lacc, acc, lacc, o_fp32=1, kv_begin=a, kv_end=b)
    out = torch.empty(q.shape, dtype=out_dtype, device=DEV)
    lout = torch.empty((B, T, H, S), dtype=torch.float32, device=DEV)
    f32 = 1 if out_dtype == torch.float32 else 0
    st.st_attn_spatial_merge(q, k, v, acc, lacc, out, lout, o_fp32=f32, kv_begin=edges[-2], kv_end=edges[-1])
    torch.cuda.synchronize()
    assert st.st_check_device_status() == st.ST_OK
    return out, lout


@pytest.mark.parametrize("D", [64, 72, 96, 128])
def test_fused_merge_chain(st, D):
    w = synth.Workload("m", 21, B=1, T=2, S=700, H=2, D=D, dtype="bf16")
    q, k, v = synth.qkv(w)
    out, lout = chain(st, q.to(DEV), k.to(DEV), v.to(DEV), [0, 128, 300, 301, 700], torch.bfloat16)
    ro, rl = oracle.spatial(q, k, v)
    assert_close(out.cpu(), ro, "bf16", f"fused merge D={D}")
    assert_lse_close(lout.cpu(), rl, f"fused merge lse D={D}")


def test_fused_merge_two_chunks_ragged_tiles(st):
    """S not a multiple of the 128-row tile nor of the 64-key step."""
    w = synth.Workload("m", 22, B=1, T=3, S=333, H=3, D=72, dtype="bf16")
    q, k, v = synth.qkv(w)
    out, lout = chain(st, q.to(DEV), k.to(DEV), v.to(DEV), [0, 170, 333], torch.bfloat16)
    ro, rl = oracle.spatial(q, k, v)
    assert_close(out.cpu(), ro, "bf16", "fused merge ragged")
    assert_lse_close(lout.cpu(), rl, "fused merge ragged lse")


def test_fused_merge_fp32_result_in_place(st):
    """The accumulator carries all chunks as an fp32 partial (o = o_acc)."""
    w = synth.Workload("m", 23, B=1, T=1, S=520, H=2, D=128, dtype="bf16")
    q, k, v = synth.qkv(w)
    out, lout = chain(st, q.to(DEV), k.to(DEV), v.to(DEV), [0, 64, 200, 520], torch.float32)
    ro, rl = oracle.spatial(q, k, v)
    assert_close(out.cpu(), ro, "bf16", "fused merge fp32 out")
    assert_lse_close(lout.cpu(), rl, "fused merge fp32 lse")


def test_fused_merge_empty_chunk_keeps_accumulator(st):
    w = synth.Workload("m", 24, B=1, T=1, S=200, H=2, D=72, dtype="bf16")
    q, k, v = (x.to(DEV) for x in synth.qkv(w))
    acc = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    lacc = torch.empty((1, 1, 2, 200), dtype=torch.float32, device=DEV)
    st.st_attn_spatial(q, k, v, acc, lacc, o_fp32=1, kv_begin=0, kv_end=200)
    out = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    lout = torch.empty_like(lacc)
    st.st_attn_spatial_merge(q, k, v, acc, lacc, out, lout, o_fp32=1, kv_begin=50, kv_end=50)
    torch.cuda.synchronize()
    assert torch.equal(out, acc) and torch.equal(lout, lacc)


def test_fused_merge_empty_accumulator_is_not_read(st):
    """lse_acc = -inf means nothing accumulated: o_acc (NaN here) must not leak."""
    w = synth.Workload("m", 25, B=1, T=2, S=300, H=2, D=72, dtype="bf16")
    q, k, v = synth.qkv(w)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    acc = torch.full(q.shape, float("nan"), dtype=torch.float32, device=DEV)
    lacc = torch.full((1, 2, 2, 300), float("-inf"), dtype=torch.float32, device=DEV)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=DEV)
    lout = torch.empty_like(lacc)
    st.st_attn_spatial_merge(qd, kd, vd, acc, lacc, out, lout, kv_begin=0, kv_end=300)
    torch.cuda.synchronize()
    ro, rl = oracle.spatial(q, k, v)
    assert_close(out.cpu(), ro, "bf16", "empty accumulator")
    assert_lse_close(lout.cpu(), rl, "empty accumulator lse")


def test_fused_merge_fp32_fma_path(st):
    w = synth.BY_NAME["tiny"]
    q, k, v = synth.qkv(w)
    out, lout = chain(st, q.to(DEV), k.to(DEV), v.to(DEV), [0, 17, 40, 64], torch.float32)
    ro, rl = oracle.spatial(q, k, v)
    assert_close(out.cpu(), ro, "f32", "fused merge fp32 path")
    assert_lse_close(lout.cpu(), rl, "fused merge fp32 path lse")


def test_fused_merge_bf16_output_may_not_alias(st):
    w = synth.Workload("m", 26, B=1, T=1, S=64, H=1, D=64, dtype="bf16")
    q, k, v = (x.to(DEV) for x in synth.qkv(w))
    acc = torch.zeros(q.shape, dtype=torch.float32, device=DEV)
    lacc = torch.zeros((1, 1, 1, 64), dtype=torch.float32, device=DEV)
    r = st.st_attn_spatial_merge(q, k, v, acc, lacc, acc, lacc, raw=True, kv_begin=0, kv_end=64)
    assert r == st.ST_ERR_SHAPE


def test_fused_merge_opensora_sampled(st):
    """The bench's two-chunk chain at the full opensora_low shape, checked on
    sampled frames against the oracle."""
    w = synth.BY_NAME["opensora_low"]
    q, k, v = synth.qkv(w)
    half = w.S // 2
    out, lout = chain(st, q.to(DEV), k.to(DEV), v.to(DEV), [0, half, w.S], torch.bfloat16)
    frames = [0, 7, 15]
    ro, rl = oracle.spatial(q, k, v, frames=frames)
    assert_close(out.cpu()[:, frames], ro, "bf16", "opensora fused merge")
    assert_lse_close(lout.cpu()[:, frames], rl, "opensora fused merge lse")


@pytest.mark.parametrize("D,S,edges", [(72, 3300, [0, 1540, 1541, 3300]), (80, 3100, [0, 1600, 3100])])
def test_fused_merge_long_chunks_q_in_tmem(st, D, S, edges):
    """Chunks of 24 or more 64-key steps take the kernel that keeps Q in TMEM
    (head dims 72 and 80), also in merge mode; the last query block of each
    frame leaves the second tile empty."""
    w = synth.Workload("m", 23, B=1, T=1, S=S, H=2, D=D, dtype="bf16")
    q, k, v = synth.qkv(w)
    out, lout = chain(st, q.to(DEV), k.to(DEV), v.to(DEV), edges, torch.bfloat16)
    rows = np.sort(np.random.default_rng(D).choice(S, 300, replace=False))
    ro, rl = oracle.spatial(q, k, v, rows=rows)
    r = torch.from_numpy(rows)
    assert_close(out.cpu()[:, :, r], ro, "bf16", f"long chunks D={D}")
    assert_lse_close(lout.cpu()[:, :, :, r], rl, f"long chunks lse D={D}")
