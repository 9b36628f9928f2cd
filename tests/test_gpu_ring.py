"""GPU parity of st_attn_ring, full attention over R KV ring chunks walked in
one launch (each query block from its own chunk onwards, the running row
statistics carried across the chunk boundaries), against the fp64 oracle:
ragged chunks and ragged query tiles, chunks of whole 64-key steps, every
supported head dim, one chunk (bit-equal to the plain call), the chunk-by-chunk merge chain, and the
image-DiT 4096px shape on sampled rows."""
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


def ring(st, q, k, v, R, o_fp32=0):
    B, T, S, H, D = q.shape
    o = torch.empty(q.shape, dtype=torch.float32 if o_fp32 else q.dtype, device=DEV)
    L = torch.empty((B, T, H, S), dtype=torch.float32, device=DEV)
    st.st_attn_ring(q, k, v, o, L, R, o_fp32=o_fp32)
    torch.cuda.synchronize()
    assert st.st_check_device_status() == st.ST_OK
    return o, L


CASES = [(1, 2, 700, 2, 72, 3), (1, 1, 1030, 2, 128, 8), (2, 1, 513, 1, 64, 5), (1, 3, 390, 2, 96, 4),
         (1, 1, 260, 3, 80, 7), (1, 2, 333, 2, 32, 2), (1, 1, 2048, 2, 128, 8), (1, 1, 130, 1, 128, 64),
         (1, 1, 1800, 2, 72, 3), (1, 2, 1700, 1, 80, 5),          # >= 24 steps per item: Q in TMEM
         # every chunk a whole number of 64-key steps (the walk is a rotation of the one-range walk)
         (1, 2, 1536, 2, 72, 3), (2, 1, 512, 2, 64, 2), (1, 1, 768, 2, 96, 3), (1, 1, 640, 2, 80, 5),
         (1, 1, 1024, 2, 128, 16), (1, 1, 4096, 1, 128, 8)]


@pytest.mark.parametrize("B,T,S,H,D,R", CASES)
def test_ring_matches_oracle(st, B, T, S, H, D, R):
    """Chunk edges floor(c*S/R) fall inside 64-key steps and 256-row blocks."""
    w = synth.Workload("r", 21, B=B, T=T, S=S, H=H, D=D, dtype="bf16")
    q, k, v = synth.qkv(w)
    o, L = ring(st, q.to(DEV), k.to(DEV), v.to(DEV), R)
    ro, rl = oracle.spatial(q, k, v)
    assert_close(o.cpu(), ro, "bf16", f"ring {B,T,S,H,D,R}")
    assert_lse_close(L.cpu(), rl, "ring lse")


def test_ring_equals_merge_of_chunk_partials(st):
    """The ring result is the log-sum-exp merge of the R per-chunk partials
    (oracle definition of the merge on oracle partials)."""
    w = synth.Workload("r", 22, B=1, T=1, S=900, H=2, D=128, dtype="bf16")
    q, k, v = synth.qkv(w)
    R = 6
    edges = [c * w.S // R for c in range(R + 1)]
    parts = [oracle.spatial(q, k, v, kv=(a, b)) for a, b in zip(edges[:-1], edges[1:])]
    # partial o is [B, T, S, H, D] and its lse [B, T, H, S]: merge per (b, t, s, h)
    mo, ml = oracle.merge_chunks([p[0] for p in parts], [p[1].transpose(0, 1, 3, 2) for p in parts])
    ml = ml.transpose(0, 1, 3, 2)
    o, L = ring(st, q.to(DEV), k.to(DEV), v.to(DEV), R, o_fp32=1)
    assert_close(o.cpu(), mo, "bf16", "ring vs merged partials")
    assert_lse_close(L.cpu(), ml, "ring lse vs merged")


@pytest.mark.parametrize("S", [777, 768])
def test_ring_one_chunk_is_the_plain_call(st, S):
    """R = 1 walks the same keys in the same order as st_attn_spatial: same
    bits (a ragged last step, and whole 64-key steps only)."""
    w = synth.Workload("r", 23, B=1, T=2, S=S, H=2, D=128, dtype="bf16")
    q, k, v = (x.to(DEV) for x in synth.qkv(w))
    o1, L1 = ring(st, q, k, v, 1)
    o2 = torch.empty_like(q)
    L2 = torch.empty_like(L1)
    st.st_attn_spatial(q, k, v, o2, L2)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(L1, L2)


def test_ring_chunk_count_changes_only_rounding(st):
    """Different chunk counts give the same attention within the bf16 bar of each other."""
    w = synth.Workload("r", 24, B=1, T=1, S=1500, H=2, D=72, dtype="bf16")
    q, k, v = (x.to(DEV) for x in synth.qkv(w))
    outs = [ring(st, q, k, v, R, o_fp32=1)[0].cpu() for R in (1, 2, 5, 8)]
    for o in outs[1:]:
        assert_close(o, outs[0].double().numpy(), "bf16", "chunk counts")


def test_ring_fp32(st):
    """fp32 inputs take the fp32 kernel over the whole key range."""
    w = synth.BY_NAME["tiny"]
    q, k, v = synth.qkv(w)
    o, L = ring(st, q.to(DEV), k.to(DEV), v.to(DEV), w.R)
    ro, rl = oracle.spatial(q, k, v)
    assert_close(o.cpu(), ro, "f32", "ring fp32")
    assert_lse_close(L.cpu(), rl, "ring fp32 lse")


def test_ring_image_4096px_sampled(st):
    """The image-DiT shape (N = 65536, 24 heads x 128, R = 8) on sampled rows,
    among them rows at the chunk edges."""
    w = synth.BY_NAME["image_4096px"]
    q, k, v = synth.qkv(w)
    o, L = ring(st, q.to(DEV), k.to(DEV), v.to(DEV), w.R)
    N = w.S
    edges = [c * N // w.R for c in range(w.R)]
    rng = np.random.default_rng(31)
    rows = np.unique(np.concatenate([rng.choice(N, 96, replace=False), np.array(edges), np.array(edges[1:]) - 1,
                                     [N - 1]]))
    ro, rl = oracle.spatial(q, k, v, rows=rows)
    r = torch.from_numpy(rows)
    assert_close(o.cpu()[:, :, r], ro, "bf16", "image ring")
    assert_lse_close(L.cpu()[:, :, :, r], rl, "image ring lse")
