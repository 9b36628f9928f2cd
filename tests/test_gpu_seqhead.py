"""GPU parity of the sequence <-> head exchange (ulysses_relayout SEQ2HEAD /
HEAD2SEQ) against the oracle on every row width and batch layout its kernels
handle: rows of 8, 16 and 32 sixteen-byte vectors (the row-walking kernel),
other widths (the segment kernel), B = 1 and B > 1 (shards stacked outermost,
batches inside), with and without the fused per-head RMSNorm, and the round
trip."""
import pytest
import torch

import oracle
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


def data(rows, D, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(rows, D, generator=g, dtype=torch.float32).to(dtype)


# (P, B, N, H, D, dtype): row bytes 128 / 256 / 512 take the row-walking kernel, the others the segment kernel
SHAPES = [(8, 1, 4096, 24, 128, torch.bfloat16), (2, 2, 96, 4, 64, torch.bfloat16), (4, 3, 64, 8, 128, torch.bfloat16),
          (2, 2, 40, 6, 128, torch.float32), (4, 1, 64, 4, 32, torch.float32), (2, 3, 30, 2, 72, torch.bfloat16),
          (3, 2, 33, 9, 96, torch.bfloat16), (2, 1, 10, 2, 64, torch.float32)]


@pytest.mark.parametrize("P,B,N,H,D,dtype", SHAPES)
@pytest.mark.parametrize("mode", ["SEQ2HEAD", "HEAD2SEQ"])
def test_seq_head_copy_bit_exact(st, P, B, N, H, D, dtype, mode):
    x = data(B * N * H, D, dtype, 5 + N)
    out = torch.full_like(x, float("nan"), device=DEV)
    st.ulysses_relayout(mode, x.to(DEV), out, P, B, N, H, D)
    torch.cuda.synchronize()
    dst, src = oracle.seq_head_row_pairs(mode, P, B, N, H)
    assert torch.equal(bits(out)[torch.from_numpy(dst)], bits(x)[torch.from_numpy(src)])


@pytest.mark.parametrize("P,B,N,H,D,dtype", SHAPES)
def test_seq_head_round_trip(st, P, B, N, H, D, dtype):
    x = data(B * N * H, D, dtype, 7 + H).to(DEV)
    y, z = torch.empty_like(x), torch.empty_like(x)
    st.ulysses_relayout("SEQ2HEAD", x, y, P, B, N, H, D)
    st.ulysses_relayout("HEAD2SEQ", y, z, P, B, N, H, D)
    torch.cuda.synchronize()
    assert torch.equal(bits(z), bits(x))


@pytest.mark.parametrize("P,B,N,H,D,dtype", SHAPES)
@pytest.mark.parametrize("mode", ["SEQ2HEAD", "HEAD2SEQ"])
def test_seq_head_fused_rmsnorm(st, P, B, N, H, D, dtype, mode):
    x = data(B * N * H, D, dtype, 11 + D)
    gamma = 1.0 + 0.1 * data(1, D, torch.float32, 3).reshape(D)
    out = torch.empty_like(x, device=DEV)
    st.ulysses_relayout(mode, x.to(DEV), out, P, B, N, H, D, rms_gamma=gamma.to(DEV), rms_head_dim=D, rms_eps=1e-6)
    torch.cuda.synchronize()
    ref = oracle.seq_head_relayout(mode, x, P, B, N, H, D, rms=(gamma, D, 1e-6))
    assert_close(out.reshape(-1), ref, "bf16" if dtype == torch.bfloat16 else "f32", f"{mode} rms {P,B,N,H,D}")
