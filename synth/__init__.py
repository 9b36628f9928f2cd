"""Seeded synthetic inputs for the spatial-temporal attention hot path.

This module is shared by the tests, the benchmark and the oracle checks. It
holds the workload table and random-number recipes only: no attention, no
relayout, no masking arithmetic. Every tensor is drawn on the CPU from a
``torch.Generator`` so that the CUDA path and the CPU oracle see identical
bits.

Workloads (shapes follow the pages' workloads; there are no datasets or
trained weights, so every tensor is synthetic):

* ``tiny``          ST-DiT block, B=1 T=4 S=64 (8x8) H=2 D=32, fp32.
* ``opensora_low``  ST-DiT block like OpenSora at low resolution:
                    T=16 S=1200 (30x40) H=16 D=72, bf16.
* ``video_1080p``   1080p long-video ST-DiT block: T=32 S=8160 (68x120)
                    H=16 D=72, bf16.
* ``image_4096px``  image-DiT full attention: N=65536 (256x256) H=24 D=128.
* ``vmajor_2304px`` V-Major selective path: N=20736 (144x144) H=24 D=128.

Seeds: workload k (0-based) uses base seed 1000+k+1; tensor ``name`` uses
sub-seed SUBSEED[name]; the generator seed is base*100 + sub-seed.  Draws are
fp32 N(0,1) and are rounded to bf16 (round to nearest even) for bf16
workloads.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

SUBSEED = {"q": 0, "k": 1, "v": 2, "prev": 3, "noise": 4, "sigma": 5,
           "gamma": 6, "kprev": 7, "knoise": 8, "qt": 9, "kt": 10, "vt": 11}


@dataclass(frozen=True)
class Workload:
    name: str
    index: int                # 0-based position in the workload table
    B: int
    T: int
    S: int
    H: int
    D: int
    dtype: str                # "f32" | "bf16"
    P: int = 1                # virtual partition count for the relayout
    n_t: int = 1              # N_T temporal slices
    n_s: int = 1              # N_S spatial slices
    L_T: int = 0              # hoisted temporal partitions
    L_S: int = 0              # hoisted spatial partitions
    R: int = 1                # KV chunks merged by log-sum-exp
    rms: bool = False         # per-head RMSNorm on Q/K
    vmajor_f: tuple = ()      # target active fractions for the V-Major mask
    sigma_range: tuple = (1e-4, 1e-1)
    rms_eps: float = 1e-6

    @property
    def C(self) -> int:
        return self.H * self.D

    @property
    def seed(self) -> int:
        return 1000 + self.index + 1

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def spatial_flops(self, n_keys: int | None = None) -> float:
        """4 * rows * keys * D per head (2 for QK^T, 2 for PV)."""
        keys = self.S if n_keys is None else n_keys
        return 4.0 * self.B * self.T * self.S * keys * self.H * self.D

    def temporal_flops(self) -> float:
        return 4.0 * self.B * self.S * self.T * self.T * self.H * self.D

    def tensor_bytes(self) -> int:
        return self.B * self.T * self.S * self.C * self.elem_bytes


WORKLOADS = [
    Workload("tiny", 0, B=1, T=4, S=64, H=2, D=32, dtype="f32", P=2, n_t=2,
             n_s=2, R=2, rms=True, vmajor_f=(0.5,)),
    Workload("opensora_low", 1, B=1, T=16, S=1200, H=16, D=72, dtype="bf16",
             P=4, n_t=4, n_s=4, L_T=1, L_S=3, R=2, rms=True, vmajor_f=(0.5,)),
    Workload("video_1080p", 2, B=1, T=32, S=8160, H=16, D=72, dtype="bf16",
             P=8, n_t=4, n_s=4, L_T=1, L_S=3, R=2, vmajor_f=(0.5,)),
    Workload("image_4096px", 3, B=1, T=1, S=65536, H=24, D=128, dtype="bf16",
             P=8, R=8, rms=True),
    Workload("vmajor_2304px", 4, B=1, T=1, S=20736, H=24, D=128, dtype="bf16",
             vmajor_f=(0.5, 0.1, 0.9)),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def generator(w: Workload, name: str) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed * 100 + SUBSEED[name])
    return g


def randn(w: Workload, name: str, shape, dtype=None) -> torch.Tensor:
    """fp32 N(0,1) draws, rounded to the workload dtype (RNE for bf16)."""
    x = torch.randn(*shape, generator=generator(w, name), dtype=torch.float32)
    return x.to(dtype or w.torch_dtype)


def qkv(w: Workload, names=("q", "k", "v")):
    """Q, K, V in the natural layout [B, T, S, H, D]."""
    shape = (w.B, w.T, w.S, w.H, w.D)
    return tuple(randn(w, n, shape) for n in names)


def rms_gamma(w: Workload) -> torch.Tensor:
    """Per head-dim gain, N(1, 0.1) (no trained weights exist), fp32 [D]."""
    g = torch.randn(w.D, generator=generator(w, "gamma"), dtype=torch.float32)
    return 1.0 + 0.1 * g


def token_sigma(w: Workload, n_tokens: int) -> torch.Tensor:
    """Per-token noise std, log-uniform in ``w.sigma_range``, fp32 [n]."""
    lo, hi = (math.log10(x) for x in w.sigma_range)
    u = torch.rand(n_tokens, generator=generator(w, "sigma"), dtype=torch.float64)
    return (10.0 ** (lo + (hi - lo) * u)).to(torch.float32)


def vmajor_pair(w: Workload, n_tokens: int, C: int, prev="prev", noise="noise"):
    """(cur, prev): prev ~ N(0,1); cur = prev + N(0, sigma_n) per token.

    Both are rounded to the workload dtype, so a small perturbation may round
    back to the stored value of ``prev``.
    """
    p32 = torch.randn(n_tokens, C, generator=generator(w, prev), dtype=torch.float32)
    z = torch.randn(n_tokens, C, generator=generator(w, noise), dtype=torch.float32)
    sig = token_sigma(w, n_tokens)
    cur32 = p32 + z * sig[:, None]
    return cur32.to(w.torch_dtype), p32.to(w.torch_dtype)


def index_tagged(n_rows: int, row_len: int, dtype=torch.float32) -> torch.Tensor:
    """Rows whose values encode (row, column): value = row * row_len + col.

    Exact in fp32 while the tensor has fewer than 2**24 elements; used to
    check that a permutation writes every element exactly once.
    """
    assert n_rows * row_len < (1 << 24) or dtype in (torch.float64, torch.int32)
    return torch.arange(n_rows * row_len, dtype=torch.float64).reshape(n_rows, row_len).to(dtype)
