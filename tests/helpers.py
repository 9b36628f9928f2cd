"""Shared helpers of the GPU parity tests (tolerances from the method's bar)."""
import numpy as np
import torch

# bf16 in / fp32 accumulate: max abs <= 2e-2 and relative Frobenius <= 5e-3;
# fp32 path: relative Frobenius <= 1e-4.
BF16_MAX_ABS = 2e-2
BF16_REL_FRO = 5e-3
F32_REL_FRO = 1e-4


def f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu").to(torch.float64).numpy()


def rel_fro(a, b) -> float:
    a, b = f64(a), f64(b)
    den = np.linalg.norm(b.ravel())
    return float(np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0))


def assert_close(got, ref, dtype: str, what: str = ""):
    """The float bar for a result computed in ``dtype`` ("bf16" or "f32")."""
    g, r = f64(got), f64(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    rf = rel_fro(g, r)
    if dtype == "bf16":
        ma = float(np.max(np.abs(g - r))) if g.size else 0.0
        assert ma <= BF16_MAX_ABS and rf <= BF16_REL_FRO, f"{what}: max abs {ma:.3e}, rel fro {rf:.3e}"
    else:
        assert rf <= F32_REL_FRO, f"{what}: rel fro {rf:.3e}"


def assert_lse_close(got, ref, what=""):
    """LSE is fp32 on both paths: absolute error well inside the bf16 bar."""
    g, r = f64(got), f64(ref)
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: -inf pattern differs"
    if fin.any():
        err = float(np.max(np.abs(g[fin] - r[fin])))
        assert err <= 2e-3, f"{what}: lse max abs {err:.3e}"
