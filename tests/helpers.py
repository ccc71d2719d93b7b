"""Shared helpers of the GPU parity tests (tolerances, sampling, transfers)."""
import numpy as np
import torch

# Tolerances stated for the path: attention outputs max-abs 2e-2 (bf16) or
# 1e-4 (fp32); log-sum-exp max-abs 1e-3.
O_TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
LSE_TOL = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    """Inputs exactly as stored, widened to fp64, on the host."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def sample_rows(n: int, boundaries=(), count: int = 8, seed: int = 0) -> np.ndarray:
    """Deterministic sample of rows of an n-row host: the ends, tile edges
    (127/128/255/256), the given boundaries +-1 and `count` seeded rows."""
    rng = np.random.default_rng(seed)
    rows = {0, 1, 2, 31, 32, 63, 64, 127, 128, 129, 255, 256, n - 2, n - 1}
    for b in boundaries:
        rows |= {b - 1, b, b + 1}
    rows |= set(rng.integers(0, n, size=count).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < n), dtype=np.int64)


def assert_close(got, want, tol, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    both_inf = np.isinf(got) & np.isinf(want) & (np.sign(got) == np.sign(want))
    with np.errstate(invalid="ignore"):
        err = np.where(both_inf, 0.0, np.abs(got - want))
    m = float(np.nanmax(err)) if err.size else 0.0
    assert not np.isnan(err).any(), f"{what}: NaN"
    assert m <= tol, f"{what}: max-abs error {m:.3e} > {tol:.1e}"
    return m
