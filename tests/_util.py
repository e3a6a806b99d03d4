"""Helpers shared by the tests: tolerances and oracle comparisons."""
import numpy as np

# Normwise relative error bar for the products: max|y - r| / max|r|.
TOL = 2e-3
# Unit roundoff of the output formats: a bf16 / fp16 output adds its own
# rounding of up to u * |r| per element on top of the computation's error.
UNIT_ROUNDOFF = {"float32": 0.0, "bfloat16": 2.0 ** -8, "float16": 2.0 ** -11}


def normwise_err(y: np.ndarray, r: np.ndarray) -> float:
    scale = np.abs(r).max()
    return float(np.abs(y - r).max() / scale) if scale > 0 else float(np.abs(y).max())


def assert_close(y: np.ndarray, r: np.ndarray, out_dtype: str, tol: float = TOL):
    """y (float64 copy of the device output) against the fp64 oracle r."""
    y = np.asarray(y, np.float64)
    r = np.asarray(r, np.float64)
    assert y.shape == r.shape, (y.shape, r.shape)
    assert np.isfinite(y).all()
    scale = np.abs(r).max()
    if scale == 0:
        assert np.abs(y).max() == 0
        return
    bound = tol * scale + UNIT_ROUNDOFF[out_dtype] * np.abs(r)
    bad = np.abs(y - r) > bound
    assert not bad.any(), (
        f"{bad.sum()} of {bad.size} outside the bound; normwise err {normwise_err(y, r):.3e}")
    return normwise_err(y, r)


def sample_rows(n: int, k: int, seed: int = 0) -> np.ndarray:
    """First, last and a seeded sample of output rows."""
    if n <= k:
        return np.arange(n)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, n - 1), size=k - 2, replace=False)
    return np.unique(np.concatenate([[0, n - 1], mid]))
