"""Helpers shared by the GPU parity tests (conversion and tolerances)."""
import numpy as np
import torch

from oracle import bf16_bits_to_f64

# bf16 inputs, fp32 accumulation: element-wise bar on outputs against the
# fp64 oracle (max and mean absolute error).
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor, as uint16 numpy (copied to host)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 widening of a bf16 tensor."""
    return bf16_bits_to_f64(bits(t))


def assert_close(got: np.ndarray, want: np.ndarray, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what=""):
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    assert err.max() <= max_abs, f"{what}: max abs err {err.max():.3e} > {max_abs}"
    assert err.mean() <= mean_abs, f"{what}: mean abs err {err.mean():.3e} > {mean_abs}"
    return float(err.max()), float(err.mean())


def assert_bf16_rounding(got: np.ndarray, want: np.ndarray, what=""):
    """got is want (exact, fp64) rounded to bf16, allowing one unit in the last place.

    fp32 arithmetic on the device may land on the other side of a rounding
    boundary than the exact value, so one ulp (2^-7 relative) is allowed.
    """
    err = np.abs(got - want)
    bound = np.abs(want) * 2.0 ** -7 + 1e-6
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements beyond 1 bf16 ulp (max err {err.max():.3e})"
