"""Shared helpers for the GPU parity tests (comparison metrics and tolerances)."""
import numpy as np
import pytest
import torch

# Acceptance bars: bf16 inputs, fp32 accumulation, bf16 outputs.
OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 5e-3
CACHE_MAX_ABS = 1e-2


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, ref: np.ndarray):
    diff = got - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    den = float(np.sqrt((ref ** 2).sum()))
    rel = float(np.sqrt((diff ** 2).sum()) / den) if den > 0 else 0.0
    return max_abs, rel


def assert_close_out(got: np.ndarray, ref: np.ndarray, what: str):
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    max_abs, rel = errors(got, ref)
    assert max_abs <= OUT_MAX_ABS and rel <= OUT_REL_L2, \
        f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def assert_close_cache(got: np.ndarray, ref: np.ndarray, what: str):
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    max_abs, _ = errors(got, ref)
    assert max_abs <= CACHE_MAX_ABS, f"{what}: max_abs={max_abs:.3e}"
    return max_abs
