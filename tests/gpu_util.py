"""Shared helpers for the GPU parity tests (comparisons against the oracle)."""
import numpy as np
import torch

# Attention outputs (bf16 in, fp32 accumulate) against the fp64 oracle.
MAX_ABS_TOL = 2e-2
MEAN_ABS_TOL = 2e-3
# LSE (fp32 log-sum-exp of up to 256K terms) against fp64.
LSE_ABS_TOL = 2e-3


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close_attention(got: np.ndarray, ref: np.ndarray, what: str):
    err = np.abs(got - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert np.all(np.isfinite(got)), "%s: non-finite output" % what
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (
        "%s: max-abs %.3g (tol %.1g), mean-abs %.3g (tol %.1g)"
        % (what, mx, MAX_ABS_TOL, mean, MEAN_ABS_TOL))
    return mx, mean


def zero_status(device="cuda"):
    return torch.zeros(1, dtype=torch.int32, device=device)
