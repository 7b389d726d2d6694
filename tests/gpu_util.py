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


# Gradients (bf16 inputs, P and dS rounded to bf16 before their MMAs, fp32
# accumulation, bf16 outputs) against the fp64 chain rule: each element is a
# sum of products with one factor carrying a bf16 rounding error (relative
# 2^-9) and the result is rounded once more, so the error scales with the
# tensor's own magnitude.  Bounds relative to the reference's scale:
GRAD_MAX_REL = 2e-2     # max |err| / max |ref|
GRAD_MEAN_REL = 1e-2    # mean |err| / mean |ref|


def assert_close_grad(got: np.ndarray, ref: np.ndarray, what: str):
    err = np.abs(got - ref)
    mref, aref = max(float(np.abs(ref).max()), 1e-6), max(float(np.abs(ref).mean()), 1e-9)
    mx, mean = float(err.max()) / mref, float(err.mean()) / aref
    assert np.all(np.isfinite(got)), "%s: non-finite output" % what
    print("%s: max-rel %.3g mean-rel %.3g (max|ref| %.3g mean|ref| %.3g)"
          % (what, mx, mean, mref, aref))
    assert mx <= GRAD_MAX_REL and mean <= GRAD_MEAN_REL, (
        "%s: max-abs/max|ref| %.3g (tol %.1g), mean-abs/mean|ref| %.3g (tol %.1g)"
        % (what, mx, GRAD_MAX_REL, mean, GRAD_MEAN_REL))
    return mx, mean
