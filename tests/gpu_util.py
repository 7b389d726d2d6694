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


# ------------------------------------------------------------- canaries
# The sanitizer's out-of-bounds checks are not available here, so the
# kernels' writes are fenced by sentinels instead: an output (or workspace)
# is a view into a larger buffer whose head and tail hold a sentinel bit
# pattern, and the output itself starts as NaN.  After the call the head and
# tail must hold the sentinel still (no write past either end) and every
# output element must be finite (no element left unwritten).
_SENTINEL = {torch.bfloat16: (torch.int16, 0x7FA5),           # a NaN bit pattern
             torch.float32: (torch.int32, 0x7FC0A5A5),        # a NaN bit pattern
             torch.uint8: (torch.uint8, 0xA5)}


class Guarded:
    def __init__(self, shape, dtype, pad=4096, device="cuda"):
        n = 1
        for s in shape:
            n *= int(s)
        self.n, self.pad = n, pad
        self.buf = torch.empty(n + 2 * pad, dtype=dtype, device=device)
        view_dtype, pattern = _SENTINEL[dtype]
        self.buf.view(view_dtype).fill_(pattern)
        self.t = self.buf[pad:pad + n].view(*shape)
        self._pattern = self.buf.view(view_dtype)[:pad].clone()

    def check_fences(self, what):
        vd = self._pattern.dtype
        head = self.buf.view(vd)[:self.pad]
        tail = self.buf.view(vd)[self.pad + self.n:]
        assert torch.equal(head, self._pattern), "%s: write before the start" % what
        assert torch.equal(tail, self._pattern), "%s: write past the end" % what

    def check_all_written(self, what):
        self.check_fences(what)
        assert bool(torch.isfinite(self.t.float()).all()), "%s: element left unwritten" % what
