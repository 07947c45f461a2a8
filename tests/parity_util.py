"""Helpers for GPU-vs-oracle parity tests: tolerances and conversions."""
import numpy as np
import torch

# Tolerances the hot path is held to (bf16 outputs with fp32 accumulation).
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 1e-3
# A tighter check on top: the error of each output row relative to the row's
# largest magnitude. bf16 rounding alone is below 2^-8 of it. The small absolute
# floor covers rows that average ~1e6 random values (|o| ~ 1e-4), where fp32
# summation error, not rounding of the output, sets the error.
ROW_REL = 1e-2
ROW_FLOOR = 2e-5


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def check_rows(o_gpu: np.ndarray, o_ref: np.ndarray, lse_gpu=None, lse_ref=None, what=""):
    """o_*: [..., d]; lse_*: matching [...] (or None)."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (what, o_gpu.shape, o_ref.shape)
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    max_abs, mean_abs = float(err.max()), float(err.mean())
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e}"
    assert mean_abs <= MEAN_ABS, f"{what}: mean-abs {mean_abs:.3e}"
    scale = np.abs(o_ref).max(axis=-1, keepdims=True) + ROW_FLOOR / ROW_REL
    rel = float((err / scale).max())
    assert rel <= ROW_REL, f"{what}: row-relative error {rel:.3e}"
    if lse_gpu is not None:
        lg = np.asarray(lse_gpu, dtype=np.float64)
        lr = np.asarray(lse_ref, dtype=np.float64)
        assert lg.shape == lr.shape, (what, lg.shape, lr.shape)
        lerr = float(np.abs(lg - lr).max())
        assert lerr <= LSE_ABS, f"{what}: lse max-abs {lerr:.3e}"
    return max_abs, mean_abs
