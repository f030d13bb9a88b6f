"""Helpers for the GPU parity tests (comparison only; no attention math)."""
import numpy as np
import torch

BF16_TOL = 2e-2   # max abs error, bf16 inputs/outputs with fp32 accumulation
F32_TOL = 1e-5    # max abs error, fp32 path


def dev():
    return torch.device("cuda:0")


def to_np(t):
    return t.detach().float().cpu().double().numpy()


def max_err(got, ref):
    got = to_np(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "non-finite output"
    return float(np.abs(got - ref).max()) if got.size else 0.0


def tol_for(dtype):
    return BF16_TOL if dtype == torch.bfloat16 else F32_TOL


def poison_unfilled(k_cache, v_cache, filled):
    """Set to NaN every ring slot a sequence has not reached yet: slots
    filled[b] .. W-1 of row b (CPU tensors, in place).  A reader that touches
    one of them, even to mask it afterwards, turns its output into NaN."""
    W = k_cache.shape[2]
    for b, n in enumerate(int(x) for x in filled):
        if n < W:
            k_cache[b, :, n:] = float("nan")
            v_cache[b, :, n:] = float("nan")
