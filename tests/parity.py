"""Comparison helpers for CUDA-vs-oracle parity tests.

Error metric (per tensor): max_i |x_i - r_i| / max_i |r_i|, the maximum error
normalised by the tensor's largest reference magnitude.  Bars: 1e-4 on the
float32 path, 2e-2 on the bf16-in / float32-accumulate path."""
from __future__ import annotations

import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def np64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def max_rel_err(x, ref) -> float:
    x, ref = np64(x), np64(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    scale = float(np.max(np.abs(ref)))
    err = float(np.max(np.abs(x - ref)))
    if not np.isfinite(err):
        return float("inf")
    return err / scale if scale > 0 else err


def assert_close(x, ref, tol, what):
    e = max_rel_err(x, ref)
    assert e <= tol, f"{what}: max rel err {e:.3e} > {tol:.1e}"
    return e
