"""Comparison helpers for CUDA-vs-oracle parity tests.

Error metric (per tensor): max_i |x_i - r_i| / max_i |r_i|, the maximum error
normalised by the tensor's largest reference magnitude.  Bars: 1e-4 on the
float32 path, 2e-2 on the bf16-in / float32-accumulate path.

Beside the bar every comparison also computes an element-wise diagnostic,
max_i |x_i - r_i| / (|r_i| + 1e-3 * rms(r)): the worst error of one element
relative to that element's own magnitude (with a floor of a thousandth of the
tensor's rms so that exact zeros do not divide by zero).  It is reported, not
enforced: small entries of a gradient can carry a large relative error while
the tensor as a whole meets its bar, and this figure makes that visible."""
from __future__ import annotations

import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}

# every comparison made in this process: (what, max rel err, element-wise diagnostic)
REPORT: list = []


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


def elementwise_err(x, ref) -> float:
    """max_i |x_i - r_i| / (|r_i| + 1e-3 * rms(r))."""
    x, ref = np64(x), np64(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    floor = 1e-3 * rms if rms > 0 else 1e-30
    e = np.abs(x - ref) / (np.abs(ref) + floor)
    m = float(np.max(e))
    return m if np.isfinite(m) else float("inf")


def assert_close(x, ref, tol, what):
    e = max_rel_err(x, ref)
    d = elementwise_err(x, ref)
    REPORT.append((what, e, d))
    assert e <= tol, f"{what}: max rel err {e:.3e} > {tol:.1e} (element-wise {d:.3e})"
    return e
