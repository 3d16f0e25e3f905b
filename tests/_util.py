"""Shared helpers of the test suite: tolerances and device transfers."""
import numpy as np
import torch


def close_rel_rms(g, o, tol):
    """|g - o| <= tol * (|o| + rms(o)) element-wise (per-tensor scale floor).

    The pages give no tolerance; this is the layer's stated 2e-2 (outputs) /
    3e-2 (gradients) read as relative to the element with the tensor's RMS as
    the floor, so that values near zero are not held to a pure relative test.
    Returns (ok, worst_ratio)."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    rms = float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    bound = tol * (np.abs(o) + rms)
    err = np.abs(g - o)
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if o.size else 0.0
    return bool(np.all(err <= bound)), ratio


def close_scores(g, o, tol=1e-5):
    """fp32 score tolerance: |g - o| <= tol * max(|o|, rms(o))."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    rms = float(np.sqrt(np.mean(o * o)))
    bound = tol * np.maximum(np.abs(o), rms)
    err = np.abs(g - o)
    return bool(np.all(err <= bound)), float(np.max(err / bound))


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def dev(x, dtype=None):
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        x = x.to(dtype)
    return x.contiguous().cuda()
