"""Error metric and helpers shared by the GPU parity tests.

Tolerance metric (the reading of "max relative error" used throughout): for each
(b, h) slice, max |x - x_ref| / max |x_ref| over the slice (y: all t and channels;
a state or snapshot: all i, j); the reported error is the max over slices.
Bounds: 2e-3 for bf16 inputs, 1e-5 for fp32 inputs (fp32 state throughout).
"""
import numpy as np
import torch

TOL = {"bf16": 2e-3, "f32": 1e-5}


def as_np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def slice_rel_err(got, ref, slice_axes):
    """Max over slices of max|got-ref| / max|ref|; slice_axes index the slice (e.g. (0, 2))."""
    got, ref = as_np(got), as_np(ref)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    red = tuple(i for i in range(ref.ndim) if i not in slice_axes)
    num = np.max(np.abs(got - ref), axis=red)
    den = np.maximum(np.max(np.abs(ref), axis=red), 1e-30)
    if not np.all(np.isfinite(got)):
        return float("inf")
    return float(np.max(num / den))


def y_err(got, ref):       # [B, T, H, N]
    return slice_rel_err(got, ref, (0, 2))


def state_err(got, ref):   # [B, H, N, N]
    return slice_rel_err(got, ref, (0, 1))


def snaps_err(got, ref):   # [B, M, H, N, N]
    return slice_rel_err(got, ref, (0, 1, 2))


def heads_slice(d, pairs):
    """Sub-batch of the sampled (b, h) pairs: token tensors -> [len, T, 1, N], S0 -> [len, 1, N, N]."""
    out = {}
    for name in ("r", "w", "k", "v", "kk", "a"):
        out[name] = torch.stack([d[name][b, :, h] for b, h in pairs])[:, :, None, :]
    out["S0"] = None if d.get("S0") is None else torch.stack([d["S0"][b, h] for b, h in pairs])[:, None]
    return out
