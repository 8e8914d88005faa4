"""Shared test helpers: the tolerance metric and device read-back."""

from __future__ import annotations

import numpy as np


def rel_err(g, r) -> float:
    """max_i |g_i - r_i| / max(|r_i|, rms(r)): the per-element relative error
    with an RMS floor, so that values near zero do not dominate."""
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    if r.size == 0:
        return 0.0
    floor = max(float(np.sqrt((r * r).mean())), 1e-300)
    return float((np.abs(g - r) / np.maximum(np.abs(r), floor)).max())


def norm_err(g, r) -> float:
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    return float(np.abs(g - r).max() / max(np.abs(r).max(), 1e-300))


# Tolerances (max relative error, metric above): fp32 outputs 1e-3, bf16
# outputs 2e-2.
TOL_F32 = 1e-3
TOL_BF16 = 2e-2


def ws_array(torch, ws, offset: int, dtype, shape):
    """numpy copy of a typed region of a device workspace."""
    n = int(np.prod(shape))
    itemsize = torch.empty((), dtype=dtype).element_size()
    start = ws.addr - ws.buf.data_ptr() + offset
    t = ws.buf[start:start + n * itemsize].view(dtype).reshape(shape)
    if dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy()


def to_np(t):
    import torch
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()
