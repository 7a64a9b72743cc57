"""Shared helpers of the GPU parity tests: error metrics and oracle/GPU runners.

The error metric is normwise per (batch, head): max|x - y| / max|y| over that head's
block of the tensor, worst case over heads.  Elementwise relative error is ill-posed
near zero; a per-head normwise figure is the strictest well-posed reading of "max
relative error".
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from chunked_linear_attention_chunk_b200 import synth

G_MIN = -5.0
TOL_BF16_O = 2e-2
TOL_BF16_S = 1e-2
TOL_F32 = 1e-4


def err_o(x, y):
    """x, y: [B, T, H, dv] -> worst per-(b, h) normwise relative error."""
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    num = np.max(np.abs(x - y), axis=(1, 3))
    den = np.maximum(np.max(np.abs(y), axis=(1, 3)), 1e-30)
    return float(np.max(num / den))


def err_s(x, y):
    """x, y: [B, H, dk, dv] -> worst per-(b, h) normwise relative error."""
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    num = np.max(np.abs(x - y), axis=(2, 3))
    den = np.maximum(np.max(np.abs(y), axis=(2, 3)), 1e-30)
    return float(np.max(num / den))


NAMES = ("q", "k", "v", "a", "beta")


def oracle_run(x, S0=None, g_min=G_MIN, heads=None, kind=oracle.GATE_BOUNDED):
    """Run the fp64 oracle recurrence on CPU inputs ``x`` (dict of tensors).  ``heads``
    restricts the run to a list of head indices (all batches)."""
    arrs = {n: synth.to_numpy32(x[n]) for n in NAMES}
    s0 = None if S0 is None else np.asarray(S0.cpu() if torch.is_tensor(S0) else S0, np.float64)
    if heads is not None:
        arrs = {n: np.ascontiguousarray(v[:, :, heads]) for n, v in arrs.items()}
        if s0 is not None:
            s0 = np.ascontiguousarray(s0[:, heads])
    return oracle.recurrence(*(arrs[n] for n in NAMES), g_min, S0=s0, kind=kind)


def to_dev(x, device="cuda"):
    return {n: (t.to(device) if torch.is_tensor(t) else t) for n, t in x.items()}
