"""Per-segment steps of the sequence-parallel forward computed by the fp64 oracle (CPU),
so the orchestration in chunked_linear_attention_chunk_b200.sp can be run by gloo ranks
without a GPU.  The transfer map M of a segment is the oracle's recurrence run from the
identity with v = 0 (the write term vanishes, leaving the product of the per-token maps)."""
from __future__ import annotations

import numpy as np
import torch

import oracle

NAMES = ("q", "k", "v", "a", "beta")


def _np(t):
    return t.detach().to(torch.float32).numpy()


class OracleSegmentOps:
    def __init__(self, g_min: float = -5.0):
        self.g_min = g_min

    def maps(self, q, k, v, a, beta):
        x = [_np(t) for t in (q, k, v, a, beta)]
        B, T, H, dk = x[0].shape
        _, S_zero = oracle.recurrence(*x, self.g_min)
        eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
        _, M = oracle.recurrence(x[0], x[1], np.zeros_like(x[2]), x[3], x[4], self.g_min, S0=eye)
        return x, torch.from_numpy(S_zero), torch.from_numpy(M)

    def combine(self, M, S_zero, S0):
        R = M.shape[0]
        S = torch.zeros_like(S_zero[0]) if S0 is None else S0.to(torch.float64)
        out = [S]
        for r in range(R):
            S = torch.einsum("bhik,bhkj->bhij", M[r], S) + S_zero[r]
            out.append(S)
        return torch.stack(out)

    def forward(self, x, S_in):
        o, S_T = oracle.recurrence(*x, self.g_min, S0=S_in.numpy())
        return torch.from_numpy(o), torch.from_numpy(S_T)

    def backward(self, tokens, S_in, dO, dS_T):
        x = [_np(t) for t in tokens]
        r = oracle.backward(*x, _np(dO), self.g_min, S0=S_in.numpy(),
                            dST=None if dS_T is None else dS_T.to(torch.float64).numpy())
        return {n: torch.from_numpy(v) for n, v in r.items()}
