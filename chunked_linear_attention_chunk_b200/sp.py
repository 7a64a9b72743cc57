"""Sequence-parallel chunked forward: one long sequence split into consecutive segments,
one per rank ("Breaking Through ..." section 3 splits the million-token sequences across
GPUs).

Over a segment the state map is affine, S_out = M S_in + S_zero.  Every rank
  1. preps its segment and computes its own (S_zero, M)          -- local, libkda,
  2. all-gathers (S_zero, M) from every rank                      -- the one exchange,
  3. forms every segment's incoming state by the prefix
     S_in[r + 1] = M[r] S_in[r] + S_zero[r]                        -- libkda,
  4. scans its segment again from S_in[rank] and writes o         -- libkda.
The exchanged maps are tiny next to the tokens (2 d^2 floats per head per rank), so a
plain NCCL all-gather over NVLink is the whole collective.

The per-segment steps are an object with three methods, so the same orchestration runs
with the CUDA library (``LibkdaSegmentOps``) or, in CPU tests, with any other
implementation of the steps.  This module holds no arithmetic of the method.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

import chunked_linear_attention_chunk_b200 as kda


class LibkdaSegmentOps:
    """The per-segment steps on this rank's GPU, through libkda (bf16 tokens)."""

    def __init__(self, g_min: float = -5.0, A_log=None, gate: int = kda.KDA_GATE_BOUNDED):
        self.g_min, self.A_log, self.gate = g_min, A_log, gate

    def maps(self, q, k, v, a, beta):
        """Prep the segment; returns (handle, S_zero, M)."""
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        ws = torch.empty(kda.kda_chunk_fwd_workspace(B, T, H, dk, dv), dtype=torch.uint8, device=q.device)
        kda.kda_chunk_fwd_prep(q, k, v, a, beta, ws, self.g_min, self.gate, A_log=self.A_log)
        S_zero, M = kda.kda_chunk_fwd_scan_affine(ws, B, T, H, dk, dv)
        return (ws, (B, T, H, dk, dv)), S_zero, M

    def combine(self, M, S_zero, S0):
        return kda.kda_state_combine(M.contiguous(), S_zero.contiguous(), S0)

    def forward(self, handle, S_in):
        ws, (B, T, H, dk, dv) = handle
        return kda.kda_chunk_fwd_scan(ws, B, T, H, dk, dv, S0=S_in.contiguous())


def sp_chunk_fwd(q, k, v, a, beta, S0=None, group=None, ops=None):
    """This rank's segment of a sequence-parallel chunked forward.

    q, k, a [B, T_r, H, dk]; v [B, T_r, H, dv]; beta [B, T_r, H]: the segment of every
    batch sequence this rank holds; rank r holds the r-th segment in sequence order
    (segments may differ in length).  S0 [B, H, dk, dv] is the sequence's initial state,
    the same on every rank (or None for zeros).  Returns (o for this segment, the whole
    sequence's final state), the latter identical on every rank."""
    ops = ops if ops is not None else LibkdaSegmentOps()
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    handle, S_zero, M = ops.maps(q, k, v, a, beta)
    if world > 1:
        Zs = [torch.empty_like(S_zero) for _ in range(world)]
        Ms = [torch.empty_like(M) for _ in range(world)]
        dist.all_gather(Zs, S_zero.contiguous(), group=group)
        dist.all_gather(Ms, M.contiguous(), group=group)
    else:
        Zs, Ms = [S_zero], [M]
    S_in = ops.combine(torch.stack(Ms), torch.stack(Zs), S0)
    o, _ = ops.forward(handle, S_in[rank])
    return o, S_in[world]
