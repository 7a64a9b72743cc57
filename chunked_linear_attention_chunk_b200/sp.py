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

The backward (``sp_chunk_bwd``) runs on the same maps.  The gradient of a segment's
incoming state is affine in the gradient of its outgoing one, dS_in = M^T dS_out + dZ, where
dZ is the segment's backward from a zero outgoing gradient.  Every rank
  1. forms its incoming state as in the forward (maps, all-gather, prefix),
  2. runs its segment's backward from a zero outgoing gradient and keeps dZ   -- libkda,
  3. all-gathers dZ                                                            -- exchange,
  4. forms every segment's outgoing gradient by the suffix
     dS_out[r] = M[r+1]^T dS_out[r+1] + dZ[r+1], dS_out[R-1] = dS_T           -- libkda,
  5. runs its segment's backward again with dS_out[rank]: the token gradients -- libkda.

The per-segment steps are an object with a few methods, so the same orchestration runs with
the CUDA library (``LibkdaSegmentOps``) or, in CPU tests, with any other implementation of
the steps.  This module holds no arithmetic of the method.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

import chunked_linear_attention_chunk_b200 as kda


class DistComm:
    """The exchange steps over torch.distributed (the default): all-gather and all-reduce in
    ``group``; a single process without a process group is world 1."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0

    def all_gather(self, x):
        if self.world == 1:
            return [x]
        xs = [torch.empty_like(x) for _ in range(self.world)]
        dist.all_gather(xs, x.contiguous(), group=self.group)
        return xs

    def all_reduce_(self, x):
        if self.world > 1:
            dist.all_reduce(x, group=self.group)
        return x


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

    def backward(self, tokens, S_in, dO, dS_T):
        """The segment's gradients (dict of kda_chunk_bwd) from S_in, given dO and dS_T."""
        if self.gate != kda.KDA_GATE_BOUNDED:
            raise ValueError("the backward supports the bounded gate only")
        return kda.kda_chunk_bwd(*tokens, dO, self.g_min, S0=S_in.contiguous(),
                                 dS_T=None if dS_T is None else dS_T.contiguous(), A_log=self.A_log)


def sp_chunk_fwd(q, k, v, a, beta, S0=None, group=None, ops=None, comm=None):
    """This rank's segment of a sequence-parallel chunked forward.

    q, k, a [B, T_r, H, dk]; v [B, T_r, H, dv]; beta [B, T_r, H]: the segment of every
    batch sequence this rank holds; rank r holds the r-th segment in sequence order
    (segments may differ in length).  S0 [B, H, dk, dv] is the sequence's initial state,
    the same on every rank (or None for zeros).  Returns (o for this segment, the whole
    sequence's final state), the latter identical on every rank.  ``comm`` replaces the
    torch.distributed exchange (``DistComm(group)``) with another one of the same methods."""
    ops = ops if ops is not None else LibkdaSegmentOps()
    comm = comm if comm is not None else DistComm(group)
    handle, S_zero, M = ops.maps(q, k, v, a, beta)
    Zs, Ms = comm.all_gather(S_zero), comm.all_gather(M)
    S_in = ops.combine(torch.stack(Ms), torch.stack(Zs), S0)
    o, _ = ops.forward(handle, S_in[comm.rank])
    return o, S_in[comm.world]


def sp_chunk_bwd(q, k, v, a, beta, dO, S0=None, dS_T=None, group=None, ops=None, comm=None):
    """This rank's segment of a sequence-parallel backward (the segments as in
    ``sp_chunk_fwd``; dO is this segment's dL/do, dS_T the gradient of the whole sequence's
    final state, the same on every rank, or None).  Returns the ``kda_chunk_bwd`` dict of
    this segment's token gradients, with dS0 the gradient of the sequence's initial state
    (identical on every rank) and, given A_log, dA_log summed over all segments."""
    ops = ops if ops is not None else LibkdaSegmentOps()
    comm = comm if comm is not None else DistComm(group)
    world, rank = comm.world, comm.rank
    tokens = (q, k, v, a, beta)
    _, S_zero, M = ops.maps(*tokens)
    Ms = comm.all_gather(M)
    S_in = ops.combine(torch.stack(Ms), torch.stack(comm.all_gather(S_zero)), S0)
    dZ = ops.backward(tokens, S_in[rank], dO, None)["dS0"]
    dZs = comm.all_gather(dZ)
    # suffix over the segments in reverse order: X[j + 1] = M[R-1-j]^T X[j] + dZ[R-1-j], X[0] = dS_T
    Mt = torch.stack([Ms[world - 1 - j].transpose(-1, -2) for j in range(world)])
    X = ops.combine(Mt, torch.stack([dZs[world - 1 - j] for j in range(world)]), dS_T)
    g = ops.backward(tokens, S_in[rank], dO, X[world - 1 - rank])
    g["dS0"] = X[world]
    if g.get("dA_log") is not None:
        comm.all_reduce_(g["dA_log"])
    return g
