"""Sequence-parallel pieces on the GPU: the segment maps (S_zero, M), the prefix combine,
and the whole path with segments emulated on one GPU (the exchange is a list), against
the fp64 oracle run over the whole sequence.  Tolerances are the bf16 path's."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import synth
from chunked_linear_attention_chunk_b200.sp import LibkdaSegmentOps, sp_chunk_fwd
from helpers import G_MIN, NAMES, TOL_BF16_O, TOL_BF16_S, err_o, err_s, oracle_run, to_dev

pytestmark = pytest.mark.gpu


def test_combine_matches_fp64_prefix():
    gen = torch.Generator().manual_seed(5)
    R, B, H, D = 4, 2, 3, 128
    M = torch.randn(R, B, H, D, D, generator=gen) / D ** 0.5
    Z = torch.randn(R, B, H, D, D, generator=gen)
    S0 = torch.randn(B, H, D, D, generator=gen)
    S_in = kda.kda_state_combine(M.cuda(), Z.cuda(), S0.cuda()).cpu().double()
    S = S0.double()
    assert torch.equal(S_in[0], S)
    for r in range(R):
        S = M[r].double() @ S + Z[r].double()
        assert torch.allclose(S_in[r + 1], S, rtol=1e-4, atol=1e-4), r


@pytest.mark.parametrize("D", [64, 128])
def test_segment_maps_against_oracle(D):
    """S_zero is the run from a zero state; M S_in + S_zero is the run from any S_in."""
    B, T, H = 1, 150, 2
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=1400 + D, s0_std=0.3)
    d = to_dev(x)
    _, S_zero, M = LibkdaSegmentOps(G_MIN).maps(*(d[n] for n in NAMES))
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    _, S_ref0 = oracle_run(x, None)
    assert err_s(S_zero.cpu().numpy(), S_ref0) <= TOL_BF16_S
    _, S_refX = oracle_run(x, x["S0"])
    S_aff = torch.einsum("bhik,bhkj->bhij", M.double().cpu(), x["S0"].double()) + S_zero.double().cpu()
    assert err_s(S_aff.numpy(), S_refX) <= TOL_BF16_S


def test_three_segments_on_one_gpu_match_one_run():
    B, T, H, D = 1, 400, 2, 128
    cut = [0, 130, 131, 400]  # a one-token segment in the middle
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=1410, s0_std=0.1)
    d = to_dev(x)
    ops = LibkdaSegmentOps(G_MIN)
    # beta slices at odd token offsets are 2-byte aligned only, which the library accepts
    parts = [ops.maps(*(d[n][:, cut[r]:cut[r + 1]] for n in NAMES)) for r in range(3)]
    S_in = ops.combine(torch.stack([p[2] for p in parts]), torch.stack([p[1] for p in parts]), d["S0"])
    o = torch.cat([ops.forward(parts[r][0], S_in[r])[0] for r in range(3)], dim=1)
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    o_ref, S_ref = oracle_run(x, x["S0"])
    eo, es = err_o(o.float().cpu().numpy(), o_ref), err_s(S_in[3].cpu().numpy(), S_ref)
    assert eo <= TOL_BF16_O and es <= TOL_BF16_S, (eo, es)


def test_sp_entry_with_a_real_process_group():
    """World size 1 over NCCL: the segment is the whole sequence; o equals kda_chunk_fwd."""
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        x = to_dev(synth.make_inputs(1, 200, 2, 128, 128, "bf16", seed=1420, s0_std=0.1))
        o, S_T = sp_chunk_fwd(*(x[n] for n in NAMES), S0=x["S0"])
        o1, S1 = kda.kda_chunk_fwd(*(x[n] for n in NAMES), G_MIN, S0=x["S0"])
        torch.cuda.synchronize()
        assert torch.equal(o, o1)
        assert err_s(S_T.cpu().numpy(), S1.cpu().numpy().astype(np.float64)) <= TOL_BF16_S
    finally:
        dist.destroy_process_group()


class ThreadComm:
    """The exchange of R ranks emulated by R host threads of one process on one GPU: every
    rank's library calls are ordinary launches (no kernel waits on another rank), and the
    all-gather / all-reduce are host barriers after a device synchronisation, so the ranks'
    tensors are complete when another thread reads them."""

    def __init__(self, world, rank, shared):
        self.world, self.rank, self.shared = world, rank, shared

    def _exchange(self, x):
        torch.cuda.synchronize()
        sh = self.shared
        sh["slots"][self.rank] = x
        sh["barrier"].wait()
        got = list(sh["slots"])
        sh["barrier"].wait()  # every rank has read the slots before they are reused
        return got

    def all_gather(self, x):
        return [t.clone() for t in self._exchange(x.contiguous())]

    def all_reduce_(self, x):
        total = sum(t.double() for t in self._exchange(x.clone()))
        x.copy_(total.to(x.dtype))
        return x


def _run_ranks(world, fn):
    import threading
    shared = {"slots": [None] * world, "barrier": threading.Barrier(world, timeout=120)}
    out, errs = [None] * world, []

    def body(r):
        try:
            out[r] = fn(ThreadComm(world, r, shared), r)
        except BaseException as e:  # noqa: BLE001 -- reported below
            errs.append(e)
            shared["barrier"].abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    if errs:
        raise errs[0]
    return out


def test_sp_backward_three_segments_on_one_gpu_match_the_oracle():
    """sp_chunk_bwd itself, with three ranks emulated by threads on one GPU (segments of 130,
    1 and 269 tokens, so one rank holds a single token), against the fp64 oracle's backward
    over the whole sequence: every token gradient, dS0 and the per-head dA_log summed over
    the ranks (the gate with a per-head scale, checked through the chain rule)."""
    import oracle
    from chunked_linear_attention_chunk_b200.sp import sp_chunk_bwd

    B, T, H, D = 1, 400, 2, 128
    cut = [0, 130, 131, 400]
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=1430, s0_std=0.1)
    gen = torch.Generator().manual_seed(1431)
    dO = torch.randn((B, T, H, D), generator=gen).to(torch.bfloat16)
    dST = torch.randn((B, H, D, D), generator=gen) * 0.5
    A_log = torch.tensor([0.3, -0.4])
    d = to_dev(x)
    dO_d, dST_d, A_d = dO.cuda(), dST.cuda(), A_log.cuda()
    ops = LibkdaSegmentOps(G_MIN, A_log=A_d)

    def rank_fn(comm, r):
        seg = [d[n][:, cut[r]:cut[r + 1]].contiguous() for n in NAMES]
        return sp_chunk_bwd(*seg, dO_d[:, cut[r]:cut[r + 1]].contiguous(), S0=d["S0"], dS_T=dST_d, ops=ops,
                            comm=comm)

    gs = _run_ranks(3, rank_fn)
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    # oracle: the bounded gate of x = e^{A_h} a, then the chain rule for da and dA_log
    scale = torch.exp(A_log).view(1, 1, H, 1)
    xs = {n: synth.to_numpy32(x[n]) for n in NAMES}
    xa = (x["a"].float() * scale).numpy()
    ref = oracle.backward(xs["q"], xs["k"], xs["v"], xa, xs["beta"], synth.to_numpy32(dO), G_MIN,
                          S0=x["S0"].numpy().astype(np.float64), dST=dST.numpy().astype(np.float64))
    ref_da = ref["da"] * scale.numpy()
    got = {n: torch.cat([g[n] for g in gs], dim=1).cpu().numpy() for n in ("dq", "dk", "dv", "da", "dbeta")}
    want = {"dq": ref["dq"], "dk": ref["dk"], "dv": ref["dv"], "da": ref_da, "dbeta": ref["dbeta"]}
    for n in got:
        e = err_o(got[n], want[n]) if got[n].ndim == 4 else \
            float(np.max(np.abs(got[n] - want[n])) / np.max(np.abs(want[n])))
        assert e <= 2e-2, (n, e)
    for g in gs:  # dS0 is the same on every rank
        assert err_s(g["dS0"].cpu().numpy(), ref["dS0"]) <= 2e-2
    # dL/dA_h = sum over the head's tokens and channels of dL/dx * x, summed over the ranks
    dx = ref["da"]
    dA_ref = np.einsum("bthc,bthc->h", dx, xa.astype(np.float64))
    scale_ref = np.einsum("bthc->h", np.abs(dx * xa))
    for g in gs:
        assert np.all(np.abs(g["dA_log"].cpu().numpy() - dA_ref) <= 2e-2 * scale_ref), (g["dA_log"], dA_ref)
