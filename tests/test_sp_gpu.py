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
