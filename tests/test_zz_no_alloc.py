"""kda_chunk_fwd_noalloc: the chunked forward for callers that cannot allocate device
memory (graph capture, allocation-free serving loops, memory owned by another
allocator).  It must give the same o and S_T as kda_chunk_fwd with a caller workspace,
call after call, on the same inputs.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import synth
from helpers import G_MIN, NAMES, TOL_BF16_O, TOL_BF16_S, err_o, err_s

pytestmark = pytest.mark.gpu


def _inputs(B, T, H, seed):
    x = synth.make_inputs(B, T, H, 128, 128, "bf16", seed=seed, s0_std=0.1)
    return {n: t.cuda() for n, t in x.items()}


def _compare(x, S0):
    o_ref, S_ref = kda.kda_chunk_fwd(*(x[n] for n in NAMES), G_MIN, S0=S0)
    o, S_T = kda.kda_chunk_fwd_noalloc(*(x[n] for n in NAMES), G_MIN, S0=S0)
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    eo = err_o(o.float().cpu().numpy(), o_ref.float().cpu().numpy())
    es = err_s(S_T.cpu().numpy(), S_ref.cpu().numpy())
    assert eo <= TOL_BF16_O and es <= TOL_BF16_S, (eo, es)
    return o, S_T


def test_noalloc_matches_workspace_path_two_calls():
    """32 heads: the 64 MiB scratch holds 20 chunks, so T = 3000 runs as three stretches
    per batch element; two calls in a row, the second continuing from the first's state."""
    x1 = _inputs(2, 3000, 32, seed=900)
    o1, S1 = _compare(x1, x1["S0"])
    x2 = _inputs(2, 1000, 32, seed=901)
    _compare(x2, S1)


def test_noalloc_without_state_output_and_small_problem():
    x = _inputs(1, 333, 4, seed=902)
    o_ref, _ = kda.kda_chunk_fwd(*(x[n] for n in NAMES), G_MIN, S0=None)
    o, S_T = kda.kda_chunk_fwd_noalloc(*(x[n] for n in NAMES), G_MIN, S0=None, return_state=False)
    torch.cuda.synchronize()
    assert S_T is None
    assert err_o(o.float().cpu().numpy(), o_ref.float().cpu().numpy()) <= TOL_BF16_O


def test_noalloc_rejects_problems_beyond_the_scratch():
    """One chunk of every head must fit the fixed scratch; 1024 heads of 128 x 128 do not."""
    assert kda.lib().kda_chunk_fwd_noalloc_max_scratch() == 64 << 20
    x = _inputs(1, 64, 1024, seed=903)
    with pytest.raises(kda.KdaError) as e:
        kda.kda_chunk_fwd_noalloc(*(x[n] for n in NAMES), G_MIN, S0=None)
    assert e.value.status == 7  # KDA_ERR_WORKSPACE
