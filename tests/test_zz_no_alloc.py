"""kda_chunk_fwd_noalloc: the chunked forward for callers that cannot allocate device
memory -- code running under CUDA graph capture, serving loops that must never call
cudaMalloc, hosts whose device memory belongs to another allocator.  It runs the same
kernels as kda_chunk_fwd over stretches of whole 64-token chunks with the float32 state
carried between them, so its o and S_T must equal kda_chunk_fwd's bit for bit, call after
call.  This file is collected last on purpose: a failure here leaves every other test run."""
import pytest
import torch

import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import synth
from helpers import G_MIN, NAMES

pytestmark = pytest.mark.gpu


def _inputs(B, T, H, seed, d=128, dtype="bf16"):
    x = synth.make_inputs(B, T, H, d, d, dtype, seed=seed, s0_std=0.1)
    return {n: t.cuda() for n, t in x.items()}


def _same(x, S0, return_state=True):
    """kda_chunk_fwd (caller workspace) and kda_chunk_fwd_noalloc on the same stream and
    inputs: o and S_T must be bitwise equal."""
    o_ref, S_ref = kda.kda_chunk_fwd(*(x[n] for n in NAMES), G_MIN, S0=S0, return_state=return_state)
    o, S_T = kda.kda_chunk_fwd_noalloc(*(x[n] for n in NAMES), G_MIN, S0=S0, return_state=return_state)
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    assert torch.equal(o, o_ref)
    if return_state:
        assert torch.equal(S_T, S_ref)
    else:
        assert S_T is None
    return o, S_T


def test_noalloc_equals_workspace_path_two_calls():
    """32 heads at d = 128: the 64 MiB scratch holds 20 chunks of every head, so T = 3000
    runs as three stretches per batch element; two calls in a row, the second continuing
    from the first's state."""
    x1 = _inputs(2, 3000, 32, seed=900)
    _, S1 = _same(x1, x1["S0"])
    x2 = _inputs(2, 1000, 32, seed=901)
    _same(x2, S1)


def test_noalloc_without_state_output_reuses_the_carry_slot():
    """No S_T: the state between stretches goes through the library's carry slot, which
    every batch element reuses; three batch elements of three stretches each."""
    x = _inputs(3, 2600, 32, seed=904)
    _same(x, x["S0"], return_state=False)
    _same(x, None, return_state=False)


def test_noalloc_state_in_place():
    """S_T given as S0 itself (in-place carry) over several stretches."""
    x = _inputs(2, 2000, 32, seed=905)
    o_ref, S_ref = kda.kda_chunk_fwd(*(x[n] for n in NAMES), G_MIN, S0=x["S0"])
    S = x["S0"].clone()
    o, S_T = kda.kda_chunk_fwd_noalloc(*(x[n] for n in NAMES), G_MIN, S0=S, S_T=S)
    torch.cuda.synchronize()
    assert S_T.data_ptr() == S.data_ptr()
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


def test_noalloc_head_dim_64_and_small_problem():
    x = _inputs(2, 5000, 80, seed=906, d=64)  # 80 heads of 64 x 64 records: four stretches
    _same(x, x["S0"])
    y = _inputs(1, 333, 4, seed=902)
    _same(y, None, return_state=False)


def test_noalloc_float32_passes_through():
    """The float32 path needs no scratch; it is the same call."""
    x = _inputs(1, 200, 2, seed=907, d=64, dtype="f32")
    _same(x, x["S0"])


def test_noalloc_rejects_problems_beyond_the_scratch():
    """One chunk of every head must fit the fixed scratch; 1024 heads of 128 x 128 do not."""
    assert kda.kda_chunk_fwd_noalloc_max_scratch() == 64 << 20
    x = _inputs(1, 64, 1024, seed=903)
    with pytest.raises(kda.KdaError) as e:
        kda.kda_chunk_fwd_noalloc(*(x[n] for n in NAMES), G_MIN, S0=None)
    assert e.value.status == 7  # KDA_ERR_WORKSPACE
