"""The ablation path kda_chunk_fwd_logsigmoid (unbounded gate g = log sigmoid(a), diagonal
16x16 tiles element by element) on the GPU against the fp64 oracle run with the same gate.

Tolerances are the bf16 path's: o <= 2e-2 and S_T <= 1e-2 normwise per head."""
import numpy as np
import pytest
import torch

import chunked_linear_attention_chunk_b200 as kda
import oracle
from chunked_linear_attention_chunk_b200 import synth
from helpers import NAMES, TOL_BF16_O, TOL_BF16_S, err_o, err_s, oracle_run, to_dev

pytestmark = pytest.mark.gpu


def _check(x, S0=True):
    d = to_dev(x)
    o, ST = kda.kda_chunk_fwd_logsigmoid(*(d[n] for n in NAMES), S0=d["S0"] if S0 else None)
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    o_ref, S_ref = oracle_run(x, x["S0"] if S0 else None, kind=oracle.GATE_LOGSIGMOID)
    o_np = o.float().cpu().numpy()
    assert np.isfinite(o_np).all() and np.isfinite(ST.cpu().numpy()).all()
    eo, es = err_o(o_np, o_ref), err_s(ST.cpu().numpy(), S_ref)
    assert eo <= TOL_BF16_O and es <= TOL_BF16_S, (eo, es)
    return eo, es


@pytest.mark.parametrize("B,T,H,D", [(2, 300, 3, 128), (1, 129, 2, 64), (1, 512, 1, 128)])
def test_logsig_several_chunks_ragged_tail(B, T, H, D):
    _check(synth.make_inputs(B, T, H, D, D, "bf16", seed=700 + T, s0_std=0.1))


@pytest.mark.parametrize("T", [1, 16, 17, 64, 65, 129])
def test_logsig_edge_lengths(T):
    _check(synth.make_inputs(1, T, 2, 128, 128, "bf16", seed=800 + T, s0_std=0.1))


def test_logsig_steep_decay_beyond_any_bound():
    """a ~ -12: g ~ -12 on every channel, a 16-token tile spans e^{-190}, beyond float32 and
    bfloat16 range for a single reference.  The element-wise diagonal must stay finite."""
    x = synth.make_inputs(1, 256, 2, 128, 128, "bf16", seed=810, s0_std=0.1)
    x["a"] = (x["a"].float() - 12.0).to(torch.bfloat16)
    _check(x)


def test_logsig_weak_decay():
    """a = +8: g ~ -3.4e-4, nearly the pure delta rule."""
    x = synth.make_inputs(1, 200, 2, 128, 128, "bf16", seed=811, s0_std=0.1)
    x["a"] = torch.full_like(x["a"], 8.0)
    _check(x)


def test_logsig_null_state_equals_zero_state():
    x = synth.make_inputs(1, 100, 2, 64, 64, "bf16", seed=812, s0_std=0.0)
    d = to_dev(x)
    o1, S1 = kda.kda_chunk_fwd_logsigmoid(*(d[n] for n in NAMES), S0=None)
    o2, S2 = kda.kda_chunk_fwd_logsigmoid(*(d[n] for n in NAMES), S0=torch.zeros_like(d["S0"]))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
