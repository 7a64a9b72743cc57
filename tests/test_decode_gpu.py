"""kda_decode_step on the GPU against the fp64 oracle, and against the chunk path."""
import numpy as np
import pytest
import torch

import oracle
import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import synth
from helpers import G_MIN, NAMES, TOL_BF16_O, TOL_F32, err_s

pytestmark = pytest.mark.gpu


def _err_tok(x, y):
    """[N, H, d] -> worst per-(n, h) normwise relative error."""
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    return float(np.max(np.max(np.abs(x - y), axis=2) / np.maximum(np.max(np.abs(y), axis=2), 1e-30)))


def test_decode_config_chained_steps():
    """N=256, H=32, d=128, fp32 state ~N(0, 0.1): 3 chained steps vs the oracle."""
    w = synth.DECODE
    S_cpu = synth.decode_state(w)
    S = S_cpu.cuda()
    S_ref = S_cpu.numpy().astype(np.float64)
    for step in range(3):
        tok = synth.decode_tokens(w, step)
        d = {n: t.cuda() for n, t in tok.items()}
        o = kda.kda_decode_step(*(d[n] for n in NAMES), S, G_MIN)
        torch.cuda.synchronize()
        o_ref, S_ref = oracle.decode(*(synth.to_numpy32(tok[n]) for n in NAMES), S_ref, G_MIN)
        assert _err_tok(o.float().cpu().numpy(), o_ref) <= TOL_BF16_O
        # the state stays float32: error is rounding of a few float32 operations
        assert err_s(S.cpu().numpy(), S_ref) <= 1e-5


@pytest.mark.parametrize("D", [64, 128])
def test_decode_f32(D):
    x = synth.make_inputs(5, 1, 3, D, D, "f32", seed=600 + D, s0_std=0.1)
    tok = {n: x[n][:, 0].contiguous() for n in NAMES}
    S = x["S0"].cuda()
    o = kda.kda_decode_step(*(tok[n].cuda() for n in NAMES), S, G_MIN)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.decode(*(synth.to_numpy32(tok[n]) for n in NAMES), x["S0"].numpy(), G_MIN)
    assert _err_tok(o.cpu().numpy(), o_ref) <= TOL_F32
    assert err_s(S.cpu().numpy(), S_ref) <= TOL_F32


def test_decode_matches_chunk_path_single_token():
    """A decode step and a one-token chunk forward compute the same thing."""
    x = synth.make_inputs(4, 1, 8, 128, 128, "bf16", seed=610, s0_std=0.1)
    d = {n: t.cuda() for n, t in x.items()}
    o_c, S_c = kda.kda_chunk_fwd(*(d[n] for n in NAMES), G_MIN, S0=d["S0"])
    S = d["S0"].clone()
    o_d = kda.kda_decode_step(*(d[n][:, 0].contiguous() for n in NAMES), S, G_MIN)
    torch.cuda.synchronize()
    assert _err_tok(o_d.float().cpu().numpy(), o_c[:, 0].float().cpu().numpy()) <= TOL_BF16_O
    assert err_s(S.cpu().numpy(), S_c.cpu().numpy()) <= 1e-2


def test_decode_chain_matches_chunk_path():
    """T chained decode steps approximate one chunk forward over the same T tokens."""
    x = synth.make_inputs(2, 40, 4, 128, 128, "bf16", seed=611, s0_std=0.1)
    d = {n: t.cuda() for n, t in x.items()}
    o_c, S_c = kda.kda_chunk_fwd(*(d[n] for n in NAMES), G_MIN, S0=d["S0"])
    S = d["S0"].clone()
    outs = []
    for t in range(40):
        outs.append(kda.kda_decode_step(*(d[n][:, t].contiguous() for n in NAMES), S, G_MIN))
    torch.cuda.synchronize()
    o_d = torch.stack(outs, 1)
    num = (o_d.float() - o_c.float()).abs().amax(dim=(1, 3))
    den = o_c.float().abs().amax(dim=(1, 3))
    assert float((num / den).max()) <= TOL_BF16_O
    assert err_s(S.cpu().numpy(), S_c.cpu().numpy()) <= 1e-2


@pytest.mark.parametrize("N,H,D", [(303, 1, 128), (7, 45, 64), (1, 1, 128)])
def test_decode_uneven_units(N, H, D):
    """The persistent decode kernel gives CTAs different numbers of (n, h) units (303 units
    over the resident CTAs), one unit, and the d = 64 bf16 shape; two chained steps."""
    x = synth.make_inputs(N, 2, H, D, D, "bf16", seed=620 + N + D, s0_std=0.1)
    S = x["S0"].cuda()
    S_ref = x["S0"].numpy().astype(np.float64)
    for t in range(2):
        tok = {n: x[n][:, t].contiguous() for n in NAMES}
        o = kda.kda_decode_step(*(tok[n].cuda() for n in NAMES), S, G_MIN)
        torch.cuda.synchronize()
        o_ref, S_ref = oracle.decode(*(synth.to_numpy32(tok[n]) for n in NAMES), S_ref, G_MIN)
        assert _err_tok(o.float().cpu().numpy(), o_ref) <= TOL_BF16_O
        assert err_s(S.cpu().numpy(), S_ref) <= 1e-5
    assert kda.kda_device_status() == 0
