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


def test_decode_config_1000_chained_steps():
    """The decode workload as configured: N=256 sequences x H=32 heads, d=128, fp32 state
    ~N(0, 0.1), 1000 chained steps, each with its own seeded token set, the state updated in
    place on the GPU.  The (n, h) units are independent, so the fp64 oracle follows a sample
    of 64 of the 8192 units through all 1000 steps: o is compared at 11 sampled steps and
    the state after the last step.

    Tolerance for the state after 1000 steps: every step rounds a handful of float32
    operations (decay, two dot products, the rank-1 update: relative 2^-24 each, a few ulp
    for the fast exponential), and the step map is non-expansive (decay factors <= 1, the
    erase I - beta k k^T with |k| = 1 and 0 < beta < 1), so rounding errors add up at most
    linearly: 1000 steps x ~2^-20 ~ 1e-3 of the state's scale.  o is bf16 (2e-2)."""
    w = synth.DECODE
    steps = 1000
    rng = np.random.default_rng(1234)
    units = np.unique(np.concatenate([[0, w.N * w.H - 1], rng.choice(w.N * w.H, 62, replace=False)]))
    un, uh = units // w.H, units % w.H
    S_cpu = synth.decode_state(w)
    S = S_cpu.cuda()
    S_ref = S_cpu.numpy()[un, uh].astype(np.float64)[:, None]  # [units, 1, dk, dv]
    check_at = set(range(0, steps, 100)) | {steps - 1}
    worst_o = 0.0
    for step, tok in enumerate(synth.decode_token_sets(w, range(steps))):
        d = {n: t.cuda(non_blocking=False) for n, t in tok.items()}
        o = kda.kda_decode_step(*(d[n] for n in NAMES), S, G_MIN)
        sub = {n: synth.to_numpy32(tok[n])[un, uh][:, None] for n in NAMES}
        o_ref, S_ref = oracle.decode(*(sub[n] for n in NAMES), S_ref, G_MIN)
        if step in check_at:
            got = o.float().cpu().numpy()[un, uh][:, None]
            worst_o = max(worst_o, _err_tok(got, o_ref))
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    assert worst_o <= TOL_BF16_O, worst_o
    es = err_s(S.cpu().numpy()[un, uh][:, None], S_ref)
    assert es <= 1e-3, es


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
