"""kda_chunk_fwd_varlen on the GPU: packed variable-length batches against the fp64 oracle
run on every sequence separately, equal lengths against kda_chunk_fwd bit for bit, and an
invalid cu_seqlens reported through the device status word.

Tolerances are the bf16 path's: o <= 2e-2 and S_T <= 1e-2 normwise per (sequence, head)."""
import numpy as np
import pytest
import torch

import chunked_linear_attention_chunk_b200 as kda
import oracle
from chunked_linear_attention_chunk_b200 import synth
from helpers import G_MIN, NAMES, TOL_BF16_O, TOL_BF16_S, err_o, err_s, oracle_run, to_dev

pytestmark = pytest.mark.gpu


def _packed(lengths, H, D, seed):
    T = int(sum(lengths))
    x = synth.make_inputs(1, max(T, 1), H, D, D, "bf16", seed=seed, s0_std=0.0)
    x = {n: x[n][:, :T] for n in NAMES}
    S0 = synth.make_inputs(len(lengths), 1, H, D, D, "bf16", seed=seed + 1, s0_std=0.1)["S0"]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return x, S0, cu


def _check(lengths, H=3, D=128, seed=1200, gate=kda.KDA_GATE_BOUNDED):
    x, S0, cu = _packed(lengths, H, D, seed)
    d = to_dev(x)
    o, ST = kda.kda_chunk_fwd_varlen(*(d[n][0] for n in NAMES), torch.from_numpy(cu).cuda(), G_MIN, gate,
                                     S0=S0.cuda())
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    o, ST = o.float().cpu().numpy(), ST.cpu().numpy()
    kind = oracle.GATE_BOUNDED if gate == kda.KDA_GATE_BOUNDED else oracle.GATE_LOGSIGMOID
    worst = (0.0, 0.0)
    for s, L in enumerate(lengths):
        a, b = int(cu[s]), int(cu[s + 1])
        xs = {n: x[n][:, a:b] for n in NAMES}
        if L == 0:
            assert np.array_equal(ST[s], S0[s].numpy())  # empty sequence: the state passes through
            continue
        o_ref, S_ref = oracle_run(xs, S0[s:s + 1], kind=kind)
        eo, es = err_o(o[None, a:b], o_ref), err_s(ST[s:s + 1], S_ref)
        assert eo <= TOL_BF16_O and es <= TOL_BF16_S, (s, L, eo, es)
        worst = (max(worst[0], eo), max(worst[1], es))
    return worst


def test_varlen_mixed_lengths():
    _check([130, 0, 1, 63, 64, 65, 200, 17])


def test_varlen_d64_and_single_sequence():
    _check([300], H=2, D=64, seed=1210)
    _check([5, 128, 77], H=2, D=64, seed=1211)


def test_varlen_logsigmoid_gate():
    _check([100, 64, 1, 90], seed=1220, gate=kda.KDA_GATE_LOGSIGMOID)


def test_varlen_many_short_sequences():
    rng = np.random.default_rng(5)
    _check(list(rng.integers(0, 40, size=60)), H=2, seed=1230)


def test_equal_lengths_match_regular_batch_bitwise():
    B, T, H, D = 3, 150, 2, 128
    x = to_dev(synth.make_inputs(B, T, H, D, D, "bf16", seed=1240, s0_std=0.1))
    o1, S1 = kda.kda_chunk_fwd(*(x[n] for n in NAMES), G_MIN, S0=x["S0"])
    cu = torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device="cuda")
    packed = [x[n].reshape(B * T, *x[n].shape[2:]) for n in NAMES]
    o2, S2 = kda.kda_chunk_fwd_varlen(*packed, cu, G_MIN, S0=x["S0"])
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    assert torch.equal(o1.reshape(B * T, H, D), o2) and torch.equal(S1, S2)


def test_invalid_cu_seqlens_is_reported_on_device():
    x, S0, _ = _packed([40, 40], 2, 64, 1250)
    d = to_dev(x)
    cu = torch.tensor([0, 60, 50], dtype=torch.int32, device="cuda")  # decreasing, and cu[N] != T
    o = torch.zeros((80, 2, 64), dtype=torch.bfloat16, device="cuda")
    _, ST = kda.kda_chunk_fwd_varlen(*(d[n][0] for n in NAMES), cu, G_MIN, S0=S0.cuda(), o=o)
    assert kda.kda_device_status() == 1           # KDA_ERR_INVALID_ARG, from the device
    assert torch.equal(ST.cpu(), S0)              # nothing ran: the state passes through
    assert not o.any()                            # and no output was written
    assert kda.kda_device_status() == 0


@pytest.mark.parametrize("gate", [kda.KDA_GATE_BOUNDED, kda.KDA_GATE_LOGSIGMOID])
def test_varlen_tail_chunk_ignores_the_next_sequence(gate):
    """A sequence whose last chunk is partial gets the next sequence's tokens in the rest of
    that chunk's tiles (the tensor copies read the packed axis); the prep must mask them.  With
    the next sequence all NaN, the first sequence's o and S_T must equal a packed batch of the
    first sequence alone, bit for bit; lengths 70 and 1 leave 58 and 63 foreign rows in the
    tail chunk."""
    H, D = 2, 128
    for L0 in (70, 1):
        x, S0, _ = _packed([L0, 90], H, D, seed=1240 + L0)
        cu2 = torch.tensor([0, L0, L0 + 90], dtype=torch.int32, device="cuda")
        cu1 = torch.tensor([0, L0], dtype=torch.int32, device="cuda")
        d = to_dev(x)
        poisoned = {n: d[n][0].clone() for n in NAMES}
        for n in NAMES:
            poisoned[n][L0:] = float("nan")
        o2, S2 = kda.kda_chunk_fwd_varlen(*(poisoned[n] for n in NAMES), cu2, G_MIN, gate, S0=S0.cuda())
        o1, S1 = kda.kda_chunk_fwd_varlen(*(d[n][0][:L0].contiguous() for n in NAMES), cu1, G_MIN, gate,
                                          S0=S0[:1].cuda())
        torch.cuda.synchronize()
        assert kda.kda_device_status() == 0
        assert torch.equal(o2[:L0], o1), L0
        assert torch.equal(S2[0], S1[0]), L0
        assert torch.isnan(S2[1]).any()          # the second sequence did run on its NaN tokens


def test_varlen_backward_tail_chunk_ignores_the_next_sequence():
    """The same for the packed backward: with the next sequence all NaN (inputs and dL/do),
    every gradient of the first sequence equals the packed backward of that sequence alone."""
    H, D, L0 = 2, 128, 70
    x, S0, _ = _packed([L0, 90], H, D, seed=1250)
    cu2 = torch.tensor([0, L0, L0 + 90], dtype=torch.int32, device="cuda")
    cu1 = torch.tensor([0, L0], dtype=torch.int32, device="cuda")
    d = to_dev(x)
    gen = torch.Generator().manual_seed(1251)
    dO = torch.randn((L0 + 90, H, D), generator=gen).to(torch.bfloat16).cuda()
    poisoned = {n: d[n][0].clone() for n in NAMES}
    dOp = dO.clone()
    for t in list(poisoned.values()) + [dOp]:
        t[L0:] = float("nan")
    g2 = kda.kda_chunk_bwd_varlen(*(poisoned[n] for n in NAMES), dOp, cu2, G_MIN, S0=S0.cuda())
    g1 = kda.kda_chunk_bwd_varlen(*(d[n][0][:L0].contiguous() for n in NAMES), dO[:L0].contiguous(), cu1, G_MIN,
                                  S0=S0[:1].cuda())
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    for n in ("dq", "dk", "dv", "da", "dbeta"):
        assert torch.equal(g2[n][:L0], g1[n]), n
    assert torch.equal(g2["dS0"][0], g1["dS0"][0])
