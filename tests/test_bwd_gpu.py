"""kda_chunk_bwd on the GPU against the fp64 oracle's backward (the reverse-mode
derivative of the recurrence, itself pinned by finite differences).

Tolerance: every gradient, dS0 included, within 2e-2 normwise per (batch, head).  The
state gradient walks the chunks through bfloat16 operands (the records' N and Q' and a
bfloat16 copy of dS'), like the forward's state through its bfloat16 copy; each rounding
is 2^-9 relative and the 192-term sums of a chunk step compound a few of them, so the
bound of the forward's output (2e-2) is the one that applies, not its float32 state's."""
import numpy as np
import pytest
import torch

import oracle
import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import synth
from helpers import G_MIN, NAMES

pytestmark = pytest.mark.gpu

TOL_BWD = 2e-2
GRADS = ("dq", "dk", "dv", "da", "dbeta", "dS0")


def _err(x, y):
    """Worst per-(b, h) normwise relative error of [B,T,H,d] or [B,T,H] tensors."""
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    axes = (1, 3) if x.ndim == 4 else (1,)
    num = np.abs(x - y).max(axis=axes)
    den = np.maximum(np.abs(y).max(axis=axes), 1e-30)
    return float((num / den).max())


def _err_state(x, y):
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    num = np.abs(x - y).max(axis=(-2, -1))
    den = np.maximum(np.abs(y).max(axis=(-2, -1)), 1e-30)
    return float((num / den).max())


def _case(B, T, H, D, seed, with_state=True):
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=seed, s0_std=0.1)
    rng = np.random.default_rng(seed)
    dO = torch.from_numpy(rng.normal(size=(B, T, H, D)).astype(np.float32)).to(torch.bfloat16)
    dST = torch.from_numpy((rng.normal(size=(B, H, D, D)) * 0.5).astype(np.float32)) if with_state else None
    S0 = x["S0"] if with_state else None
    return x, dO, dST, S0


def _oracle(x, dO, dST, S0):
    xn = {n: synth.to_numpy32(x[n]) for n in NAMES}
    return oracle.backward(*(xn[n] for n in NAMES), synth.to_numpy32(dO), G_MIN,
                           S0=None if S0 is None else S0.numpy(),
                           dST=None if dST is None else dST.numpy().astype(np.float64))


def _gpu(x, dO, dST, S0, workspace=None):
    d = {n: x[n].cuda() for n in NAMES}
    g = kda.kda_chunk_bwd(*(d[n] for n in NAMES), dO.cuda(), G_MIN,
                          S0=None if S0 is None else S0.cuda(), dS_T=None if dST is None else dST.cuda(),
                          workspace=workspace)
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    return {n: t.cpu().numpy() for n, t in g.items() if t is not None}


def _check(got, ref):
    for n in GRADS:
        e = _err_state(got[n], ref[n]) if n == "dS0" else _err(got[n], ref[n])
        assert e <= TOL_BWD, f"{n}: {e:.3e}"


@pytest.mark.parametrize("B,T,H,D", [(1, 1, 1, 64), (1, 64, 1, 128), (2, 150, 2, 64), (1, 200, 2, 128),
                                     (2, 333, 3, 128), (1, 1000, 2, 64)])
def test_bwd_matches_oracle(B, T, H, D):
    """Single token, one full chunk, ragged tails, several chunks and heads, both head dims."""
    x, dO, dST, S0 = _case(B, T, H, D, seed=700 + T + D)
    _check(_gpu(x, dO, dST, S0), _oracle(x, dO, dST, S0))


def test_bwd_zero_state_and_no_state_gradient():
    x, dO, _, _ = _case(2, 130, 2, 128, seed=711, with_state=False)
    _check(_gpu(x, dO, None, None), _oracle(x, dO, None, None))


@pytest.mark.parametrize("B,T,H,D", [(2, 150, 2, 64), (1, 200, 2, 128)])
def test_bwd_saved_states_and_state_gradients(B, T, H, D):
    """The workspace's chunk states match the oracle's state after 64 n tokens, and the
    state gradients match the oracle backward of the remaining suffix (its dS0)."""
    x, dO, dST, S0 = _case(B, T, H, D, seed=720 + T)
    NT = (T + 63) // 64
    ws = torch.zeros(kda.kda_chunk_bwd_workspace(B, T, H, D, D), dtype=torch.uint8, device="cuda")
    _gpu(x, dO, dST, S0, workspace=ws)
    so, dso = kda.kda_chunk_bwd_offsets(B, T, H, D, D)
    nb = B * H * NT * D * D * 4
    Hs = ws[so:so + nb].view(torch.float32).view(B, H, NT, D, D).cpu().numpy()
    dHs = ws[dso:dso + nb].view(torch.float32).view(B, H, NT, D, D).cpu().numpy()
    xn = {n: synth.to_numpy32(x[n]) for n in NAMES}
    dOn = synth.to_numpy32(dO)
    for n in range(NT):
        t0, t1 = 64 * n, min(T, 64 * (n + 1))
        if n == 0:
            S_ref = S0.numpy().astype(np.float64)
        else:
            _, S_ref = oracle.recurrence(*(xn[m][:, :t0] for m in NAMES), G_MIN, S0=S0.numpy())
        assert _err_state(Hs[:, :, n], S_ref) <= 1e-2, f"state entering chunk {n}"
        if t1 == T:
            dS_ref = dST.numpy().astype(np.float64)
        else:
            _, S1 = oracle.recurrence(*(xn[m][:, :t1] for m in NAMES), G_MIN, S0=S0.numpy())
            dS_ref = oracle.backward(*(xn[m][:, t1:] for m in NAMES), dOn[:, t1:], G_MIN, S0=S1,
                                     dST=dST.numpy().astype(np.float64))["dS0"]
        assert _err_state(dHs[:, :, n], dS_ref) <= TOL_BWD, f"state gradient after chunk {n}"


def test_bwd_empty_sequence_copies_state_gradient():
    B, H, D = 2, 3, 64
    q = torch.empty(B, 0, H, D, dtype=torch.bfloat16, device="cuda")
    v = torch.empty(B, 0, H, D, dtype=torch.bfloat16, device="cuda")
    beta = torch.empty(B, 0, H, dtype=torch.bfloat16, device="cuda")
    dST = torch.randn(B, H, D, D, device="cuda")
    g = kda.kda_chunk_bwd(q, q, v, q, beta, v, G_MIN, dS_T=dST)
    torch.cuda.synchronize()
    assert torch.equal(g["dS0"], dST)
    g = kda.kda_chunk_bwd(q, q, v, q, beta, v, G_MIN)
    torch.cuda.synchronize()
    assert torch.count_nonzero(g["dS0"]) == 0


def test_bwd_repeatable():
    """Two calls on the same inputs give identical gradients (no reduction-order freedom)."""
    x, dO, dST, S0 = _case(1, 300, 2, 128, seed=730)
    a = _gpu(x, dO, dST, S0)
    b = _gpu(x, dO, dST, S0)
    for n in GRADS:
        assert np.array_equal(a[n], b[n]), n


def test_bwd_repeatable_full_size_and_packed():
    """Five calls at the full 64K-token stage (B1 T65536 H32 d128, 1024 chunks per head over
    the 148 persistent gradient CTAs, each CTA reusing its scratch slot for about 220
    chunks) and three over a packed batch with the per-head gate scale: every gradient is
    bitwise the same from call to call.  Each element of every gradient is produced by one
    thread from values written before a CTA barrier, with no atomics, so nothing may vary."""
    w = synth.STAGE_64K
    x = synth.workload_inputs(w)
    rng = np.random.default_rng(741)
    dO = torch.from_numpy(rng.normal(size=(w.B, w.T, w.H, w.dv)).astype(np.float32)).to(torch.bfloat16).cuda()
    d = {n: x[n].cuda() for n in NAMES}
    S0 = x["S0"].cuda()
    ws = torch.empty(kda.kda_chunk_bwd_workspace(w.B, w.T, w.H, w.dk, w.dv), dtype=torch.uint8, device="cuda")
    first = None
    for _ in range(5):
        g = kda.kda_chunk_bwd(*(d[n] for n in NAMES), dO, G_MIN, S0=S0, workspace=ws)
        torch.cuda.synchronize()
        assert kda.kda_device_status() == 0
        if first is None:
            first = {n: t.clone() for n, t in g.items() if t is not None}
        else:
            for n, t in first.items():
                assert torch.equal(g[n], t), n
    del first, g, ws, d, dO
    lengths = [700, 1, 64, 3000, 129]
    xp, dOp, dSTp, S0p, cu = _packed(lengths, 4, 128, seed=742)
    A_log = torch.from_numpy((np.random.default_rng(743).normal(size=4) * 0.5).astype(np.float32)).cuda()
    dp = {n: xp[n][0].cuda() for n in NAMES}
    cu_d = torch.from_numpy(cu).cuda()
    ref = None
    for _ in range(3):
        g = kda.kda_chunk_bwd_varlen(*(dp[n] for n in NAMES), dOp[0].cuda(), cu_d, G_MIN, S0=S0p.cuda(),
                                     dS_T=dSTp.cuda(), A_log=A_log)
        torch.cuda.synchronize()
        assert kda.kda_device_status() == 0
        if ref is None:
            ref = {n: t.clone() for n, t in g.items() if t is not None}
        else:
            for n, t in ref.items():
                assert torch.equal(g[n], t), n


def test_bwd_full_size_sampled_heads():
    """The 64K-token stage (B1 T65536 H32 d128, bench inputs) against the oracle on two
    sampled heads (the oracle runs them alone: heads are independent)."""
    w = synth.STAGE_64K
    x = synth.workload_inputs(w)
    rng = np.random.default_rng(740)
    dO = torch.from_numpy(rng.normal(size=(w.B, w.T, w.H, w.dv)).astype(np.float32)).to(torch.bfloat16)
    got = _gpu(x, dO, None, x["S0"])
    for h in (0, w.H - 1):
        xs = {n: x[n][:, :, h:h + 1] for n in NAMES}
        ref = _oracle(xs, dO[:, :, h:h + 1], None, x["S0"][:, h:h + 1])
        for n in GRADS:
            gh = got[n][:, h:h + 1] if n == "dS0" else got[n][:, :, h:h + 1]
            e = _err_state(gh, ref[n]) if n == "dS0" else _err(gh, ref[n])
            assert e <= TOL_BWD, f"head {h} {n}: {e:.3e}"


def _oracle_scaled(x, dO, dST, S0, A_log):
    """The oracle on the gate's scaled argument: g = g_min sigma(e^{A_h} a) is the bounded gate
    of a' = e^{A_h} a, so da = e^{A_h} da' and dL/dA_log[h] = sum over the head of da' a'."""
    scale = np.exp(A_log.astype(np.float64))
    a_s = (synth.to_numpy32(x["a"]).astype(np.float64) * scale[None, None, :, None]).astype(np.float32)
    xs = dict(x)
    xs["a"] = torch.from_numpy(a_s)
    ref = _oracle(xs, dO, dST, S0)
    dA = np.einsum("bthc,bthc->h", ref["da"], a_s.astype(np.float64))
    terms = np.einsum("bthc->h", np.abs(ref["da"] * a_s.astype(np.float64)))
    ref["da"] = ref["da"] * scale[None, None, :, None]
    return ref, dA, terms


@pytest.mark.parametrize("B,T,H,D", [(2, 150, 3, 64), (1, 200, 2, 128)])
def test_bwd_head_scaled_gate(B, T, H, D):
    """A_log given: every gradient against the oracle run on e^{A_h} a, and dL/dA_log against
    the chain rule (the sum of da' a' over the head), within 2e-2 of the sum of |da' a'|."""
    x, dO, dST, S0 = _case(B, T, H, D, seed=750 + T)
    A_log = (np.random.default_rng(751).normal(size=H) * 0.5).astype(np.float32)
    d = {n: x[n].cuda() for n in NAMES}
    g = kda.kda_chunk_bwd(*(d[n] for n in NAMES), dO.cuda(), G_MIN, S0=S0.cuda(), dS_T=dST.cuda(),
                          A_log=torch.from_numpy(A_log).cuda())
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    got = {n: t.cpu().numpy() for n, t in g.items()}
    ref, dA, terms = _oracle_scaled(x, dO, dST, S0, A_log)
    _check(got, ref)
    assert np.all(np.abs(got["dA_log"] - dA) <= TOL_BWD * terms), (got["dA_log"], dA, terms)
    # the reduction is the sum of the kernel's own da * a
    own = np.einsum("bthc,bthc->h", got["da"].astype(np.float64), synth.to_numpy32(x["a"]).astype(np.float64))
    assert np.all(np.abs(got["dA_log"] - own) <= 1e-4 * np.abs(got["da"] * synth.to_numpy32(x["a"])).sum((0, 1, 3)))


def _packed(lengths, H, D, seed):
    T = int(sum(lengths))
    x = synth.make_inputs(1, T, H, D, D, "bf16", seed=seed, s0_std=0.1)
    N = len(lengths)
    rng = np.random.default_rng(seed)
    S0 = torch.from_numpy((rng.normal(size=(N, H, D, D)) * 0.1).astype(np.float32))
    dST = torch.from_numpy((rng.normal(size=(N, H, D, D)) * 0.5).astype(np.float32))
    dO = torch.from_numpy(rng.normal(size=(1, T, H, D)).astype(np.float32)).to(torch.bfloat16)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return x, dO, dST, S0, cu


@pytest.mark.parametrize("lengths,H,D,with_A", [([70, 0, 129, 64], 2, 64, False), ([1, 200, 63], 2, 128, True)])
def test_bwd_varlen_matches_oracle(lengths, H, D, with_A):
    """Packed sequences (one empty, a single token, tails, exact chunks): each sequence against
    the oracle on its own slice with its own S0 and dS_T."""
    x, dO, dST, S0, cu = _packed(lengths, H, D, seed=760 + D)
    A_log = (np.random.default_rng(761).normal(size=H) * 0.5).astype(np.float32) if with_A else None
    pk = {n: x[n][0].cuda() for n in NAMES}
    g = kda.kda_chunk_bwd_varlen(*(pk[n] for n in NAMES), dO[0].cuda(), torch.from_numpy(cu).cuda(), G_MIN,
                                 S0=S0.cuda(), dS_T=dST.cuda(),
                                 A_log=None if A_log is None else torch.from_numpy(A_log).cuda())
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    got = {n: (None if t is None else t.cpu().numpy()) for n, t in g.items()}
    dA_tot, terms_tot = np.zeros(H), np.zeros(H)
    for s in range(len(lengths)):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        if t1 == t0:
            assert np.array_equal(got["dS0"][s], dST[s].numpy()), "empty sequence passes dS_T through"
            continue
        xs = {n: x[n][:, t0:t1] for n in NAMES}
        if with_A:
            ref, dA, terms = _oracle_scaled(xs, dO[:, t0:t1], dST[s:s + 1], S0[s:s + 1], A_log)
            dA_tot += dA
            terms_tot += terms
        else:
            ref = _oracle(xs, dO[:, t0:t1], dST[s:s + 1], S0[s:s + 1])
        gs = {n: got[n][None, t0:t1] for n in ("dq", "dk", "dv", "da", "dbeta")}
        gs["dS0"] = got["dS0"][s:s + 1]
        _check(gs, ref)
    if with_A:
        assert np.all(np.abs(got["dA_log"] - dA_tot) <= TOL_BWD * terms_tot)


def test_bwd_varlen_equal_lengths_equals_regular_batch():
    """B equal-length sequences packed give exactly the regular batch's gradients."""
    B, T, H, D = 3, 130, 2, 128
    x, dO, dST, S0 = _case(B, T, H, D, seed=770)
    reg = _gpu(x, dO, dST, S0)
    cu = torch.arange(0, (B + 1) * T, T, dtype=torch.int32).cuda()
    pk = {n: x[n].reshape(B * T, *x[n].shape[2:]).cuda() for n in NAMES}
    g = kda.kda_chunk_bwd_varlen(*(pk[n] for n in NAMES), dO.reshape(B * T, H, D).cuda(), cu, G_MIN,
                                 S0=S0.cuda(), dS_T=dST.cuda())
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    for n in ("dq", "dk", "dv", "da", "dbeta"):
        assert np.array_equal(g[n].cpu().numpy().reshape(reg[n].shape), reg[n]), n
    assert np.array_equal(g["dS0"].cpu().numpy(), reg["dS0"])
