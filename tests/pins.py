"""Pins of the fp64 oracle against facts fixed by the pages and by the mathematics.

Each ``pin_*`` function takes an oracle ctypes library (the real one, or a deliberately
broken build made by the mutation test) and raises ``AssertionError`` when the oracle
disagrees with the fact it checks.  None of them re-types the oracle's own formula:
each compares against an independent closed form, a library routine, brute force on a
tiny input, an exact invariant, or a second formulation (chunked vs recurrent).

Facts used (the recurrence S_t = (I - beta k k^T) Diag(e^{g_t}) S_{t-1} + beta k v^T,
o_t = S_t^T q_t, with the bounded gate g = g_min * sigmoid(a) of "Trillion-Scale MoE
Multimodal Models ..." section 3.2 / "Breaking Through Trillion-Parameter Multimodal
MoE ..." section 2.1):
* the gate is g_min * logistic(a) with range [g_min, 0) -- "Breaking Through ..." 2.1;
* with beta = 0 nothing is written and the state only decays: a closed-form decayed sum;
* to first order in beta -> 0 (zero initial state) the output is the decayed causal
  linear-attention sum, and with g = 0 plain causal linear attention, both O(T^2)
  brute force;
* delta-rule retrieval: after writing (k, v) with beta = 1 and a unit key, reading with
  k returns v;
* linearity in (v, S0) jointly;
* the chunked form equals the recurrence at every chunk size; a sequence split into
  segments with the state carried equals one call ("Trillion-Parameter MoE Multimodal
  Models: Engineering ..." section 3.2: training recurses in chunks);
* the range claim of "Trillion-Scale ..." section 3.2: with g >= -5 the factored 1/Gamma
  inside a 16-token tile is finite in float32; with the unbounded log-sigmoid form it
  overflows.
"""
from __future__ import annotations

import numpy as np
import scipy.special

import oracle
from chunked_linear_attention_chunk_b200 import synth

G_MIN = -5.0


def _inputs(B, T, H, d, seed, s0_std=0.1, dv=None):
    x = synth.make_inputs(B, T, H, d, dv or d, "f32", seed, s0_std)
    return {n: synth.to_numpy32(t) for n, t in x.items()}


def _cumG(a, g_min, kind=oracle.GATE_BOUNDED, lib=None):
    """Inclusive cumulative log-decay over tokens from the oracle's gate, [B,T,H,dk]."""
    return np.cumsum(oracle.gate_f64(a, g_min, kind, lib=lib), axis=1)


def _rel(x, y):
    return float(np.max(np.abs(x - y)) / max(np.max(np.abs(y)), 1e-300))


# ---------------------------------------------------------------------------- gate
def pin_gate_special_values(lib):
    a = np.array([0.0, np.inf, -np.inf, np.nan, 100.0, -200.0], np.float32)
    g = oracle.gate(a, G_MIN, lib=lib)
    assert g[0] == np.float32(G_MIN / 2), "sigmoid(0) = 1/2"
    assert g[1] == np.float32(G_MIN), "a = +inf gives g_min"
    assert g[2] == 0.0 and np.signbit(g[2]), "a = -inf gives -0"
    assert np.isnan(g[3]), "NaN propagates"
    assert g[4] == np.float32(G_MIN), "sigmoid rounds to 1"
    assert g[5] == 0.0 and np.signbit(g[5]), "sigmoid underflows to +0, g to -0"
    # log sigmoid: log(1/2) at 0
    l0 = oracle.gate(np.zeros(1, np.float32), G_MIN, oracle.GATE_LOGSIGMOID, lib=lib)
    assert l0[0] == np.float32(-np.log(2.0))


def pin_gate_vs_library(lib):
    """g_min * logistic(a) against scipy's expit / log_expit (a different implementation)."""
    bits = np.arange(65536, dtype=np.uint32) << 16
    a = bits.view(np.float32)
    a = a[np.isfinite(a)]
    for g_min in (-5.0, -1.0, -5.4):
        g = oracle.gate(a, g_min, lib=lib).astype(np.float64)
        ref = g_min * scipy.special.expit(a.astype(np.float64))
        ok = np.isclose(g, ref, rtol=2**-23, atol=1e-45)
        assert ok.all(), f"bounded gate differs from g_min*expit at {a[~ok][:4]}"
    lg = oracle.gate(a, G_MIN, oracle.GATE_LOGSIGMOID, lib=lib).astype(np.float64)
    ref = scipy.special.log_expit(a.astype(np.float64))
    ok = np.isclose(lg, ref, rtol=2**-22, atol=1e-45)
    assert ok.all(), "log-sigmoid gate differs from log_expit"


def pin_gate_range_exhaustive(lib):
    """Every bf16 input: g in [g_min, -0]; strictly negative for |a| <= 16; monotone."""
    bits = np.arange(65536, dtype=np.uint32) << 16
    a = bits.view(np.float32)
    g = oracle.gate(a, G_MIN, lib=lib)
    fin = ~np.isnan(a)
    assert np.isnan(g[~fin]).all()
    gf, af = g[fin], a[fin]
    assert (gf >= np.float32(G_MIN)).all() and (gf <= 0.0).all()
    assert (gf[np.abs(af) <= 16] < 0).all()
    order = np.argsort(af, kind="stable")
    assert (np.diff(gf[order].astype(np.float64)) <= 0).all(), "g must not increase with a"
    # the unbounded gate leaves [-5, 0) for strongly negative a (it is unbounded below)
    lg = oracle.gate(np.array([-8.0], np.float32), G_MIN, oracle.GATE_LOGSIGMOID, lib=lib)
    assert lg[0] < -8.0


# ---------------------------------------------------------------------- recurrence
def pin_beta_zero_closed_form(lib):
    """beta = 0: S_t = Diag(Gamma_t) S0 and o_t = S0^T (Gamma_t * q_t), Gamma_t = e^{G_t}."""
    x = _inputs(2, 37, 2, 16, seed=11)
    beta = np.zeros_like(x["beta"])
    o, ST = oracle.recurrence(x["q"], x["k"], x["v"], x["a"], beta, G_MIN, S0=x["S0"], lib=lib)
    G = _cumG(x["a"], G_MIN, lib=lib)                          # [B,T,H,dk]
    o_ref = np.einsum("bthc,bhcj->bthj", np.exp(G) * x["q"], x["S0"].astype(np.float64))
    ST_ref = np.exp(G[:, -1])[..., None] * x["S0"].astype(np.float64)
    assert _rel(o, o_ref) < 1e-12 and _rel(ST, ST_ref) < 1e-12


def _decayed_linear_attention(q, k, v, G):
    """o_t = sum_{j<=t} sum_c q_tc k_jc e^{G_tc - G_jc} v_j, O(T^2) brute force, fp64."""
    B, T, H, dk = q.shape
    o = np.zeros(v.shape, np.float64)
    for t in range(T):
        w = np.einsum("bhc,bjhc->bjh", q[:, t].astype(np.float64),
                      k[:, : t + 1].astype(np.float64) * np.exp(G[:, t : t + 1] - G[:, : t + 1]))
        o[:, t] = np.einsum("bjh,bjhv->bhv", w, v[:, : t + 1].astype(np.float64))
    return o


def pin_small_beta_is_linear_attention(lib):
    """S0 = 0, beta = eps: o/eps -> decayed causal linear attention (O(eps T) error);
    with a -> -inf (g = 0) it is plain causal linear attention sum_j (q_t . k_j) v_j."""
    eps = np.float32(1e-7)
    for a_fill in (None, -np.inf):
        x = _inputs(1, 48, 2, 8, seed=12, s0_std=0.0)
        a = x["a"] if a_fill is None else np.full_like(x["a"], a_fill)
        beta = np.full_like(x["beta"], eps)
        o, _ = oracle.recurrence(x["q"], x["k"], x["v"], a, beta, G_MIN, lib=lib)
        if a_fill is None:
            ref = _decayed_linear_attention(x["q"], x["k"], x["v"], _cumG(a, G_MIN, lib=lib))
        else:
            qk = np.einsum("bthc,bjhc->bhtj", x["q"].astype(np.float64), x["k"].astype(np.float64))
            qk = np.tril(qk)
            ref = np.einsum("bhtj,bjhv->bthv", qk, x["v"].astype(np.float64))
        assert _rel(o / np.float64(eps), ref) < 1e-4


def pin_delta_rule_retrieval(lib):
    """beta = 1 and exactly-unit keys: S_t^T k_t = v_t, so q = k reads back v."""
    rng = np.random.default_rng(13)
    B, T, H, d = 1, 40, 1, 16
    k = np.zeros((B, T, H, d), np.float32)
    for t in range(T):  # four entries of +-1/2 on random channels: |k| = 1 exactly
        ch = rng.choice(d, 4, replace=False)
        k[0, t, 0, ch] = rng.choice([-0.5, 0.5], 4)
    x = _inputs(B, T, H, d, seed=13)
    o, _ = oracle.recurrence(k, k, x["v"], x["a"], np.ones_like(x["beta"]), G_MIN, S0=x["S0"], lib=lib)
    assert _rel(o, x["v"].astype(np.float64)) < 1e-12


def pin_delta_rule_general_beta(lib):
    """For any beta: S_t^T k = (1 - beta k.k) (D_t S_{t-1})^T k + beta (k.k) v  (exact)."""
    x = _inputs(1, 30, 2, 16, seed=14)
    T = x["q"].shape[1]
    _, S_prev = oracle.recurrence(*(x[n][:, : T - 1] for n in ("q", "k", "v", "a", "beta")),
                                  G_MIN, S0=x["S0"], lib=lib)
    _, S_t = oracle.recurrence(*(x[n] for n in ("q", "k", "v", "a", "beta")), G_MIN, S0=x["S0"], lib=lib)
    k = x["k"][0, T - 1].astype(np.float64)                 # [H, dk]
    v = x["v"][0, T - 1].astype(np.float64)
    b = x["beta"][0, T - 1].astype(np.float64)              # [H]
    D = np.exp(oracle.gate_f64(x["a"][0, T - 1], G_MIN, lib=lib))  # [H, dk]
    kk = np.sum(k * k, axis=-1)
    lhs = np.einsum("hcj,hc->hj", S_t[0], k)
    rhs = (1 - b * kk)[:, None] * np.einsum("hcj,hc->hj", D[..., None] * S_prev[0], k) + (b * kk)[:, None] * v
    assert _rel(lhs, rhs) < 1e-12


def pin_basis_key_hand_cases(lib):
    """Hand-computed two-token cases with basis keys (dk = dv = 2).
    Token 1 writes v1 under e1 with beta1; token 2 writes v2 under e1 with beta2.  With the
    decay d_t = e^{g_t} on channel 1 applied before the erase:
      S_2 row 1 = (1 - beta2) d2 beta1 v1 + beta2 v2,  row 2 = 0;  o_2 = S_2^T q."""
    g_min = -1.0
    a = np.zeros((1, 2, 1, 2), np.float32)
    a[0, :, 0, 0] = [0.0, 2.0]
    k = np.zeros((1, 2, 1, 2), np.float32)
    k[0, :, 0, 0] = 1.0
    v = np.array([[[[1.0, 2.0]], [[-3.0, 0.5]]]], np.float32)
    beta = np.array([[[0.75], [0.25]]], np.float32)
    q = np.array([[[[1.0, 1.0]], [[0.5, -1.0]]]], np.float32)
    o, ST = oracle.recurrence(q, k, v, a, beta, g_min, lib=lib)
    d2 = np.exp(g_min / (1 + np.exp(-2.0)))
    row1_t1 = 0.75 * np.array([1.0, 2.0])
    row1_t2 = (1 - 0.25) * d2 * row1_t1 + 0.25 * np.array([-3.0, 0.5])
    assert np.allclose(ST[0, 0, 0], row1_t2, rtol=1e-14) and np.all(ST[0, 0, 1] == 0)
    assert np.allclose(o[0, 0, 0], row1_t1 * 1.0, rtol=1e-14)
    assert np.allclose(o[0, 1, 0], row1_t2 * 0.5, rtol=1e-14)
    # an initial state on channel 2 only decays (k never touches it)
    S0 = np.zeros((1, 1, 2, 2))
    S0[0, 0, 1] = [4.0, -2.0]
    _, ST = oracle.recurrence(q, k, v, a, beta, g_min, S0=S0, lib=lib)
    d_ch2 = np.exp(2 * g_min / 2)  # a = 0 on channel 2 at both tokens
    assert np.allclose(ST[0, 0, 1], d_ch2 * np.array([4.0, -2.0]), rtol=1e-14)


def pin_linearity(lib):
    """o and S_T are linear in (v, S0) jointly.  Values are dyadic so that
    v = v1/2 + v2 and S0 = S01/2 + S02 hold exactly in the inputs' precision."""
    x1 = _inputs(1, 33, 2, 16, seed=15)
    x2 = _inputs(1, 33, 2, 16, seed=16)
    v1 = (np.round(x1["v"] * 64) / 64).astype(np.float32)
    v2 = (np.round(x2["v"] * 64) / 64).astype(np.float32)
    v = (0.5 * v1 + v2).astype(np.float32)
    S0 = 0.5 * x1["S0"].astype(np.float64) + x2["S0"].astype(np.float64)
    args = (x1["q"], x1["k"])
    o, ST = oracle.recurrence(*args, v, x1["a"], x1["beta"], G_MIN, S0=S0, lib=lib)
    o1, ST1 = oracle.recurrence(*args, v1, x1["a"], x1["beta"], G_MIN, S0=x1["S0"], lib=lib)
    o2, ST2 = oracle.recurrence(*args, v2, x1["a"], x1["beta"], G_MIN, S0=x2["S0"], lib=lib)
    assert _rel(o, 0.5 * o1 + o2) < 1e-12 and _rel(ST, 0.5 * ST1 + ST2) < 1e-12


def pin_decay_nonincreasing(lib):
    """Gamma_t = e^{G_t} is non-increasing in t on every channel (bounded gate)."""
    x = _inputs(1, 200, 2, 16, seed=17)
    G = _cumG(x["a"], G_MIN, lib=lib)
    assert (np.diff(G, axis=1) <= 0).all() and (G >= G_MIN * np.arange(1, 201)[None, :, None, None] - 1e-9).all()


# ------------------------------------------------------------------- chunked form
def pin_chunked_equals_recurrence(lib, sizes=(1, 2, 3, 4, 8, 16, 32, 64, 256), lengths=(1, 17, 256)):
    for T in lengths:
        x = _inputs(1, T, 2, 8, seed=20 + T)
        o_r, S_r = oracle.recurrence(*(x[n] for n in ("q", "k", "v", "a", "beta")), G_MIN, S0=x["S0"], lib=lib)
        for C in sizes:
            o_c, S_c = oracle.chunked(C, *(x[n] for n in ("q", "k", "v", "a", "beta")), G_MIN, S0=x["S0"], lib=lib)
            assert _rel(o_c, o_r) < 1e-12 and _rel(S_c, S_r) < 1e-12, f"C={C} T={T}"
    # wider head dims and both gate kinds at a 64-token chunk
    x = _inputs(1, 150, 1, 32, seed=29)
    for kind in (oracle.GATE_BOUNDED, oracle.GATE_LOGSIGMOID):
        o_r, S_r = oracle.recurrence(*(x[n] for n in ("q", "k", "v", "a", "beta")), G_MIN, S0=x["S0"], kind=kind, lib=lib)
        o_c, S_c = oracle.chunked(64, *(x[n] for n in ("q", "k", "v", "a", "beta")), G_MIN, S0=x["S0"], kind=kind, lib=lib)
        assert _rel(o_c, o_r) < 1e-12 and _rel(S_c, S_r) < 1e-12


def pin_segment_carry(lib):
    """Two calls with the state carried equal one call, for both formulations."""
    x = _inputs(2, 100, 2, 16, seed=30)
    names = ("q", "k", "v", "a", "beta")
    o, ST = oracle.recurrence(*(x[n] for n in names), G_MIN, S0=x["S0"], lib=lib)
    o1, S1 = oracle.recurrence(*(x[n][:, :37] for n in names), G_MIN, S0=x["S0"], lib=lib)
    o2, S2 = oracle.recurrence(*(x[n][:, 37:] for n in names), G_MIN, S0=S1, lib=lib)
    assert _rel(np.concatenate([o1, o2], 1), o) < 1e-13 and _rel(S2, ST) < 1e-13
    c1, T1 = oracle.chunked(16, *(x[n][:, :64] for n in names), G_MIN, S0=x["S0"], lib=lib)
    c2, T2 = oracle.chunked(16, *(x[n][:, 64:] for n in names), G_MIN, S0=T1, lib=lib)
    assert _rel(np.concatenate([c1, c2], 1), o) < 1e-12 and _rel(T2, ST) < 1e-12


# ------------------------------------------------------------------------- decode
def pin_decode_step(lib):
    """A decode step is the recurrence for one token; a chain of steps is the sequence."""
    x = _inputs(3, 5, 2, 16, seed=40)
    names = ("q", "k", "v", "a", "beta")
    o_seq, S_seq = oracle.recurrence(*(x[n] for n in names), G_MIN, S0=x["S0"], lib=lib)
    S = x["S0"].astype(np.float64)
    for t in range(5):
        o_t, S = oracle.decode(*(x[n][:, t] for n in names), S, G_MIN, lib=lib)
        assert _rel(o_t, o_seq[:, t]) < 1e-13
    assert _rel(S, S_seq) < 1e-13


# ------------------------------------------------------------------- range claim
def pin_range_claim(lib):
    """Bounded gate: 16-token tiles factor densely in float32 without inf/NaN/subnormal,
    even at g ~ g_min (a = +8) with the mid-tile reference and with the tile-start one.
    Unbounded log-sigmoid at a = -8: the same dense factorisation overflows."""
    rng = np.random.default_rng(50)
    n, dk = 16, 128
    k = rng.standard_normal((n, dk)).astype(np.float32)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    for a_val in (8.0, 0.0, -8.0):
        a = np.full((n, dk), a_val, np.float32)
        g = oracle.gate(a, G_MIN, lib=lib)
        # lower triangle of the dense product against the pairwise exponential in fp64
        G = np.cumsum(g.astype(np.float64), axis=0)
        pair = np.einsum("rc,jc,rjc->rj", k.astype(np.float64), k.astype(np.float64),
                         np.exp(G[:, None, :] - G[None, :, :]))
        low = np.tril(np.ones((n, n), bool))
        for ref in (n // 2 - 1, 0):
            (bad, sub, bad_prod), prod = oracle.tile_factors_f32(g, k, ref, lib=lib, return_products=True)
            assert bad == 0 and bad_prod == 0, (a_val, ref)
            assert np.max(np.abs(prod[low] - pair[low])) < 1e-5 * np.max(np.abs(pair[low])), (a_val, ref)
            if ref == n // 2 - 1:  # the mid-tile reference also keeps factors normal
                assert sub == 0, (a_val, ref)
    a = np.full((n, dk), -8.0, np.float32)
    g = oracle.gate(a, G_MIN, oracle.GATE_LOGSIGMOID, lib=lib)
    assert (g < -8.0).all()
    bad, _, bad_prod = oracle.tile_factors_f32(g, k, n // 2 - 1, lib=lib)
    assert bad_prod > 0, "unbounded decay must overflow the dense factorisation"
    bad, _, _ = oracle.tile_factors_f32(g, k, 0, lib=lib)
    assert bad > 0


def pin_gate_head_scale(lib):
    """g_min * sigmoid(e^A * a) per head ("Trillion-Scale ..." 3.2): A = 0 is the plain gate
    bit for bit; other A against scipy's expit of the scaled argument (within one float32
    ulp: e^{log s} is s only to double rounding)."""
    rng = np.random.default_rng(77)
    a = (rng.standard_normal((5, 3, 16)) * 3).astype(np.float32)
    g0 = oracle.gate_heads(a, np.zeros(3, np.float32), G_MIN, lib=lib)
    assert np.array_equal(g0, oracle.gate(a, G_MIN, lib=lib))
    A_log = np.array([np.log(0.5), 0.0, np.log(3.0)], np.float32)
    g = oracle.gate_heads(a, A_log, G_MIN, lib=lib).astype(np.float64)
    scale = np.exp(A_log.astype(np.float64))[None, :, None]
    ref = (G_MIN * scipy.special.expit(a.astype(np.float64) * scale)).astype(np.float32).astype(np.float64)
    assert np.all(np.abs(g - ref) <= np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)), \
        "per-head scaled gate differs from g_min*expit(e^A a)"


# ---------------------------------------------------------------------------- backward
# The backward is the derivative of the recurrence: it is pinned by central finite
# differences of the (separately pinned) forward, by the exact Euler identities of the
# inputs the outputs are linear in, and by a hand-derived closed form at T = 1.


def _grid_inputs(B, T, H, d, seed):
    """Inputs on a 2^-8 grid (|x| < 4), so that x +- 2^-14 is exact in float32."""
    rng = np.random.default_rng(seed)

    def g8(x):
        return (np.round(np.clip(x, -3.9, 3.9) * 256) / 256).astype(np.float32)

    return dict(
        q=g8(rng.normal(size=(B, T, H, d)) * 0.3), k=g8(rng.normal(size=(B, T, H, d)) * 0.3),
        v=g8(rng.normal(size=(B, T, H, d))), a=g8(rng.normal(size=(B, T, H, d)) * 1.5),
        beta=g8(rng.uniform(0.05, 0.95, size=(B, T, H))),
        S0=g8(rng.normal(size=(B, H, d, d)) * 0.2).astype(np.float64),
        dO=g8(rng.normal(size=(B, T, H, d))), dST=g8(rng.normal(size=(B, H, d, d))).astype(np.float64))


def _loss(x, kind, lib):
    o, ST = oracle.recurrence(x["q"], x["k"], x["v"], x["a"], x["beta"], G_MIN, S0=x["S0"], kind=kind, lib=lib)
    return float(np.sum(o * x["dO"]) + np.sum(ST * x["dST"]))


def pin_backward_finite_differences(lib):
    """Every gradient against a central difference of L = <dO, o> + <dST, S_T>, at sampled
    entries, for both gates; T = 70 spans the oracle's 64-token recompute segments."""
    h = 2.0 ** -14
    names = {"q": "dq", "k": "dk", "v": "dv", "a": "da", "beta": "dbeta", "S0": "dS0"}
    for kind in (oracle.GATE_BOUNDED, oracle.GATE_LOGSIGMOID):
        x = _grid_inputs(1, 70, 2, 8, seed=40 + kind)
        grads = oracle.backward(x["q"], x["k"], x["v"], x["a"], x["beta"], x["dO"], G_MIN, S0=x["S0"],
                                dST=x["dST"], kind=kind, lib=lib)
        rng = np.random.default_rng(7 + kind)
        for n, gname in names.items():
            for _ in range(8):
                idx = tuple(int(rng.integers(0, m)) for m in x[n].shape)
                xp, xm = dict(x), dict(x)
                xp[n] = x[n].copy()
                xm[n] = x[n].copy()
                xp[n][idx] += h
                xm[n][idx] -= h
                fd = (_loss(xp, kind, lib) - _loss(xm, kind, lib)) / (2 * h)
                got = grads[gname][idx]
                assert abs(got - fd) <= 1e-6 * max(abs(fd), 1e-3), f"d{n}{idx} (kind {kind}): {got} vs {fd}"


def pin_backward_linear_inputs(lib):
    """o and S_T are linear in (v, S0) jointly and o is linear in q, so (Euler) the loss
    equals <dv, v> + <dS0, S0> exactly, and with dST = 0 it equals <dq, q>."""
    x = _inputs(2, 45, 2, 16, seed=41)
    rng = np.random.default_rng(42)
    dO = rng.normal(size=x["v"].shape).astype(np.float32)
    dST = rng.normal(size=x["S0"].shape)
    o, ST = oracle.recurrence(x["q"], x["k"], x["v"], x["a"], x["beta"], G_MIN, S0=x["S0"], lib=lib)
    g = oracle.backward(x["q"], x["k"], x["v"], x["a"], x["beta"], dO, G_MIN, S0=x["S0"], dST=dST, lib=lib)
    L = np.sum(o * dO) + np.sum(ST * dST)
    euler_vs = np.sum(g["dv"] * x["v"]) + np.sum(g["dS0"] * x["S0"])
    assert abs(L - euler_vs) <= 1e-10 * max(abs(L), 1.0), (L, euler_vs)
    g0 = oracle.backward(x["q"], x["k"], x["v"], x["a"], x["beta"], dO, G_MIN, S0=x["S0"], lib=lib)
    Lo = np.sum(o * dO)
    assert abs(Lo - np.sum(g0["dq"] * x["q"])) <= 1e-10 * max(abs(Lo), 1.0)


def pin_backward_single_token_closed_form(lib):
    """T = 1 from a zero state, by hand: o = b (k.q) v and S_T = b k v^T, so with weights
    w = dO, W = dST the gradients are dq = b (v.w) k, dk = b (v.w) q + b W v,
    dv = b (k.q) w + b W^T k, dbeta = (k.q)(v.w) + k^T W v and da = 0; and since
    S_T = (I - b k k^T) D S0 + b k v^T, dS0 = D (I - b k k^T) (q w^T + W), D = Diag(e^g)."""
    rng = np.random.default_rng(43)
    d = 5
    q, k, v, a, w = (rng.normal(size=(1, 1, 1, d)).astype(np.float32) for _ in range(5))
    beta = np.array([[[0.625]]], np.float32)
    W = rng.normal(size=(1, 1, d, d))
    g = oracle.backward(q, k, v, a, beta, w, G_MIN, dST=W, lib=lib)
    qq, kk, vv, ww = (np.asarray(x, np.float64).reshape(-1) for x in (q, k, v, w))
    WW = W[0, 0]
    b = 0.625
    kq, vw = kk @ qq, vv @ ww
    assert np.allclose(g["dq"].reshape(-1), b * vw * kk, rtol=1e-12, atol=1e-14)
    assert np.allclose(g["dk"].reshape(-1), b * vw * qq + b * WW @ vv, rtol=1e-12, atol=1e-14)
    assert np.allclose(g["dv"].reshape(-1), b * kq * ww + b * WW.T @ kk, rtol=1e-12, atol=1e-14)
    assert np.isclose(g["dbeta"].reshape(()), kq * vw + kk @ WW @ vv, rtol=1e-12, atol=1e-14)
    assert np.all(g["da"] == 0.0)
    D = np.exp(G_MIN * scipy.special.expit(np.asarray(a, np.float64).reshape(-1)))
    ref = D[:, None] * ((np.eye(d) - b * np.outer(kk, kk)) @ (np.outer(qq, ww) + WW))
    assert np.allclose(g["dS0"][0, 0], ref, rtol=1e-12, atol=1e-14)


def pin_backward_chunked_equals_recurrence(lib):
    """The chunked form of the backward (fp64 numpy, chunk algebra written out) equals the
    token-level derivative at every chunk size, both gates, ragged tails included."""
    from oracle.chunked_backward import chunked_backward
    for kind in (oracle.GATE_BOUNDED, oracle.GATE_LOGSIGMOID):
        for C, T in ((1, 5), (7, 64), (16, 37), (64, 150)):
            x = _inputs(2, T, 2, 8, seed=80 + C + T, s0_std=0.2)
            rng = np.random.default_rng(C + T)
            dO = rng.normal(size=x["v"].shape).astype(np.float32)
            dST = rng.normal(size=x["S0"].shape)
            ref = oracle.backward(x["q"], x["k"], x["v"], x["a"], x["beta"], dO, G_MIN, S0=x["S0"], dST=dST,
                                  kind=kind, lib=lib)
            got = chunked_backward(C, x["q"], x["k"], x["v"], x["a"], x["beta"], dO, G_MIN, S0=x["S0"], dST=dST,
                                   kind=kind)
            for n in ref:
                assert _rel(got[n], ref[n]) < 1e-11, (kind, C, T, n, _rel(got[n], ref[n]))


ALL_PINS = [
    pin_gate_special_values,
    pin_gate_vs_library,
    pin_gate_range_exhaustive,
    pin_beta_zero_closed_form,
    pin_small_beta_is_linear_attention,
    pin_delta_rule_retrieval,
    pin_delta_rule_general_beta,
    pin_basis_key_hand_cases,
    pin_linearity,
    pin_decay_nonincreasing,
    pin_chunked_equals_recurrence,
    pin_segment_carry,
    pin_decode_step,
    pin_range_claim,
    pin_gate_head_scale,
    pin_backward_finite_differences,
    pin_backward_linear_inputs,
    pin_backward_single_token_closed_form,
    pin_backward_chunked_equals_recurrence,
]
