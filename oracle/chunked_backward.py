"""Chunked form of the backward, fp64 numpy -- TEST INFRASTRUCTURE ONLY (like the rest of
``oracle/``): only ``tests/`` may call it.

It states, in plain fp64 array code, the algebra the chunked backward computes: the
derivative of the chunked forward ("Trillion-Scale MoE Multimodal Models ..." section 3.1,
the chunked computation with a cumulative decay; "Trillion-Parameter MoE Multimodal Models:
Engineering ..." section 3.2, training recursing in chunks), taken chunk by chunk in reverse.
It is pinned against ``oracle.backward`` (the token-level derivative, itself pinned by finite
differences), so the chunk algebra is checked independently of any GPU code.

Inside a chunk of L tokens with entering state S, G the inclusive cumulative log-decay and
E_rs = e^{G_r - G_s} per channel:
    A'_rs = sum_c k_rc k_sc E_rsc (s < r),   P_rs = sum_c q_rc k_sc E_rsc (s <= r)
    T = (I + diag(beta) A')^{-1},  W = T diag(beta) Kbar,  Utilde = T diag(beta) V
    U = Utilde - W S,  O = Qbar S + P U,  S' = Diag(e^{G_last}) S + Khat^T U
with Kbar = k e^{G}, Qbar = q e^{G}, Khat = k e^{G_last - G}.  Given dO and dS' the reverse is
written out step by step below.
"""
from __future__ import annotations

import numpy as np

GATE_BOUNDED = 0
GATE_LOGSIGMOID = 1


def _gate(a, g_min, kind):
    s = 1.0 / (1.0 + np.exp(-a))
    if kind == GATE_BOUNDED:
        return g_min * s, g_min * s * (1.0 - s)
    return -np.logaddexp(0.0, -a), 1.0 - s


def _chunk_forward(q, k, v, g, beta, S):
    """The chunk's quantities (all fp64) and its exit state."""
    L = q.shape[0]
    G = np.cumsum(g, axis=0)
    Gl = G[L - 1]
    # [r, s, c]; only s <= r is used, where G_r - G_s <= 0 (g <= 0); the clamp keeps the
    # unused upper part finite
    E = np.exp(np.minimum(G[:, None, :] - G[None, :, :], 0.0))
    low = np.tril(np.ones((L, L)), -1)
    Ap = np.einsum("rc,sc,rsc->rs", k, k, E) * low
    P = np.einsum("rc,sc,rsc->rs", q, k, E) * (low + np.eye(L))
    T = np.linalg.inv(np.eye(L) + beta[:, None] * Ap)
    Kb, Qb, Kh = k * np.exp(G), q * np.exp(G), k * np.exp(Gl - G)
    W = T @ (beta[:, None] * Kb)
    Ut = T @ (beta[:, None] * v)
    U = Ut - W @ S
    S_next = np.exp(Gl)[:, None] * S + Kh.T @ U
    return dict(G=G, Gl=Gl, E=E, Ap=Ap, P=P, T=T, Kb=Kb, Qb=Qb, Kh=Kh, W=W, U=U), S_next


def _chunk_backward(q, k, v, a, beta, dO, S, dSn, f, g_min, kind):
    """Reverse of one chunk: gradients of its tokens and of its entering state."""
    L = q.shape[0]
    low = np.tril(np.ones((L, L)), -1)
    T, Kb, Kh, Qb, U, W, P, Ap, E, G, Gl = (f[n] for n in ("T", "Kb", "Kh", "Qb", "U", "W", "P", "Ap", "E", "G",
                                                           "Gl"))
    # S' = Diag(Gamma) S + Khat^T U
    dU = Kh @ dSn
    dKh = U @ dSn.T
    dGam = np.sum(dSn * S, axis=1)
    dS = np.exp(Gl)[:, None] * dSn
    # O = Qbar S + P U
    dQb = dO @ S.T
    dS += Qb.T @ dO
    dP = (dO @ U.T) * (low + np.eye(L))
    dU += P.T @ dO
    # U = Utilde - W S
    dW = -dU @ S.T
    dS -= W.T @ dU
    # W = T Bk, Utilde = T Bv (Bk = diag(beta) Kbar, Bv = diag(beta) V), T = (I + A)^{-1}
    dBk, dBv = T.T @ dW, T.T @ dU
    dT = dW @ (beta[:, None] * Kb).T + dU @ (beta[:, None] * v).T
    dA = -(T.T @ dT @ T.T) * low
    dbeta = np.sum(dBk * Kb, axis=1) + np.sum(dBv * v, axis=1) + np.sum(dA * Ap, axis=1)
    dv = beta[:, None] * dBv
    dKb = beta[:, None] * dBk
    dAp = beta[:, None] * dA
    # the pairwise products: d/dq, d/dk and d/dG of sum_c x_rc y_sc E_rsc
    dq = np.einsum("rs,sc,rsc->rc", dP, k, E)
    dk_row = np.einsum("rs,sc,rsc->rc", dAp, k, E)
    dk_col = np.einsum("rs,rc,rsc->sc", dP, q, E) + np.einsum("rs,rc,rsc->sc", dAp, k, E)
    dG = q * dq + k * dk_row - k * dk_col
    dk = dk_row + dk_col
    # Qbar = q e^G, Kbar = k e^G, Khat = k e^{G_last - G}, Gamma = e^{G_last}
    eG, eh = np.exp(G), np.exp(Gl - G)
    dq = dq + dQb * eG
    dk = dk + dKb * eG + dKh * eh
    dG += dQb * Qb + dKb * Kb - dKh * Kh
    dG[L - 1] += np.sum(dKh * Kh, axis=0) + dGam * np.exp(Gl)
    # G = cumsum(g): dg is the reverse cumulative sum; then through the gate
    dg = np.cumsum(dG[::-1], axis=0)[::-1]
    _, gp = _gate(a, g_min, kind)
    return dq, dk, dv, dg * gp, dbeta, dS


def chunked_backward(C, q, k, v, a, beta, dO, g_min=-5.0, S0=None, dST=None, kind=GATE_BOUNDED):
    """The backward in chunks of C tokens.  Shapes as ``oracle.backward``; returns the same dict."""
    q, k, v, a, dO = (np.asarray(x, np.float64) for x in (q, k, v, a, dO))
    beta = np.asarray(beta, np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = {"dq": np.zeros((B, T, H, dk)), "dk": np.zeros((B, T, H, dk)), "dv": np.zeros((B, T, H, dv)),
           "da": np.zeros((B, T, H, dk)), "dbeta": np.zeros((B, T, H)), "dS0": np.zeros((B, H, dk, dv))}
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.asarray(S0[b, h], np.float64).copy()
            spans = [(t0, min(T, t0 + C)) for t0 in range(0, T, C)]
            saved = []
            for t0, t1 in spans:
                g, _ = _gate(a[b, t0:t1, h], g_min, kind)
                f, S_next = _chunk_forward(q[b, t0:t1, h], k[b, t0:t1, h], v[b, t0:t1, h], g, beta[b, t0:t1, h], S)
                saved.append((f, S))
                S = S_next
            dS = np.zeros((dk, dv)) if dST is None else np.asarray(dST[b, h], np.float64).copy()
            for (t0, t1), (f, S_in) in zip(reversed(spans), reversed(saved)):
                r = _chunk_backward(q[b, t0:t1, h], k[b, t0:t1, h], v[b, t0:t1, h], a[b, t0:t1, h],
                                    beta[b, t0:t1, h], dO[b, t0:t1, h], S_in, dS, f, g_min, kind)
                (out["dq"][b, t0:t1, h], out["dk"][b, t0:t1, h], out["dv"][b, t0:t1, h], out["da"][b, t0:t1, h],
                 out["dbeta"][b, t0:t1, h], dS) = r
            out["dS0"][b, h] = dS
    return out
