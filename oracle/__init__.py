"""fp64 CPU oracle for the KDA forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The CUDA library never imports, links or calls it, and the
two share no code: the oracle is plain C (``kda_oracle.c``) compiled with gcc and
called through ctypes on host numpy arrays.

Functions (each wraps the C routine of the same name; see ``kda_oracle.c`` for the
passages of the pages each one follows):

* ``gate(a, g_min, kind)``      -- g = g_min * sigmoid(a) (or log sigmoid(a)), fp64
  rounded once to float32.
* ``recurrence(...)``           -- the token-by-token recurrence, fp64.
* ``chunked(C, ...)``           -- the chunked form with pairwise exponentials, fp64.
* ``decode(...)``               -- one decode step, state updated in place.
* ``backward(...)``             -- gradients of the recurrence (reverse mode, by hand).

``oracle.chunked_backward`` (fp64 numpy) writes the same gradients out in the chunked form,
chunk by chunk in reverse; it is pinned equal to ``backward``.
* ``tile_factors_f32(...)``     -- counts of non-finite / subnormal values when a
  16-token tile's pairwise decay is factored densely in float32.

Layouts: q, k, a ``[B, T, H, dk]``; v, o ``[B, T, H, dv]``; beta ``[B, T, H]``;
state ``[B, H, dk, dv]``.  Inputs are float32 (bf16 values are exact in float32).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

GATE_BOUNDED = 0
GATE_LOGSIGMOID = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libkda_oracle.so")

# Plain optimisation only; AVX2/FMA is present on every host this runs on.
CFLAGS = ["-O3", "-march=x86-64-v3", "-fPIC", "-shared", "-std=c11", "-pthread"]


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the oracle with gcc into ``out`` (skipped when up to date)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if (
        not extra_flags
        and os.path.exists(out)
        and os.path.getmtime(out) >= os.path.getmtime(src)
    ):
        return out
    cmd = ["gcc", *CFLAGS, *extra_flags, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double
_L = ctypes.c_int64


def load(path: str | None = None) -> ctypes.CDLL:
    """Load (building first if needed) an oracle shared library."""
    if path is None:
        path = build()
    lib = ctypes.CDLL(path)
    lib.oracle_gate_f32.argtypes = [_P, _L, _D, _I, _P]
    lib.oracle_gate_f32.restype = None
    lib.oracle_gate_f64.argtypes = [_P, _L, _D, _I, _P]
    lib.oracle_gate_f64.restype = None
    lib.oracle_recurrence.argtypes = [_I] * 5 + [_P] * 5 + [_D, _I, _P, _P, _P, _I]
    lib.oracle_recurrence.restype = _I
    lib.oracle_chunked.argtypes = [_I] * 6 + [_P] * 5 + [_D, _I, _P, _P, _P, _I]
    lib.oracle_chunked.restype = _I
    lib.oracle_decode.argtypes = [_I] * 4 + [_P] * 5 + [_D, _I, _P, _P, _I]
    lib.oracle_decode.restype = _I
    lib.oracle_tile_factors_f32.argtypes = [_P, _P, _I, _I, _I, _P, _P]
    lib.oracle_tile_factors_f32.restype = _I
    lib.oracle_gate_heads_f32.argtypes = [_P, _L, _I, _I, _D, _P, _P]
    lib.oracle_gate_heads_f32.restype = None
    lib.oracle_backward.argtypes = [_I] * 5 + [_P] * 5 + [_D, _I] + [_P] * 9 + [_I]
    lib.oracle_backward.restype = _I
    return lib


_lib = None


def _get(lib):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = load()
    return _lib


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(x):
    return x.ctypes.data_as(ctypes.c_void_p) if x is not None else None


def gate(a, g_min: float = -5.0, kind: int = GATE_BOUNDED, lib=None) -> np.ndarray:
    """g = g_min * sigmoid(a) (kind 0) or log(sigmoid(a)) (kind 1), fp64 -> float32."""
    a = _f32(a)
    g = np.empty(a.shape, np.float32)
    _get(lib).oracle_gate_f32(_ptr(a), a.size, float(g_min), int(kind), _ptr(g))
    return g


def gate_f64(a, g_min: float = -5.0, kind: int = GATE_BOUNDED, lib=None) -> np.ndarray:
    a = _f32(a)
    g = np.empty(a.shape, np.float64)
    _get(lib).oracle_gate_f64(_ptr(a), a.size, float(g_min), int(kind), _ptr(g))
    return g


def gate_heads(a, A_log, g_min: float = -5.0, lib=None) -> np.ndarray:
    """g = g_min * sigmoid(e^{A_log[h]} * a) for a [..., H, dk] (fp64, rounded once)."""
    a = _f32(a)
    A_log = _f32(A_log)
    H, dk = a.shape[-2], a.shape[-1]
    assert A_log.shape == (H,), "A_log is one value per head"
    g = np.empty(a.shape, np.float32)
    _get(lib).oracle_gate_heads_f32(_ptr(a), a.size // (H * dk), H, dk, float(g_min), _ptr(A_log), _ptr(g))
    return g


def _seq_args(q, k, v, a, beta, S0):
    q, k, v, a, beta = (_f32(x) for x in (q, k, v, a, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and a.shape == q.shape, "q, k, a must share [B,T,H,dk]"
    assert v.shape == (B, T, H, dv), "v must be [B,T,H,dv]"
    assert beta.shape == (B, T, H), "beta must be [B,T,H]"
    if S0 is not None:
        S0 = np.ascontiguousarray(S0, dtype=np.float64)
        assert S0.shape == (B, H, dk, dv), "S0 must be [B,H,dk,dv]"
    return q, k, v, a, beta, S0, (B, T, H, dk, dv)


def recurrence(q, k, v, a, beta, g_min=-5.0, S0=None, kind=GATE_BOUNDED, nthreads=0, lib=None):
    """Token-by-token recurrence. Returns (o [B,T,H,dv] fp64, S_T [B,H,dk,dv] fp64)."""
    q, k, v, a, beta, S0, (B, T, H, dk, dv) = _seq_args(q, k, v, a, beta, S0)
    o = np.empty((B, T, H, dv), np.float64)
    ST = np.empty((B, H, dk, dv), np.float64)
    st = _get(lib).oracle_recurrence(
        B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta),
        float(g_min), int(kind), _ptr(S0), _ptr(o), _ptr(ST), int(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle_recurrence failed with status {st}")
    return o, ST


def chunked(C, q, k, v, a, beta, g_min=-5.0, S0=None, kind=GATE_BOUNDED, nthreads=0, lib=None):
    """Chunked form with chunk size C. Returns (o, S_T) like ``recurrence``."""
    q, k, v, a, beta, S0, (B, T, H, dk, dv) = _seq_args(q, k, v, a, beta, S0)
    o = np.empty((B, T, H, dv), np.float64)
    ST = np.empty((B, H, dk, dv), np.float64)
    st = _get(lib).oracle_chunked(
        int(C), B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta),
        float(g_min), int(kind), _ptr(S0), _ptr(o), _ptr(ST), int(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle_chunked failed with status {st}")
    return o, ST


def backward(q, k, v, a, beta, dO, g_min=-5.0, S0=None, dST=None, kind=GATE_BOUNDED, nthreads=0, lib=None):
    """Gradients of a loss L given dO = dL/do [B,T,H,dv] and dST = dL/dS_T (None: zero).

    Returns a dict of fp64 arrays: dq, dk, da [B,T,H,dk], dv [B,T,H,dv], dbeta [B,T,H],
    dS0 [B,H,dk,dv] (the gradient with respect to the initial state, zero or not)."""
    q, k, v, a, beta, S0, (B, T, H, dk, dv) = _seq_args(q, k, v, a, beta, S0)
    dO = _f32(dO)
    assert dO.shape == (B, T, H, dv), "dO must be [B,T,H,dv]"
    if dST is not None:
        dST = np.ascontiguousarray(dST, dtype=np.float64)
        assert dST.shape == (B, H, dk, dv), "dST must be [B,H,dk,dv]"
    out = {
        "dq": np.zeros((B, T, H, dk)), "dk": np.zeros((B, T, H, dk)), "dv": np.zeros((B, T, H, dv)),
        "da": np.zeros((B, T, H, dk)), "dbeta": np.zeros((B, T, H)), "dS0": np.zeros((B, H, dk, dv)),
    }
    st = _get(lib).oracle_backward(
        B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta), float(g_min), int(kind),
        _ptr(S0), _ptr(dO), _ptr(dST), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
        _ptr(out["da"]), _ptr(out["dbeta"]), _ptr(out["dS0"]), int(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle_backward failed with status {st}")
    return out


def decode(q, k, v, a, beta, S, g_min=-5.0, kind=GATE_BOUNDED, nthreads=0, lib=None):
    """One decode step on [N,H,d] tokens. Returns (o [N,H,dv], S' [N,H,dk,dv]); S is not modified."""
    q, k, v, a, beta = (_f32(x) for x in (q, k, v, a, beta))
    N, H, dk = q.shape
    dv = v.shape[-1]
    S_new = np.array(S, dtype=np.float64, copy=True, order="C")
    assert S_new.shape == (N, H, dk, dv)
    o = np.empty((N, H, dv), np.float64)
    st = _get(lib).oracle_decode(
        N, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta),
        float(g_min), int(kind), _ptr(S_new), _ptr(o), int(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle_decode failed with status {st}")
    return o, S_new


def tile_factors_f32(g_tile, k_tile, ref: int, lib=None, return_products=False):
    """(non-finite factors, subnormal factors, non-finite dense products) for one tile;
    with ``return_products`` also the [n, n] float32 dense products."""
    g_tile, k_tile = _f32(g_tile), _f32(k_tile)
    n, dk = g_tile.shape
    counts = np.zeros(3, np.int64)
    prod = np.empty((n, n), np.float32)
    st = _get(lib).oracle_tile_factors_f32(_ptr(g_tile), _ptr(k_tile), n, dk, int(ref), _ptr(counts), _ptr(prod))
    if st != 0:
        raise RuntimeError(f"oracle_tile_factors_f32 failed with status {st}")
    c = tuple(int(x) for x in counts)
    return (c, prod) if return_products else c
