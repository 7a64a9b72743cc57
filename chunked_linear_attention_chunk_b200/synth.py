"""Seeded synthetic inputs shaped like the pages' 8K -> 64K -> 256K -> 1M context stages.

This module is shared by the tests, the benchmark and the oracle checks; it holds none
of the method's arithmetic.  It only draws random numbers and puts them in the form the
library's contract asks for:

* q, k ~ N(0, 1), L2-normalised per [dk] head vector in float32 (the caller normalises;
  the library does not), then cast to the compute dtype;
* v ~ N(0, 1);
* beta = sigmoid(N(0, 1)) (beta is passed post-activation, in (0, 1));
* a ~ N(0, 2) (standard deviation 2), the gate pre-activation;
* S0 ~ N(0, 0.1) (standard deviation 0.1) or zero;
* for the 64K stage, one contiguous run of ceil(5% of T) tokens starting at token 32773
  (deliberately not 16-aligned) has a = +8 on every head and channel, so g sits at the
  lower bound there and tiles straddle the run's edges.

Every tensor comes from its own numpy ``default_rng([seed, stream_id, block])`` streams
(one per block of 2^22 elements), so a tensor depends neither on which other tensors
were drawn nor on how many threads drew it.  bf16 rounding is
round-to-nearest-even (torch's float32 -> bfloat16 cast).  All tensors are returned on
the CPU; bf16 values are exact in float32, which is what the oracle consumes.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch

# Stream ids: one independent random stream per tensor.
_Q, _K, _V, _A, _BETA, _S0 = 1, 2, 3, 4, 5, 6


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str  # "bf16" or "f32"
    seed: int
    s0_std: float
    adversarial: bool = False
    segment: int = 0  # >0: processed as T/segment calls with the state carried


# The five workloads (the pages' context stages plus a tiny debug case and decode).
TINY = Workload("tiny_B1_H2_T256_d64_f32", 1, 256, 2, 64, 64, "f32", 1000, 0.0)
STAGE_8K = Workload("8k_B4_H16_T8192_d128_bf16", 4, 8192, 16, 128, 128, "bf16", 1001, 0.1)
STAGE_64K = Workload("64k_B1_H32_T65536_d128_bf16_adv5pct", 1, 65536, 32, 128, 128, "bf16", 1002, 0.1, adversarial=True)
# a quarter of the 64K stage (its 32 heads, 16384 tokens): a small case of the same kernel forms
PROFILE_16K = Workload("16k_B1_H32_T16384_d128_bf16", 1, 16384, 32, 128, 128, "bf16", 1005, 0.1)
STAGE_1M = Workload("1m_B1_H16_T1048576_d128_bf16_seg64k", 1, 1048576, 16, 128, 128, "bf16", 1004, 0.1, segment=65536)


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    N: int
    H: int
    dk: int
    dv: int
    seed: int
    s_std: float
    steps: int


DECODE = DecodeWorkload("decode_N256_H32_d128_fp32state", 256, 32, 128, 128, 1003, 0.1, 1000)

ADV_START = 32773
ADV_FRACTION = 0.05
ADV_VALUE = 8.0


_BLOCK = 1 << 22  # elements per independently seeded block


def _normal(seed, stream, shape, std=1.0):
    """N(0, std^2) float32 draws; block i of the flattened array comes from
    default_rng([seed, stream, i]), so the values do not depend on the thread count."""
    n = int(np.prod(shape))
    x = np.empty(n, np.float32)

    def fill(i):
        lo, hi = i * _BLOCK, min(n, (i + 1) * _BLOCK)
        np.random.default_rng([int(seed), int(stream), i]).standard_normal(out=x[lo:hi], dtype=np.float32)
        if std != 1.0:
            x[lo:hi] *= np.float32(std)

    nb = (n + _BLOCK - 1) // _BLOCK
    if nb <= 1:
        for i in range(nb):
            fill(i)
    else:
        with ThreadPoolExecutor(max_workers=min(nb, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(nb)))
    return x.reshape(shape)


def _unit_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float32) ** 2, axis=-1, keepdims=True, dtype=np.float32))
    return (x / np.maximum(n, np.float32(1e-30))).astype(np.float32)


def _sigmoid32(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _cast(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.bfloat16) if dtype == "bf16" else t.to(torch.float32)


def adversarial_range(T: int):
    """The [start, stop) token range that carries a = +8 in the 64K stage."""
    n = int(math.ceil(ADV_FRACTION * T))
    start = min(ADV_START, max(T - n, 0))
    return start, min(start + n, T)


def make_inputs(B, T, H, dk, dv, dtype="bf16", seed=0, s0_std=0.1, adversarial=False):
    """Draw one batch.  Returns a dict of CPU tensors:
    q, k, a [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H] (all ``dtype``); S0 [B,H,dk,dv] float32
    (zeros when ``s0_std`` is 0; left out when it is None)."""
    q = _unit_rows(_normal(seed, _Q, (B, T, H, dk)))
    k = _unit_rows(_normal(seed, _K, (B, T, H, dk)))
    v = _normal(seed, _V, (B, T, H, dv))
    a = _normal(seed, _A, (B, T, H, dk), std=2.0)
    if adversarial:
        s, e = adversarial_range(T)
        a[:, s:e] = np.float32(ADV_VALUE)
    beta = _sigmoid32(_normal(seed, _BETA, (B, T, H)))
    out = {n: _cast(x, dtype) for n, x in (("q", q), ("k", k), ("v", v), ("a", a), ("beta", beta))}
    if s0_std is None:  # token tensors only
        return out
    if s0_std > 0:
        S0 = _normal(seed, _S0, (B, H, dk, dv), std=s0_std)
    else:
        S0 = np.zeros((B, H, dk, dv), np.float32)
    out["S0"] = torch.from_numpy(S0)
    return out


def workload_inputs(w: Workload, segment_index: int | None = None, T: int | None = None):
    """Inputs of a workload.  For segmented workloads pass ``segment_index``: each segment
    of ``w.segment`` tokens is drawn from its own seed (seed*1000 + index) so segments can be
    regenerated independently; the initial state belongs to segment 0's draw."""
    if w.segment and segment_index is not None:
        seed = w.seed * 1000 + segment_index
        return make_inputs(w.B, T or w.segment, w.H, w.dk, w.dv, w.dtype, seed, w.s0_std, False)
    return make_inputs(w.B, T or w.T, w.H, w.dk, w.dv, w.dtype, w.seed, w.s0_std, w.adversarial)


def decode_state(w: DecodeWorkload):
    """Initial fp32 decode state [N,H,dk,dv] ~ N(0, s_std)."""
    return torch.from_numpy(_normal(w.seed, _S0, (w.N, w.H, w.dk, w.dv), std=w.s_std))


def decode_tokens(w: DecodeWorkload, step: int, dtype="bf16"):
    """Token set of one decode step: q, k, a [N,H,dk]; v [N,H,dv]; beta [N,H]."""
    seed = w.seed * 1000 + step
    x = make_inputs(w.N, 1, w.H, w.dk, w.dv, dtype, seed, None, False)
    return {n: x[n][:, 0].contiguous() for n in ("q", "k", "v", "a", "beta")}


def decode_token_sets(w: DecodeWorkload, steps, seed_of=None, workers=None):
    """Token sets of consecutive decode steps, in order (``decode_tokens(w, seed_of(i))`` for
    each i in ``steps``), drawn a bounded number of steps ahead on a thread pool."""
    steps = list(steps)
    seed_of = seed_of or (lambda i: i)
    workers = workers or min(16, os.cpu_count() or 1)
    ahead = 2 * workers
    with ThreadPoolExecutor(max_workers=workers) as ex:
        futs = [ex.submit(decode_tokens, w, seed_of(i)) for i in steps[:ahead]]
        for j in range(len(steps)):
            if j + ahead < len(steps):
                futs.append(ex.submit(decode_tokens, w, seed_of(steps[j + ahead])))
            yield futs[j].result()
            futs[j] = None


def to_numpy32(t: torch.Tensor) -> np.ndarray:
    """Exact float32 copy of a (bf16 or f32) CPU tensor, for the oracle."""
    return t.detach().to("cpu", torch.float32).contiguous().numpy()


# ---------------------------------------------------------------------------- packed batches
# Packed variable-length stage: documents of mixed length packed back to back to fill one
# 64K-token axis.  Lengths are log-uniform between 16 and 16384 tokens (most documents are
# short, most tokens sit in long ones), drawn from their own stream; the last document is
# cut to fill the axis exactly.  Token tensors are the 64K stage's draw (without the a = +8
# run); every document starts from its own S0 slice.
VARLEN_64K_T = 65536
VARLEN_64K_H = 32
VARLEN_SEED = 1005


def document_lengths(T: int, seed: int = VARLEN_SEED, lo: int = 16, hi: int = 16384) -> np.ndarray:
    rng = np.random.default_rng([seed, 99])
    out, total = [], 0
    while total < T:
        L = int(np.exp(rng.uniform(np.log(lo), np.log(hi))))
        L = min(L, T - total)
        out.append(L)
        total += L
    return np.asarray(out, np.int64)


def cu_seqlens(lengths) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
