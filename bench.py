#!/usr/bin/env python
"""Benchmark of libkda's chunked KDA forward at the 64K context stage.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {libkda,reference}]

One step = one chunked forward over the 64K-stage batch (B=1, H=32, T=65536,
dk=dv=128, bf16 inputs, fp32 state, the 5% a=+8 slice): gate, cumulative decay,
dense 16-token tile products, WY/UT solve and the state scan, i.e. the whole hot path.
It is issued as kda_chunk_fwd_prep + kda_chunk_fwd_scan (the same launches kda_chunk_fwd
makes: the gate table and the prep, then the scan) so that CUDA events between them time
each stage during the timed steps.  The 8K and 1M context stages are timed too, under
``stages``.
Inputs (2.69 GB) exceed the 126 MB L2, so no flush is needed between steps.
The log-sigmoid ablation (element-wise diagonal tiles) is timed on the same inputs and
reported under ``ablation``.

Prints ONE JSON line (rank 0).  ``value`` is whole-job tokens/s with inputs resident in
HBM; ``e2e`` is the same metric through the C ABI with pinned host buffers (H2D of every
input and D2H of o and S_T inside the timed region).  The decode step (N=256, H=32,
d=128, fp32 state) is measured in the same run and reported under ``decode``.

Multi-GPU (torchrun): every rank runs its own 64K batch (independent sequences, no
data-path collective: weak scaling); the step time is the max over ranks.
``--impl reference`` times the fp64 CPU oracle (the only reference this method has) on
a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from chunked_linear_attention_chunk_b200 import synth  # noqa: E402

METRIC = "KDA chunk-fwd tokens/s & TFLOP/s (% of B200 BF16 peak) at T=64K; decode HBM GB/s"
UNIT = "tokens/s"
G_MIN = -5.0
# Algorithmic cost of the path per token-head at d = 128 (bf16 token tensors):
# q, k, v, a (256 B each), beta (2 B), o (256 B); states add 2 * dk*dv*4 B per head.
BYTES_PER_TOKEN_HEAD = 4 * 256 + 2 + 256
# The prep kernel's share of them (it reads the inputs; the scan writes o and the states).
# The workspace records between the two kernels are the implementation's own traffic.
PREP_BYTES_PER_TOKEN_HEAD = 4 * 256 + 2
# Backward, per token-head at d = 128: q, k, v, a, dO read (bf16) and beta; dq, dk, dv, da
# written (float32) and dbeta.
BWD_BYTES_PER_TOKEN_HEAD = 5 * 256 + 2 + 4 * 512 + 4
# The per-chunk gradient kernel also reads the chunk's saved state and state gradient
# (2 x dk dv x 4 B per 64 tokens).
BWD_CHUNK_BYTES_PER_TOKEN_HEAD = BWD_BYTES_PER_TOKEN_HEAD + 2 * 128 * 128 * 4 // 64
# Triangle-aware flops per token-head at the 16-token tile (state products W S, Qbar S,
# Khat^T U: 6 dk dv; tile products and W: dk (3C - 1); Utilde and P U: 2 C dv; solve
# C^2/3; Gamma scaling dk dv / C), C = 16.
FLOPS_PER_TOKEN_HEAD = 6 * 128 * 128 + 128 * (3 * 16 - 1) + 2 * 16 * 128 + 16 * 16 / 3 + 128 * 128 / 16
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "chunk_fwd_traffic.json")
WORKLOADS = {"64k": synth.STAGE_64K, "8k": synth.STAGE_8K, "16k": synth.PROFILE_16K}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


KERNEL_SOURCES = ("chunk_bf16.cu", "kda_common.cuh", "tcgen05.cuh")


def strip_comments(src: str) -> str:
    """C/C++/CUDA source without its // and /* */ comments (string and character literals
    kept as they are), so that a comment edit leaves the hash of the code unchanged."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "".join(out)


def kernel_source_hash() -> str:
    """Hash of the chunk kernels' code (comments removed, whitespace collapsed): a traffic
    figure is valid only for this code."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "chunked_linear_attention_chunk_b200", "csrc")
    for f in KERNEL_SOURCES:
        code = " ".join(strip_comments(open(os.path.join(csrc, f)).read()).split())  # layout-free
        h.update(code.encode())
    return h.hexdigest()[:16]


def measured_traffic_per_token_head(kernel: str):
    """DRAM bytes (read + write) per token-head of one launch of ``kernel`` ("prep", "scan",
    "bwd_chunk" or "dscan") from the committed ncu summary, or None when the kernels changed
    since."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    d = json.load(open(PROFILE_TRAFFIC))
    if d.get("source_hash") != kernel_source_hash() or kernel not in d:
        return None
    return float(d[kernel]["dram_bytes_per_token_head"])


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        # raw samples go to KDA_BENCH_OUT (default: the system temp directory); their summary
        # goes into the JSON line
        out = os.environ.get("KDA_BENCH_OUT") or tempfile.gettempdir()
        os.makedirs(out, exist_ok=True)
        self.path = os.path.join(out, f"clocks_rank{self.gpu}_{os.getpid()}.csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- dist
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own independent batch (weak scaling over sequences)."""
    return base + 7919 * rank


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------- arms
def time_steps(fn, steps: int, warmup: int, world: int, device, timed_flag=None):
    for _ in range(warmup):
        fn()
    if timed_flag is not None:
        timed_flag["on"] = True
    torch.cuda.synchronize(device)
    barrier(world)
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier(world)
    ms = e0.elapsed_time(e1) / steps
    return max_over_ranks(ms, world, device)


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def normwise_err(x, y, axes):
    """Worst per-head normwise relative error max|x - y| / max|y| (the parity metric)."""
    import numpy as np
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    num = np.max(np.abs(x - y), axis=axes)
    den = np.maximum(np.max(np.abs(y), axis=axes), 1e-30)
    return float(np.max(num / den))


def cpu_baseline(x, sample_tokens: int, gpu_out=None):
    """The fp64 oracle, as it stands, on the first ``sample_tokens`` tokens of every head,
    plus its chunked form (C = 16) on a shorter sample as a second CPU figure.  When the
    sample is the whole workload and ``gpu_out`` = (o, S_T) of the GPU on the same inputs, the
    line also records their parity with the oracle."""
    import oracle
    from chunked_linear_attention_chunk_b200.synth import to_numpy32
    names = ("q", "k", "v", "a", "beta")
    arrs = [to_numpy32(x[n][:, :sample_tokens]) for n in names]
    S0 = x["S0"].numpy().astype("float64")
    B, _, H, _ = arrs[0].shape
    cores = min(os.cpu_count() or 1, B * H)
    oracle.recurrence(*(a[:, :16] for a in arrs), G_MIN, S0=S0)  # build/load outside timing
    t = time.perf_counter()
    o_ref, S_ref = oracle.recurrence(*arrs, G_MIN, S0=S0, nthreads=cores)
    dt = time.perf_counter() - t
    parity = None
    if gpu_out is not None and sample_tokens >= x["q"].shape[1]:
        o_gpu, S_gpu = gpu_out
        parity = {"o_max_rel": normwise_err(o_gpu.float().cpu().numpy(), o_ref, (1, 3)),
                  "S_T_max_rel": normwise_err(S_gpu.cpu().numpy(), S_ref, (2, 3)),
                  "metric": "worst per-head max|gpu - oracle| / max|oracle| over the full workload",
                  "tolerance": {"o": 2e-2, "S_T": 1e-2}}
    del o_ref, S_ref
    short = min(sample_tokens, 8192)
    t = time.perf_counter()
    oracle.chunked(16, *(a[:, :short] for a in arrs), G_MIN, S0=S0, nthreads=cores)
    dtc = time.perf_counter() - t
    return {"value": B * sample_tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "nproc": os.cpu_count(), "cpu_model": cpu_model(),
            "sample": f"first {sample_tokens} of {x['q'].shape[1]} tokens, all {B * H} (batch, head) pairs "
                      f"of the 64K stage; fp64 token-by-token recurrence, {dt:.2f} s",
            "chunked_c16": {"value": B * short / dtc, "unit": UNIT,
                            "sample": f"first {short} tokens, fp64 chunked form with C = 16, {dtc:.2f} s"},
            "parity": parity}


def cpu_baseline_bwd(x, dO, sample_tokens: int):
    """The fp64 oracle's backward, as it stands, on the first ``sample_tokens`` tokens of every
    (batch, head) pair of the same inputs and dL/do (dL/dS_T = 0), on the host's cores."""
    import oracle
    from chunked_linear_attention_chunk_b200.synth import to_numpy32
    names = ("q", "k", "v", "a", "beta")
    arrs = [to_numpy32(x[n][:, :sample_tokens].cpu()) for n in names]
    dOs = to_numpy32(dO[:, :sample_tokens].cpu())
    S0 = x["S0"].cpu().numpy().astype("float64")
    B, Ts, H, _ = arrs[0].shape
    cores = min(os.cpu_count() or 1, B * H)
    oracle.backward(*(a[:, :4] for a in arrs), dOs[:, :4], G_MIN, S0=S0)  # build/load outside timing
    t = time.perf_counter()
    oracle.backward(*arrs, dOs, G_MIN, S0=S0, nthreads=cores)
    dt = time.perf_counter() - t
    return {"value": B * Ts / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"first {Ts} of {x['q'].shape[1]} tokens, all {B * H} (batch, head) pairs; fp64 "
                      f"token-by-token backward with 64-token recompute, {dt:.2f} s"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = synth.STAGE_64K
    sample = 2048
    x = synth.make_inputs(w.B, sample, w.H, w.dk, w.dv, w.dtype, w.seed, w.s0_std, False)
    import oracle
    from chunked_linear_attention_chunk_b200.synth import to_numpy32
    names = ("q", "k", "v", "a", "beta")
    arrs = [to_numpy32(x[n]) for n in names]
    S0 = x["S0"].numpy().astype("float64")
    cores = min(os.cpu_count() or 1, w.B * w.H)
    for _ in range(args.warmup):
        oracle.recurrence(*(a[:, :64] for a in arrs), G_MIN, S0=S0, nthreads=cores)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.recurrence(*arrs, G_MIN, S0=S0, nthreads=cores)
    dt = (time.perf_counter() - t) / args.steps
    value = w.B * sample / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "sample_tokens_per_step": sample, "note":
                   "fp64 CPU oracle of the recurrence; each step is a bounded sample of the 64K workload"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"first {sample} tokens x {w.B * w.H} (batch, head) pairs per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def stage_metrics(tokens, token_heads, states, ms, world, hbm_peak, bf16_peak, peak_kind):
    """tokens/s, TFLOP/s and the path roofline of one chunked-forward step of ``ms``."""
    alg = token_heads * BYTES_PER_TOKEN_HEAD + 2 * states * 128 * 128 * 4
    gbs = alg / (ms * 1e-3) / 1e9
    tflops = token_heads * FLOPS_PER_TOKEN_HEAD / (ms * 1e-3) / 1e12
    return {"ms_per_step": ms, "value": world * tokens / (ms * 1e-3), "unit": UNIT, "tflops": tflops,
            "pct_bf16_peak": tflops / bf16_peak,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "peak_kind": peak_kind, "kernels": "prep + scan of every kda_chunk_fwd call of the step",
                         "algorithmic_bytes": alg}}


def time_stage(kda, sw, rank, world, device, hbm_peak, bf16_peak, peak_kind, args):
    """One step of a context stage on its own seeded inputs: the 8K stage is one kda_chunk_fwd
    over B4 H16 T8192; the 1M stage is one sequence of 16 consecutive 64K segments (each drawn
    from its own seed), the state carried from segment to segment.  The 1M step is one
    kda_chunk_fwd_segmented call (64K stretches, each stretch's prep overlapping the scan of the
    one before); the same work as 16 kda_chunk_fwd calls is timed beside it
    (`sequential_calls`) and both are checked to give the same final state bit for bit."""
    names = ("q", "k", "v", "a", "beta")
    B, H, D = sw.B, sw.H, sw.dk
    seq = None
    if sw.segment:
        nseg, seg = sw.T // sw.segment, sw.segment
        full = {n: torch.empty((B, sw.T, H) + (() if n == "beta" else (D,)), dtype=torch.bfloat16, device=device)
                for n in names}
        for i in range(nseg):
            if rank == 0:
                xi = synth.workload_inputs(sw, segment_index=i)
            else:  # every rank its own sequence
                xi = synth.make_inputs(B, seg, H, D, D, sw.dtype, rank_seed(sw.seed * 1000 + i, rank), sw.s0_std)
            for n in names:
                full[n][:, i * seg:(i + 1) * seg].copy_(xi[n])
            if i == 0:
                S0 = xi["S0"].to(device)
            del xi
        o = torch.empty((B, sw.T, H, D), dtype=torch.bfloat16, device=device)
        S = torch.empty_like(S0)
        ws = torch.empty(kda.kda_chunk_fwd_workspace(B, seg, H, D, D), dtype=torch.uint8, device=device)
        ws2 = torch.empty(kda.kda_chunk_fwd_segmented_workspace(B, sw.T, H, D, D, seg), dtype=torch.uint8,
                          device=device)

        def step_calls():
            S.copy_(S0)
            for i in range(nseg):
                sl = slice(i * seg, (i + 1) * seg)
                kda.kda_chunk_fwd(*(full[n][:, sl] for n in names), G_MIN, S0=S, o=o[:, sl], S_T=S, workspace=ws)

        def step():
            S.copy_(S0)
            kda.kda_chunk_fwd_segmented(*(full[n] for n in names), seg, G_MIN, S0=S, o=o, S_T=S, workspace=ws2)

        steps = max(2, min(args.steps, 3))
        ms_calls = time_steps(step_calls, steps, 3, world, device)
        S_calls = S.clone()
        seq = {"ms_per_step": ms_calls, "value": B * sw.T * world / (ms_calls * 1e-3), "unit": "tokens/s",
               "calls_per_step": nseg}
        calls = 1
    else:
        xi = synth.make_inputs(B, sw.T, H, D, D, sw.dtype, rank_seed(sw.seed, rank), sw.s0_std, sw.adversarial)
        x = {n: xi[n].to(device) for n in names}
        S0 = xi["S0"].to(device)
        del xi
        S = torch.empty_like(S0)
        o = torch.empty((B, sw.T, H, D), dtype=torch.bfloat16, device=device)
        ws = torch.empty(kda.kda_chunk_fwd_workspace(B, sw.T, H, D, D), dtype=torch.uint8, device=device)
        nseg, calls = 1, 1

        def step():
            S.copy_(S0)
            kda.kda_chunk_fwd(*(x[n] for n in names), G_MIN, S0=S, o=o, S_T=S, workspace=ws)

        steps = max(2, min(args.steps, 10))
    with ClockSampler(device.index) as clk:
        ms = time_steps(step, steps, 3, world, device)
    assert kda.kda_device_status(device) == 0
    out = {"workload": sw.name, "B": B, "T": sw.T, "H": H, "dk": D, "dv": D, "steps": steps,
           "calls_per_step": calls, "gpu_launches_per_step": 3 * nseg,
           "l2": "inputs exceed the 126 MB L2; no flush"}
    if seq is not None:
        out["entry"] = f"kda_chunk_fwd_segmented, {sw.segment}-token stretches"
        seq["same_final_state"] = bool(torch.equal(S, S_calls))
        out["sequential_calls"] = seq
    out.update(stage_metrics(B * sw.T, B * sw.T * H, B * H, ms, world, hbm_peak, bf16_peak, peak_kind))
    out["clocks"] = clk.summary()
    return out


def run_libkda(args):
    import chunked_linear_attention_chunk_b200 as kda

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    hbm_peak, bf16_peak, peak_kind = peaks()

    w = WORKLOADS[args.workload]
    x = synth.make_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, rank_seed(w.seed, rank), w.s0_std, w.adversarial)
    names = ("q", "k", "v", "a", "beta")
    d = {n: x[n].to(device) for n in names}
    S0 = x["S0"].to(device)
    B, T, H, D = w.B, w.T, w.H, w.dk
    o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=device)
    S_T = torch.empty((B, H, D, D), dtype=torch.float32, device=device)
    need = kda.kda_chunk_fwd_workspace(B, T, H, D, D)
    ws = torch.empty(need, dtype=torch.uint8, device=device)

    # One step is kda_chunk_fwd issued as its two stages (the same launches the single
    # call makes), with CUDA events around each on the launching stream during the timed
    # steps, so each kernel's own duration is measured live.
    stream = torch.cuda.current_stream(device)
    timed = {"on": False, "ev": []}

    def step():
        ev = None
        if timed["on"]:
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            ev[0].record(stream)
        kda.kda_chunk_fwd_prep(*(d[n] for n in names), ws, G_MIN)
        if ev:
            ev[1].record(stream)
        kda.kda_chunk_fwd_scan(ws, B, T, H, D, D, S0=S0, o=o, S_T=S_T)
        if ev:
            ev[2].record(stream)
            timed["ev"].append(ev)

    prep_ms = scan_ms = float("nan")
    if args.only == "decode":
        ms = float("nan")
        clocks = {}
    else:
        with ClockSampler(local) as clk:
            ms = time_steps(step, args.steps, args.warmup, world, device, timed)
        assert kda.kda_device_status(device) == 0
        clocks = clk.summary()
        prep_ms = max_over_ranks(statistics.fmean(e[0].elapsed_time(e[1]) for e in timed["ev"]), world, device)
        scan_ms = max_over_ranks(statistics.fmean(e[1].elapsed_time(e[2]) for e in timed["ev"]), world, device)
    tokens = B * T
    value = world * tokens / (ms * 1e-3)
    token_heads = B * T * H
    alg_bytes = token_heads * BYTES_PER_TOKEN_HEAD + 2 * B * H * D * D * 4
    achieved_gbs = alg_bytes / (ms * 1e-3) / 1e9
    prep_bytes = token_heads * PREP_BYTES_PER_TOKEN_HEAD
    prep_gbs = prep_bytes / (prep_ms * 1e-3) / 1e9
    tflops = token_heads * FLOPS_PER_TOKEN_HEAD / (ms * 1e-3) / 1e12
    prep_traffic = measured_traffic_per_token_head("prep")
    scan_traffic = measured_traffic_per_token_head("scan")

    # ---- the other context stages: 8K (B4 H16 T8192) and 1M (B1 H16 T1048576 as 16 calls of
    # 64K tokens with the state carried in place), each through kda_chunk_fwd on its own inputs
    stages = None
    if args.only != "decode" and not args.no_stages:
        stages = {}
        for key, sw in (("8k", synth.STAGE_8K), ("1m", synth.STAGE_1M)):
            if key == "8k" and w is synth.STAGE_8K:
                continue
            stages[key] = time_stage(kda, sw, rank, world, device, hbm_peak, bf16_peak, peak_kind, args)

    # ---- the ablation: unbounded log-sigmoid gate, element-wise diagonal tiles (same inputs)
    abl = None
    if args.only != "decode" and not args.no_ablation:
        def abl_step():
            kda.kda_chunk_fwd_logsigmoid(*(d[n] for n in names), S0=S0, o=o, S_T=S_T, workspace=ws)

        abl_ms = time_steps(abl_step, max(2, min(args.steps, 5)), 3, world, device)
        assert kda.kda_device_status(device) == 0
        abl = {"gate": "g = log sigmoid(a), diagonal 16x16 tiles element by element", "ms_per_step": abl_ms,
               "value": world * tokens / (abl_ms * 1e-3), "unit": UNIT, "slowdown_vs_bounded": abl_ms / ms}

    # ---- packed variable-length batch: documents of mixed length on the same 64K token axis
    vl = None
    if args.only != "decode" and not args.no_varlen and (B, T, H) == (1, synth.VARLEN_64K_T, synth.VARLEN_64K_H):
        lengths = synth.document_lengths(T)
        cu = torch.from_numpy(synth.cu_seqlens(lengths)).to(device)
        Nd = len(lengths)
        S0v = synth.make_inputs(Nd, 1, H, D, D, "bf16", synth.VARLEN_SEED, 0.1)["S0"].to(device)
        S_Tv = torch.empty_like(S0v)
        packed = [d[n][0] for n in names]
        ws_v = torch.empty(kda.kda_chunk_fwd_varlen_workspace(Nd, T, H, D, D), dtype=torch.uint8, device=device)

        def vl_step():
            kda.kda_chunk_fwd_varlen(*packed, cu, G_MIN, S0=S0v, o=o[0], S_T=S_Tv, workspace=ws_v)

        vl_ms = time_steps(vl_step, max(3, min(args.steps, 10)), 3, world, device)
        assert kda.kda_device_status(device) == 0
        vl = {"workload": f"packed 64K axis, H={H} d={D}: {Nd} documents, log-uniform lengths 16..16384 "
                          f"(min {int(lengths.min())}, max {int(lengths.max())})",
              "ms_per_step": vl_ms, "value": world * tokens / (vl_ms * 1e-3), "unit": UNIT, "gpu_launches_per_step": 4,
              "roofline_path_frac": (token_heads * BYTES_PER_TOKEN_HEAD + 2 * Nd * H * D * D * 4) / (vl_ms * 1e-3)
              / 1e9 / hbm_peak}

    # ---- sequence parallel: one 64K sequence split into world consecutive segments, one per
    # rank (the same seeded sequence on every rank; rank r takes its slice)
    spl = None
    if args.only != "decode" and not args.no_sp and B == 1 and T % world == 0:
        from chunked_linear_attention_chunk_b200.sp import sp_chunk_fwd
        xs = x if world == 1 else synth.make_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.seed, w.s0_std,
                                                    w.adversarial)
        seg = T // world
        sd = [xs[n][:, rank * seg:(rank + 1) * seg].contiguous().to(device) for n in names]
        S0s = xs["S0"].to(device)

        def sp_step():
            sp_chunk_fwd(*sd, S0=S0s)

        sp_ms = time_steps(sp_step, max(3, min(args.steps, 10)), 3, world, device)
        assert kda.kda_device_status(device) == 0
        spl = {"workload": f"one {T}-token sequence in {world} segment(s) of {seg}, H={H} d={D}",
               "ms_per_step": sp_ms, "value": tokens / (sp_ms * 1e-3), "unit": UNIT, "segments": world,
               "gpu_launches_per_step": 5, "collectives_per_step": 2 if world > 1 else 0}
        del sd, xs

    # ---- backward: the gradients of every input for the same workload and inputs, one
    # kda_chunk_bwd per step (prep, state-saving scan, reverse state-gradient scan, per-chunk
    # gradients: four launches), dL/do seeded normal, no gradient on the final state
    bwd = None
    if args.only != "decode" and not args.no_bwd:
        gen = torch.Generator().manual_seed(rank_seed(w.seed + 17, rank))
        dO = torch.randn((B, T, H, D), generator=gen).to(torch.bfloat16).to(device)
        ws_b = torch.empty(kda.kda_chunk_bwd_workspace(B, T, H, D, D), dtype=torch.uint8, device=device)
        gout = {}

        def bwd_step():
            gout.update(kda.kda_chunk_bwd(*(d[n] for n in names), dO, G_MIN, S0=S0, workspace=ws_b,
                                          out=gout or None))

        bwd_ms = time_steps(bwd_step, max(3, min(args.steps, 5)), 3, world, device)
        assert kda.kda_device_status(device) == 0
        bwd_bytes = token_heads * BWD_BYTES_PER_TOKEN_HEAD + 2 * B * H * D * D * 4
        bwd_traffic = measured_traffic_per_token_head("bwd_chunk")
        bwd_gbs = bwd_bytes / (bwd_ms * 1e-3) / 1e9
        bwd_cpu = None
        if world == 1 and rank == 0 and not args.no_cpu_baseline:
            bwd_cpu = cpu_baseline_bwd(x, dO, min(T, 8192))
        bwd = {"what": "kda_chunk_bwd: dq, dk, dv, da, dbeta, dS0 (float32) from dL/do",
               "cpu_baseline": bwd_cpu,
               "ms_per_step": bwd_ms, "value": world * tokens / (bwd_ms * 1e-3), "unit": UNIT,
               "gpu_launches_per_step": 5, "vs_forward_time": bwd_ms / ms, "workspace_bytes": ws_b.numel(),
               "roofline": {"bound": "hbm", "achieved": bwd_gbs, "peak": hbm_peak, "unit": "GB/s",
                            "frac": bwd_gbs / hbm_peak, "peak_kind": peak_kind,
                            "kernels": "the whole backward path (five launches)",
                            "algorithmic_bytes_per_step": bwd_bytes},
               "dominant_kernel": {"kernel": "bwd_chunk_kernel (per-chunk gradients)",
                                   "algorithmic_bytes_per_token_head": BWD_CHUNK_BYTES_PER_TOKEN_HEAD,
                                   "traffic": None if bwd_traffic is None else bwd_traffic * token_heads}}
        # a training step's two calls on these inputs: the forward, then the backward; the forward
        # writes its records into the backward's workspace, which kda_chunk_bwd_recorded reuses
        # instead of running the prep again (kda_chunk_bwd recomputes them)
        o_t = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=device)

        def train_step(recorded):
            kda.kda_chunk_fwd(*(d[n] for n in names), G_MIN, S0=S0, o=o_t, workspace=ws_b, return_state=False)
            if recorded:
                gout.update(kda.kda_chunk_bwd_recorded(*(d[n] for n in names), dO, ws_b, G_MIN, S0=S0, out=gout))
            else:
                gout.update(kda.kda_chunk_bwd(*(d[n] for n in names), dO, G_MIN, S0=S0, workspace=ws_b, out=gout))

        n_tr = max(3, min(args.steps, 5))
        tr_plain = time_steps(lambda: train_step(False), n_tr, 3, world, device)
        tr_rec = time_steps(lambda: train_step(True), n_tr, 3, world, device)
        assert kda.kda_device_status(device) == 0
        bwd["training_step"] = {"what": "kda_chunk_fwd then kda_chunk_bwd_recorded (the backward reusing the "
                                        "forward's records from its workspace)",
                                "ms_per_step": tr_rec, "value": world * tokens / (tr_rec * 1e-3), "unit": UNIT,
                                "ms_with_kda_chunk_bwd": tr_plain, "gpu_launches_per_step": 6}
        del ws_b, gout, o_t
        # the same over the packed batch of the varlen leg (documents of mixed length)
        if (B, T, H) == (1, synth.VARLEN_64K_T, synth.VARLEN_64K_H):
            lengths = synth.document_lengths(T)
            cu_b = torch.from_numpy(synth.cu_seqlens(lengths)).to(device)
            ws_vb = torch.empty(kda.kda_chunk_bwd_varlen_workspace(len(lengths), T, H, D, D), dtype=torch.uint8,
                                device=device)
            packed = [d[n][0] for n in names]
            gv = {}

            def bwd_vl_step():
                gv.update(kda.kda_chunk_bwd_varlen(*packed, dO[0], cu_b, G_MIN, workspace=ws_vb, out=gv or None))

            bvl_ms = time_steps(bwd_vl_step, max(3, min(args.steps, 5)), 3, world, device)
            assert kda.kda_device_status(device) == 0
            bwd["packed"] = {"workload": f"the varlen leg's {len(lengths)} documents on the 64K axis",
                             "ms_per_step": bvl_ms, "value": world * tokens / (bvl_ms * 1e-3), "unit": UNIT,
                             "gpu_launches_per_step": 6}
            del ws_vb, gv
        del dO

    # ---- end to end through the C ABI with pinned host buffers, pipelined across steps:
    # every step copies its inputs host -> device on one stream, runs kda_chunk_fwd on a
    # second, and reads o and S_T back on a third; device and host buffers are double-
    # buffered, so step i's read-back overlaps step i+1's upload (PCIe is full duplex).
    hx = {n: x[n].pin_memory() for n in names}
    hS0 = x["S0"].pin_memory()
    e2e_ms = float("nan")
    if not args.no_e2e and args.only != "decode":
        sets = []
        for _ in range(2):
            st = {n: torch.empty_like(d[n]) for n in names}
            st.update(S0=torch.empty_like(S0), o=torch.empty_like(o), S_T=torch.empty_like(S_T),
                      ho=torch.empty(o.shape, dtype=o.dtype).pin_memory(),
                      hST=torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory())
            sets.append(st)
        s_in, s_run, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_run = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        count = [0]

        def e2e_step():
            i = count[0]
            count[0] += 1
            bsel = i % 2
            st = sets[bsel]
            s_in.wait_event(ev_run[bsel])  # step i-2 is done reading this input set
            with torch.cuda.stream(s_in):
                for n in names:
                    st[n].copy_(hx[n], non_blocking=True)
                st["S0"].copy_(hS0, non_blocking=True)
            ev_in[bsel].record(s_in)
            s_run.wait_event(ev_in[bsel])
            s_run.wait_event(ev_out[bsel])  # step i-2's outputs have been read back
            with torch.cuda.stream(s_run):
                kda.kda_chunk_fwd(*(st[n] for n in names), G_MIN, S0=st["S0"], o=st["o"], S_T=st["S_T"],
                                  workspace=ws)
            ev_run[bsel].record(s_run)
            s_out.wait_event(ev_run[bsel])
            with torch.cuda.stream(s_out):
                st["ho"].copy_(st["o"], non_blocking=True)
                st["hST"].copy_(st["S_T"], non_blocking=True)
            ev_out[bsel].record(s_out)

        def time_e2e(steps, warmup):
            for _ in range(warmup):
                e2e_step()
            torch.cuda.synchronize(device)
            barrier(world)
            torch.cuda.synchronize(device)
            cur = torch.cuda.current_stream(device)
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(cur)
            s_in.wait_event(t0)  # nothing of the timed steps starts before t0
            last = None
            for _ in range(steps):
                e2e_step()
                last = ev_out[(count[0] - 1) % 2]
            cur.wait_event(last)  # the last read-back depends on every earlier step
            t1.record(cur)
            torch.cuda.synchronize(device)
            barrier(world)
            return max_over_ranks(t0.elapsed_time(t1) / steps, world, device)

        e2e_ms = time_e2e(max(3, min(args.steps, 6)), max(3, min(args.warmup, 3)))
        assert kda.kda_device_status(device) == 0
        del sets
    h2d = sum(hx[n].numel() * hx[n].element_size() for n in names) + hS0.numel() * 4
    d2h = o.numel() * o.element_size() + S_T.numel() * 4

    # ---- decode step: N=256, H=32, d=128, fp32 state, chained steps
    dw = synth.DECODE
    # (the configured 1000 chained steps, every step with its own seeded token set, all of them
    # resident on the device: 8.4 GB of tokens; the warm-up steps have sets of their own)
    dec_steps = dw.steps if args.only != "decode" else max(args.steps, 1)
    dec_warm = max(args.warmup, 3)
    dec_ms = float("nan")
    dclk = None
    if args.only != "chunk":
        S = synth.decode_state(dw).to(device)
        toks = []
        for t in synth.decode_token_sets(dw, range(dec_warm + dec_steps), seed_of=lambda i: rank_seed(i, rank)):
            toks.append({n: t[n].to(device) for n in names})
        od = torch.empty((dw.N, dw.H, dw.dv), dtype=torch.bfloat16, device=device)
        counter = [0]

        def dec_step():
            t = toks[counter[0]]
            counter[0] += 1
            kda.kda_decode_step(*(t[n] for n in names), S, G_MIN, o=od)

        with ClockSampler(local) as dclk:
            dec_ms = time_steps(dec_step, dec_steps, dec_warm, world, device)
        assert kda.kda_device_status(device) == 0
        del toks
    units = dw.N * dw.H
    dec_bytes = units * (2 * dw.dk * dw.dv * 4 + 3 * dw.dk * 2 + dw.dv * 2 + 2 + dw.dv * 2)
    dec_gbs = world * dec_bytes / (dec_ms * 1e-3) / 1e9

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "gpu": torch.cuda.get_device_name(device),
        "config": {"workload": w.name, "B": B, "T": T, "H": H, "dk": D, "dv": D, "chunk": 64, "tile": 16,
                   "g_min": G_MIN, "global_batch": world * B, "seq_len": T, "parallelism": f"replicas{world}",
                   "l2": "inputs exceed the 126 MB L2; no flush"},
        "clocks": clocks,
        "e2e": {"value": world * tokens / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "how": "kda_chunk_fwd from pinned host buffers; upload, compute and read-back on three "
                       "streams, double-buffered, so step i's read-back overlaps step i+1's upload"},
        "gpu_launches": 3 * args.steps,
        "roofline": {"bound": "hbm", "achieved": prep_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": prep_gbs / hbm_peak, "peak_kind": peak_kind,
                     "kernel": "prep_kernel (dominant; one launch per step, timed with the 3-us gate-table launch before it)",
                     "algorithmic_bytes_per_launch": prep_bytes, "ms_per_launch": prep_ms,
                     "traffic": None if prep_traffic is None else prep_traffic * token_heads,
                     "path": {"kernels": "prep + scan (one kda_chunk_fwd)", "achieved": achieved_gbs,
                              "frac": achieved_gbs / hbm_peak, "algorithmic_bytes": alg_bytes}},
        "kernels": {"prep_kernel": {"ms_per_launch": prep_ms, "share": prep_ms / (prep_ms + scan_ms)},
                    "scan_kernel": {"ms_per_launch": scan_ms, "share": scan_ms / (prep_ms + scan_ms),
                                    "traffic": None if scan_traffic is None else scan_traffic * token_heads}},
        "chunk_fwd": {"tflops": tflops, "pct_bf16_peak": tflops / bf16_peak, "bf16_peak_tflops": bf16_peak,
                      "flops_per_token_head": FLOPS_PER_TOKEN_HEAD},
        "decode": {"metric": "decode HBM GB/s", "value": dec_gbs, "unit": "GB/s", "ms_per_step": dec_ms,
                   "steps": dec_steps, "workload": dw.name, "gpu_launches": dec_steps,
                   "roofline": {"bound": "hbm", "achieved": dec_gbs / world, "peak": hbm_peak, "unit": "GB/s",
                                "frac": dec_gbs / world / hbm_peak, "peak_kind": peak_kind},
                   "clocks": dclk.summary() if dclk is not None else {}},
    }
    if abl is not None:
        line["ablation"] = abl
    if stages:
        line["stages"] = stages
    if vl is not None:
        line["varlen"] = vl
    if spl is not None:
        line["sequence_parallel"] = spl
    if bwd is not None:
        line["backward"] = bwd
    if world == 1 and rank == 0 and not args.no_cpu_baseline and args.only != "decode":
        # a fresh run of the main path on this exact input (later legs reuse o and S_T)
        o_p, S_p = kda.kda_chunk_fwd(*(d[n] for n in names), G_MIN, S0=S0, workspace=ws)
        torch.cuda.synchronize(device)
        line["cpu_baseline"] = cpu_baseline(x, args.cpu_sample_tokens, gpu_out=(o_p, S_p))
        del o_p, S_p
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("libkda", "reference"), default="libkda")
    ap.add_argument("--cpu-sample-tokens", type=int, default=65536)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="64k",
                    help="64k (the benchmark workload); 8k or 16k (smaller cases for profiler captures; 16k has the 64K stage's 32 heads, so its scan takes the same one-block form)")
    ap.add_argument("--only", choices=("all", "chunk", "decode"), default="all")
    ap.add_argument("--no-ablation", action="store_true", help="skip timing the log-sigmoid ablation path")
    ap.add_argument("--no-varlen", action="store_true", help="skip timing the packed variable-length batch")
    ap.add_argument("--no-sp", action="store_true", help="skip timing the sequence-parallel leg")
    ap.add_argument("--no-bwd", action="store_true", help="skip timing the backward leg")
    ap.add_argument("--no-stages", action="store_true", help="skip timing the 8K and 1M context stages")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args)
    return run_libkda(args)


if __name__ == "__main__":
    sys.exit(main())
