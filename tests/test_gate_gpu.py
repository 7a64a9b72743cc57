"""K1 gate on the GPU against the fp64 oracle: bit-exact g."""
import numpy as np
import pytest
import torch

import oracle
import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import synth

pytestmark = pytest.mark.gpu


def _all_bf16():
    bits = torch.arange(65536, dtype=torch.int32)
    bits = torch.where(bits >= 32768, bits - 65536, bits).to(torch.int16)
    return bits.view(torch.bfloat16)


def _same_bits(g_gpu: np.ndarray, g_ref: np.ndarray):
    nan = np.isnan(g_ref)
    assert (np.isnan(g_gpu) == nan).all()
    a = g_gpu[~nan].view(np.uint32)
    b = g_ref[~nan].view(np.uint32)
    bad = np.nonzero(a != b)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first at {bad[:5]}"


@pytest.mark.parametrize("g_min", [-5.0, -1.0, -5.4, -0.25])
def test_gate_bf16_exhaustive_bit_exact(g_min):
    """g_min crosses the C ABI as float32, so the oracle gets the same float32 value."""
    g_min = float(np.float32(g_min))
    a = _all_bf16()
    g = kda.kda_gate_fwd(a.cuda(), g_min).cpu().numpy()
    ref = oracle.gate(a.float().numpy(), g_min)
    _same_bits(g, ref)
    fin = ~np.isnan(ref)
    assert (g[fin] >= np.float32(g_min)).all() and (g[fin] <= 0).all()


def test_gate_f32_bit_exact():
    rng = np.random.default_rng(7)
    a = np.concatenate([
        rng.standard_normal(1 << 20).astype(np.float32) * 2,
        rng.standard_normal(1 << 16).astype(np.float32) * 40,
        np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e-30, -1e-30, 88.0, -88.0, 104.0, -104.0], np.float32),
    ])
    x = synth.workload_inputs(synth.TINY)["a"].numpy().reshape(-1)
    a = np.concatenate([a, x])
    g = kda.kda_gate_fwd(torch.from_numpy(a).cuda(), -5.0).cpu().numpy()
    _same_bits(g, oracle.gate(a, -5.0))


@pytest.mark.parametrize("n", [1, 7, 8, 9, 15, 1000003])
def test_gate_ragged_lengths(n):
    a = _all_bf16()[:n] if n <= 65536 else _all_bf16().repeat(n // 65536 + 1)[:n]
    a = a.clone()
    g = kda.kda_gate_fwd(a.cuda(), -5.0).cpu().numpy()
    _same_bits(g, oracle.gate(a.float().numpy(), -5.0))


def test_gate_writes_nothing_past_n():
    a = torch.randn(13, dtype=torch.bfloat16, device="cuda")
    out = torch.full((32,), 7.0, device="cuda")
    kda.kda_gate_fwd(a, -5.0, out=out[:13])
    assert (out[13:] == 7.0).all()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gate_heads_bit_exact(dtype):
    """g_min * sigmoid(e^{A_h} a) per head, bit-exact against the fp64 oracle."""
    gen = torch.Generator().manual_seed(31)
    a = (torch.randn(37, 6, 128, generator=gen) * 3).to(dtype)
    A_log = torch.randn(6, generator=gen) * 0.7
    g = kda.kda_gate_fwd_heads(a.cuda(), A_log.cuda(), -5.0)
    torch.cuda.synchronize()
    ref = oracle.gate_heads(a.float().numpy(), A_log.numpy(), -5.0)
    assert np.array_equal(g.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def _records_bytes(B, T, H, D):
    rec = D * D * 2 + 64 * D * 2 + D * 4 + D * D * 2 + 64 * D * 2
    return B * H * ((T + 63) // 64) * rec


@pytest.mark.parametrize("g_min", [-5.0, -0.25])
def test_chunk_path_gate_table_is_bit_exact(g_min):
    """The chunk path reads g from a table of the gate at all 65536 bfloat16 inputs, which the
    prep writes into the workspace (after the records) with the fp64 function of kda_gate_fwd.
    The table equals the oracle's gate bit for bit, so every g the hot path uses does too."""
    g_min = float(np.float32(g_min))
    B, T, H, D = 1, 200, 2, 128
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=41, s0_std=0.1)
    d = {n: x[n].cuda() for n in ("q", "k", "v", "a", "beta")}
    ws = torch.zeros(kda.kda_chunk_fwd_workspace(B, T, H, D, D), dtype=torch.uint8, device="cuda")
    kda.kda_chunk_fwd_prep(d["q"], d["k"], d["v"], d["a"], d["beta"], ws, g_min)
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    off = _records_bytes(B, T, H, D)
    assert ws.numel() >= off + 65536 * 4
    tab = ws[off:off + 65536 * 4].cpu().numpy().view(np.float32)
    a = _all_bf16()
    _same_bits(tab, oracle.gate(a.float().numpy(), g_min))
    # the table is indexed by the input's bits: entry i is the gate of bf16 pattern i
    assert tab[0] == np.float32(oracle.gate(np.zeros(1, np.float32), g_min)[0])


def test_chunk_path_gate_table_per_head_is_bit_exact():
    """With the per-head scale the prep writes one table per head, each equal to
    kda_gate_fwd_heads (and the oracle) at every bfloat16 input of that head."""
    B, T, H, D = 1, 70, 3, 64
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=42, s0_std=0.1)
    d = {n: x[n].cuda() for n in ("q", "k", "v", "a", "beta")}
    A_log = torch.tensor([0.4, -0.7, 1.1])
    ws = torch.zeros(kda.kda_chunk_fwd_workspace(B, T, H, D, D), dtype=torch.uint8, device="cuda")
    kda.kda_chunk_fwd_prep(d["q"], d["k"], d["v"], d["a"], d["beta"], ws, -5.0, A_log=A_log.cuda())
    torch.cuda.synchronize()
    off = _records_bytes(B, T, H, D)
    tab = ws[off:off + H * 65536 * 4].cpu().numpy().view(np.float32).reshape(H, 65536)
    a = _all_bf16().float().numpy()
    for h in range(H):
        ref = oracle.gate_heads(a.reshape(1, 1, 65536), A_log[h:h + 1].numpy(), -5.0).reshape(-1)
        _same_bits(tab[h], ref)
