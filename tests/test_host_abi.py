"""Host-side checks of the C ABI (CPU only): the library loads, exports every entry
point include/kda.h declares, sizes workspaces, and rejects bad arguments with the
documented status before any CUDA call is made."""
import ctypes
import os
import re
import subprocess

import pytest

import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

OK, INVALID, UNSUPPORTED, ALIGN, ALIAS, CUDA, TIMEOUT, WS = range(8)


@pytest.fixture(scope="module")
def L():
    build.build()
    return kda.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(kda_[a-z0-9_]+)\s*\(", text, re.M)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("kda_gate_fwd", "kda_chunk_fwd_workspace", "kda_chunk_fwd", "kda_decode_step",
              "kda_device_status", "kda_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", kda.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(kda_[a-z0-9_]+)$", out, re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(L, n)
    assert set(kda.EXPORTS) <= set(declared_functions())


def test_status_strings(L):
    for code, name in kda.STATUS.items():
        assert L.kda_status_string(code).decode() == name
    assert L.kda_status_string(99).decode() == "KDA_ERR_UNKNOWN"
    assert L.kda_version() >= 100


def test_workspace_size(L):
    f = L.kda_chunk_fwd_workspace
    # per chunk record: N (D x D) + Q' (64 x D) bf16, Gamma (D f32), Bm (D x D) + O' (64 x D) bf16;
    # after the records, one gate table of 65536 floats per head
    rec128 = 128 * 128 * 2 + 64 * 128 * 2 + 128 * 4 + 128 * 128 * 2 + 64 * 128 * 2
    tab = 65536 * 4
    assert f(1, 64, 1, 128, 128, kda.KDA_BF16) == rec128 + tab
    assert f(2, 65, 3, 128, 128, kda.KDA_BF16) == 2 * 3 * 2 * rec128 + 3 * tab
    assert f(1, 65536, 32, 128, 128, kda.KDA_BF16) == 32 * 1024 * rec128 + 32 * tab
    rec64 = 64 * 64 * 2 + 64 * 64 * 2 + 64 * 4 + 64 * 64 * 2 + 64 * 64 * 2
    assert f(1, 100, 1, 64, 64, kda.KDA_BF16) == 2 * rec64 + tab
    assert f(1, 100, 1, 64, 64, kda.KDA_F32) == 0
    assert f(1, 0, 1, 128, 128, kda.KDA_BF16) == 0
    assert f(0, 64, 1, 128, 128, kda.KDA_BF16) == 0
    assert f(1, 64, 1, 96, 96, kda.KDA_BF16) == 0


# Fake, never-dereferenced device addresses: validation must reject before any launch.
BASE = 1 << 40


def _chunk(L, B=1, T=64, H=1, dk=128, dv=128, dt=kda.KDA_BF16, q=None, k=None, v=None, a=None, beta=None,
           g_min=-5.0, S0=None, o=None, ST=None, ws=None, ws_bytes=None):
    es = 2 if dt == kda.KDA_BF16 else 4
    n = B * T * H * max(dk, 1) * es
    q = BASE if q is None else q
    k = BASE + 1 * (n + 4096) if k is None else k
    v = BASE + 2 * (n + 4096) if v is None else v
    a = BASE + 3 * (n + 4096) if a is None else a
    beta = BASE + 4 * (n + 4096) if beta is None else beta
    o = BASE + 5 * (n + 4096) if o is None else o
    if ws is None:
        ws = BASE + 6 * (n + 4096)
    need = L.kda_chunk_fwd_workspace(B, T, H, dk, dv, dt)
    ws_bytes = need if ws_bytes is None else ws_bytes
    P = ctypes.c_void_p
    return L.kda_chunk_fwd(B, T, H, dk, dv, dt, P(q), P(k), P(v), P(a), P(beta), ctypes.c_float(g_min),
                           P(S0), P(o), P(ST), P(ws), ws_bytes, None)


def test_chunk_fwd_rejects_bad_arguments(L):
    assert _chunk(L, B=0) == INVALID
    assert _chunk(L, T=-1) == INVALID
    assert _chunk(L, dt=7) == INVALID
    assert _chunk(L, g_min=0.0) == INVALID
    assert _chunk(L, g_min=1.0) == INVALID
    assert _chunk(L, g_min=float("nan")) == INVALID
    assert _chunk(L, g_min=float("-inf")) == INVALID
    assert _chunk(L, g_min=-6.0) == UNSUPPORTED
    assert _chunk(L, dk=96, dv=96) == UNSUPPORTED
    assert _chunk(L, dk=128, dv=64) == UNSUPPORTED
    assert _chunk(L, q=0) == INVALID  # null input with T > 0
    assert _chunk(L, o=0) == INVALID
    assert _chunk(L, q=BASE + 8) == ALIGN
    assert _chunk(L, S0=BASE * 3 + 4) == ALIGN
    assert _chunk(L, ws=0) == WS
    assert _chunk(L, ws_bytes=100) == WS
    assert _chunk(L, B=300, H=300) == UNSUPPORTED  # B*H beyond the grid limit


def test_chunk_fwd_rejects_aliasing(L):
    n = 64 * 128 * 2
    assert _chunk(L, o=BASE) == ALIAS                       # o is q
    assert _chunk(L, o=BASE + 16) == ALIAS                  # o overlaps q
    S = BASE * 2
    assert _chunk(L, S0=S, ST=S + 4096) == ALIAS            # partial overlap of states
    assert _chunk(L, ST=BASE + n + 4096) == ALIAS            # S_T overlaps k
    assert _chunk(L, ws=BASE + 2 * (n + 4096)) == ALIAS      # workspace overlaps v
    assert _chunk(L, o=BASE * 3, ST=BASE * 3 + 1024) == ALIAS


def _decode(L, N=2, H=2, dk=128, dv=128, dt=kda.KDA_BF16, g_min=-5.0, S=None, o=None, q=None):
    P = ctypes.c_void_p
    step = 1 << 24
    q = BASE if q is None else q
    S = BASE + 6 * step if S is None else S
    o = BASE + 5 * step if o is None else o
    return L.kda_decode_step(N, H, dk, dv, dt, P(q), P(BASE + step), P(BASE + 2 * step), P(BASE + 3 * step),
                             P(BASE + 4 * step), ctypes.c_float(g_min), P(S), P(o), None)


def test_decode_rejects_bad_arguments(L):
    assert _decode(L, N=0) == INVALID
    assert _decode(L, g_min=0.5) == INVALID
    assert _decode(L, g_min=-10.0) == UNSUPPORTED
    assert _decode(L, dk=32, dv=32) == UNSUPPORTED
    assert _decode(L, S=0) == INVALID
    assert _decode(L, S=BASE + 6 * (1 << 24) + 8) == ALIGN
    assert _decode(L, o=BASE) == ALIAS
    assert _decode(L, S=BASE + (1 << 24)) == ALIAS


def test_gate_rejects_bad_arguments(L):
    P = ctypes.c_void_p
    assert L.kda_gate_fwd(P(BASE), kda.KDA_BF16, ctypes.c_float(-5.0), P(BASE * 2), -1, None) == INVALID
    assert L.kda_gate_fwd(P(BASE), kda.KDA_BF16, ctypes.c_float(-5.0), P(BASE * 2), 0, None) == OK
    assert L.kda_gate_fwd(P(BASE), 3, ctypes.c_float(-5.0), P(BASE * 2), 16, None) == INVALID
    assert L.kda_gate_fwd(P(BASE), kda.KDA_BF16, ctypes.c_float(0.0), P(BASE * 2), 16, None) == INVALID
    assert L.kda_gate_fwd(P(BASE), kda.KDA_BF16, ctypes.c_float(-5.5), P(BASE * 2), 16, None) == UNSUPPORTED
    assert L.kda_gate_fwd(P(0), kda.KDA_BF16, ctypes.c_float(-5.0), P(BASE * 2), 16, None) == INVALID
    assert L.kda_gate_fwd(P(BASE + 2), kda.KDA_BF16, ctypes.c_float(-5.0), P(BASE * 2), 16, None) == ALIGN
    assert L.kda_gate_fwd(P(BASE), kda.KDA_BF16, ctypes.c_float(-5.0), P(BASE + 16), 16, None) == ALIAS


def test_python_binding_has_no_cpu_fallback():
    """The binding refuses CPU tensors instead of computing anything itself."""
    import torch
    x = torch.zeros(16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        kda.kda_gate_fwd(x)
    q = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16)
    beta = torch.zeros(1, 8, 1, dtype=torch.bfloat16)
    for call in (lambda: kda.kda_chunk_fwd(q, q, q, q, beta),
                 lambda: kda.kda_chunk_bwd(q, q, q, q, beta, q),
                 lambda: kda.kda_chunk_bwd_varlen(q[0], q[0], q[0], q[0], beta[0], q[0],
                                                  torch.tensor([0, 8], dtype=torch.int32)),
                 lambda: kda.kda_decode_step(q[:, 0], q[:, 0], q[:, 0], q[:, 0], beta[:, 0],
                                             torch.zeros(1, 1, 64, 64))):
        with pytest.raises(ValueError):
            call()


def _chunk_logsig(L, B=1, T=64, H=1, dk=128, dv=128, dt=kda.KDA_BF16, q=None, o=None, S0=None, ST=None, ws=None,
                  ws_bytes=None):
    es = 2 if dt == kda.KDA_BF16 else 4
    n = B * T * H * max(dk, 1) * es
    q = BASE if q is None else q
    o = BASE + 5 * (n + 4096) if o is None else o
    ws = BASE + 6 * (n + 4096) if ws is None else ws
    need = L.kda_chunk_fwd_workspace(B, T, H, dk, dv, dt)
    ws_bytes = need if ws_bytes is None else ws_bytes
    P = ctypes.c_void_p
    return L.kda_chunk_fwd_logsigmoid(B, T, H, dk, dv, dt, P(q), P(BASE + (n + 4096)), P(BASE + 2 * (n + 4096)),
                                      P(BASE + 3 * (n + 4096)), P(BASE + 4 * (n + 4096)), P(S0), P(o), P(ST),
                                      P(ws), ws_bytes, None)


def test_logsigmoid_entry_validates_like_chunk_fwd(L):
    """The ablation entry shares kda_chunk_fwd's checks, takes no g_min, and has no fp32 path."""
    assert _chunk_logsig(L, B=0) == INVALID
    assert _chunk_logsig(L, dt=kda.KDA_F32) == UNSUPPORTED
    assert _chunk_logsig(L, dk=96, dv=96) == UNSUPPORTED
    assert _chunk_logsig(L, q=0) == INVALID
    assert _chunk_logsig(L, q=BASE + 8) == ALIGN
    assert _chunk_logsig(L, ws=0) == WS
    assert _chunk_logsig(L, o=BASE + 16) == ALIAS


def test_prep_and_scan_entries_validate(L):
    P = ctypes.c_void_p
    B, T, H, D = 1, 64, 1, 128
    n = B * T * H * D * 2
    need = L.kda_chunk_fwd_workspace(B, T, H, D, D, kda.KDA_BF16)
    ins = [BASE + i * (n + 4096) for i in range(5)]
    ws = BASE + 6 * (n + 4096)

    def prep(gate=kda.KDA_GATE_BOUNDED, g_min=-5.0, q=ins[0], w=ws, wb=need, dk=D):
        return L.kda_chunk_fwd_prep(B, T, H, dk, dk, gate, ctypes.c_float(g_min), None, P(q), P(ins[1]), P(ins[2]),
                                    P(ins[3]), P(ins[4]), P(w), wb, None)

    def scan(w=ws, wb=need, S0=None, o=BASE + 5 * (n + 4096), ST=None):
        return L.kda_chunk_fwd_scan(B, T, H, D, D, P(w), wb, P(S0), P(o), P(ST), None)

    assert prep(g_min=0.0) == INVALID
    assert prep(g_min=-6.0) == UNSUPPORTED
    assert prep(gate=7) == INVALID
    assert prep(q=0) == INVALID
    assert prep(q=BASE + 8) == ALIGN
    assert prep(w=0) == WS
    assert prep(wb=need - 1) == WS
    assert prep(w=ins[2]) == ALIAS                     # workspace over v
    assert prep(dk=96) == UNSUPPORTED
    assert scan(o=0) == INVALID
    assert scan(w=0) == WS
    assert scan(S0=BASE * 3 + 4) == ALIGN
    assert scan(o=ws + 1024) == ALIAS                  # o inside the records
    S = BASE * 2
    assert scan(S0=S, ST=S + 4096) == ALIAS
    assert scan(ST=ws) == ALIAS


def test_selftest_timeout_rejects_bad_limits(L):
    assert L.kda_selftest_device_timeout(0, None) == INVALID
    assert L.kda_selftest_device_timeout(2000001, None) == INVALID


def test_varlen_entry_validates(L):
    P = ctypes.c_void_p
    N, T, H, D = 2, 100, 2, 128
    n = T * H * D * 2
    ws_need = L.kda_chunk_fwd_varlen_workspace(N, T, H, D, D, kda.KDA_BF16)
    rec = 128 * 128 * 2 + 64 * 128 * 2 + 128 * 4 + 128 * 128 * 2 + 64 * 128 * 2
    assert ws_need == H * ((T + 63) // 64 + N) * rec + 256 + H * 65536 * 4  # records, chunk table, gate tables
    assert L.kda_chunk_fwd_varlen_workspace(N, T, H, D, D, kda.KDA_F32) == 0
    ins = [BASE + i * (n + 4096) for i in range(5)]
    cu = BASE * 2
    ws = BASE + 6 * (n + 4096)

    def call(N=N, cu=cu, dt=kda.KDA_BF16, gate=kda.KDA_GATE_BOUNDED, g_min=-5.0, o=BASE + 5 * (n + 4096), w=ws,
             wb=ws_need, H=H):
        return L.kda_chunk_fwd_varlen(N, P(cu), T, H, D, D, dt, gate, ctypes.c_float(g_min), None, *(P(p) for p in ins),
                                      None, P(o), None, P(w), wb, None)

    assert call(N=0) == INVALID
    assert call(cu=0) == INVALID
    assert call(cu=cu + 2) == ALIGN
    assert call(dt=kda.KDA_F32) == UNSUPPORTED
    assert call(g_min=-9.0) == UNSUPPORTED
    assert call(gate=5) == INVALID
    assert call(N=40000) == UNSUPPORTED          # N * H beyond the grid limit
    assert call(w=0) == WS
    assert call(wb=ws_need - 1) == WS
    assert call(o=ins[1]) == ALIAS
    assert call(cu=ws + 64) == ALIAS              # cu_seqlens inside the workspace


def test_binding_has_a_function_for_every_export():
    """The Python binding carries the C names: one function per exported entry point."""
    missing = [n for n in kda.EXPORTS if not callable(getattr(kda, n, None))]
    assert not missing, missing
    assert set(kda.EXPORTS) == set(declared_functions())


def test_gate_heads_validates(L):
    P = ctypes.c_void_p
    f = lambda a=BASE, g=BASE * 2, A=BASE * 3, n=10, H=2, dk=64, g_min=-5.0, dt=kda.KDA_BF16: \
        L.kda_gate_fwd_heads(P(a), dt, ctypes.c_float(g_min), P(A), n, H, dk, P(g), None)
    assert f(n=0) == OK
    assert f(H=0) == INVALID
    assert f(A=0) == INVALID
    assert f(dk=12) == UNSUPPORTED
    assert f(g_min=-7.0) == UNSUPPORTED
    assert f(a=BASE + 8) == ALIGN
    assert f(A=BASE * 3 + 2) == ALIGN
    assert f(g=BASE + 64) == ALIAS
    assert f(A=BASE * 2 + 16) == ALIAS


def test_sp_entries_validate(L):
    P = ctypes.c_void_p
    assert L.kda_chunk_fwd_scan_affine(1, 64, 1, 128, 128, P(BASE), 1 << 20, None, P(BASE * 2), None) == INVALID
    assert L.kda_chunk_fwd_scan_affine(1, 64, 1, 96, 96, P(BASE), 1 << 20, P(BASE * 3), P(BASE * 2), None) == UNSUPPORTED
    assert L.kda_chunk_fwd_scan_affine(1, 64, 1, 128, 128, P(BASE), 10, P(BASE * 3), P(BASE * 2), None) == WS
    assert L.kda_chunk_fwd_scan_affine(1, 64, 1, 128, 128, P(BASE), 1 << 20, P(BASE * 3), P(BASE * 3 + 64), None) == ALIAS
    assert L.kda_state_combine(-1, 1, 1, 128, 128, P(BASE), P(BASE * 2), None, P(BASE * 3), None) == INVALID
    assert L.kda_state_combine(2, 1, 1, 128, 128, P(BASE), P(BASE * 2), None, None, None) == INVALID
    assert L.kda_state_combine(2, 1, 1, 128, 128, P(BASE + 4), P(BASE * 2), None, P(BASE * 3), None) == ALIGN
    assert L.kda_state_combine(2, 1, 1, 128, 128, P(BASE), P(BASE * 2), None, P(BASE + 4096), None) == ALIAS


def test_beta_needs_only_its_element_size():
    """beta may start at any token offset: 2-byte alignment passes the alignment check (the
    call then stops on the too-small workspace, before any launch); 1 byte does not."""
    L = kda.lib()
    n = 1 * 64 * 1 * 128 * 2
    beta = BASE + 4 * (n + 4096)
    assert _chunk(L, beta=beta + 2, ws_bytes=100) == WS
    assert _chunk(L, beta=beta + 1) == ALIGN


def test_debug_build_exports_the_same_entry_points():
    """libkda_debug.so (KDA_DEBUG_CHECKS) is the same ABI."""
    path = build.build(debug_checks=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(kda_[a-z0-9_]+)$", out, re.M))
    assert set(declared_functions()) <= exported


@pytest.mark.parametrize("entry", ["kda_chunk_bwd", "kda_chunk_bwd_recorded"])
def test_chunk_bwd_entry_validates(L, entry):
    """kda_chunk_bwd (and kda_chunk_bwd_recorded, which shares its checks) rejects every bad
    argument before a launch (fake pointers: none of these calls may pass validation)."""
    P = ctypes.c_void_p
    B, T, H, D = 1, 64, 1, 128
    nb = B * T * H * D * 2
    need = L.kda_chunk_bwd_workspace(B, T, H, D, D, kda.KDA_BF16)
    assert need > L.kda_chunk_fwd_workspace(B, T, H, D, D, kda.KDA_BF16)
    assert L.kda_chunk_bwd_workspace(B, T, H, D, D, kda.KDA_F32) == 0
    assert L.kda_chunk_bwd_workspace(B, T, H, 96, 96, kda.KDA_BF16) == 0
    step = nb * 2 + 4096
    ins = [BASE + i * step for i in range(6)]          # q, k, v, a, beta, dO
    outs = [BASE + (6 + i) * step for i in range(5)]   # dq, dk, dv, da, dbeta
    ws = BASE + 12 * step

    def bwd(dtype=kda.KDA_BF16, g_min=-5.0, q=ins[0], dO=ins[5], dq=outs[0], dbeta=outs[4], w=ws, wb=need,
            S0=None, dST=None, dS0=None, dk=D, A=None, dA=None):
        return getattr(L, entry)(B, T, H, dk, dk, dtype, P(q), P(ins[1]), P(ins[2]), P(ins[3]), P(ins[4]),
                                 ctypes.c_float(g_min), P(A), P(S0), P(dO), P(dST), P(dq), P(outs[1]), P(outs[2]),
                                 P(outs[3]), P(dbeta), P(dS0), P(dA), P(w), wb, None)

    assert bwd(dtype=kda.KDA_F32) == UNSUPPORTED
    assert bwd(dk=96) == UNSUPPORTED
    # the saved state arrays are (records x dk) rows addressed with 32-bit row indices
    big = lambda T_, H_, dk_: getattr(L, entry)(1, T_, H_, dk_, dk_, kda.KDA_BF16, *([P(BASE)] * 5), ctypes.c_float(-5.0),
                                              None, None, P(BASE), None, *([P(BASE)] * 5), None, None, P(BASE), 1, None)
    assert big(64 * (1 << 16), 256, 128) == UNSUPPORTED   # 2^24 records x 128 rows each
    assert big(64 * (1 << 16), 256, 64) != UNSUPPORTED    # 2^24 records x 64 rows: within range
    assert bwd(g_min=0.0) == INVALID
    assert bwd(q=0) == INVALID
    assert bwd(dO=0) == INVALID
    assert bwd(dq=0) == INVALID
    assert bwd(q=BASE + 8) == ALIGN
    assert bwd(dq=outs[0] + 4) == ALIGN
    assert bwd(dbeta=outs[4] + 2) == ALIGN
    assert bwd(w=0) == WS
    assert bwd(wb=need - 1) == WS
    assert bwd(dq=ins[2]) == ALIAS                        # an output over v
    assert bwd(dq=outs[1]) == ALIAS                       # two outputs on one buffer
    assert bwd(w=outs[3] - 1024) == ALIAS                 # workspace over da
    S = BASE * 2
    assert bwd(S0=S, dS0=S) == ALIAS
    assert bwd(dST=S, dS0=S + 4096) == ALIAS
    assert bwd(dA=BASE * 3) == INVALID                    # dA_log needs A_log
    assert bwd(A=BASE * 3 + 2) == ALIGN
    assert bwd(A=BASE * 3, dA=BASE * 3) == ALIAS
    assert bwd(A=BASE * 3, dA=outs[0]) == ALIAS           # dA_log inside dq
    sa, sb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert L.kda_chunk_bwd_offsets(B, T, H, D, D, ctypes.byref(sa), ctypes.byref(sb)) == OK
    assert sa.value >= L.kda_chunk_fwd_workspace(B, T, H, D, D, kda.KDA_BF16) and sa.value % 16 == 0
    assert sb.value == sa.value + B * H * D * D * 4
    assert L.kda_chunk_bwd_offsets(B, T, H, D, D, None, ctypes.byref(sb)) == INVALID


def test_chunk_bwd_varlen_entry_validates(L):
    """kda_chunk_bwd_varlen rejects bad arguments before a launch (fake pointers)."""
    P = ctypes.c_void_p
    N, T, H, D = 3, 200, 2, 64
    nb = T * H * D * 2
    need = L.kda_chunk_bwd_varlen_workspace(N, T, H, D, D, kda.KDA_BF16)
    assert need > L.kda_chunk_bwd_workspace(1, T, H, D, D, kda.KDA_BF16)
    assert L.kda_chunk_bwd_varlen_workspace(0, T, H, D, D, kda.KDA_BF16) == 0
    step = nb * 2 + 4096
    ins = [BASE + i * step for i in range(6)]
    outs = [BASE + (6 + i) * step for i in range(5)]
    ws = BASE + 12 * step
    cu = BASE + 13 * step

    def bwd(n=N, cu_=cu, q=ins[0], dq=outs[0], w=ws, wb=need, g_min=-5.0, dk=D, A=None, dA=None):
        return L.kda_chunk_bwd_varlen(n, P(cu_), T, H, dk, dk, kda.KDA_BF16, ctypes.c_float(g_min), P(A), P(q),
                                      P(ins[1]), P(ins[2]), P(ins[3]), P(ins[4]), None, P(ins[5]), None, P(dq),
                                      P(outs[1]), P(outs[2]), P(outs[3]), P(outs[4]), None, P(dA), P(w), wb, None)

    assert bwd(n=0) == INVALID
    assert bwd(cu_=0) == INVALID
    assert bwd(cu_=cu + 2) == ALIGN
    assert bwd(g_min=0.0) == INVALID
    assert bwd(dk=96) == UNSUPPORTED
    assert bwd(q=0) == INVALID
    assert bwd(dq=outs[0] + 4) == ALIGN
    assert bwd(w=0) == WS
    assert bwd(wb=need - 1) == WS
    assert bwd(dq=ins[1]) == ALIAS
    assert bwd(w=cu) == ALIAS                             # workspace over cu_seqlens
    assert bwd(dA=BASE * 3) == INVALID


def _noalloc(L, B=2, T=64, H=1, dk=128, dv=128, dt=kda.KDA_BF16, q=None, S0=None, o=None, ST=None, g_min=-5.0):
    es = 2 if dt == kda.KDA_BF16 else 4
    n = B * T * H * dk * es
    q = BASE if q is None else q
    o = BASE + 5 * (n + 4096) if o is None else o
    P = ctypes.c_void_p
    return L.kda_chunk_fwd_noalloc(B, T, H, dk, dv, dt, P(q), P(BASE + (n + 4096)), P(BASE + 2 * (n + 4096)),
                                   P(BASE + 3 * (n + 4096)), P(BASE + 4 * (n + 4096)), ctypes.c_float(g_min),
                                   P(S0), P(o), P(ST), None)


def test_noalloc_validates_the_whole_problem_before_launching(L):
    """The no-workspace entry runs its batch elements one by one, but every check covers
    the whole (B, T) problem first: an overlap that only exists between different batch
    elements is refused with ALIAS, before anything is launched (no GPU is needed to see it)."""
    B, T, H, d = 2, 64, 1, 128
    per_o = T * H * d * 2           # bytes of o per batch element
    per_s = H * d * d * 4           # bytes of S per batch element
    O = BASE * 2
    # S0 of batch element 1 starts where o (element 0) starts: o[0] overlaps S0[1] only
    assert O - per_s + per_s == O and per_o > 0
    assert _noalloc(L, B=B, S0=O - per_s, o=O, ST=BASE * 4) == ALIAS
    S = BASE * 3
    # S_T of element 0 lies on q of element 1
    q_elem1 = BASE + T * H * d * 2
    assert _noalloc(L, B=B, ST=q_elem1, S0=None) == ALIAS
    # the same problems through kda_chunk_fwd are refused the same way
    assert _chunk(L, B=B, ST=q_elem1) == ALIAS
    # and the ordinary argument checks hold
    assert _noalloc(L, g_min=-6.0) == UNSUPPORTED
    assert _noalloc(L, dk=96, dv=96) == UNSUPPORTED
    assert _noalloc(L, q=BASE + 8) == ALIGN
    assert _noalloc(L, o=BASE) == ALIAS
    assert _noalloc(L, S0=S, ST=S + 4096) == ALIAS


def _segmented(L, B=1, T=1000, H=2, dk=128, dv=128, dt=kda.KDA_BF16, seg=256, q=None, o=None, S0=None,
               ST=BASE * 3, ws=None, ws_bytes=None, g_min=-5.0):
    es = 2 if dt == kda.KDA_BF16 else 4
    n = B * T * H * max(dk, 1) * es
    q = BASE if q is None else q
    k, v, a, beta = (BASE + i * (n + 4096) for i in (1, 2, 3, 4))
    o = BASE + 5 * (n + 4096) if o is None else o
    ws = BASE + 6 * (n + 4096) if ws is None else ws
    need = L.kda_chunk_fwd_segmented_workspace(B, T, H, dk, dv, seg)
    ws_bytes = need if ws_bytes is None else ws_bytes
    P = ctypes.c_void_p
    return L.kda_chunk_fwd_segmented(B, T, H, dk, dv, dt, seg, P(q), P(k), P(v), P(a), P(beta), ctypes.c_float(g_min),
                                     P(S0), P(o), P(ST), P(ws), ws_bytes, None)


def test_segmented_entry_sizes_and_validates(L):
    """kda_chunk_fwd_segmented: two stretches' records of workspace, and every argument check
    (its own and kda_chunk_fwd's) before any launch."""
    f = L.kda_chunk_fwd_segmented_workspace
    one = L.kda_chunk_fwd_workspace(1, 256, 2, 128, 128, kda.KDA_BF16)
    assert f(1, 1000, 2, 128, 128, 256) == 2 * ((one + 255) // 256 * 256)
    assert f(3, 1000, 2, 128, 128, 256) == f(1, 1000, 2, 128, 128, 256)  # per stretch, not per batch
    short = L.kda_chunk_fwd_workspace(1, 100, 2, 128, 128, kda.KDA_BF16)
    assert f(1, 100, 2, 128, 128, 256) == 2 * ((short + 255) // 256 * 256)  # T < seg_T
    for bad in (0, 32, 100, -64):
        assert f(1, 1000, 2, 128, 128, bad) == 0
        assert _segmented(L, seg=bad) == INVALID
    assert _segmented(L, ST=None) == INVALID                 # S_T carries the state
    assert _segmented(L, dt=kda.KDA_F32) == UNSUPPORTED
    assert _segmented(L, dk=96, dv=96) == UNSUPPORTED
    assert _segmented(L, g_min=-6.0) == UNSUPPORTED
    assert _segmented(L, q=BASE + 8) == ALIGN
    assert _segmented(L, ws_bytes=f(1, 1000, 2, 128, 128, 256) - 1) == WS
    assert _segmented(L, ws=0) == WS
    assert _segmented(L, o=BASE) == ALIAS                    # o over q
    assert _segmented(L, S0=BASE * 3, ST=BASE * 3 + 4096) == ALIAS
