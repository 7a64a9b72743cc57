"""libkda Python binding: chunked KDA forward (bounded-decay gated delta rule) on B200.

A thin ctypes layer over ``libkda.so`` (built in-tree by ``build.py``).  Each function
has the name of the C entry point it calls and does argument marshalling only: it
checks tensor devices, dtypes, shapes and contiguity, then passes raw device pointers
and the current CUDA stream.  Every step of the computation runs in the library's
CUDA kernels; there is no fallback.  If ``libkda.so`` is missing or the library returns
an error, these functions raise.

PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# KDA_DEBUG_CHECKS=1 selects the build with the kernels' index checks (libkda_debug.so)
LIB_PATH = os.path.join(HERE, "libkda_debug.so" if os.environ.get("KDA_DEBUG_CHECKS") == "1" else "libkda.so")

KDA_BF16 = 0
KDA_F32 = 1
KDA_CHUNK = 64
KDA_TILE = 16
KDA_G_MIN_LOWEST = -5.4
KDA_GATE_BOUNDED = 0
KDA_GATE_LOGSIGMOID = 1

STATUS = {
    0: "KDA_OK",
    1: "KDA_ERR_INVALID_ARG",
    2: "KDA_ERR_UNSUPPORTED",
    3: "KDA_ERR_ALIGNMENT",
    4: "KDA_ERR_ALIAS",
    5: "KDA_ERR_CUDA",
    6: "KDA_ERR_DEVICE_TIMEOUT",
    7: "KDA_ERR_WORKSPACE",
    8: "KDA_ERR_DEVICE_BOUNDS",
}

EXPORTS = (
    "kda_gate_fwd",
    "kda_chunk_fwd_workspace",
    "kda_chunk_fwd",
    "kda_decode_step",
    "kda_device_status",
    "kda_status_string",
    "kda_version",
    "kda_chunk_fwd_noalloc",
    "kda_chunk_fwd_noalloc_max_scratch",
    "kda_chunk_fwd_logsigmoid",
    "kda_chunk_fwd_prep",
    "kda_chunk_fwd_scan",
    "kda_selftest_device_timeout",
    "kda_chunk_fwd_varlen_workspace",
    "kda_chunk_fwd_varlen",
    "kda_gate_fwd_heads",
    "kda_chunk_fwd_scan_affine",
    "kda_state_combine",
    "kda_chunk_bwd_workspace",
    "kda_chunk_bwd_offsets",
    "kda_chunk_bwd",
    "kda_chunk_bwd_varlen_workspace",
    "kda_chunk_bwd_varlen",
    "kda_chunk_fwd_segmented_workspace",
    "kda_chunk_fwd_segmented",
    "kda_chunk_bwd_recorded",
)


class KdaError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call} failed: {STATUS.get(status, status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libkda.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{os.path.basename(LIB_PATH)} not found at {LIB_PATH}; build it with "
            "`python -m chunked_linear_attention_chunk_b200.build` (add --debug-checks for the debug build)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, L64, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int64, ctypes.c_size_t
    L.kda_gate_fwd.argtypes = [P, I, F, P, L64, P]
    L.kda_gate_fwd.restype = I
    L.kda_chunk_fwd_workspace.argtypes = [I, I, I, I, I, I]
    L.kda_chunk_fwd_workspace.restype = S
    L.kda_chunk_fwd.argtypes = [I, I, I, I, I, I, P, P, P, P, P, F, P, P, P, P, S, P]
    L.kda_chunk_fwd.restype = I
    L.kda_decode_step.argtypes = [I, I, I, I, I, P, P, P, P, P, F, P, P, P]
    L.kda_decode_step.restype = I
    L.kda_device_status.argtypes = [P]
    L.kda_device_status.restype = I
    L.kda_status_string.argtypes = [I]
    L.kda_status_string.restype = ctypes.c_char_p
    L.kda_version.argtypes = []
    L.kda_version.restype = I
    L.kda_chunk_fwd_noalloc.argtypes = [I, I, I, I, I, I, P, P, P, P, P, F, P, P, P, P]
    L.kda_chunk_fwd_noalloc.restype = I
    L.kda_chunk_fwd_noalloc_max_scratch.argtypes = []
    L.kda_chunk_fwd_noalloc_max_scratch.restype = S
    L.kda_chunk_fwd_logsigmoid.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, S, P]
    L.kda_chunk_fwd_logsigmoid.restype = I
    L.kda_chunk_fwd_prep.argtypes = [I, I, I, I, I, I, F, P, P, P, P, P, P, P, S, P]
    L.kda_chunk_fwd_prep.restype = I
    L.kda_chunk_fwd_scan.argtypes = [I, I, I, I, I, P, S, P, P, P, P]
    L.kda_chunk_fwd_scan.restype = I
    L.kda_selftest_device_timeout.argtypes = [ctypes.c_uint32, P]
    L.kda_selftest_device_timeout.restype = I
    L.kda_chunk_fwd_varlen_workspace.argtypes = [I, I, I, I, I, I]
    L.kda_chunk_fwd_varlen_workspace.restype = S
    L.kda_chunk_fwd_varlen.argtypes = [I, P, I, I, I, I, I, I, F, P, P, P, P, P, P, P, P, P, P, S, P]
    L.kda_gate_fwd_heads.argtypes = [P, I, F, P, L64, I, I, P, P]
    L.kda_gate_fwd_heads.restype = I
    L.kda_chunk_fwd_scan_affine.argtypes = [I, I, I, I, I, P, S, P, P, P]
    L.kda_chunk_fwd_scan_affine.restype = I
    L.kda_state_combine.argtypes = [I, I, I, I, I, P, P, P, P, P]
    L.kda_state_combine.restype = I
    L.kda_chunk_fwd_varlen.restype = I
    L.kda_chunk_bwd_workspace.argtypes = [I, I, I, I, I, I]
    L.kda_chunk_bwd_workspace.restype = S
    L.kda_chunk_bwd_offsets.argtypes = [I, I, I, I, I, P, P]
    L.kda_chunk_bwd_offsets.restype = I
    L.kda_chunk_bwd.argtypes = [I, I, I, I, I, I, P, P, P, P, P, F, P, P, P, P, P, P, P, P, P, P, P, P, S, P]
    L.kda_chunk_bwd.restype = I
    L.kda_chunk_bwd_varlen_workspace.argtypes = [I, I, I, I, I, I]
    L.kda_chunk_bwd_varlen_workspace.restype = S
    L.kda_chunk_bwd_varlen.argtypes = [I, P, I, I, I, I, I, F, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P]
    L.kda_chunk_bwd_varlen.restype = I
    L.kda_chunk_fwd_segmented_workspace.argtypes = [I, I, I, I, I, I]
    L.kda_chunk_fwd_segmented_workspace.restype = S
    L.kda_chunk_fwd_segmented.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, F, P, P, P, P, S, P]
    L.kda_chunk_fwd_segmented.restype = I
    L.kda_chunk_bwd_recorded.argtypes = L.kda_chunk_bwd.argtypes
    L.kda_chunk_bwd_recorded.restype = I
    _lib = L
    return L


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("libkda takes CUDA tensors only")
        if not t.is_contiguous():
            raise ValueError("libkda takes contiguous tensors only")


def _raise(st: int, call: str):
    if st != 0:
        raise KdaError(st, call)


def kda_gate_fwd(a: torch.Tensor, g_min: float = -5.0, out: torch.Tensor | None = None) -> torch.Tensor:
    """g = g_min * sigmoid(a) as float32 (fp64 evaluation, one rounding)."""
    _check_cuda(a, out)
    g = out if out is not None else torch.empty(a.shape, dtype=torch.float32, device=a.device)
    st = lib().kda_gate_fwd(_ptr(a), _dtype_code(a), float(g_min), _ptr(g), a.numel(), _stream(a.device))
    _raise(st, "kda_gate_fwd")
    return g


def kda_gate_fwd_heads(a: torch.Tensor, A_log: torch.Tensor, g_min: float = -5.0, out=None) -> torch.Tensor:
    """g = g_min * sigmoid(e^{A_log[h]} * a) for a [..., H, dk] (fp64 evaluation, one rounding)."""
    _check_cuda(a, A_log, out)
    H, dk = a.shape[-2], a.shape[-1]
    if A_log.dtype != torch.float32 or A_log.shape != (H,):
        raise ValueError("A_log must be float32 [H]")
    g = out if out is not None else torch.empty(a.shape, dtype=torch.float32, device=a.device)
    st = lib().kda_gate_fwd_heads(_ptr(a), _dtype_code(a), float(g_min), _ptr(A_log), a.numel() // (H * dk), H, dk,
                                  _ptr(g), _stream(a.device))
    _raise(st, "kda_gate_fwd_heads")
    return g


def kda_chunk_fwd_workspace(B: int, T: int, H: int, dk: int, dv: int, dtype=torch.bfloat16) -> int:
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(lib().kda_chunk_fwd_workspace(B, T, H, dk, dv, code))


def kda_chunk_fwd(q, k, v, a, beta, g_min: float = -5.0, S0=None, o=None, S_T=None,
                  workspace=None, return_state: bool = True):
    """Chunked forward.  q, k, a [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H] (bf16 or f32).
    S0 [B,H,dk,dv] float32 or None (zeros).  Returns (o, S_T); S_T is None when
    ``return_state`` is False and no S_T buffer is given.  S_T may be S0 (in place)."""
    _check_cuda(q, k, v, a, beta, S0, o, S_T, workspace)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    code = _dtype_code(q)
    for t in (k, v, a, beta):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, a, beta must share one dtype")
    if k.shape != q.shape or a.shape != q.shape or v.shape != (B, T, H, dv) or beta.shape != (B, T, H):
        raise ValueError("shape mismatch: q,k,a [B,T,H,dk], v [B,T,H,dv], beta [B,T,H]")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    need = int(lib().kda_chunk_fwd_workspace(B, T, H, dk, dv, code))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().kda_chunk_fwd(B, T, H, dk, dv, code, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta),
                             float(g_min), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace), ws_bytes,
                             _stream(q.device))
    _raise(st, "kda_chunk_fwd")
    return o, S_T


def kda_chunk_fwd_segmented_workspace(B: int, T: int, H: int, dk: int, dv: int, seg_T: int) -> int:
    return int(lib().kda_chunk_fwd_segmented_workspace(B, T, H, dk, dv, seg_T))


def kda_chunk_fwd_segmented(q, k, v, a, beta, seg_T: int, g_min: float = -5.0, S0=None, o=None, S_T=None,
                            workspace=None):
    """``kda_chunk_fwd`` (bf16) taken ``seg_T`` tokens at a time (a multiple of 64), the prep of
    each stretch overlapping the scan of the one before; bit for bit the same result.  Returns
    (o, S_T); S_T may be S0 (in place)."""
    _check_cuda(q, k, v, a, beta, S0, o, S_T, workspace)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    code = _dtype_code(q)
    for t in (k, v, a, beta):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, a, beta must share one dtype")
    if k.shape != q.shape or a.shape != q.shape or v.shape != (B, T, H, dv) or beta.shape != (B, T, H):
        raise ValueError("shape mismatch: q,k,a [B,T,H,dk], v [B,T,H,dv], beta [B,T,H]")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    need = int(lib().kda_chunk_fwd_segmented_workspace(B, T, H, dk, dv, int(seg_T)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().kda_chunk_fwd_segmented(B, T, H, dk, dv, code, int(seg_T), _ptr(q), _ptr(k), _ptr(v), _ptr(a),
                                       _ptr(beta), float(g_min), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace),
                                       ws_bytes, _stream(q.device))
    _raise(st, "kda_chunk_fwd_segmented")
    return o, S_T


def kda_chunk_bwd_workspace(B: int, T: int, H: int, dk: int, dv: int, dtype=torch.bfloat16) -> int:
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(lib().kda_chunk_bwd_workspace(B, T, H, dk, dv, code))


def kda_chunk_bwd_offsets(B: int, T: int, H: int, dk: int, dv: int):
    """Byte offsets in the backward workspace of the saved chunk states and of the state
    gradients (float32 [B, H, NT, dk, dv] each, NT = ceil(T / 64))."""
    a, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
    st = lib().kda_chunk_bwd_offsets(B, T, H, dk, dv, ctypes.byref(a), ctypes.byref(b))
    _raise(st, "kda_chunk_bwd_offsets")
    return int(a.value), int(b.value)


def _bwd_outputs(q, v, beta, n_state, H, dk, dv, return_dS0, A_log, out):
    dev = q.device
    shapes = {"dq": q.shape, "dk": q.shape, "dv": v.shape, "da": q.shape, "dbeta": beta.shape,
              "dS0": (n_state, H, dk, dv), "dA_log": (H,)}
    g = dict(out or {})
    for name, shp in shapes.items():
        if name in g:
            continue
        if (name == "dS0" and not return_dS0) or (name == "dA_log" and A_log is None):
            g[name] = None
        else:
            g[name] = torch.empty(shp, dtype=torch.float32, device=dev)
    _check_cuda(*g.values())
    return g


def _bwd_checks(q, k, v, a, beta, dO, A_log, token_dims):
    if any(t.dtype != torch.bfloat16 for t in (q, k, v, a, beta, dO)):
        raise TypeError("the backward takes bfloat16 q, k, v, a, beta, dO")
    if k.shape != q.shape or a.shape != q.shape or dO.shape != v.shape or \
            v.shape[:token_dims] != q.shape[:token_dims] or beta.shape != q.shape[:token_dims + 1]:
        raise ValueError("shape mismatch: q, k, a [.., H, dk], v, dO [.., H, dv], beta [.., H]")
    if A_log is not None and (A_log.dtype != torch.float32 or A_log.shape != (q.shape[-2],)):
        raise ValueError("A_log must be float32 [H]")


def kda_chunk_bwd(q, k, v, a, beta, dO, g_min: float = -5.0, S0=None, dS_T=None, workspace=None,
                  return_dS0: bool = True, out=None, A_log=None, _recorded: bool = False):
    """Gradients of the bf16 chunked forward.  q, k, a [B,T,H,dk], v and dO [B,T,H,dv],
    beta [B,T,H] (bfloat16); S0 and dS_T [B,H,dk,dv] float32 or None (zeros); A_log float32
    [H] or None (the gate's per-head scale e^{A_log[h]}).  Returns a dict of float32 tensors
    dq, dk, dv, da, dbeta, dS0 (None unless ``return_dS0``) and dA_log (None without
    A_log); ``out`` may supply some of those tensors."""
    _check_cuda(q, k, v, a, beta, dO, S0, dS_T, workspace, A_log)
    _bwd_checks(q, k, v, a, beta, dO, A_log, 2)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    g = _bwd_outputs(q, v, beta, B, H, dk, dv, return_dS0, A_log, out)
    need = int(lib().kda_chunk_bwd_workspace(B, T, H, dk, dv, KDA_BF16))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fn = lib().kda_chunk_bwd_recorded if _recorded else lib().kda_chunk_bwd
    st = fn(B, T, H, dk, dv, KDA_BF16, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta),
            float(g_min), _ptr(A_log), _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(g["dq"]), _ptr(g["dk"]),
            _ptr(g["dv"]), _ptr(g["da"]), _ptr(g["dbeta"]), _ptr(g["dS0"]), _ptr(g["dA_log"]),
            _ptr(workspace), ws_bytes, _stream(q.device))
    _raise(st, "kda_chunk_bwd_recorded" if _recorded else "kda_chunk_bwd")
    return g


def kda_chunk_bwd_recorded(q, k, v, a, beta, dO, workspace, g_min: float = -5.0, S0=None, dS_T=None,
                           return_dS0: bool = True, out=None, A_log=None):
    """``kda_chunk_bwd`` when ``workspace`` (at least ``kda_chunk_bwd_workspace`` bytes) already
    holds the records a bf16 ``kda_chunk_fwd`` (or ``kda_chunk_fwd_prep``) wrote into it for the
    same inputs, g_min and A_log: the backward's own prep is skipped."""
    if workspace is None:
        raise ValueError("kda_chunk_bwd_recorded needs the workspace the forward wrote its records to")
    return kda_chunk_bwd(q, k, v, a, beta, dO, g_min, S0=S0, dS_T=dS_T, workspace=workspace, return_dS0=return_dS0,
                         out=out, A_log=A_log, _recorded=True)


def kda_chunk_bwd_varlen_workspace(N: int, T: int, H: int, dk: int, dv: int) -> int:
    return int(lib().kda_chunk_bwd_varlen_workspace(N, T, H, dk, dv, KDA_BF16))


def kda_chunk_bwd_varlen(q, k, v, a, beta, dO, cu_seqlens, g_min: float = -5.0, S0=None, dS_T=None,
                         workspace=None, return_dS0: bool = True, out=None, A_log=None):
    """Backward over a packed batch: q, k, a [T,H,dk], v and dO [T,H,dv], beta [T,H]
    (bfloat16); cu_seqlens int32 [N+1] on the device; S0, dS_T [N,H,dk,dv] float32 or None.
    Returns the dict of ``kda_chunk_bwd`` with token gradients [T,H,.] and dS0 [N,H,dk,dv]."""
    _check_cuda(q, k, v, a, beta, dO, cu_seqlens, S0, dS_T, workspace, A_log)
    _bwd_checks(q, k, v, a, beta, dO, A_log, 1)
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    T, H, dk = q.shape
    dv = v.shape[-1]
    N = cu_seqlens.numel() - 1
    g = _bwd_outputs(q, v, beta, N, H, dk, dv, return_dS0, A_log, out)
    need = int(lib().kda_chunk_bwd_varlen_workspace(N, T, H, dk, dv, KDA_BF16))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().kda_chunk_bwd_varlen(N, _ptr(cu_seqlens), T, H, dk, dv, KDA_BF16, float(g_min), _ptr(A_log),
                                    _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta), _ptr(S0), _ptr(dO), _ptr(dS_T),
                                    _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["da"]), _ptr(g["dbeta"]),
                                    _ptr(g["dS0"]), _ptr(g["dA_log"]), _ptr(workspace), ws_bytes, _stream(q.device))
    _raise(st, "kda_chunk_bwd_varlen")
    return g


def kda_chunk_fwd_logsigmoid(q, k, v, a, beta, S0=None, o=None, S_T=None, workspace=None,
                             return_state: bool = True):
    """The ablation path: ``kda_chunk_fwd`` with the unbounded gate g = log(sigmoid(a)) and
    element-wise diagonal tiles (bf16 only).  Same shapes and return value."""
    _check_cuda(q, k, v, a, beta, S0, o, S_T, workspace)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    code = _dtype_code(q)
    for t in (k, v, a, beta):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, a, beta must share one dtype")
    if k.shape != q.shape or a.shape != q.shape or v.shape != (B, T, H, dv) or beta.shape != (B, T, H):
        raise ValueError("shape mismatch: q,k,a [B,T,H,dk], v [B,T,H,dv], beta [B,T,H]")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    need = int(lib().kda_chunk_fwd_workspace(B, T, H, dk, dv, code))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().kda_chunk_fwd_logsigmoid(B, T, H, dk, dv, code, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta),
                                        _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace), ws_bytes,
                                        _stream(q.device))
    _raise(st, "kda_chunk_fwd_logsigmoid")
    return o, S_T


def kda_chunk_fwd_varlen_workspace(N: int, T: int, H: int, dk: int, dv: int, dtype=torch.bfloat16) -> int:
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(lib().kda_chunk_fwd_varlen_workspace(N, T, H, dk, dv, code))


def kda_chunk_fwd_varlen(q, k, v, a, beta, cu_seqlens, g_min: float = -5.0, gate: int = KDA_GATE_BOUNDED,
                         S0=None, o=None, S_T=None, workspace=None, return_state: bool = True, A_log=None):
    """Chunked forward over a packed batch: q, k, a [T,H,dk]; v [T,H,dv]; beta [T,H] (bf16);
    cu_seqlens int32 [N+1] on the device (sequence s = tokens cu[s]..cu[s+1]-1).  S0 / S_T
    are [N,H,dk,dv] float32.  Returns (o [T,H,dv], S_T)."""
    _check_cuda(q, k, v, a, beta, cu_seqlens, S0, o, S_T, workspace, A_log)
    if q.dim() == 4 and q.shape[0] == 1:
        q, k, v, a, beta = (t[0] for t in (q, k, v, a, beta))
    T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
        raise TypeError("cu_seqlens must be a 1-D int32 tensor")
    N = cu_seqlens.numel() - 1
    code = _dtype_code(q)
    if o is None:
        o = torch.empty((T, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None and return_state:
        S_T = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    need = int(lib().kda_chunk_fwd_varlen_workspace(N, T, H, dk, dv, code))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().kda_chunk_fwd_varlen(N, _ptr(cu_seqlens), T, H, dk, dv, code, int(gate), float(g_min), _ptr(A_log),
                                    _ptr(q),
                                    _ptr(k), _ptr(v), _ptr(a), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_T),
                                    _ptr(workspace), ws_bytes, _stream(q.device))
    _raise(st, "kda_chunk_fwd_varlen")
    return o, S_T


def kda_chunk_fwd_prep(q, k, v, a, beta, workspace, g_min: float = -5.0, gate: int = KDA_GATE_BOUNDED,
                       A_log=None):
    """First stage of the bf16 chunked forward: one record per (batch*head, chunk) into
    ``workspace`` (uint8, at least ``kda_chunk_fwd_workspace`` bytes).  ``A_log`` (float32
    [H], optional) scales the gate's argument by e^{A_log[h]}."""
    _check_cuda(q, k, v, a, beta, workspace, A_log)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype != torch.bfloat16 or any(t.dtype != torch.bfloat16 for t in (k, v, a, beta)):
        raise TypeError("kda_chunk_fwd_prep takes bfloat16 tensors")
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib().kda_chunk_fwd_prep(B, T, H, dk, dv, int(gate), float(g_min), _ptr(A_log), _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(a),
                                  _ptr(beta), _ptr(workspace), ws_bytes, _stream(q.device))
    _raise(st, "kda_chunk_fwd_prep")


def kda_chunk_fwd_scan(workspace, B: int, T: int, H: int, dk: int, dv: int, S0=None, o=None, S_T=None,
                       return_state: bool = True):
    """Second stage: the chunk recursion over the records of ``kda_chunk_fwd_prep``.
    Returns (o, S_T) like ``kda_chunk_fwd``."""
    _check_cuda(workspace, S0, o, S_T)
    dev = workspace.device
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib().kda_chunk_fwd_scan(B, T, H, dk, dv, _ptr(workspace), ws_bytes, _ptr(S0), _ptr(o), _ptr(S_T),
                                  _stream(dev))
    _raise(st, "kda_chunk_fwd_scan")
    return o, S_T


def kda_chunk_fwd_scan_affine(workspace, B: int, T: int, H: int, dk: int, dv: int, S_zero=None, M=None):
    """Affine map of the segment whose records ``workspace`` holds: returns (S_zero, M) with
    S_out = M S_in + S_zero; S_zero [B,H,dk,dv], M [B,H,dk,dk] (float32)."""
    _check_cuda(workspace, S_zero, M)
    dev = workspace.device
    if S_zero is None:
        S_zero = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    if M is None:
        M = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib().kda_chunk_fwd_scan_affine(B, T, H, dk, dv, _ptr(workspace), ws_bytes, _ptr(S_zero), _ptr(M),
                                         _stream(dev))
    _raise(st, "kda_chunk_fwd_scan_affine")
    return S_zero, M


def kda_state_combine(M, S_zero, S0=None, S_in=None):
    """Incoming states of R consecutive segments from their maps: M, S_zero [R,B,H,d,d];
    returns S_in [R+1,B,H,d,d] with S_in[0] = S0 (or 0) and S_in[R] the final state."""
    _check_cuda(M, S_zero, S0, S_in)
    R, B, H, dk, dv = S_zero.shape
    if S_in is None:
        S_in = torch.empty((R + 1, B, H, dk, dv), dtype=torch.float32, device=M.device)
    st = lib().kda_state_combine(R, B, H, dk, dv, _ptr(M), _ptr(S_zero), _ptr(S0), _ptr(S_in), _stream(M.device))
    _raise(st, "kda_state_combine")
    return S_in


def kda_chunk_fwd_noalloc(q, k, v, a, beta, g_min: float = -5.0, S0=None, o=None, S_T=None,
                          return_state: bool = True):
    """Like ``kda_chunk_fwd`` but with the library's built-in scratch instead of a
    workspace (for callers that cannot allocate device memory; see include/kda.h)."""
    _check_cuda(q, k, v, a, beta, S0, o, S_T)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t in (k, v, a, beta):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, a, beta must share one dtype")
    if k.shape != q.shape or a.shape != q.shape or v.shape != (B, T, H, dv) or beta.shape != (B, T, H):
        raise ValueError("shape mismatch: q,k,a [B,T,H,dk], v [B,T,H,dv], beta [B,T,H]")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    st = lib().kda_chunk_fwd_noalloc(B, T, H, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(a),
                                     _ptr(beta), float(g_min), _ptr(S0), _ptr(o), _ptr(S_T), _stream(q.device))
    _raise(st, "kda_chunk_fwd_noalloc")
    return o, S_T


def kda_chunk_fwd_noalloc_max_scratch() -> int:
    """Bytes of the built-in device scratch kda_chunk_fwd_noalloc uses."""
    return int(lib().kda_chunk_fwd_noalloc_max_scratch())


def kda_decode_step(q, k, v, a, beta, S, g_min: float = -5.0, o=None):
    """One decode token.  q, k, a [N,H,dk]; v [N,H,dv]; beta [N,H]; S [N,H,dk,dv] float32,
    updated in place.  Returns o [N,H,dv]."""
    _check_cuda(q, k, v, a, beta, S, o)
    N, H, dk = q.shape
    dv = v.shape[-1]
    if S.dtype != torch.float32 or S.shape != (N, H, dk, dv):
        raise ValueError("S must be float32 [N,H,dk,dv]")
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    st = lib().kda_decode_step(N, H, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta),
                               float(g_min), _ptr(S), _ptr(o), _stream(q.device))
    _raise(st, "kda_decode_step")
    return o


def kda_device_status(device=None) -> int:
    """Synchronise the current stream and return/clear the device status word."""
    dev = device if device is not None else torch.cuda.current_device()
    return int(lib().kda_device_status(_stream(dev)))


def kda_selftest_device_timeout(limit_us: int = 20000, device=None) -> None:
    """Launch the library's bounded-wait self-test: a kernel whose wait runs out after
    ``limit_us`` and records KDA_ERR_DEVICE_TIMEOUT (read it with kda_device_status)."""
    dev = device if device is not None else torch.cuda.current_device()
    _raise(lib().kda_selftest_device_timeout(int(limit_us), _stream(dev)), "kda_selftest_device_timeout")


def kda_status_string(status: int) -> str:
    return lib().kda_status_string(int(status)).decode()


def kda_version() -> int:
    return int(lib().kda_version())
