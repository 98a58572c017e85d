"""KDA (fine-grained gated delta rule) for B200: Python binding of libkda.so.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/kda.h. PyTorch provides device
memory and the current CUDA stream. There is no CPU fallback: if the library
cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["load", "chunk_fwd", "chunk_fwd_varlen", "chunk_bwd", "chunk_fwd_noalloc", "noalloc_status", "decode_step",
           "workspace_size", "workspace_status", "chunk_fwd_timeout_test", "KDAError", "library_path", "STATUS"]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libkda.so")

STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_CUDA",
          4: "KDA_ERR_TIMEOUT"}
_DTYPE = {"f32": 0, "bf16": 1}
_ALGO = {"auto": 0, "simt": 1, "tc": 2, "tc_scan": 3}
# Variant switches (include/kda.h): gate "channel" = log_alpha [.., dk], "scalar" =
# one per token and head, "none" = no decay (log_alpha may be None).
GATES = {"channel": 0, "scalar": 1, "none": 2}


class KDAError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} -> {STATUS.get(code, code)}: {msg}")
        self.code = code


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load(build_if_stale: bool = True):
    """Load libkda.so (building it in-tree with nvcc if it is missing or older
    than its sources). Raises if it cannot be built or loaded."""
    global _lib
    if _lib is not None:
        return _lib
    if build_if_stale:
        from . import build as _build
        if not _build.up_to_date():
            _build.build()
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libkda.so not found at {_LIB_PATH}; run python -m gated_delta_rule_134_b200.build")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.kda_status_string.argtypes = [I]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_chunk_fwd_workspace_size.argtypes = [I] * 8
    lib.kda_chunk_fwd_workspace_size.restype = Z
    lib.kda_chunk_fwd.argtypes = [P] * 8 + [I] * 7 + [P, Z, P]
    lib.kda_chunk_fwd.restype = I
    lib.kda_chunk_fwd_ex.argtypes = [P] * 8 + [I] * 7 + [P, Z, I, P]
    lib.kda_chunk_fwd_ex.restype = I
    lib.kda_workspace_status.argtypes = [P, Z, P]
    lib.kda_chunk_fwd_timeout_test.argtypes = [P] * 8 + [I] * 7 + [P, Z, ctypes.c_longlong, P]
    lib.kda_chunk_fwd_timeout_test.restype = I
    lib.kda_workspace_status.restype = I
    lib.kda_decode_step.argtypes = [P] * 8 + [I] * 5 + [P]
    lib.kda_decode_step.restype = I
    lib.kda_chunk_fwd_noalloc.argtypes = [P] * 8 + [I] * 7 + [P]
    lib.kda_chunk_fwd_noalloc.restype = I
    lib.kda_noalloc_status.argtypes = [P]
    lib.kda_noalloc_status.restype = I
    lib.kda_chunk_fwd_v.argtypes = [P] * 8 + [I] * 9 + [P, Z, I, P]
    lib.kda_chunk_fwd_v.restype = I
    lib.kda_decode_step_v.argtypes = [P] * 8 + [I] * 7 + [P]
    lib.kda_decode_step_v.restype = I
    lib.kda_chunk_fwd_varlen.argtypes = [P] * 9 + [I] * 9 + [P, Z, I, P]
    lib.kda_chunk_fwd_varlen.restype = I
    lib.kda_chunk_bwd_workspace_size.argtypes = [I] * 5
    lib.kda_chunk_bwd_workspace_size.restype = Z
    lib.kda_chunk_bwd.argtypes = [P] * 14 + [I] * 8 + [P, Z, P]
    lib.kda_chunk_bwd.restype = I
    lib.kda_chunk_bwd_ex.argtypes = [P] * 14 + [I] * 9 + [P, Z, P]
    lib.kda_chunk_bwd_ex.restype = I
    lib.kda_chunk_bwd_workspace_size_ex.argtypes = [I] * 6
    lib.kda_chunk_bwd_workspace_size_ex.restype = Z
    _lib = lib
    return lib


def _check(fn: str, code: int):
    if code != 0:
        raise KDAError(fn, code, load().kda_status_string(code).decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_of(t) -> str:
    import torch
    if t.dtype == torch.float32:
        return "f32"
    if t.dtype == torch.bfloat16:
        return "bf16"
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _stream(stream, device=None):
    """The stream handle to pass: the given torch stream, else the current
    stream of `device` (the tensors' device), else of the current device."""
    import torch
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _on(device):
    """Make the tensors' device current for the call: the library launches on
    the current device (and the allocation-free entry point looks up its
    scratch array there), so it must be the device the pointers live on."""
    import torch
    return torch.cuda.device(device)


def _need(t, name, shape, dtype, device):
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor (this library has no CPU path)")
    if t.device != device or t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)} on {device}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def workspace_size(B, T, H, dk, dv, chunk=64, dtype="bf16", algo="auto") -> int:
    return int(load().kda_chunk_fwd_workspace_size(B, T, H, dk, dv, chunk, _DTYPE[dtype], _ALGO[algo]))


def _gate_shape(gate, lead, dk):
    if gate not in GATES:
        raise ValueError(f"gate must be one of {sorted(GATES)}")
    return None if gate == "none" else (tuple(lead) + (dk,) if gate == "channel" else tuple(lead))


def chunk_fwd(q, k, v, log_alpha, beta, S0=None, *, chunk: int = 64, algo: str = "auto",
              output_final_state: bool = True, o=None, S_T=None, workspace=None, stream=None,
              erase: bool = True, gate: str = "channel"):
    """kda_chunk_fwd(q, k, v, log_alpha, beta, S0 -> o, S_T) on CUDA tensors.

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; beta: [B,T,H]; log_alpha: [B,T,H,dk]
    (gate "channel"), [B,T,H] (gate "scalar") or None (gate "none"), all
    float32 or all bfloat16; S0: [B,H,dk,dv] float32 or None. erase=False
    selects the additive-write variants (kda_chunk_fwd_v). Returns (o, S_T)
    with S_T None when output_final_state is False."""
    import torch
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    _need(q, "q", (B, T, H, dk), dt, dev)
    _need(k, "k", (B, T, H, dk), dt, dev)
    gshape = _gate_shape(gate, (B, T, H), dk)
    if gshape is not None:
        _need(log_alpha, "log_alpha", gshape, dt, dev)
    _need(v, "v", (B, T, H, dv), dt, dev)
    _need(beta, "beta", (B, T, H), dt, dev)
    if S0 is not None:
        _need(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=dt, device=dev)
    _need(o, "o", (B, T, H, dv), dt, dev)
    if output_final_state and S_T is None:
        S_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", (B, H, dk, dv), torch.float32, dev)
    dts = _dtype_of(q)
    ws_bytes = workspace_size(B, T, H, dk, dv, chunk, dts, algo)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    la = log_alpha if gshape is not None else None
    with _on(dev):
        code = lib.kda_chunk_fwd_v(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(S0), _ptr(o),
                                   _ptr(S_T), B, T, H, dk, dv, chunk, _DTYPE[dts], int(bool(erase)), GATES[gate],
                                   _ptr(workspace), ws_len, _ALGO[algo], _stream(stream, dev))
    _check("kda_chunk_fwd_v", code)
    return o, S_T


def chunk_fwd_varlen(q, k, v, log_alpha, beta, cu_seqlens, S0=None, *, chunk: int = 64, algo: str = "auto",
                     output_final_state: bool = True, o=None, S_T=None, workspace=None, stream=None,
                     erase: bool = True, gate: str = "channel"):
    """kda_chunk_fwd_varlen: N packed sequences. q, k [total_T,H,dk]; v
    [total_T,H,dv]; beta [total_T,H]; log_alpha [total_T,H,dk] / [total_T,H] /
    None by gate; cu_seqlens int32 CUDA tensor [N+1]; S0 [N,H,dk,dv] float32
    or None. Returns (o [total_T,H,dv], S_T [N,H,dk,dv] or None)."""
    import torch
    lib = load()
    TT, H, dk = q.shape
    dv = v.shape[-1]
    N = cu_seqlens.numel() - 1
    dt, dev = q.dtype, q.device
    _need(q, "q", (TT, H, dk), dt, dev)
    _need(k, "k", (TT, H, dk), dt, dev)
    gshape = _gate_shape(gate, (TT, H), dk)
    if gshape is not None:
        _need(log_alpha, "log_alpha", gshape, dt, dev)
    _need(v, "v", (TT, H, dv), dt, dev)
    _need(beta, "beta", (TT, H), dt, dev)
    _need(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, dev)
    if S0 is not None:
        _need(S0, "S0", (N, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(TT, H, dv, dtype=dt, device=dev)
    _need(o, "o", (TT, H, dv), dt, dev)
    if output_final_state and S_T is None:
        S_T = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", (N, H, dk, dv), torch.float32, dev)
    dts = _dtype_of(q)
    # packed batches never take the segment scan: size the workspace for one pass
    ws_bytes = workspace_size(N, TT, H, dk, dv, chunk, dts, "tc" if algo == "auto" and dts == "bf16" and
                              dk == dv == 128 and chunk == 64 else algo)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    la = log_alpha if gshape is not None else None
    with _on(dev):
        code = lib.kda_chunk_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(S0), _ptr(o),
                                        _ptr(S_T), _ptr(cu_seqlens), N, TT, H, dk, dv, chunk, _DTYPE[dts],
                                        int(bool(erase)), GATES[gate], _ptr(workspace), ws_len, _ALGO[algo],
                                        _stream(stream, dev))
    _check("kda_chunk_fwd_varlen", code)
    return o, S_T


BWD_MODES = {"auto": 0, "all": 1, "low": 2}


def chunk_bwd(q, k, v, log_alpha, beta, S0, dO, dS_T=None, *, erase: bool = True, gate: str = "channel",
              want_dS0: bool = True, workspace=None, stream=None, memory: str = "auto") -> dict:
    """kda_chunk_bwd_ex: gradients of a loss with dL/do = dO [B,T,H,dv] and
    dL/dS_T = dS_T [B,H,dk,dv] (None: 0). Inputs as for chunk_fwd. memory:
    "auto", "all" (keep every chunk's state) or "low" (one per 64 tokens and a
    recompute sweep). Returns dict dq, dk, dv, dlog_alpha (None without a
    gate), dbeta, dS0 (None unless want_dS0)."""
    import torch
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    _need(q, "q", (B, T, H, dk), dt, dev)
    _need(k, "k", (B, T, H, dk), dt, dev)
    gshape = _gate_shape(gate, (B, T, H), dk)
    if gshape is not None:
        _need(log_alpha, "log_alpha", gshape, dt, dev)
    _need(v, "v", (B, T, H, dv), dt, dev)
    _need(beta, "beta", (B, T, H), dt, dev)
    _need(dO, "dO", (B, T, H, dv), dt, dev)
    if S0 is not None:
        _need(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    if dS_T is not None:
        _need(dS_T, "dS_T", (B, H, dk, dv), torch.float32, dev)
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
         "dlog_alpha": None if gshape is None else torch.empty(gshape, dtype=dt, device=dev),
         "dbeta": torch.empty_like(beta),
         "dS0": torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev) if want_dS0 else None}
    mode = BWD_MODES[memory]
    ws_bytes = int(lib.kda_chunk_bwd_workspace_size_ex(B, T, H, dk, dv, mode))
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    la = log_alpha if gshape is not None else None
    with _on(dev):
        code = lib.kda_chunk_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(S0), _ptr(dO),
                                    _ptr(dS_T), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlog_alpha"]),
                                    _ptr(g["dbeta"]), _ptr(g["dS0"]), B, T, H, dk, dv, _DTYPE[_dtype_of(q)],
                                    int(bool(erase)), GATES[gate], mode, _ptr(workspace), ws_len,
                                    _stream(stream, dev))
    _check("kda_chunk_bwd_ex", code)
    return g


def workspace_status(workspace, stream=None) -> int:
    """Synchronise and return the device-side status word of a workspace."""
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    dev = None if workspace is None else workspace.device
    with _on(dev):
        return int(load().kda_workspace_status(_ptr(workspace), ws_len, _stream(stream, dev)))


def decode_step(q, k, v, log_alpha, beta, S, *, S_out=None, o=None, stream=None, erase: bool = True,
                gate: str = "channel"):
    """kda_decode_step(q, k, v, log_alpha, beta, S -> o, S'): one token per
    sequence. q, k [N,H,dk]; log_alpha [N,H,dk] / [N,H] / None by gate; v
    [N,H,dv]; beta [N,H]; S [N,H,dk,dv] float32. S_out defaults to S
    (in-place update). Returns (o, S_out)."""
    import torch
    lib = load()
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    _need(q, "q", (N, H, dk), dt, dev)
    _need(k, "k", (N, H, dk), dt, dev)
    gshape = _gate_shape(gate, (N, H), dk)
    if gshape is not None:
        _need(log_alpha, "log_alpha", gshape, dt, dev)
    _need(v, "v", (N, H, dv), dt, dev)
    _need(beta, "beta", (N, H), dt, dev)
    _need(S, "S", (N, H, dk, dv), torch.float32, dev)
    if S_out is None:
        S_out = S
    _need(S_out, "S_out", (N, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(N, H, dv, dtype=dt, device=dev)
    _need(o, "o", (N, H, dv), dt, dev)
    la = log_alpha if gshape is not None else None
    with _on(dev):
        code = lib.kda_decode_step_v(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(S), _ptr(S_out),
                                     _ptr(o), N, H, dk, dv, _DTYPE[_dtype_of(q)], int(bool(erase)), GATES[gate],
                                     _stream(stream, dev))
    _check("kda_decode_step_v", code)
    return o, S_out


def chunk_fwd_noalloc(q, k, v, log_alpha, beta, S0=None, *, o, S_T=None, chunk: int = 64, stream=None):
    """kda_chunk_fwd_noalloc: the tensor-core prefill without a workspace.

    For callers that must not allocate device memory where they run the
    prefill: the library keeps the kernel's small scratch in a fixed array of
    its own, so only inputs and caller-owned outputs (o, and S_T if wanted)
    are passed. bf16 inputs, dk = dv = 128, chunk = 64. Calls that overlap on
    the GPU share that array and race; noalloc_status reads its status word.
    Returns (o, S_T)."""
    import torch
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    _need(q, "q", (B, T, H, dk), dt, dev)
    _need(k, "k", (B, T, H, dk), dt, dev)
    _need(log_alpha, "log_alpha", (B, T, H, dk), dt, dev)
    _need(v, "v", (B, T, H, dv), dt, dev)
    _need(beta, "beta", (B, T, H), dt, dev)
    _need(o, "o", (B, T, H, dv), dt, dev)
    if S0 is not None:
        _need(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    if S_T is not None:
        _need(S_T, "S_T", (B, H, dk, dv), torch.float32, dev)
    with _on(dev):
        code = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                                         _ptr(o), _ptr(S_T), B, T, H, dk, dv, chunk, _DTYPE[_dtype_of(q)],
                                         _stream(stream, dev))
    _check("kda_chunk_fwd_noalloc", code)
    return o, S_T


def chunk_fwd_timeout_test(q, k, v, log_alpha, beta, S0=None, *, o, S_T, workspace, wait_budget_cycles: int,
                           stream=None):
    """kda_chunk_fwd_timeout_test: the tensor-core prefill with its first k/q
    load withheld and every wait bounded by wait_budget_cycles SM cycles, so
    the kernel gives up and records KDA_ERR_TIMEOUT in `workspace` (read it
    with workspace_status). A test hook for the timeout path; o and S_T are
    left undefined."""
    import torch
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt, dev = q.dtype, q.device
    _need(q, "q", (B, T, H, dk), dt, dev)
    _need(k, "k", (B, T, H, dk), dt, dev)
    _need(log_alpha, "log_alpha", (B, T, H, dk), dt, dev)
    _need(v, "v", (B, T, H, dv), dt, dev)
    _need(beta, "beta", (B, T, H), dt, dev)
    _need(o, "o", (B, T, H, dv), dt, dev)
    _need(S_T, "S_T", (B, H, dk, dv), torch.float32, dev)
    if S0 is not None:
        _need(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    ws_len = workspace.numel() * workspace.element_size()
    with _on(dev):
        code = lib.kda_chunk_fwd_timeout_test(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                                              _ptr(o), _ptr(S_T), B, T, H, dk, dv, 64, _DTYPE[_dtype_of(q)],
                                              _ptr(workspace), ws_len, int(wait_budget_cycles),
                                              _stream(stream, dev))
    _check("kda_chunk_fwd_timeout_test", code)
    return o, S_T


def noalloc_status(device=None, stream=None) -> int:
    """kda_noalloc_status: synchronise and return the status word the last
    chunk_fwd_noalloc on `device` left in the library's own scratch array
    (0 = KDA_OK, 4 = KDA_ERR_TIMEOUT). Allocates nothing."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with _on(dev):
        return int(load().kda_noalloc_status(_stream(stream, dev)))
