"""Thin ctypes binding of libgret (argument marshalling only).

``gret_prefill``, ``gret_decode_step``, ``gret_prefill_workspace_size``,
``gret_prefill_path``, ``gret_last_device_status``, ``gret_status_string`` and
``gret_version`` call the C ABI of ``include/gret.h`` one to one with raw
pointers.  ``prefill`` and ``decode_step`` are conveniences for torch CUDA
tensors: they check dtypes and shapes, allocate outputs and scratch with
torch's allocator and pass the current stream.  Every step of the mixer runs
in the CUDA library; there is no fallback, and a missing library raises.
"""
from __future__ import annotations

import ctypes
import enum
import os
import threading
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgret.so")
_lib = None
_lock = threading.Lock()


class Status(enum.IntEnum):
    OK = 0
    ERR_INVALID_ARG = 1
    ERR_UNSUPPORTED = 2
    ERR_CUDA = 3
    ERR_TIMEOUT = 4


class Dtype(enum.IntEnum):
    F32 = 0
    BF16 = 1


class Epilogue(enum.IntEnum):
    GN_SWISH = 0
    NONE = 1


class Path(enum.IntEnum):
    NONE = 0
    SIMT = 1
    TC = 2


class GretError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = Status(status)
        super().__init__(f"{what}: {self.status.name}" if what else self.status.name)


# Exported C symbols and their signatures.
_VP, _FP, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "gret_prefill": (_I, [_VP, _VP, _VP, _FP, _VP, _F, _I, _VP, _FP, _I, _I, _I, _I, _I, _I, _F, _I,
                          _VP, _SZ, _VP]),
    "gret_prefill_noalloc": (_I, [_VP, _VP, _VP, _FP, _VP, _F, _I, _VP, _FP, _I, _I, _I, _I, _I, _I, _F,
                                  _I, _VP]),
    "gret_prefill_from_state": (_I, [_VP, _VP, _VP, _FP, _VP, _FP, _F, _I, _VP, _FP, _I, _I, _I, _I, _I, _I,
                                     _F, _I, _VP, _SZ, _VP]),
    "gret_prefill_resume": (_I, [_VP, _VP, _VP, _FP, _VP, _FP, _F, _I, _VP, _FP, _I, _I, _I, _I, _I, _I,
                                 _F, _I, _VP, _SZ, _VP]),
    "gret_prefill_state_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "gret_prefill_state": (_I, [_VP, _VP, _FP, _F, _I, _FP, _FP, _I, _I, _I, _I, _I, _I, _VP, _SZ, _VP]),
    "gret_state_fold": (_I, [_FP, _FP, _I, _I, _FP, _FP, _I, _I, _I, _I, _VP]),
    "gret_prefill_backward_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "gret_prefill_backward_launches": (_I, [_I, _I, _I, _I, _I, _I]),
    "gret_prefill_backward": (_I, [_VP, _VP, _VP, _FP, _VP, _FP, _VP, _FP, _F, _F, _I, _VP, _VP, _VP, _FP, _VP, _FP,
                                   _I, _I, _I, _I, _I, _I, _VP, _SZ, _VP]),
    "gret_prefill_varlen": (_I, [_VP, _VP, _VP, _FP, _VP, _FP, _VP, _I, _I, _I, _F, _I, _VP, _FP, _I, _I, _I, _I,
                                 _F, _I, _VP, _SZ, _VP]),
    "gret_prefill_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "gret_prefill_varlen_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "gret_prefill_varlen_launches": (_I, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "gret_prefill_launches": (_I, [_I, _I, _I, _I, _I, _I, _I]),
    "gret_prefill_path": (_I, [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_int)]),
    "gret_decode_step": (_I, [_VP, _VP, _VP, _FP, _VP, _FP, _VP, _I, _I, _I, _I, _F, _I, _F, _I, _VP]),
    "gret_last_device_status": (_I, [_VP]),
    "gret_set_profile_events": (None, [_VP, _VP]),
    "gret_debug_inject_timeout": (None, [_I]),
    "gret_set_gate_profile_events": (None, [_VP, _VP]),
    "gret_prefill_projected": (_I, [_VP, _VP, _VP, _VP, _FP, _I, _VP, _F, _I, _VP, _FP, _I, _I, _I, _I, _I, _I,
                                    _F, _I, _VP, _SZ, _VP]),
    "gret_prefill_projected_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "gret_status_string": (ctypes.c_char_p, [_I]),
    "gret_version": (_I, []),
}


def load():
    """Load libgret.so (built by ``gated_retention_sequence_b200.build``); raises if absent."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libgret.so is not built ({LIB_PATH}); run __graft_entry__.build()")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


# ---------------------------------------------------------------- raw C calls
def gret_prefill(Q, K, V, gate_logits, G, tau, chunk, O, S_final, B, H, N, dk, dv, io_dtype, eps,
                 epi, workspace, workspace_bytes, stream) -> int:
    return load().gret_prefill(Q, K, V, gate_logits, G, tau, chunk, O, S_final, B, H, N, dk, dv,
                               int(io_dtype), eps, int(epi), workspace, workspace_bytes, stream)


def gret_prefill_from_state(Q, K, V, gate_logits, G, S0, tau, chunk, O, S_final, B, H, N, dk, dv, io_dtype,
                            eps, epi, workspace, workspace_bytes, stream) -> int:
    return load().gret_prefill_from_state(Q, K, V, gate_logits, G, S0, tau, chunk, O, S_final, B, H, N, dk, dv,
                                          int(io_dtype), eps, int(epi), workspace, workspace_bytes, stream)


def gret_prefill_resume(Q, K, V, gate_logits, G, S0, tau, chunk, O, S_final, B, H, N, dk, dv, io_dtype,
                        eps, epi, workspace, workspace_bytes, stream) -> int:
    return load().gret_prefill_resume(Q, K, V, gate_logits, G, S0, tau, chunk, O, S_final, B, H, N, dk, dv,
                                      int(io_dtype), eps, int(epi), workspace, workspace_bytes, stream)


def gret_prefill_varlen(Q, K, V, gate_logits, G, S0, cu_seqlens, num_seqs, total_tokens, max_seqlen, tau, chunk,
                        O, S_final, H, dk, dv, io_dtype, eps, epi, workspace, workspace_bytes, stream) -> int:
    return load().gret_prefill_varlen(Q, K, V, gate_logits, G, S0, cu_seqlens, num_seqs, total_tokens, max_seqlen,
                                      tau, chunk, O, S_final, H, dk, dv, int(io_dtype), eps, int(epi), workspace,
                                      workspace_bytes, stream)


def gret_prefill_state_workspace_size(B, H, N, dk, dv, chunk, io_dtype) -> int:
    return load().gret_prefill_state_workspace_size(B, H, N, dk, dv, chunk, int(io_dtype))


def gret_prefill_state(K, V, gate_logits, tau, chunk, dS, decay, B, H, N, dk, dv, io_dtype, workspace,
                       workspace_bytes, stream) -> int:
    return load().gret_prefill_state(K, V, gate_logits, tau, chunk, dS, decay, B, H, N, dk, dv, int(io_dtype),
                                     workspace, workspace_bytes, stream)


def gret_state_fold(dS_all, decay_all, num_slices, slice_, S0, S_in, B, H, dk, dv, stream) -> int:
    return load().gret_state_fold(dS_all, decay_all, num_slices, slice_, S0, S_in, B, H, dk, dv, stream)


def gret_prefill_backward_workspace_size(B, H, N, dk, dv, io_dtype) -> int:
    return load().gret_prefill_backward_workspace_size(B, H, N, dk, dv, int(io_dtype))


def gret_prefill_backward_launches(B, H, N, dk, dv, io_dtype) -> int:
    return load().gret_prefill_backward_launches(B, H, N, dk, dv, int(io_dtype))


def gret_prefill_backward(Q, K, V, gate_logits, G, S0, dO, dS_final, tau, eps, epi, dQ, dK, dV, dz, dG, dS0, B, H,
                          N, dk, dv, io_dtype, workspace, workspace_bytes, stream) -> int:
    return load().gret_prefill_backward(Q, K, V, gate_logits, G, S0, dO, dS_final, tau, eps, int(epi), dQ, dK, dV,
                                        dz, dG, dS0, B, H, N, dk, dv, int(io_dtype), workspace, workspace_bytes,
                                        stream)


def gret_prefill_noalloc(Q, K, V, gate_logits, G, tau, chunk, O, S_final, B, H, N, dk, dv, io_dtype, eps,
                         epi, stream) -> int:
    return load().gret_prefill_noalloc(Q, K, V, gate_logits, G, tau, chunk, O, S_final, B, H, N, dk, dv,
                                       int(io_dtype), eps, int(epi), stream)


def gret_prefill_workspace_size(B, H, N, dk, dv, chunk, io_dtype) -> int:
    return load().gret_prefill_workspace_size(B, H, N, dk, dv, chunk, int(io_dtype))


def gret_prefill_varlen_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, chunk, io_dtype) -> int:
    return load().gret_prefill_varlen_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, chunk,
                                                     int(io_dtype))


def gret_prefill_varlen_launches(num_seqs, total_tokens, max_seqlen, H, dk, dv, chunk, io_dtype) -> int:
    return load().gret_prefill_varlen_launches(num_seqs, total_tokens, max_seqlen, H, dk, dv, chunk, int(io_dtype))


def gret_prefill_launches(B, H, N, dk, dv, chunk, io_dtype) -> int:
    return load().gret_prefill_launches(B, H, N, dk, dv, chunk, int(io_dtype))


def gret_prefill_path(B, H, N, dk, dv, chunk, io_dtype) -> Tuple[Path, int]:
    segs = ctypes.c_int(0)
    p = load().gret_prefill_path(B, H, N, dk, dv, chunk, int(io_dtype), ctypes.byref(segs))
    return Path(p), segs.value


def gret_decode_step(q, k, v, gate_logit, g, S_inout, o, num_seqs, H, dk, dv, tau, io_dtype, eps,
                     epi, stream) -> int:
    return load().gret_decode_step(q, k, v, gate_logit, g, S_inout, o, num_seqs, H, dk, dv, tau,
                                   int(io_dtype), eps, int(epi), stream)


def gret_last_device_status(stream=None) -> int:
    return load().gret_last_device_status(stream)


def gret_set_profile_events(start, stop) -> None:
    load().gret_set_profile_events(start, stop)


def gret_debug_inject_timeout(calls: int) -> None:
    load().gret_debug_inject_timeout(int(calls))


def gret_set_gate_profile_events(start, stop) -> None:
    load().gret_set_gate_profile_events(start, stop)


def gret_prefill_projected(Q, K, V, X, W_gamma, d_model, G, tau, chunk, O, S_final, B, H, N, dk, dv, io_dtype, eps,
                           epi, workspace, workspace_bytes, stream) -> int:
    return load().gret_prefill_projected(Q, K, V, X, W_gamma, d_model, G, tau, chunk, O, S_final, B, H, N, dk, dv,
                                         int(io_dtype), eps, int(epi), workspace, workspace_bytes, stream)


def gret_prefill_projected_workspace_size(B, H, N, dk, dv, chunk, d_model, io_dtype) -> int:
    return load().gret_prefill_projected_workspace_size(B, H, N, dk, dv, chunk, d_model, int(io_dtype))


def gret_status_string(status: int) -> str:
    return load().gret_status_string(int(status)).decode()


def gret_version() -> int:
    return load().gret_version()


# ---------------------------------------------------------------- torch helpers
def _torch():
    import torch
    return torch


def _io_of(t) -> Dtype:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return Dtype.BF16
    if t.dtype == torch.float32:
        return Dtype.F32
    raise TypeError(f"unsupported io dtype {t.dtype}")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _scratch(workspace, ws_bytes, dev, st):
    """The caller's workspace when it is large enough, else a new one from
    torch's allocator.  A new one is allocated on the current stream but used
    by kernels on ``st``; it is dropped when the call returns, so it is
    recorded on ``st`` to keep the caching allocator from handing its memory
    out again before those kernels finish."""
    torch = _torch()
    if not ws_bytes:
        return workspace
    if workspace is not None and workspace.numel() * workspace.element_size() >= ws_bytes:
        return workspace
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if st != torch.cuda.current_stream(dev):
        workspace.record_stream(st)
    return workspace


def _need_g(G, epi, name="G"):
    if epi == Epilogue.GN_SWISH and G is None:
        raise ValueError(f"{name} is required for epilogue 'gn_swish' (pass epilogue='none' for the pre-norm Y)")


def _check(t, name, dtype, shape, device):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def prefill(Q, K, V, z, G, tau: float, chunk: int, eps: float = 1e-5, epilogue: str = "gn_swish",
            O=None, S_final=None, want_state: bool = True, workspace=None, stream=None, S0=None,
            resume: bool = False):
    """Chunkwise prefill from the zero state, or from ``S0`` (gret_prefill_from_state).

    ``resume=True`` (gret_prefill_resume) reuses the decay sums and state-pass
    pieces that ``prefill_state`` left in ``workspace`` for the same K, V, z.

    Q, K [B,N,H,dk] and V, G [B,N,H,dv] in bf16 or fp32; z [B,N,H] fp32 gate logits;
    S0 [B,H,dk,dv] fp32 or None.
    Returns (O [B,N,H,dv] in the io dtype, S_final [B,H,dk,dv] fp32 or None).
    ``epilogue='none'`` returns the pre-norm Y in O (G may be None).
    """
    torch = _torch()
    B, N, H, dk = Q.shape
    dv = V.shape[-1]
    dev = Q.device
    io = _io_of(Q)
    epi = Epilogue.NONE if epilogue == "none" else Epilogue.GN_SWISH
    _need_g(G, epi)
    _check(Q, "Q", Q.dtype, (B, N, H, dk), dev)
    _check(K, "K", Q.dtype, (B, N, H, dk), dev)
    _check(V, "V", Q.dtype, (B, N, H, dv), dev)
    _check(z, "z", torch.float32, (B, N, H), dev)
    if G is not None:
        _check(G, "G", Q.dtype, (B, N, H, dv), dev)
    if O is None:
        O = torch.empty((B, N, H, dv), dtype=Q.dtype, device=dev)
    _check(O, "O", Q.dtype, (B, N, H, dv), dev)
    if S_final is None and want_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    if S_final is not None:
        _check(S_final, "S_final", torch.float32, (B, H, dk, dv), dev)
    if S0 is not None:
        _check(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    if resume and workspace is None:
        raise ValueError("resume=True needs the workspace prefill_state wrote")
    with torch.cuda.device(dev):
        ws_bytes = (gret_prefill_state_workspace_size if resume else gret_prefill_workspace_size)(
            B, H, N, dk, dv, chunk, io)
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        if resume and ws_bytes and workspace.numel() * workspace.element_size() < ws_bytes:
            raise ValueError("the workspace is smaller than gret_prefill_state_workspace_size")
        workspace = _scratch(workspace, ws_bytes, dev, st)
        ws = _ptr(workspace) if ws_bytes else None
        if resume:
            status = gret_prefill_resume(_ptr(Q), _ptr(K), _ptr(V), _ptr(z), _ptr(G), _ptr(S0), float(tau),
                                         int(chunk), _ptr(O), _ptr(S_final), B, H, N, dk, dv, io, float(eps), epi,
                                         ws, ws_bytes, st.cuda_stream)
        elif S0 is None:
            status = gret_prefill(_ptr(Q), _ptr(K), _ptr(V), _ptr(z), _ptr(G), float(tau), int(chunk),
                                  _ptr(O), _ptr(S_final), B, H, N, dk, dv, io, float(eps), epi, ws, ws_bytes,
                                  st.cuda_stream)
        else:
            status = gret_prefill_from_state(_ptr(Q), _ptr(K), _ptr(V), _ptr(z), _ptr(G), _ptr(S0), float(tau),
                                             int(chunk), _ptr(O), _ptr(S_final), B, H, N, dk, dv, io,
                                             float(eps), epi, ws, ws_bytes, st.cuda_stream)
    if status != Status.OK:
        raise GretError(status, "gret_prefill_resume" if resume else
                        "gret_prefill" if S0 is None else "gret_prefill_from_state")
    return O, S_final


def prefill_projected(Q, K, V, X, W_gamma, G, tau: float, chunk: int, eps: float = 1e-5, epilogue: str = "gn_swish",
                      O=None, S_final=None, want_state: bool = True, workspace=None, stream=None):
    """Prefill with the gate logits computed from z = X W_gamma (gret_prefill_projected).

    Q, K [B,N,H,dk]; V, G [B,N,H,dv]; X [B,N,d_model] (all bf16 or all fp32);
    W_gamma [d_model,H] fp32.  Returns (O, S_final) as ``prefill`` does."""
    torch = _torch()
    B, N, H, dk = Q.shape
    dv = V.shape[-1]
    d_model = X.shape[-1]
    dev = Q.device
    io = _io_of(Q)
    epi = Epilogue.NONE if epilogue == "none" else Epilogue.GN_SWISH
    _need_g(G, epi)
    _check(K, "K", Q.dtype, (B, N, H, dk), dev)
    _check(V, "V", Q.dtype, (B, N, H, dv), dev)
    _check(X, "X", Q.dtype, (B, N, d_model), dev)
    _check(W_gamma, "W_gamma", torch.float32, (d_model, H), dev)
    if G is not None:
        _check(G, "G", Q.dtype, (B, N, H, dv), dev)
    if O is None:
        O = torch.empty((B, N, H, dv), dtype=Q.dtype, device=dev)
    _check(O, "O", Q.dtype, (B, N, H, dv), dev)
    if S_final is None and want_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    if S_final is not None:
        _check(S_final, "S_final", torch.float32, (B, H, dk, dv), dev)
    with torch.cuda.device(dev):
        ws_bytes = gret_prefill_projected_workspace_size(B, H, N, dk, dv, chunk, d_model, io)
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        workspace = _scratch(workspace, ws_bytes, dev, st)
        status = gret_prefill_projected(_ptr(Q), _ptr(K), _ptr(V), _ptr(X), _ptr(W_gamma), d_model, _ptr(G),
                                        float(tau), int(chunk), _ptr(O), _ptr(S_final), B, H, N, dk, dv, io,
                                        float(eps), epi, _ptr(workspace) if ws_bytes else None, ws_bytes,
                                        st.cuda_stream)
    if status != Status.OK:
        raise GretError(status, "gret_prefill_projected")
    return O, S_final


def prefill_varlen(Q, K, V, z, G, cu_seqlens, max_seqlen: int, tau: float, chunk: int, eps: float = 1e-5,
                   epilogue: str = "gn_swish", O=None, S_final=None, want_state: bool = True, workspace=None,
                   stream=None, S0=None):
    """Prefill of a packed batch of sequences (gret_prefill_varlen).

    Q, K [T,H,dk]; V, G [T,H,dv] (bf16 or fp32); z [T,H] fp32; cu_seqlens int32 [S+1] on the
    device (sequence b is rows cu_seqlens[b] .. cu_seqlens[b+1]-1); S0 [S,H,dk,dv] fp32 or None.
    Returns (O [T,H,dv], S_final [S,H,dk,dv] fp32 or None).
    """
    torch = _torch()
    T, H, dk = Q.shape
    dv = V.shape[-1]
    S = cu_seqlens.numel() - 1
    dev = Q.device
    io = _io_of(Q)
    epi = Epilogue.NONE if epilogue == "none" else Epilogue.GN_SWISH
    _need_g(G, epi)
    _check(Q, "Q", Q.dtype, (T, H, dk), dev)
    _check(K, "K", Q.dtype, (T, H, dk), dev)
    _check(V, "V", Q.dtype, (T, H, dv), dev)
    _check(z, "z", torch.float32, (T, H), dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, (S + 1,), dev)
    if G is not None:
        _check(G, "G", Q.dtype, (T, H, dv), dev)
    if O is None:
        O = torch.empty((T, H, dv), dtype=Q.dtype, device=dev)
    _check(O, "O", Q.dtype, (T, H, dv), dev)
    if S_final is None and want_state:
        S_final = torch.empty((S, H, dk, dv), dtype=torch.float32, device=dev)
    if S_final is not None:
        _check(S_final, "S_final", torch.float32, (S, H, dk, dv), dev)
    if S0 is not None:
        _check(S0, "S0", torch.float32, (S, H, dk, dv), dev)
    with torch.cuda.device(dev):
        ws_bytes = gret_prefill_varlen_workspace_size(S, T, max_seqlen, H, dk, dv, chunk, io)
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        workspace = _scratch(workspace, ws_bytes, dev, st)
        status = gret_prefill_varlen(_ptr(Q), _ptr(K), _ptr(V), _ptr(z), _ptr(G), _ptr(S0), _ptr(cu_seqlens), S, T,
                                     int(max_seqlen), float(tau), int(chunk), _ptr(O), _ptr(S_final), H, dk, dv, io,
                                     float(eps), epi, _ptr(workspace) if ws_bytes else None, ws_bytes,
                                     st.cuda_stream)
    if status != Status.OK:
        raise GretError(status, "gret_prefill_varlen")
    return O, S_final


def prefill_state(K, V, z, tau: float, chunk: int, workspace=None, stream=None):
    """State increment and total log-decay of a token slice (gret_prefill_state).

    K [B,N,H,dk], V [B,N,H,dv] (bf16 or fp32), z [B,N,H] fp32.
    Returns (dS [B,H,dk,dv] fp32, decay [B,H] fp32)."""
    torch = _torch()
    B, N, H, dk = K.shape
    dv = V.shape[-1]
    dev = K.device
    io = _io_of(K)
    _check(V, "V", K.dtype, (B, N, H, dv), dev)
    _check(z, "z", torch.float32, (B, N, H), dev)
    dS = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    decay = torch.empty((B, H), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        ws_bytes = gret_prefill_state_workspace_size(B, H, N, dk, dv, chunk, io)
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        workspace = _scratch(workspace, ws_bytes, dev, st)
        status = gret_prefill_state(_ptr(K), _ptr(V), _ptr(z), float(tau), int(chunk), _ptr(dS), _ptr(decay), B, H,
                                    N, dk, dv, io, _ptr(workspace) if ws_bytes else None, ws_bytes, st.cuda_stream)
    if status != Status.OK:
        raise GretError(status, "gret_prefill_state")
    return dS, decay


def state_fold(dS_all, decay_all, slice_: int, S0=None, out=None, stream=None):
    """S_in of slice ``slice_`` from the gathered increments (gret_state_fold).

    dS_all [P,B,H,dk,dv] fp32, decay_all [P,B,H] fp32, S0 [B,H,dk,dv] fp32 or None."""
    torch = _torch()
    P, B, H, dk, dv = dS_all.shape
    dev = dS_all.device
    _check(dS_all, "dS_all", torch.float32, (P, B, H, dk, dv), dev)
    _check(decay_all, "decay_all", torch.float32, (P, B, H), dev)
    if S0 is not None:
        _check(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    if out is None:
        out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    _check(out, "out", torch.float32, (B, H, dk, dv), dev)
    with torch.cuda.device(dev):
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        status = gret_state_fold(_ptr(dS_all), _ptr(decay_all), P, int(slice_), _ptr(S0), _ptr(out), B, H, dk, dv,
                                 st.cuda_stream)
    if status != Status.OK:
        raise GretError(status, "gret_state_fold")
    return out


def prefill_backward(Q, K, V, z, G, dO, tau: float, eps: float = 1e-5, epilogue: str = "gn_swish", S0=None,
                     dS_final=None, want_dS0: bool = False, workspace=None, stream=None):
    """Gradients of <O, dO> + <S_final, dS_final> (gret_prefill_backward).

    Shapes as for ``prefill``.  Returns a dict: dQ, dK, dV (io dtype), dz (fp32),
    dG (io dtype; None for epilogue='none'), dS0 (fp32, when S0 is given or
    want_dS0)."""
    torch = _torch()
    B, N, H, dk = Q.shape
    dv = V.shape[-1]
    dev = Q.device
    io = _io_of(Q)
    epi = Epilogue.NONE if epilogue == "none" else Epilogue.GN_SWISH
    _need_g(G, epi)
    for t, name, shape in ((K, "K", (B, N, H, dk)), (V, "V", (B, N, H, dv)), (dO, "dO", (B, N, H, dv))):
        _check(t, name, Q.dtype, shape, dev)
    _check(z, "z", torch.float32, (B, N, H), dev)
    if epi == Epilogue.GN_SWISH:
        _check(G, "G", Q.dtype, (B, N, H, dv), dev)
    for t, name in ((S0, "S0"), (dS_final, "dS_final")):
        if t is not None:
            _check(t, name, torch.float32, (B, H, dk, dv), dev)
    out = {"dQ": torch.empty_like(Q), "dK": torch.empty_like(K), "dV": torch.empty_like(V),
           "dz": torch.empty_like(z), "dG": torch.empty_like(V) if epi == Epilogue.GN_SWISH else None,
           "dS0": torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if (S0 is not None or want_dS0)
           else None}
    with torch.cuda.device(dev):
        ws_bytes = gret_prefill_backward_workspace_size(B, H, N, dk, dv, io)
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        workspace = _scratch(workspace, ws_bytes, dev, st)
        status = gret_prefill_backward(_ptr(Q), _ptr(K), _ptr(V), _ptr(z), _ptr(G), _ptr(S0), _ptr(dO), _ptr(dS_final),
                                       float(tau), float(eps), epi, _ptr(out["dQ"]), _ptr(out["dK"]), _ptr(out["dV"]),
                                       _ptr(out["dz"]), _ptr(out["dG"]), _ptr(out["dS0"]), B, H, N, dk, dv, io,
                                       _ptr(workspace) if ws_bytes else None, ws_bytes, st.cuda_stream)
    if status != Status.OK:
        raise GretError(status, "gret_prefill_backward")
    return out


def decode_step(q, k, v, z, g, S, tau: float, eps: float = 1e-5, epilogue: str = "gn_swish",
                o=None, stream=None):
    """One recurrent step; S [num_seqs,H,dk,dv] fp32 is updated in place. Returns o."""
    torch = _torch()
    ns, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    io = _io_of(q)
    epi = Epilogue.NONE if epilogue == "none" else Epilogue.GN_SWISH
    _need_g(g, epi, "g")
    _check(q, "q", q.dtype, (ns, H, dk), dev)
    _check(k, "k", q.dtype, (ns, H, dk), dev)
    _check(v, "v", q.dtype, (ns, H, dv), dev)
    _check(z, "z", torch.float32, (ns, H), dev)
    if g is not None:
        _check(g, "g", q.dtype, (ns, H, dv), dev)
    _check(S, "S", torch.float32, (ns, H, dk, dv), dev)
    if o is None:
        o = torch.empty((ns, H, dv), dtype=q.dtype, device=dev)
    _check(o, "o", q.dtype, (ns, H, dv), dev)
    with torch.cuda.device(dev):
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        status = gret_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(g), _ptr(S), _ptr(o), ns, H,
                                  dk, dv, float(tau), io, float(eps), epi, st.cuda_stream)
    if status != Status.OK:
        raise GretError(status, "gret_decode_step")
    return o


def prefill_path(B, H, N, dk, dv, chunk, io: Dtype) -> Tuple[Path, int]:
    """Kernel the library would pick, and the sequence segments per unit."""
    return gret_prefill_path(B, H, N, dk, dv, chunk, io)


def check_device_status(stream=None) -> None:
    """Synchronise and raise GretError if a kernel's bounded wait gave up."""
    s = gret_last_device_status(stream)
    if s != Status.OK:
        raise GretError(s, "device status")
