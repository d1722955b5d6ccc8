"""Python face of the fp64 C oracle (``gret_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg; never by the GPU library.  The wrapper only
marshals arguments (widens stored bf16/fp32 values to fp64 and splits
(batch, head) units across threads); every step of the method is in the C file.

Parity status of each function (what pins it, checked in ``tests/test_oracle_pins.py``):
  log_gamma        spot values of sigmoid(z)^(1/tau); closed form via two routes
  recurrent        brute force vs parallel (tiny N); gamma=1 prefix sum; gamma=0
                   closed form; constant-gamma geometric series; state
                   decomposition; decode chaining
  parallel         as above (independent products of gamma)
  chunkwise        equality with recurrent for every chunk length incl. ragged
  groupnorm_swish  torch.nn.functional.group_norm and silu; mean-0 / variance
                   invariants
  decode_step      prefill(N0) + T steps == prefill(N0 + T)
  gate_project     worked value; numpy matmul as a second route; linearity
  rotate           worked values (position 0, one radian per position);
                   pair norms; R(a) R(b) = R(a + b); rotated scores depend on
                   positions only through their difference
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gret_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_gret.so")
_lock = threading.Lock()
_lib = None

__all__ = ["build", "build_variant", "source_text", "log_gamma", "recurrent", "parallel", "chunkwise", "groupnorm_swish",
           "prefill", "decode_step", "gate_project", "rotate", "prefill_projected", "as_f64", "default_threads"]


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle_gret.so`` with gcc (plain -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    """Load a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(ctypes.c_double)
    I, D, L = ctypes.c_int, ctypes.c_double, ctypes.c_long
    lib.oracle_log_gamma.argtypes = [P, L, D, P]
    lib.oracle_recurrent.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P]
    lib.oracle_parallel.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P]
    lib.oracle_chunkwise.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, P, P]
    lib.oracle_groupnorm_swish.argtypes = [P, P, L, I, D, P]
    lib.oracle_decode_step.argtypes = [P, P, P, P, P, P, I, I, I, I, D, I, I, P, P]
    lib.oracle_gate_project.argtypes = [P, P, L, I, I, P]
    lib.oracle_rotate.argtypes = [P, I, I, I, I, D, L, P]
    for f in (lib.oracle_log_gamma, lib.oracle_recurrent, lib.oracle_parallel,
              lib.oracle_chunkwise, lib.oracle_groupnorm_swish, lib.oracle_decode_step,
              lib.oracle_gate_project, lib.oracle_rotate):
        f.restype = None
    return lib


def build_variant(source_text: str, out_dir: str):
    """Compile a modified copy of the oracle source (used by mutation tests) and load it."""
    src = os.path.join(out_dir, "gret_oracle_variant.c")
    so = os.path.join(out_dir, "liboracle_variant.so")
    with open(src, "w") as f:
        f.write(source_text)
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", so, src, "-lm"])
    return _bind(so)


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _load(lib=None):
    """The oracle library (``lib`` overrides it, e.g. a mutated build in a test)."""
    global _lib
    if lib is not None:
        return lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1))


def as_f64(x) -> np.ndarray:
    """Widen a stored tensor (torch bf16/fp32 or numpy) to a contiguous fp64 array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _split(n_units: int, threads: int):
    threads = max(1, min(threads, n_units))
    step = (n_units + threads - 1) // threads
    return [(u, min(n_units, u + step)) for u in range(0, n_units, step)]


def _run_units(fn, n_units: int, threads: Optional[int]):
    ranges = _split(n_units, threads or default_threads())
    if len(ranges) == 1:
        fn(*ranges[0])
        return
    with ThreadPoolExecutor(len(ranges)) as ex:
        list(ex.map(lambda r: fn(*r), ranges))


def log_gamma(z, tau: float, lib=None) -> np.ndarray:
    z = as_f64(z)
    out = np.empty_like(z)
    _load(lib).oracle_log_gamma(_p(z), z.size, float(tau), _p(out))
    return out


def _dims(Q, V):
    B, N, H, dk = Q.shape
    dv = V.shape[-1]
    return B, N, H, dk, dv


def recurrent(Q, K, V, lg, S0=None, threads: Optional[int] = None, lib=None) -> Tuple[np.ndarray, np.ndarray]:
    """Recurrent form. Q,K [B,N,H,dk]; V [B,N,H,dv]; lg [B,N,H]; S0 [B,H,dk,dv] or None.
    Returns (Y [B,N,H,dv], S_final [B,H,dk,dv]) in fp64."""
    Q, K, V, lg = as_f64(Q), as_f64(K), as_f64(V), as_f64(lg)
    S0 = None if S0 is None else as_f64(S0)
    B, N, H, dk, dv = _dims(Q, V)
    Y = np.empty((B, N, H, dv))
    Sf = np.empty((B, H, dk, dv))
    lib = _load(lib)
    _run_units(lambda a, b: lib.oracle_recurrent(_p(Q), _p(K), _p(V), _p(lg), _p(S0), B, H, N, dk, dv,
                                                 a, b, _p(Y), _p(Sf)), B * H, threads)
    return Y, Sf


def parallel(Q, K, V, lg, S0=None, threads: Optional[int] = None, lib=None) -> np.ndarray:
    """Parallel form (small N only). Returns Y [B,N,H,dv] in fp64."""
    Q, K, V, lg = as_f64(Q), as_f64(K), as_f64(V), as_f64(lg)
    S0 = None if S0 is None else as_f64(S0)
    B, N, H, dk, dv = _dims(Q, V)
    Y = np.empty((B, N, H, dv))
    lib = _load(lib)
    _run_units(lambda a, b: lib.oracle_parallel(_p(Q), _p(K), _p(V), _p(lg), _p(S0), B, H, N, dk, dv,
                                                a, b, _p(Y)), B * H, threads)
    return Y


def chunkwise(Q, K, V, lg, chunk: int, S0=None, threads: Optional[int] = None, lib=None):
    """Chunkwise form with block length ``chunk``. Returns (Y, S_final) in fp64."""
    Q, K, V, lg = as_f64(Q), as_f64(K), as_f64(V), as_f64(lg)
    S0 = None if S0 is None else as_f64(S0)
    B, N, H, dk, dv = _dims(Q, V)
    Y = np.empty((B, N, H, dv))
    Sf = np.empty((B, H, dk, dv))
    lib = _load(lib)
    _run_units(lambda a, b: lib.oracle_chunkwise(_p(Q), _p(K), _p(V), _p(lg), _p(S0), B, H, N, dk, dv,
                                                 int(chunk), a, b, _p(Y), _p(Sf)), B * H, threads)
    return Y, Sf


def groupnorm_swish(Y, G, eps: float, lib=None) -> np.ndarray:
    """Per-row GroupNorm (no affine, biased variance) times swish(G); rows = all but last dim."""
    Y, G = as_f64(Y), as_f64(G)
    out = np.empty_like(Y)
    dv = Y.shape[-1]
    _load(lib).oracle_groupnorm_swish(_p(Y), _p(G), Y.size // dv, dv, float(eps), _p(out))
    return out


def prefill(Q, K, V, z, G, tau: float, eps: float = 1e-5, S0=None, lg=None,
            threads: Optional[int] = None, lib=None):
    """Whole prefill: gate, recurrent form, epilogue. Returns (O, Y, S_final) in fp64.
    ``lg`` (log gamma) overrides the gate when given (tests use 0 or -inf)."""
    if lg is None:
        lg = log_gamma(z, tau, lib=lib)
    Y, Sf = recurrent(Q, K, V, lg, S0=S0, threads=threads, lib=lib)
    O = groupnorm_swish(Y, G, eps, lib=lib)
    return O, Y, Sf


def decode_step(q, k, v, z, g, S, tau: float, eps: float = 1e-5, lg=None,
                threads: Optional[int] = None, lib=None):
    """One decode step. q,k [S,H,dk]; v,g [S,H,dv]; z [S,H]; S [S,H,dk,dv].
    Returns (o, y, S_new) in fp64 (S is not modified)."""
    q, k, v, g = as_f64(q), as_f64(k), as_f64(v), as_f64(g)
    if lg is None:
        lg = log_gamma(z, tau, lib=lib)
    lg = as_f64(lg)
    Sn = as_f64(S).copy()
    ns, H, dk = q.shape
    dv = v.shape[-1]
    y = np.empty((ns, H, dv))
    o = np.empty((ns, H, dv))
    lib = _load(lib)
    _run_units(lambda a, b: lib.oracle_decode_step(_p(q), _p(k), _p(v), _p(lg), _p(g), _p(Sn), ns, H,
                                                   dk, dv, float(eps), a, b, _p(y), _p(o)),
               ns * H, threads)
    return o, y, Sn


def gate_project(X, W, lib=None) -> np.ndarray:
    """Gate logits z = X W_gamma. X [..., d_model]; W [d_model, H]. Returns z [..., H] in fp64."""
    X, W = as_f64(X), as_f64(W)
    d_model, H = W.shape
    assert X.shape[-1] == d_model
    rows = X.size // d_model
    z = np.empty(X.shape[:-1] + (H,))
    _load(lib).oracle_gate_project(_p(X), _p(W), rows, d_model, H, _p(z))
    return z


def rotate(X, base: float, pos0: int = 0, lib=None) -> np.ndarray:
    """The rotation Theta (RoPE on consecutive channel pairs) of X [B, N, H, d]
    at positions pos0 .. pos0 + N - 1. Returns fp64."""
    X = as_f64(X)
    B, N, H, d = X.shape
    assert d % 2 == 0
    out = np.empty_like(X)
    _load(lib).oracle_rotate(_p(X), B, N, H, d, float(base), int(pos0), _p(out))
    return out


def prefill_projected(Q, K, V, X, W, G, tau: float, eps: float = 1e-5, theta_base: float = 0.0,
                      S0=None, threads: Optional[int] = None, lib=None):
    """Prefill whose gate logits come from the projection z = X W_gamma, and whose
    Q and K are rotated by Theta first when theta_base > 0.
    X [B, N, d_model]; W [d_model, H]. Returns (O, Y, S_final) in fp64."""
    z = gate_project(X, W, lib=lib)
    if theta_base > 0:
        Q, K = rotate(Q, theta_base, lib=lib), rotate(K, theta_base, lib=lib)
    return prefill(Q, K, V, z, G, tau, eps, S0=S0, threads=threads, lib=lib)
