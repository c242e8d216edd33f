"""fp64 CPU oracle for Exact Flow Linear Attention (test infrastructure only).

Only the tests, the smoke check and the bench's CPU-baseline leg use this package.  The
library under test never imports it, and it imports nothing from the library: the two
share no code.  The arithmetic lives in efla_oracle.c (plain sequential loops, one
(b, h) stream per OpenMP task); this module builds it with gcc, loads it with ctypes and
marshals numpy/torch arrays to float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "efla_oracle.c")
LIB = os.path.join(_HERE, "_efla_oracle.so")

EXACT = 0
EULER = 1

_lib = None


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile efla_oracle.c into a shared library (gcc, OpenMP, no fast-math)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
           "-std=c11", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def load(path: Optional[str] = None):
    """Load (building if needed) the oracle library and declare its signatures."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(path or build())
    dp = ctypes.POINTER(ctypes.c_double)
    L, I = ctypes.c_long, ctypes.c_int
    lib.efla_oracle_alpha.argtypes = [ctypes.c_double, ctypes.c_double]
    lib.efla_oracle_alpha.restype = ctypes.c_double
    lib.efla_oracle_fwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, L, L, L, L, L, I, I]
    lib.efla_oracle_fwd.restype = I
    lib.efla_oracle_step.argtypes = [dp, dp, dp, dp, dp, dp, L, L, L, L, I, I]
    lib.efla_oracle_step.restype = I
    lib.efla_oracle_fwd_gated.argtypes = [dp] * 8 + [L, L, L, L, L, I, I]
    lib.efla_oracle_fwd_gated.restype = I
    lib.efla_oracle_step_gated.argtypes = [dp] * 7 + [L, L, L, L, I, I]
    lib.efla_oracle_step_gated.restype = I
    lib.efla_oracle_dalpha_dlambda.argtypes = [ctypes.c_double, ctypes.c_double]
    lib.efla_oracle_dalpha_dlambda.restype = ctypes.c_double
    lib.efla_oracle_bwd.argtypes = [dp] * 12 + [L, L, L, L, L, I, I]
    lib.efla_oracle_bwd.restype = I
    if path is None:
        _lib = lib
    return lib


def _f64(x) -> np.ndarray:
    """Upcast a torch tensor or array-like to a C-contiguous float64 numpy array."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: exact upcast of its stored (cast) values
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def alpha(beta: float, lam: float, lib=None) -> float:
    return (lib or load()).efla_oracle_alpha(float(beta), float(lam))


def fwd(q, k, v, beta, S0=None, mode: int = EXACT, threads: Optional[int] = None, lib=None,
        want_o: bool = True):
    """Sequential fp64 forward. q, k [B,H,T,dk], v [B,H,T,dv], beta [B,H,T], S0 [B,H,dk,dv].

    Returns (o [B,H,T,dv] or None, S_T [B,H,dk,dv]) as float64 numpy arrays.
    """
    q, k, v, beta, S0 = _f64(q), _f64(k), _f64(v), _f64(beta), _f64(S0)
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape[:3] == (B, H, T) and beta.shape == (B, H, T)
    if S0 is not None:
        assert S0.shape == (B, H, dk, dv)
    o = np.empty((B, H, T, dv), dtype=np.float64) if want_o else None
    ST = np.empty((B, H, dk, dv), dtype=np.float64)
    rc = (lib or load()).efla_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S0),
                                         _ptr(o), _ptr(ST), B, H, T, dk, dv, mode,
                                         threads or default_threads())
    if rc != 0:
        raise MemoryError("oracle could not allocate its per-stream state")
    return o, ST


def step(q, k, v, beta, S, mode: int = EXACT, threads: Optional[int] = None, lib=None):
    """One decode step. q, k [N,H,dk], v [N,H,dv], beta [N,H]; S [N,H,dk,dv] float64.

    S is updated in place when it is already a C-contiguous float64 array (else a copy is
    made and returned).  Returns (o [N,H,dv], S).
    """
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    if not (isinstance(S, np.ndarray) and S.dtype == np.float64 and S.flags.c_contiguous):
        S = _f64(S).copy()
    N, H, dk = k.shape
    dv = v.shape[-1]
    o = np.empty((N, H, dv), dtype=np.float64)
    rc = (lib or load()).efla_oracle_step(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S),
                                          _ptr(o), N, H, dk, dv, mode,
                                          threads or default_threads())
    if rc != 0:
        raise MemoryError("oracle could not allocate its per-stream state")
    return o, S


def fwd_gated(q, k, v, beta, g, S0=None, mode: int = EXACT, threads: Optional[int] = None, lib=None,
              want_o: bool = True):
    """Gated forward (per-token log-decay g [B,H,T]); otherwise as fwd."""
    q, k, v, beta, g, S0 = _f64(q), _f64(k), _f64(v), _f64(beta), _f64(g), _f64(S0)
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape[:3] == (B, H, T) and beta.shape == (B, H, T) and g.shape == (B, H, T)
    if S0 is not None:
        assert S0.shape == (B, H, dk, dv)
    o = np.empty((B, H, T, dv), dtype=np.float64) if want_o else None
    ST = np.empty((B, H, dk, dv), dtype=np.float64)
    rc = (lib or load()).efla_oracle_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S0),
                                               _ptr(o), _ptr(ST), B, H, T, dk, dv, mode,
                                               threads or default_threads())
    if rc != 0:
        raise MemoryError("oracle could not allocate its per-stream state")
    return o, ST


def step_gated(q, k, v, beta, g, S, mode: int = EXACT, threads: Optional[int] = None, lib=None):
    """One gated decode step (g [N,H]); otherwise as step."""
    q, k, v, beta, g = _f64(q), _f64(k), _f64(v), _f64(beta), _f64(g)
    if not (isinstance(S, np.ndarray) and S.dtype == np.float64 and S.flags.c_contiguous):
        S = _f64(S).copy()
    N, H, dk = k.shape
    dv = v.shape[-1]
    o = np.empty((N, H, dv), dtype=np.float64)
    rc = (lib or load()).efla_oracle_step_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S),
                                                _ptr(o), N, H, dk, dv, mode, threads or default_threads())
    if rc != 0:
        raise MemoryError("oracle could not allocate its per-stream state")
    return o, S


def dalpha_dlambda(beta: float, lam: float, lib=None) -> float:
    return (lib or load()).efla_oracle_dalpha_dlambda(float(beta), float(lam))


def bwd(q, k, v, beta, dO, S0=None, dS_T=None, mode: int = EXACT, threads: Optional[int] = None,
        lib=None):
    """Reverse-mode derivative of fwd for the loss sum(dO * o) + sum(dS_T * S_T).

    Returns (dq, dk [B,H,T,dk], dv [B,H,T,dv], dbeta [B,H,T], dS0 [B,H,dk,dv]) as float64.
    Keeps every state of a running stream: (T + 1) dk dv doubles per thread.
    """
    q, k, v, beta, dO, S0, dS_T = (_f64(x) for x in (q, k, v, beta, dO, S0, dS_T))
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape[:3] == (B, H, T) and dO.shape == v.shape
    dq, dk_ = np.empty_like(q), np.empty_like(k)
    dv_, dbeta = np.empty_like(v), np.empty((B, H, T), dtype=np.float64)
    dS0 = np.empty((B, H, dk, dv), dtype=np.float64)
    rc = (lib or load()).efla_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S0), _ptr(dO),
                                         _ptr(dS_T), _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dbeta),
                                         _ptr(dS0), B, H, T, dk, dv, mode,
                                         threads or default_threads())
    if rc != 0:
        raise MemoryError("oracle could not allocate the states of a stream")
    return dq, dk_, dv_, dbeta, dS0
