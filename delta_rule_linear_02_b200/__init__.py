"""Python binding of libefla.so, the B200 Exact Flow Linear Attention forward.

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels.  PyTorch provides device memory and streams.  The names mirror the C ABI of
include/efla.h.  Importing this package loads the in-tree libefla.so and fails loudly if
it has not been built (python delta_rule_linear_02_b200/build.py).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libefla.so")
# the same entry points built with EFLA_CHECKED=1: the tensor-core forward's kernels test
# every direct global access against its buffer and report EFLA_ERR_BOUNDS through the
# workspace status instead of touching memory out of range (build.py --checked)
LIB_CHECKED_PATH = os.path.join(_PKG, "libefla_checked.so")

EFLA_OK, EFLA_ERR_INVALID_ARG, EFLA_ERR_UNSUPPORTED, EFLA_ERR_CUDA, EFLA_ERR_TIMEOUT, EFLA_ERR_BOUNDS = range(6)
EFLA_DTYPE_F32, EFLA_DTYPE_BF16 = 0, 1
EFLA_RULE_EXACT, EFLA_RULE_EULER = 0, 1     # exact-flow gate, or alpha = beta (the delta rule)
CHUNK = 64

_DTYPES = {torch.float32: EFLA_DTYPE_F32, torch.bfloat16: EFLA_DTYPE_BF16}


class EflaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {efla_status_string(status)} ({status})")


def _load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} is not built at {path}; run "
                          "`python delta_rule_linear_02_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    vp, I, L, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_size_t
    lib.efla_status_string.argtypes = [I]
    lib.efla_status_string.restype = ctypes.c_char_p
    lib.efla_gate.argtypes = [vp, vp, vp, L, I, I, vp]
    lib.efla_gate.restype = I
    lib.efla_chunk_fwd_workspace_bytes.argtypes = [I, I, I, I, I, I, I]
    lib.efla_chunk_fwd_workspace_bytes.restype = Z
    lib.efla_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, I, I, I, I, I, I, I, vp, Z, vp]
    lib.efla_chunk_fwd.restype = I
    lib.efla_chunk_fwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, I, I, I, I, I, I, I, I, vp, Z, vp]
    lib.efla_chunk_fwd_ex.restype = I
    lib.efla_chunk_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, I, I, I, I, I, I, I, vp]
    lib.efla_chunk_fwd_noalloc.restype = I
    lib.efla_workspace_status.argtypes = [vp, I, vp]
    lib.efla_workspace_status.restype = I
    lib.efla_noalloc_status.argtypes = [I, vp]
    lib.efla_noalloc_status.restype = I
    lib.efla_chunk_fwd_gated_workspace_bytes.argtypes = [I, I, I, I, I, I, I]
    lib.efla_chunk_fwd_gated_workspace_bytes.restype = Z
    lib.efla_chunk_fwd_gated.argtypes = [vp] * 8 + [I, I, I, I, I, I, I, I, vp, Z, vp]
    lib.efla_chunk_fwd_gated.restype = I
    lib.efla_recurrent_step_gated.argtypes = [vp] * 7 + [I, I, I, I, I, I, vp]
    lib.efla_recurrent_step_gated.restype = I
    lib.efla_chunk_fwd_segmented_workspace_bytes.argtypes = [I, I, I, I, I, I, I, I, I]
    lib.efla_chunk_fwd_segmented_workspace_bytes.restype = Z
    lib.efla_chunk_fwd_segmented.argtypes = [vp] * 8 + [I] * 9 + [vp, Z, vp]
    lib.efla_chunk_fwd_segmented.restype = I
    lib.efla_chunk_fwd_varlen_workspace_bytes.argtypes = [vp, I, I, I, I, I, I, I]
    lib.efla_chunk_fwd_varlen_workspace_bytes.restype = Z
    lib.efla_chunk_fwd_varlen.argtypes = [vp] * 9 + [I, I, I, I, I, I, I, vp, Z, vp]
    lib.efla_chunk_fwd_varlen.restype = I
    lib.efla_selftest_wait_timeout.argtypes = [vp, ctypes.c_longlong, vp]
    lib.efla_selftest_wait_timeout.restype = I
    lib.efla_recurrent_step.argtypes = [vp, vp, vp, vp, vp, vp, I, I, I, I, I, vp]
    lib.efla_recurrent_step.restype = I
    lib.efla_recurrent_step_ex.argtypes = [vp, vp, vp, vp, vp, vp, I, I, I, I, I, I, vp]
    lib.efla_recurrent_step_ex.restype = I
    lib.efla_backward_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.efla_backward_workspace_bytes.restype = Z
    lib.efla_backward.argtypes = [vp] * 12 + [I, I, I, I, I, I, vp, Z, vp]
    lib.efla_backward.restype = I
    lib.efla_backward_ex.argtypes = [vp] * 12 + [I, I, I, I, I, I, I, vp, Z, vp]
    lib.efla_backward_ex.restype = I
    lib.efla_train_saved_bytes.argtypes = [I, I, I, I, I, I, I]
    lib.efla_train_saved_bytes.restype = Z
    lib.efla_chunk_fwd_save.argtypes = [vp] * 7 + [I] * 8 + [vp, Z, vp]
    lib.efla_chunk_fwd_save.restype = I
    lib.efla_backward_saved_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.efla_backward_saved_workspace_bytes.restype = Z
    lib.efla_backward_saved.argtypes = [vp] * 11 + [I] * 7 + [vp, Z, vp, Z, vp]
    lib.efla_backward_saved.restype = I
    return lib


lib = _load()


def load_checked() -> ctypes.CDLL:
    """The checked build (libefla_checked.so) with the same argument types as `lib`; the
    wrappers below call whichever library the module attribute `lib` holds."""
    return _load(LIB_CHECKED_PATH)


def efla_status_string(status: int) -> str:
    return lib.efla_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _raise(status: int, where: str):
    if status != EFLA_OK:
        raise EflaError(status, where)


def efla_gate(k: torch.Tensor, beta: torch.Tensor, out: Optional[torch.Tensor] = None,
              stream=None) -> torch.Tensor:
    """alpha [...] float32 from keys k [..., d_k] and gates beta [...] (same dtype)."""
    _check(k, "k"); _check(beta, "beta", k.dtype)
    n = beta.numel()
    if out is None:
        out = torch.empty(beta.shape, device=k.device, dtype=torch.float32)
    _check(out, "out", torch.float32)
    _raise(lib.efla_gate(_ptr(k), _ptr(beta), _ptr(out), n, k.shape[-1], _DTYPES[k.dtype],
                         _stream(stream)), "efla_gate")
    return out


def efla_chunk_fwd_workspace_bytes(B, H, T, d_k, d_v, chunk=CHUNK, dtype=torch.bfloat16) -> int:
    return int(lib.efla_chunk_fwd_workspace_bytes(B, H, T, d_k, d_v, chunk, _DTYPES[dtype]))


def new_workspace(B, H, T, d_k, d_v, chunk=CHUNK, dtype=torch.bfloat16, device="cuda"):
    """A zeroed workspace tensor (uint8) sized for efla_chunk_fwd."""
    n = efla_chunk_fwd_workspace_bytes(B, H, T, d_k, d_v, chunk, dtype)
    if n == 0:
        raise EflaError(EFLA_ERR_UNSUPPORTED, "efla_chunk_fwd_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def efla_chunk_fwd(q, k, v, beta, S0=None, chunk: int = CHUNK, o=None, S_T=None,
                   workspace=None, want_state: bool = True, stream=None, rule: int = EFLA_RULE_EXACT
                   ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked EFLA forward. q, k [B,H,T,d_k], v [B,H,T,d_v], beta [B,H,T] (one dtype),
    S0 [B,H,d_k,d_v] float32 or None.  Returns (o [B,H,T,d_v], S_T or None).
    rule: EFLA_RULE_EXACT (the method) or EFLA_RULE_EULER (the delta rule, alpha = beta)."""
    dt = k.dtype
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, nme, dt)
    B, H, T, d_k = k.shape
    d_v = v.shape[-1]
    if S0 is not None:
        _check(S0, "S0", torch.float32)
    if o is None:
        o = torch.empty((B, H, T, d_v), device=k.device, dtype=dt)
    _check(o, "o", dt)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, d_k, d_v), device=k.device, dtype=torch.float32)
    if S_T is not None:
        _check(S_T, "S_T", torch.float32)
    if workspace is None:
        workspace = new_workspace(B, H, T, d_k, d_v, chunk, dt, k.device)
    st = lib.efla_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_T),
                               B, H, T, d_k, d_v, chunk, _DTYPES.get(dt, -1), int(rule), _ptr(workspace),
                               workspace.numel(), _stream(stream))
    _raise(st, "efla_chunk_fwd")
    return o, S_T


def efla_chunk_fwd_gated(q, k, v, beta, g, S0=None, chunk: int = CHUNK, o=None, S_T=None,
                         workspace=None, want_state: bool = True, stream=None, rule: int = EFLA_RULE_EXACT
                         ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Gated EFLA forward: efla_chunk_fwd plus g [B,H,T] float32, the per-token log-decay."""
    dt = k.dtype
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, nme, dt)
    _check(g, "g", torch.float32)
    B, H, T, d_k = k.shape
    d_v = v.shape[-1]
    if S0 is not None:
        _check(S0, "S0", torch.float32)
    if o is None:
        o = torch.empty((B, H, T, d_v), device=k.device, dtype=dt)
    _check(o, "o", dt)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, d_k, d_v), device=k.device, dtype=torch.float32)
    if S_T is not None:
        _check(S_T, "S_T", torch.float32)
    if workspace is None:
        n = int(lib.efla_chunk_fwd_gated_workspace_bytes(B, H, T, d_k, d_v, chunk, _DTYPES.get(dt, -1)))
        if n == 0:
            raise EflaError(EFLA_ERR_UNSUPPORTED, "efla_chunk_fwd_gated_workspace_bytes")
        workspace = torch.zeros(n, dtype=torch.uint8, device=k.device)
    st = lib.efla_chunk_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S0), _ptr(o), _ptr(S_T),
                                  B, H, T, d_k, d_v, chunk, _DTYPES.get(dt, -1), int(rule), _ptr(workspace),
                                  workspace.numel(), _stream(stream))
    _raise(st, "efla_chunk_fwd_gated")
    return o, S_T


def efla_recurrent_step_gated(q, k, v, beta, g, S, o=None, stream=None, rule: int = EFLA_RULE_EXACT):
    """One gated decode token: efla_recurrent_step plus g [N,H] float32, the log-decay."""
    dt = k.dtype
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, nme, dt)
    _check(g, "g", torch.float32)
    _check(S, "S", torch.float32)
    N, H, d_k = k.shape
    d_v = v.shape[-1]
    if o is None:
        o = torch.empty((N, H, d_v), device=k.device, dtype=dt)
    _check(o, "o", dt)
    _raise(lib.efla_recurrent_step_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S), _ptr(o),
                                         N, H, d_k, d_v, _DTYPES.get(dt, -1), int(rule), _stream(stream)),
           "efla_recurrent_step_gated")
    return o


def efla_chunk_fwd_segmented(q, k, v, beta, S0=None, g=None, segments: int = 0, chunk: int = CHUNK, o=None,
                             S_T=None, workspace=None, want_state: bool = True, stream=None,
                             rule: int = EFLA_RULE_EXACT) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """efla_chunk_fwd (or, with g, efla_chunk_fwd_gated) as a segmented scan of `segments`
    segments per stream (0: the library's choice)."""
    dt = k.dtype
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, nme, dt)
    if g is not None:
        _check(g, "g", torch.float32)
    B, H, T, d_k = k.shape
    d_v = v.shape[-1]
    if S0 is not None:
        _check(S0, "S0", torch.float32)
    if o is None:
        o = torch.empty((B, H, T, d_v), device=k.device, dtype=dt)
    _check(o, "o", dt)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, d_k, d_v), device=k.device, dtype=torch.float32)
    if S_T is not None:
        _check(S_T, "S_T", torch.float32)
    if workspace is None:
        n = int(lib.efla_chunk_fwd_segmented_workspace_bytes(B, H, T, d_k, d_v, chunk, _DTYPES.get(dt, -1),
                                                             int(g is not None), int(segments)))
        if n == 0:
            raise EflaError(EFLA_ERR_UNSUPPORTED, "efla_chunk_fwd_segmented_workspace_bytes")
        workspace = torch.zeros(n, dtype=torch.uint8, device=k.device)
    st = lib.efla_chunk_fwd_segmented(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S0), _ptr(o), _ptr(S_T),
                                      B, H, T, d_k, d_v, chunk, _DTYPES.get(dt, -1), int(rule), int(segments),
                                      _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st, "efla_chunk_fwd_segmented")
    return o, S_T


def efla_chunk_fwd_varlen(q, k, v, beta, cu_seqlens, S0=None, g=None, chunk: int = CHUNK, o=None, S_T=None,
                          workspace=None, want_state: bool = True, stream=None, rule: int = EFLA_RULE_EXACT
                          ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Packed variable-length forward: q, k [H,total_T,d_k], v [H,total_T,d_v], beta [H,total_T];
    cu_seqlens: N+1 offsets (a sequence of ints or a CPU int32 tensor); S0 [N,H,d_k,d_v] or None;
    g [H,total_T] float32 (gated flow) or None.  Returns (o, S_T [N,H,d_k,d_v] or None)."""
    dt = k.dtype
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, nme, dt)
    if g is not None:
        _check(g, "g", torch.float32)
    cu = torch.as_tensor(cu_seqlens, dtype=torch.int32, device="cpu").contiguous()
    N = cu.numel() - 1
    H, total_T, d_k = k.shape
    d_v = v.shape[-1]
    if S0 is not None:
        _check(S0, "S0", torch.float32)
    if o is None:
        o = torch.empty((H, total_T, d_v), device=k.device, dtype=dt)
    _check(o, "o", dt)
    if S_T is None and want_state:
        S_T = torch.empty((N, H, d_k, d_v), device=k.device, dtype=torch.float32)
    if S_T is not None:
        _check(S_T, "S_T", torch.float32)
    cup = ctypes.c_void_p(cu.data_ptr())
    if workspace is None:
        n = int(lib.efla_chunk_fwd_varlen_workspace_bytes(cup, N, H, d_k, d_v, chunk, _DTYPES.get(dt, -1),
                                                          int(g is not None)))
        if n == 0:
            raise EflaError(EFLA_ERR_INVALID_ARG, "efla_chunk_fwd_varlen_workspace_bytes")
        workspace = torch.zeros(n, dtype=torch.uint8, device=k.device)
    st = lib.efla_chunk_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), cup, _ptr(S0), _ptr(o),
                                   _ptr(S_T), N, H, d_k, d_v, chunk, _DTYPES.get(dt, -1), int(rule),
                                   _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st, "efla_chunk_fwd_varlen")
    return o, S_T


def efla_train_saved_bytes(B, H, T, d_k, d_v, chunk=CHUNK, dtype=torch.bfloat16) -> int:
    return int(lib.efla_train_saved_bytes(B, H, T, d_k, d_v, chunk, _DTYPES.get(dtype, -1)))


def efla_chunk_fwd_save(q, k, v, beta, S0=None, saved=None, o=None, S_T=None, want_state: bool = True,
                        stream=None, rule: int = EFLA_RULE_EXACT):
    """efla_chunk_fwd that also keeps the residuals efla_backward_saved needs (bf16, d = 128).
    Returns (o, S_T or None, saved); `saved` is a uint8 tensor of efla_train_saved_bytes."""
    dt = k.dtype
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, nme, dt)
    B, H, T, d_k = k.shape
    d_v = v.shape[-1]
    if S0 is not None:
        _check(S0, "S0", torch.float32)
    if o is None:
        o = torch.empty((B, H, T, d_v), device=k.device, dtype=dt)
    _check(o, "o", dt)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, d_k, d_v), device=k.device, dtype=torch.float32)
    if S_T is not None:
        _check(S_T, "S_T", torch.float32)
    if saved is None:
        n = efla_train_saved_bytes(B, H, T, d_k, d_v, CHUNK, dt)
        if n == 0:
            raise EflaError(EFLA_ERR_UNSUPPORTED, "efla_train_saved_bytes")
        saved = torch.zeros(n, dtype=torch.uint8, device=k.device)
    st = lib.efla_chunk_fwd_save(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_T),
                                 B, H, T, d_k, d_v, CHUNK, _DTYPES.get(dt, -1), int(rule), _ptr(saved),
                                 saved.numel(), _stream(stream))
    _raise(st, "efla_chunk_fwd_save")
    return o, S_T, saved


def efla_backward_saved(q, k, v, beta, dO, saved, dS_T=None, want_dS0: bool = True, grads=None,
                        workspace=None, stream=None, rule: int = EFLA_RULE_EXACT):
    """efla_backward from the residuals efla_chunk_fwd_save kept (no forward recompute).
    Returns (dq, dk, dv, dbeta, dS0 or None), all float32."""
    dt = k.dtype
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta"), (dO, "dO")):
        _check(t, nme, dt)
    B, H, T, d_k = k.shape
    d_v = v.shape[-1]
    if dS_T is not None:
        _check(dS_T, "dS_T", torch.float32)
    f32 = dict(device=k.device, dtype=torch.float32)
    if grads is None:
        grads = (torch.empty((B, H, T, d_k), **f32), torch.empty((B, H, T, d_k), **f32),
                 torch.empty((B, H, T, d_v), **f32), torch.empty((B, H, T), **f32),
                 torch.empty((B, H, d_k, d_v), **f32) if want_dS0 else None)
    for t, nme in zip(grads, ("dq", "dk", "dv", "dbeta", "dS0")):
        if t is not None:
            _check(t, nme, torch.float32)
    if workspace is None:
        n = int(lib.efla_backward_saved_workspace_bytes(B, H, T, d_k, d_v, _DTYPES.get(dt, -1)))
        if n == 0:
            raise EflaError(EFLA_ERR_UNSUPPORTED, "efla_backward_saved_workspace_bytes")
        workspace = torch.zeros(n, dtype=torch.uint8, device=k.device)
    st = lib.efla_backward_saved(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(dO), _ptr(dS_T),
                                 *(_ptr(g) for g in grads), B, H, T, d_k, d_v, _DTYPES.get(dt, -1), int(rule),
                                 _ptr(saved), saved.numel(), _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st, "efla_backward_saved")
    return grads


def efla_chunk_fwd_noalloc(q, k, v, beta, S0=None, chunk: int = CHUNK, o=None, S_T=None,
                           want_state: bool = True, stream=None
                           ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """efla_chunk_fwd using the library's internal static scratch instead of a workspace.
    o and S_T are allocated here when not given (pass them in to allocate nothing)."""
    dt = k.dtype
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, nme, dt)
    B, H, T, d_k = k.shape
    d_v = v.shape[-1]
    if S0 is not None:
        _check(S0, "S0", torch.float32)
    if o is None:
        o = torch.empty((B, H, T, d_v), device=k.device, dtype=dt)
    _check(o, "o", dt)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, d_k, d_v), device=k.device, dtype=torch.float32)
    if S_T is not None:
        _check(S_T, "S_T", torch.float32)
    st = lib.efla_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S0), _ptr(o),
                                    _ptr(S_T), B, H, T, d_k, d_v, chunk, _DTYPES.get(dt, -1),
                                    _stream(stream))
    _raise(st, "efla_chunk_fwd_noalloc")
    return o, S_T


def efla_workspace_status(workspace: torch.Tensor, clear: bool = False, stream=None) -> int:
    return int(lib.efla_workspace_status(_ptr(workspace), int(clear), _stream(stream)))


def efla_noalloc_status(clear: bool = False, stream=None) -> int:
    """Device error word of efla_chunk_fwd_noalloc's static scratch (current device)."""
    return int(lib.efla_noalloc_status(int(clear), _stream(stream)))


def efla_selftest_wait_timeout(workspace: torch.Tensor, limit_ns: int = 1_000_000, stream=None) -> None:
    _raise(lib.efla_selftest_wait_timeout(_ptr(workspace), int(limit_ns), _stream(stream)),
           "efla_selftest_wait_timeout")


def efla_recurrent_step(q, k, v, beta, S, o=None, stream=None, rule: int = EFLA_RULE_EXACT) -> torch.Tensor:
    """One decode token: q, k [N,H,d_k], v [N,H,d_v], beta [N,H]; S [N,H,d_k,d_v] float32
    updated in place.  Returns o [N,H,d_v].  rule as in efla_chunk_fwd."""
    dt = k.dtype
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, nme, dt)
    _check(S, "S", torch.float32)
    N, H, d_k = k.shape
    d_v = v.shape[-1]
    if o is None:
        o = torch.empty((N, H, d_v), device=k.device, dtype=dt)
    _check(o, "o", dt)
    _raise(lib.efla_recurrent_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S), _ptr(o),
                                      N, H, d_k, d_v, _DTYPES.get(dt, -1), int(rule), _stream(stream)),
           "efla_recurrent_step")
    return o


def efla_backward_workspace_bytes(B, H, T, d_k, d_v, dtype=torch.bfloat16) -> int:
    return int(lib.efla_backward_workspace_bytes(B, H, T, d_k, d_v, _DTYPES[dtype]))


def efla_backward(q, k, v, beta, dO, S0=None, dS_T=None, want_dS0: bool = True, grads=None,
                  workspace=None, stream=None, rule: int = EFLA_RULE_EXACT):
    """Gradients of efla_chunk_fwd for the loss sum(dO * o) + sum(dS_T * S_T).

    q, k [B,H,T,d_k], v, dO [B,H,T,d_v], beta [B,H,T] (one dtype); S0, dS_T [B,H,d_k,d_v]
    float32 or None.  Returns (dq, dk, dv, dbeta, dS0 or None), all float32.  `grads` may
    supply those five tensors preallocated (dS0 may be None)."""
    dt = k.dtype
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta"), (dO, "dO")):
        _check(t, nme, dt)
    B, H, T, d_k = k.shape
    d_v = v.shape[-1]
    for t, nme in ((S0, "S0"), (dS_T, "dS_T")):
        if t is not None:
            _check(t, nme, torch.float32)
    f32 = dict(device=k.device, dtype=torch.float32)
    if grads is None:
        grads = (torch.empty((B, H, T, d_k), **f32), torch.empty((B, H, T, d_k), **f32),
                 torch.empty((B, H, T, d_v), **f32), torch.empty((B, H, T), **f32),
                 torch.empty((B, H, d_k, d_v), **f32) if want_dS0 else None)
    for t, nme in zip(grads, ("dq", "dk", "dv", "dbeta", "dS0")):
        if t is not None:
            _check(t, nme, torch.float32)
    if workspace is None:
        n = efla_backward_workspace_bytes(B, H, T, d_k, d_v, dt)
        if n == 0 and B * H * T > 0:
            raise EflaError(EFLA_ERR_UNSUPPORTED, "efla_backward_workspace_bytes")
        workspace = torch.zeros(max(n, 16), dtype=torch.uint8, device=k.device)
    st = lib.efla_backward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S0), _ptr(dO), _ptr(dS_T),
                              *(_ptr(g) for g in grads), B, H, T, d_k, d_v, _DTYPES.get(dt, -1), int(rule),
                              _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st, "efla_backward")
    return grads


__all__ = ["efla_train_saved_bytes", "efla_chunk_fwd_save", "efla_backward_saved", "efla_chunk_fwd_segmented", "efla_chunk_fwd_varlen", "efla_chunk_fwd_gated", "efla_recurrent_step_gated", "efla_backward", "efla_backward_workspace_bytes", "EFLA_RULE_EXACT", "EFLA_RULE_EULER", "efla_gate", "efla_chunk_fwd", "efla_chunk_fwd_noalloc", "efla_chunk_fwd_workspace_bytes", "efla_recurrent_step",
           "efla_workspace_status", "efla_noalloc_status", "efla_status_string", "load_checked", "efla_selftest_wait_timeout", "new_workspace", "EflaError", "lib",
           "LIB_PATH", "CHUNK"]
