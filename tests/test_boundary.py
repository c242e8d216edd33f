"""The C ABI library loads, exports every declared symbol and rejects bad arguments
without launching anything (CPU only: no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "efla.h")

# validation codes
OK, INVALID, UNSUPPORTED = 0, 1, 2


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(efla_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("efla_chunk_fwd", "efla_recurrent_step", "efla_gate", "efla_status_string",
                 "efla_chunk_fwd_workspace_bytes", "efla_workspace_status"):
        assert want in names


def test_library_exports_every_declared_symbol(efla):
    lib = ctypes.CDLL(efla.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"libefla.so does not export {name}"


def test_checked_library_exports_every_declared_symbol(efla):
    """The EFLA_CHECKED=1 build of the same sources (bounds recorded, accesses skipped)."""
    from conftest import _build_library
    path = _build_library(checked=True)
    assert path == efla.LIB_CHECKED_PATH
    lib = efla.load_checked()
    for name in declared_functions():
        assert hasattr(lib, name), f"libefla_checked.so does not export {name}"
    assert lib.efla_status_string(efla.EFLA_ERR_BOUNDS) == b"EFLA_ERR_BOUNDS"


def test_status_strings(efla):
    assert efla.efla_status_string(0) == "EFLA_OK"
    assert efla.efla_status_string(4) == "EFLA_ERR_TIMEOUT"
    assert efla.efla_status_string(5) == "EFLA_ERR_BOUNDS"
    assert efla.efla_status_string(99) == "EFLA_ERR_UNKNOWN"


def test_workspace_bytes(efla):
    L = efla.lib
    assert L.efla_chunk_fwd_workspace_bytes(4, 16, 2048, 128, 128, 64, 1) >= 16
    assert L.efla_chunk_fwd_workspace_bytes(1, 1, 1, 64, 64, 64, 0) >= 16
    assert L.efla_chunk_fwd_workspace_bytes(1, 1, 1, 96, 96, 64, 0) == 0      # unsupported d
    assert L.efla_chunk_fwd_workspace_bytes(1, 1, 1, 128, 64, 64, 1) == 0     # d_k != d_v
    assert L.efla_chunk_fwd_workspace_bytes(1, 1, 1, 128, 128, 32, 1) == 0    # chunk
    assert L.efla_chunk_fwd_workspace_bytes(-1, 1, 1, 128, 128, 64, 1) == 0   # negative


def _fwd(L, ptrs, B=1, H=1, T=64, d=128, chunk=64, dtype=1, ws=256):
    q, k, v, b, s0, o, st, w = ptrs
    return L.efla_chunk_fwd(q, k, v, b, s0, o, st, B, H, T, d, d, chunk, dtype, w, ws, None)


# fake, well-separated, 16-byte aligned device addresses: validation never dereferences them
GOOD = [ctypes.c_void_p(0x10000000 * (i + 1)) for i in range(8)]


def test_chunk_fwd_rejects_bad_arguments(efla):
    L = efla.lib
    assert _fwd(L, GOOD, d=96) == UNSUPPORTED
    assert _fwd(L, GOOD, chunk=32) == UNSUPPORTED
    assert _fwd(L, GOOD, dtype=7) == UNSUPPORTED
    assert _fwd(L, GOOD, T=-1) == INVALID
    assert _fwd(L, GOOD, B=-2) == INVALID
    for i in (0, 1, 2, 3, 5):                     # q, k, v, beta, o may not be NULL
        bad = list(GOOD); bad[i] = None
        assert _fwd(L, bad) == INVALID, i
    for i in range(8):                            # every pointer must be 16-byte aligned
        bad = list(GOOD); bad[i] = ctypes.c_void_p(GOOD[i].value + 8)
        assert _fwd(L, bad) == INVALID, i
    bad = list(GOOD); bad[7] = None               # workspace required
    assert _fwd(L, bad) == INVALID
    assert _fwd(L, GOOD, ws=8) == INVALID         # workspace too small
    bad = list(GOOD); bad[5] = GOOD[0]            # o aliases q
    assert _fwd(L, bad) == INVALID
    for i in (0, 1, 2, 3, 4, 6):                  # no input or state may lie inside the workspace
        bad = list(GOOD); bad[i] = ctypes.c_void_p(GOOD[7].value + 1024)
        assert _fwd(L, bad, ws=1 << 20) == INVALID, i
    assert _fwd(L, GOOD, B=0) == OK               # nothing to do, nothing launched
    assert _fwd(L, GOOD, H=0) == OK


def test_recurrent_step_rejects_bad_arguments(efla):
    L = efla.lib
    P = GOOD
    f = lambda ptrs=P, N=4, H=2, d=128, dt=0: L.efla_recurrent_step(*ptrs[:6], N, H, d, d, dt, None)
    assert f(d=32) == UNSUPPORTED
    assert f(dt=3) == UNSUPPORTED
    assert f(N=-1) == INVALID
    assert f(N=0) == OK
    for i in range(6):
        bad = list(P); bad[i] = None
        assert f(bad) == INVALID, i
        bad = list(P); bad[i] = ctypes.c_void_p(P[i].value + 4)
        assert f(bad) == INVALID, i
    bad = list(P); bad[5] = P[4]                  # o aliases S
    assert f(bad) == INVALID
    assert L.efla_recurrent_step(P[0], P[1], P[2], P[3], P[4], P[5], 4, 2, 128, 64, 0, None) == UNSUPPORTED


def test_rule_entry_points_validate_the_rule(efla):
    """The _ex entry points take the step rule; anything but EXACT (0) or EULER (1) is an
    invalid argument and launches nothing.  With a valid rule the other checks are those
    of the plain entry points."""
    L = efla.lib
    q, k, v, b, s0, o, st, w = GOOD
    B, H, T, d, ws = 1, 2, 128, 128, 1 << 24
    fwd = lambda rule, ptrs=GOOD, **kw: L.efla_chunk_fwd_ex(*ptrs[:7], kw.get("B", B), H, T, d, d, 64, 1, rule,
                                                             ptrs[7], ws, None)
    for rule in (-1, 2, 7):
        assert fwd(rule) == INVALID
    assert fwd(0, B=0) == OK and fwd(1, B=0) == OK
    bad = list(GOOD); bad[0] = None
    assert fwd(1, bad) == INVALID
    step = lambda rule, N=4: L.efla_recurrent_step_ex(*GOOD[:6], N, 2, 128, 128, 0, rule, None)
    for rule in (-1, 2):
        assert step(rule) == INVALID
    assert step(0, N=0) == OK and step(1, N=0) == OK
    assert efla.EFLA_RULE_EXACT == 0 and efla.EFLA_RULE_EULER == 1


def test_gate_rejects_bad_arguments(efla):
    L = efla.lib
    assert L.efla_gate(GOOD[0], GOOD[1], GOOD[2], 10, 6, 0, None) == UNSUPPORTED   # 24-byte rows
    assert L.efla_gate(GOOD[0], GOOD[1], GOOD[2], -1, 64, 0, None) == INVALID
    assert L.efla_gate(None, GOOD[1], GOOD[2], 10, 64, 0, None) == INVALID
    assert L.efla_gate(GOOD[0], GOOD[1], GOOD[2], 0, 64, 0, None) == OK


def test_binding_fails_loudly_without_the_library(tmp_path):
    """The product path has no fallback: a missing libefla.so is an import error."""
    import subprocess, sys, shutil
    pkg = tmp_path / "delta_rule_linear_02_b200"
    shutil.copytree(os.path.join(ROOT, "delta_rule_linear_02_b200"), pkg,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    r = subprocess.run([sys.executable, "-c", "import delta_rule_linear_02_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libefla.so is not built" in r.stderr


def _bwd(L, ptrs, B=1, H=1, T=64, d=128, dtype=1, ws=1 << 20, rule=0):
    q, k, v, b, s0, do, dst, dq, dk, dv, db, ds0, w = ptrs
    return L.efla_backward_ex(q, k, v, b, s0, do, dst, dq, dk, dv, db, ds0, B, H, T, d, d, dtype, rule, w, ws,
                              None)


# 13 fake device addresses 16 MiB apart: no two ranges of the small problems below overlap
GOOD_B = [ctypes.c_void_p(0x10000000 + 0x1000000 * i) for i in range(13)]


def test_backward_workspace_bytes(efla):
    L = efla.lib
    # bf16, d = 128 (the chunkwise path): error word + per tile T (64 x 64 bf16), X (64 x 68 fp32),
    # S and dS' (128 x 128 bf16)
    assert L.efla_backward_workspace_bytes(4, 16, 2048, 128, 128, 1) == \
        256 + 64 * 32 * ((64 * 64 + 2 * 128 * 128) * 2 + 64 * 68 * 4)
    # the reverse sweep: residuals and the gate gradient, fp32
    assert L.efla_backward_workspace_bytes(4, 16, 2048, 128, 128, 0) == 4 * 16 * 2048 * (128 + 1) * 4
    assert L.efla_backward_workspace_bytes(1, 1, 1, 96, 96, 0) == 0      # unsupported d
    assert L.efla_backward_workspace_bytes(1, 1, 1, 128, 64, 1) == 0     # d_k != d_v
    assert L.efla_backward_workspace_bytes(1, 1, 1, 64, 64, 5) == 0      # dtype
    assert L.efla_backward_workspace_bytes(1, -1, 1, 64, 64, 0) == 0     # negative


def test_backward_rejects_bad_arguments(efla):
    L = efla.lib
    assert _bwd(L, GOOD_B, d=96) == UNSUPPORTED
    assert _bwd(L, GOOD_B, dtype=3) == UNSUPPORTED
    assert _bwd(L, GOOD_B, rule=9) == INVALID
    assert _bwd(L, GOOD_B, T=-1) == INVALID
    for i in (0, 1, 2, 3, 5, 7, 8, 9, 10):        # inputs, dO and dq, dk, dv, dbeta are required
        bad = list(GOOD_B); bad[i] = None
        assert _bwd(L, bad) == INVALID, i
    for i in range(13):                           # every pointer must be 16-byte aligned
        bad = list(GOOD_B); bad[i] = ctypes.c_void_p(GOOD_B[i].value + 4)
        assert _bwd(L, bad) == INVALID, i
    bad = list(GOOD_B); bad[12] = None            # workspace required
    assert _bwd(L, bad) == INVALID
    assert _bwd(L, GOOD_B, ws=64) == INVALID      # workspace too small
    bad = list(GOOD_B); bad[7] = GOOD_B[0]        # dq aliases q
    assert _bwd(L, bad) == INVALID
    bad = list(GOOD_B); bad[8] = GOOD_B[7]        # dk aliases dq
    assert _bwd(L, bad) == INVALID
    bad = list(GOOD_B); bad[11] = GOOD_B[4]       # dS0 aliases S0
    assert _bwd(L, bad) == INVALID
    for i in range(7):                            # no input may lie inside the workspace
        bad = list(GOOD_B); bad[i] = ctypes.c_void_p(GOOD_B[12].value + 4096)
        assert _bwd(L, bad) == INVALID, i
    assert _bwd(L, GOOD_B, B=0) == OK             # nothing to do, nothing launched
    assert _bwd(L, GOOD_B, H=0) == OK


def test_gated_entry_points_validate_arguments(efla):
    """efla_chunk_fwd_gated / efla_recurrent_step_gated: g is required, aligned and disjoint
    from the outputs and the workspace; the rest is validated as for the ungated calls."""
    L = efla.lib
    q, k, v, b, s0, o, st, w = GOOD
    gp = ctypes.c_void_p(0x90000000)
    B, H, T, d = 1, 2, 128, 128
    ws = L.efla_chunk_fwd_gated_workspace_bytes(B, H, T, d, d, 64, 1)
    assert ws >= L.efla_chunk_fwd_workspace_bytes(B, H, T, d, d, 64, 1)
    assert L.efla_chunk_fwd_gated_workspace_bytes(B, H, T, 96, 96, 64, 1) == 0
    fwd = lambda g=gp, o_=o, **kw: L.efla_chunk_fwd_gated(q, k, v, b, g, s0, o_, st, kw.get("B", B), H, T, d, d,
                                                          64, 1, kw.get("rule", 0), w, kw.get("ws", ws), None)
    assert fwd(g=None) == INVALID                              # g required
    assert fwd(g=ctypes.c_void_p(gp.value + 4)) == INVALID     # misaligned
    assert fwd(o_=gp) == INVALID                               # o overlaps g
    assert fwd(g=ctypes.c_void_p(w.value + 512), ws=1 << 24) == INVALID   # g inside the workspace
    assert fwd(rule=5) == INVALID
    assert fwd(ws=8) == INVALID
    assert fwd(B=0) == OK and fwd(g=None, B=0) == OK
    step = lambda g=gp, N=4, rule=0: L.efla_recurrent_step_gated(q, k, v, b, g, s0, o, N, 2, 128, 128, 0, rule,
                                                                   None)
    assert step(g=None) == INVALID
    assert step(g=ctypes.c_void_p(gp.value + 8)) == INVALID
    assert step(g=s0) == INVALID                               # g overlaps S
    assert step(rule=-1) == INVALID
    assert step(N=0) == OK


def test_varlen_entry_point_validates_offsets(efla):
    L = efla.lib
    import ctypes as C
    arr = lambda xs: (C.c_int * len(xs))(*xs)
    q, k, v, b, s0, o, st, w = GOOD
    ok_cu = arr([0, 64, 64, 200])
    ws = L.efla_chunk_fwd_varlen_workspace_bytes(ok_cu, 3, 2, 128, 128, 64, 1, 0)
    assert ws > 0 and L.efla_chunk_fwd_varlen_workspace_bytes(ok_cu, 3, 2, 128, 128, 64, 1, 1) > ws
    for bad in ([1, 64, 64, 200], [0, 64, 63, 200]):          # cu[0] != 0, decreasing
        assert L.efla_chunk_fwd_varlen_workspace_bytes(arr(bad), 3, 2, 128, 128, 64, 1, 0) == 0
        assert L.efla_chunk_fwd_varlen(q, k, v, b, None, arr(bad), s0, o, st, 3, 2, 128, 128, 64, 1, 0, w, 1 << 26,
                                       None) == INVALID
    call = lambda cu=ok_cu, N=3, ws_=ws, rule=0, d=128: L.efla_chunk_fwd_varlen(
        q, k, v, b, None, cu, s0, o, st, N, 2, d, d, 64, 1, rule, w, ws_, None)
    assert call(d=96) == UNSUPPORTED
    assert call(rule=4) == INVALID
    assert call(ws_=16) == INVALID
    assert call(cu=None) == INVALID
    assert call(N=0) == OK


def test_segmented_entry_point_validates_arguments(efla):
    L = efla.lib
    q, k, v, b, s0, o, st, w = GOOD
    plain = L.efla_chunk_fwd_workspace_bytes(1, 2, 4096, 128, 128, 64, 1)
    seg = L.efla_chunk_fwd_segmented_workspace_bytes(1, 2, 4096, 128, 128, 64, 1, 0, 2)
    assert seg > plain                                            # + states, transition products, R
    assert L.efla_chunk_fwd_segmented_workspace_bytes(1, 2, 4096, 128, 128, 64, 1, 0, 1) == plain
    assert L.efla_chunk_fwd_segmented_workspace_bytes(1, 2, 4096, 128, 128, 64, 1, 0, -1) == 0
    assert L.efla_chunk_fwd_segmented_workspace_bytes(1, 2, 4096, 96, 96, 64, 1, 0, 2) == 0
    call = lambda segments=2, ws=seg, rule=0, B=1: L.efla_chunk_fwd_segmented(
        q, k, v, b, None, s0, o, st, B, 2, 4096, 128, 128, 64, 1, rule, segments, w, ws, None)
    assert call(segments=-1) == INVALID
    assert call(ws=plain) == INVALID                              # too small for two segments
    assert call(rule=3) == INVALID
    assert call(B=0) == OK


def test_training_entry_points_sizes_and_validation(efla):
    """efla_chunk_fwd_save / efla_backward_saved (bf16, d = 128 only): sizes, and every
    rejection happens before anything is launched."""
    L = efla.lib
    tiles = 4 * 16 * 32
    assert L.efla_train_saved_bytes(4, 16, 2048, 128, 128, 64, 1) == \
        256 + tiles * ((64 * 64 + 128 * 128) * 2 + 64 * 68 * 4)
    assert L.efla_backward_saved_workspace_bytes(4, 16, 2048, 128, 128, 1) == 256 + tiles * 128 * 128 * 2
    for args in ((1, 1, 64, 64, 64, 64, 1), (1, 1, 64, 128, 128, 64, 0), (1, 1, 64, 128, 128, 32, 1),
                 (1, 1, -1, 128, 128, 64, 1)):
        assert L.efla_train_saved_bytes(*args) == 0, args
    assert L.efla_backward_saved_workspace_bytes(1, 1, 64, 64, 64, 1) == 0
    assert L.efla_backward_saved_workspace_bytes(1, 1, 64, 128, 128, 0) == 0
    q, k, v, b, s0, o, st, sv = GOOD
    need = L.efla_train_saved_bytes(1, 1, 64, 128, 128, 64, 1)

    def fwd(d=128, dtype=1, rule=0, saved=sv, n=need, out=o):
        return L.efla_chunk_fwd_save(q, k, v, b, s0, out, st, 1, 1, 64, d, d, 64, dtype, rule, saved, n, None)
    assert fwd(d=64) == UNSUPPORTED
    assert fwd(dtype=0) == UNSUPPORTED
    assert fwd(rule=5) == INVALID
    assert fwd(n=need - 16) == INVALID
    assert fwd(saved=None) == INVALID
    assert fwd(out=q) == INVALID                               # o aliases q
    assert fwd(saved=ctypes.c_void_p(q.value)) == INVALID      # saved covers q

    P = GOOD_B
    ws_need = L.efla_backward_saved_workspace_bytes(1, 1, 64, 128, 128, 1)

    def bwd(ptrs=P, d=128, dtype=1, rule=0, saved_n=need, ws_n=ws_need):
        qq, kk, vv, bb, do, dst, dq, dk, dv, db, ds0, saved, w = ptrs
        return L.efla_backward_saved(qq, kk, vv, bb, do, dst, dq, dk, dv, db, ds0, 1, 1, 64, d, d, dtype, rule,
                                     saved, saved_n, w, ws_n, None)
    assert bwd(d=64) == UNSUPPORTED
    assert bwd(dtype=0) == UNSUPPORTED
    assert bwd(rule=7) == INVALID
    assert bwd(saved_n=need - 16) == INVALID
    assert bwd(ws_n=ws_need - 16) == INVALID
    for i in range(13):                           # every pointer must be 16-byte aligned
        bad = list(P); bad[i] = ctypes.c_void_p(P[i].value + 4)
        assert bwd(bad) == INVALID, i
    bad = list(P); bad[6] = P[0]                  # dq aliases q
    assert bwd(bad) == INVALID
    bad = list(P); bad[12] = P[11]                # the workspace holds `saved`
    assert bwd(bad, ws_n=max(ws_need, need)) == INVALID
