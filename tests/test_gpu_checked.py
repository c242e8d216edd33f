"""The checked build (libefla_checked.so, EFLA_CHECKED=1) of the tensor-core forward and of
the chunkwise backward.

In that build the UT and chain kernels test every direct global access (loads of beta and
the log-decay, stores of T, o, S_T, the chunk states and the segment products, loads of
S0) and every computed shared-memory store against its buffer's extent, and the backward's
kernels test their direct accesses (beta, dS_T, dS0 and the gradients); an access out of
range is skipped and recorded, and efla_workspace_status then returns EFLA_ERR_BOUNDS.
Each case below runs one path through the checked library and asserts that nothing was
recorded and that the outputs still match the fp64 oracle (2e-2, relative Frobenius, bf16).
"""
import ctypes

import pytest
import torch

import oracle
import workloads
from helpers import TOL, rel_frob

pytestmark = pytest.mark.gpu

W = workloads.CHUNK_WORKLOADS


def dev(inp, cuda):
    return {k: (v.to(cuda) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def zeroed(n, cuda):
    assert n > 0
    return torch.zeros(int(n), dtype=torch.uint8, device=cuda)


def assert_clean(efla, ws):
    st = efla.efla_workspace_status(ws, clear=True)
    assert st == efla.EFLA_OK, efla.efla_status_string(st)


@pytest.mark.parametrize("over,rule", [
    ({"B": 1, "H": 2, "T": 200}, 0),      # four chunks, ragged tail, S0
    ({"B": 2, "H": 1, "T": 64}, 1),       # one full chunk per stream, Euler rule
    ({"B": 1, "H": 3, "T": 5}, 0),        # a single ragged chunk
], ids=str)
def test_checked_dense(efla_checked, cuda, over, rule):
    efla = efla_checked
    w = W["longctx_bf16"].replace(**over)
    inp = workloads.make_chunk_inputs(w)
    d = dev(inp, cuda)
    ws = efla.new_workspace(w.B, w.H, w.T, w.dk, w.dv, dtype=torch.bfloat16, device=cuda)
    o, ST = efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], workspace=ws, rule=rule)
    assert_clean(efla, ws)
    o_ref, S_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"], mode=rule)
    assert rel_frob(o, o_ref) <= TOL[w.dtype] and rel_frob(ST, S_ref) <= TOL[w.dtype]


def test_checked_gated(efla_checked, cuda):
    efla = efla_checked
    w = W["lm1p3b_bf16"].replace(B=1, H=2, T=300)
    inp = workloads.make_chunk_inputs(w)
    inp["g"] = workloads.make_log_decay((w.B, w.H, w.T), w.seed + 7)
    d = dev(inp, cuda)
    n = efla.lib.efla_chunk_fwd_gated_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, efla.CHUNK, efla.EFLA_DTYPE_BF16)
    ws = zeroed(n, cuda)
    o, ST = efla.efla_chunk_fwd_gated(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], workspace=ws)
    assert_clean(efla, ws)
    o_ref, S_ref = oracle.fwd_gated(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["S0"])
    assert rel_frob(o, o_ref) <= TOL[w.dtype] and rel_frob(ST, S_ref) <= TOL[w.dtype]


@pytest.mark.parametrize("gated", [False, True])
def test_checked_varlen(efla_checked, cuda, gated):
    efla = efla_checked
    w = W["longctx_bf16"].replace(H=2)
    mix = [1, 63, 64, 65, 200, 0, 130]
    inp = workloads.make_varlen_inputs(w, mix, with_g=gated)
    d = dev(inp, cuda)
    cu = torch.as_tensor(inp["cu"], dtype=torch.int32).contiguous()
    N = cu.numel() - 1
    n = efla.lib.efla_chunk_fwd_varlen_workspace_bytes(ctypes.c_void_p(cu.data_ptr()), N, w.H, w.dk, w.dv,
                                                       efla.CHUNK, efla.EFLA_DTYPE_BF16, int(gated))
    ws = zeroed(n, cuda)
    o, ST = efla.efla_chunk_fwd_varlen(d["q"], d["k"], d["v"], d["beta"], inp["cu"], S0=d["S0"],
                                       g=d.get("g") if gated else None, workspace=ws)
    assert_clean(efla, ws)
    for s in range(N):
        a, b = inp["cu"][s], inp["cu"][s + 1]
        sl = lambda x: x[:, a:b][None].contiguous()
        S0 = None if inp["S0"] is None else inp["S0"][s][None]
        if gated:
            o_ref, S_ref = oracle.fwd_gated(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["beta"]),
                                            sl(inp["g"]), S0)
        else:
            o_ref, S_ref = oracle.fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["beta"]), S0)
        if b > a:
            assert rel_frob(o[:, a:b], o_ref[0]) <= TOL[w.dtype], s
        assert rel_frob(ST[s], S_ref[0]) <= TOL[w.dtype], s


@pytest.mark.parametrize("segments,gated", [(2, False), (3, True)])
def test_checked_segmented(efla_checked, cuda, segments, gated):
    efla = efla_checked
    w = W["longctx_bf16"].replace(H=2, T=1300)
    inp = workloads.make_chunk_inputs(w)
    if gated:
        inp["g"] = workloads.make_log_decay((w.B, w.H, w.T), w.seed + 7)
    d = dev(inp, cuda)
    n = efla.lib.efla_chunk_fwd_segmented_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, efla.CHUNK,
                                                          efla.EFLA_DTYPE_BF16, int(gated), segments)
    ws = zeroed(n, cuda)
    o, ST = efla.efla_chunk_fwd_segmented(d["q"], d["k"], d["v"], d["beta"], d["S0"], g=d.get("g"),
                                          segments=segments, workspace=ws)
    assert_clean(efla, ws)
    if gated:
        o_ref, S_ref = oracle.fwd_gated(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["S0"])
    else:
        o_ref, S_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"])
    assert rel_frob(o, o_ref) <= TOL[w.dtype] and rel_frob(ST, S_ref) <= TOL[w.dtype]


def test_checked_backward(efla_checked, cuda):
    """The chunkwise backward (bf16, d = 128) through the checked library: the reverse chain's
    dS_T / dS0 accesses and the per-chunk kernel's beta loads and gradient stores are tested
    against their buffers, on top of the forward kernels it reuses."""
    efla = efla_checked
    w = W["lm1p3b_bf16"].replace(B=1, H=2, T=150)
    inp = workloads.make_chunk_inputs(w)
    cot = workloads.make_cotangents(w, with_state_grad=True)
    S0 = 0.1 * torch.randn(w.B, w.H, w.dk, w.dv, generator=torch.Generator().manual_seed(w.seed + 7))
    d = {k: (None if v is None else v.to(cuda)) for k, v in dict(inp, S0=S0, **cot).items()}
    ws = zeroed(efla.efla_backward_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, torch.bfloat16), cuda)
    got = efla.efla_backward(d["q"], d["k"], d["v"], d["beta"], d["dO"], S0=d["S0"], dS_T=d["dS_T"], workspace=ws)
    assert_clean(efla, ws)
    ref = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], cot["dO"], S0=S0, dS_T=cot["dS_T"])
    for g, r in zip(got, ref):
        assert rel_frob(g.cpu(), r) <= 2e-2
