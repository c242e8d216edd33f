"""The backward pass (efla_backward, CUDA) against the oracle's fp64 reverse sweep.

The oracle's backward is pinned by finite differences of the pinned forward oracle
(tests/oracle_bwd_pins.py).  Both sides take the same dtype-cast inputs.  Two CUDA paths:
  * bf16 with d = 128 runs the backward through the chunkwise form on tensor cores, whose
    products take bf16 operands (as the forward's do): 2e-2 relative Frobenius per gradient,
    the bf16 bound of the forward; at the full 1.3B-layer shape (B4 H16 T2048) every stream;
  * fp32 inputs and d = 64 run the token-by-token reverse sweep with the state and every
    gradient in fp32: 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import rel_frob

pytestmark = pytest.mark.gpu

W = workloads.CHUNK_WORKLOADS
NAMES = ("dq", "dk", "dv", "dbeta", "dS0")


def run_both(efla, cuda, w, with_state=True, rule=None, streams=None, unit_keys=False):
    inp = workloads.make_chunk_inputs(w)
    if unit_keys:   # beta ||k||^2 < 2: the explicit (Euler) step stays stable
        k = inp["k"].float()
        inp["k"] = (k / k.norm(dim=-1, keepdim=True).clamp_min(1e-30)).to(inp["k"].dtype)
    cot = workloads.make_cotangents(w, with_state_grad=with_state)
    S0 = inp["S0"]
    if with_state and S0 is None:
        S0 = 0.1 * torch.randn(w.B, w.H, w.dk, w.dv, generator=torch.Generator().manual_seed(w.seed + 7))
    if not with_state:
        S0 = None
    d = {k: (None if v is None else v.to(cuda)) for k, v in dict(inp, S0=S0, **cot).items()}
    kw = {} if rule is None else dict(rule=rule)
    got = efla.efla_backward(d["q"], d["k"], d["v"], d["beta"], d["dO"], S0=d["S0"], dS_T=d["dS_T"], **kw)
    torch.cuda.synchronize()
    mode = oracle.EULER if rule == efla.EFLA_RULE_EULER else oracle.EXACT
    if streams is None:
        ref = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], cot["dO"], S0=S0, dS_T=cot["dS_T"], mode=mode)
        return [g.cpu() for g in got], ref
    sel = lambda t: None if t is None else torch.stack([t[b, h] for b, h in streams])[None]
    ref = oracle.bwd(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(inp["beta"]), sel(cot["dO"]),
                     S0=sel(S0), dS_T=sel(cot["dS_T"]), mode=mode, threads=len(streams))
    got = [sel(g.cpu()) for g in got]
    return got, ref


CASES = [("tiny_fp32", dict(B=1, H=2, T=200)),                          # fp32, d = 64, ragged T
         ("tiny_fp32", dict(B=2, H=1, T=97, dk=128, dv=128)),             # fp32, d = 128
         ("lm1p3b_bf16", dict(B=1, H=2, T=150)),                          # bf16, d = 128
         ("lm1p3b_bf16", dict(B=1, H=3, T=64, dk=64, dv=64)),             # bf16, d = 64
         ("stiff_bf16", dict(B=1, H=2, T=300))]                           # stiff keys, corrupted tokens


def tol_for(w):
    return 2e-2 if (w.dtype == torch.bfloat16 and w.dk == 128) else 1e-4


@pytest.mark.parametrize("name,over", CASES, ids=lambda x: str(x))
def test_backward_matches_oracle(efla, cuda, name, over):
    w = W[name].replace(**over)
    got, ref = run_both(efla, cuda, w)
    for nme, g, r in zip(NAMES, got, ref):
        e = rel_frob(g, r)
        print(f"{name} {over} {nme}: {e:.3e}")
        assert e <= tol_for(w), (nme, e)


@pytest.mark.parametrize("with_state,rule,T", [(False, None, 130), (True, "euler", 200), (True, None, 1),
                                               (True, None, 64), (True, None, 65)])
def test_chunked_backward_cases(efla, cuda, with_state, rule, T):
    """bf16 d = 128 (the chunkwise path): no state tensors, the Euler rule, T = 1, one chunk, a
    ragged second chunk."""
    w = W["lm1p3b_bf16"].replace(B=1, H=2, T=T)
    r = efla.EFLA_RULE_EULER if rule == "euler" else None
    got, ref = run_both(efla, cuda, w, with_state=with_state, rule=r, unit_keys=rule == "euler")
    for nme, g, rr in zip(NAMES, got, ref):
        e = rel_frob(g, rr)
        assert e <= 2e-2, (nme, e)


def test_backward_without_state_tensors(efla, cuda):
    """No S0, no dS_T: the oracle's zero state and zero final gradient."""
    w = W["tiny_fp32"].replace(B=1, H=2, T=77)
    got, ref = run_both(efla, cuda, w, with_state=False)
    for nme, g, r in zip(NAMES, got, ref):
        assert rel_frob(g, r) <= 1e-4, nme


def test_backward_euler_rule(efla, cuda):
    """The Euler step alpha = beta differentiated (keys of unit norm, as for the forward's
    Euler test: with beta ||k||^2 up to ~64 the explicit step diverges and overflows)."""
    w = W["tiny_fp32"].replace(B=1, H=2, T=90)
    got, ref = run_both(efla, cuda, w, rule=efla.EFLA_RULE_EULER, unit_keys=True)
    for nme, g, r in zip(NAMES, got, ref):
        assert rel_frob(g, r) <= 1e-4, nme


def test_backward_single_token_and_empty(efla, cuda):
    w = W["tiny_fp32"].replace(B=1, H=3, T=1)
    got, ref = run_both(efla, cuda, w)
    for nme, g, r in zip(NAMES, got, ref):
        assert rel_frob(g, r) <= 1e-5, nme
    # T = 0: the state gradient passes straight through
    dST = torch.randn(1, 2, 64, 64, device=cuda)
    e = torch.empty(1, 2, 0, 64, device=cuda)
    out = efla.efla_backward(e, e, e, torch.empty(1, 2, 0, device=cuda), e, dS_T=dST)
    torch.cuda.synchronize()
    assert torch.equal(out[4], dST)


def test_backward_full_shape_every_stream(efla, cuda):
    """B4 H16 T2048 d128 bf16, the forward's benchmark shape: every stream against the oracle."""
    w = W["lm1p3b_bf16"]
    got, ref = run_both(efla, cuda, w)
    for nme, g, r in zip(NAMES, got, ref):
        e = rel_frob(g, r)
        print(f"full shape {nme}: {e:.3e}")
        assert e <= 2e-2, (nme, e)


def test_chunked_backward_repeats_bitwise_and_reports_ok(efla, cuda):
    """The chunkwise backward has no atomics and no order-dependent sums: two calls on the same
    inputs give the same bits, and the workspace's error word stays EFLA_OK."""
    w = W["lm1p3b_bf16"].replace(B=1, H=3, T=300)
    inp = workloads.make_chunk_inputs(w)
    cot = workloads.make_cotangents(w, with_state_grad=True)
    S0 = 0.1 * torch.randn(w.B, w.H, w.dk, w.dv, generator=torch.Generator().manual_seed(w.seed + 7))
    d = {k: (None if v is None else v.to(cuda)) for k, v in dict(inp, S0=S0, **cot).items()}
    n = efla.efla_backward_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, torch.bfloat16)
    ws = torch.zeros(n, dtype=torch.uint8, device=cuda)
    a = efla.efla_backward(d["q"], d["k"], d["v"], d["beta"], d["dO"], S0=d["S0"], dS_T=d["dS_T"], workspace=ws)
    b = efla.efla_backward(d["q"], d["k"], d["v"], d["beta"], d["dO"], S0=d["S0"], dS_T=d["dS_T"], workspace=ws)
    assert efla.efla_workspace_status(ws) == efla.EFLA_OK
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("name,over,rule", [("lm1p3b_bf16", dict(B=1, H=3, T=300), None),
                                            ("lm1p3b_bf16", dict(B=1, H=2, T=65), "euler"),
                                            ("lm1p3b_bf16", {}, None)], ids=str)
def test_training_saved_path_is_the_recompute_bit_for_bit(efla, cuda, name, over, rule):
    """efla_chunk_fwd_save gives efla_chunk_fwd's outputs, and efla_backward_saved (fed by it)
    efla_backward's gradients, bit for bit: the saved T and entering states are the ones the
    backward would recompute.  The recompute path is itself checked against the oracle above."""
    w = W[name].replace(**over)
    inp = workloads.make_chunk_inputs(w)
    if rule == "euler":
        k = inp["k"].float()
        inp["k"] = (k / k.norm(dim=-1, keepdim=True).clamp_min(1e-30)).to(inp["k"].dtype)
    cot = workloads.make_cotangents(w, with_state_grad=True)
    S0 = 0.1 * torch.randn(w.B, w.H, w.dk, w.dv, generator=torch.Generator().manual_seed(w.seed + 7))
    d = {k: (None if v is None else v.to(cuda)) for k, v in dict(inp, S0=S0, **cot).items()}
    r = efla.EFLA_RULE_EULER if rule == "euler" else efla.EFLA_RULE_EXACT
    o1, S1 = efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], rule=r)
    o2, S2, saved = efla.efla_chunk_fwd_save(d["q"], d["k"], d["v"], d["beta"], d["S0"], rule=r)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    g1 = efla.efla_backward(d["q"], d["k"], d["v"], d["beta"], d["dO"], S0=d["S0"], dS_T=d["dS_T"], rule=r)
    ws = torch.zeros(efla.lib.efla_backward_saved_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, efla.EFLA_DTYPE_BF16),
                     dtype=torch.uint8, device=cuda)
    g2 = efla.efla_backward_saved(d["q"], d["k"], d["v"], d["beta"], d["dO"], saved, dS_T=d["dS_T"], rule=r,
                                  workspace=ws)
    assert efla.efla_workspace_status(ws) == efla.EFLA_OK
    assert efla.efla_workspace_status(saved) == efla.EFLA_OK
    for nme, x, y in zip(NAMES, g1, g2):
        assert torch.equal(x, y), nme
