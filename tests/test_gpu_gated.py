"""Gated EFLA on the GPU against the gated fp64 oracle, through the C ABI (B200 only).

The gated flow (a per-token log-decay g in the zero-order-hold ODE, Section 3.4's Gated
EFLA) runs through the same chunked and decode entry points' kernels; tolerances are the
ungated ones: relative Frobenius error 1e-4 for fp32 inputs, 2e-2 for bf16.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import TOL, rel_frob

pytestmark = pytest.mark.gpu

W = workloads.CHUNK_WORKLOADS

CASES = [
    ("tiny_fp32", {}, oracle.EXACT),
    ("tiny_fp32", {"T": 200, "H": 3}, oracle.EXACT),
    ("tiny_fp32", {"dk": 128, "dv": 128, "T": 130}, oracle.EXACT),
    # Euler (the gated delta rule) only where it is stable: unit-scale keys, not tiny_fp32's ||k||^2 ~ 64
    ("lm1p3b_bf16", {"B": 1, "H": 2, "T": 150, "dk": 64, "dv": 64, "dtype": torch.float32}, oracle.EULER),
    ("lm1p3b_bf16", {"B": 1, "H": 2, "T": 333}, oracle.EXACT),
    ("lm1p3b_bf16", {"B": 2, "H": 3, "T": 64, "dk": 64, "dv": 64}, oracle.EXACT),
    ("longctx_bf16", {"H": 2, "T": 1000}, oracle.EXACT),
    ("stiff_bf16", {"B": 1, "H": 2, "T": 517}, oracle.EXACT),
    ("lm1p3b_bf16", {"B": 1, "H": 2, "T": 300}, oracle.EULER),
    ("lm1p3b_bf16", {"B": 1, "H": 1, "T": 1}, oracle.EXACT),
]


def gated_inputs(w):
    inp = workloads.make_chunk_inputs(w)
    inp["g"] = workloads.make_log_decay((w.B, w.H, w.T), w.seed + 7)
    return inp


def dev(inp, cuda):
    return {k: (None if v is None else v.to(cuda)) for k, v in inp.items()}


@pytest.mark.parametrize("name,over,mode", CASES, ids=lambda x: str(x))
def test_gated_chunk_fwd_matches_oracle(efla, cuda, name, over, mode):
    w = W[name].replace(**over)
    inp = gated_inputs(w)
    d = dev(inp, cuda)
    o, ST = efla.efla_chunk_fwd_gated(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], rule=mode)
    o_ref, ST_ref = oracle.fwd_gated(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["S0"], mode=mode)
    tol = TOL[w.dtype]
    eo, es = rel_frob(o, o_ref), rel_frob(ST, ST_ref)
    assert eo <= tol and es <= tol, (eo, es)


@pytest.mark.parametrize("name", ["tiny_fp32", "lm1p3b_bf16"])
def test_gated_with_zero_decay_is_the_ungated_forward(efla, cuda, name):
    w = W[name].replace(B=1, H=2, T=200)
    d = dev(workloads.make_chunk_inputs(w), cuda)
    g0 = torch.zeros(w.B, w.H, w.T, device=cuda)
    o, ST = efla.efla_chunk_fwd_gated(d["q"], d["k"], d["v"], d["beta"], g0, d["S0"])
    o1, S1 = efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"])
    tol = TOL[w.dtype]
    assert rel_frob(o, o1) <= tol and rel_frob(ST, S1) <= tol


def test_gated_full_size_every_stream(efla, cuda):
    """The gated flow at the 1.3B-layer shape (B4 H16 T2048 d128 bf16), every stream vs the oracle."""
    w = W["lm1p3b_bf16"]
    inp = gated_inputs(w)
    d = dev(inp, cuda)
    o, ST = efla.efla_chunk_fwd_gated(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"])
    torch.cuda.synchronize()
    o_ref, ST_ref = oracle.fwd_gated(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["S0"])
    eo, es = rel_frob(o, o_ref), rel_frob(ST, ST_ref)
    worst = max(rel_frob(o[b, h], o_ref[b, h]) for b in range(w.B) for h in range(w.H))
    print(f"gated lm1p3b: o {eo:.3e} (worst stream {worst:.3e}), S_T {es:.3e}")
    assert eo <= 2e-2 and es <= 2e-2 and worst <= 2e-2


@pytest.mark.parametrize("dtype,D,mode", [(torch.float32, 128, oracle.EXACT), (torch.float32, 64, oracle.EXACT),
                                          (torch.bfloat16, 128, oracle.EXACT), (torch.float32, 128, oracle.EULER)])
def test_gated_decode_matches_oracle(efla, cuda, dtype, D, mode):
    w = workloads.DECODE_WORKLOAD.replace(N=5, H=3, dk=D, dv=D, steps=40)
    S = workloads.make_decode_state(w)
    steps = {k: v.to(dtype) for k, v in workloads.make_decode_steps(w).items()}
    gs = workloads.make_log_decay((w.steps, w.N, w.H), 99)
    Sd = S.to(cuda)
    So = S.double().numpy().copy()
    os_, orefs = [], []
    for s in range(w.steps):
        o = efla.efla_recurrent_step_gated(steps["q"][s].to(cuda), steps["k"][s].to(cuda), steps["v"][s].to(cuda),
                                           steps["beta"][s].to(cuda), gs[s].to(cuda), Sd, rule=mode)
        oref, So = oracle.step_gated(steps["q"][s], steps["k"][s], steps["v"][s], steps["beta"][s], gs[s], So,
                                     mode=mode)
        os_.append(o.double().cpu().numpy())
        orefs.append(oref)
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    assert rel_frob(np.stack(os_), np.stack(orefs)) <= tol
    assert rel_frob(Sd, So) <= tol
