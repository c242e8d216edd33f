"""The Euler (delta-rule) step through the same kernels, against the oracle's EULER mode.

The exact-flow method replaces beta by the gate alpha; with EFLA_RULE_EULER the library
writes with alpha = beta, the explicit Euler step of the same ODE (the page's Section 2)
that the exact flow improves on.  The oracle's EULER mode is pinned to one explicit Euler
step of the ODE in the oracle's own tests.  Keys are scaled to unit norm here: with
beta in (0, 1) that keeps beta ||k||^2 < 2, where the explicit step is stable.
Tolerances as for the exact rule: 1e-4 (fp32), 2e-2 (bf16).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import TOL, rel_frob

pytestmark = pytest.mark.gpu

W = workloads.CHUNK_WORKLOADS


def unit_keys(inp):
    k = inp["k"].float()
    inp = dict(inp)
    inp["k"] = (k / k.norm(dim=-1, keepdim=True).clamp_min(1e-30)).to(inp["k"].dtype)
    return inp


CASES = [("lm1p3b_bf16", dict(B=1, H=3, T=200)),           # tcgen05 path (bf16, d = 128)
         ("lm1p3b_bf16", dict(B=1, H=2, T=65, dk=64, dv=64)),  # SIMT bf16, d = 64
         ("tiny_fp32", dict(B=1, H=2, T=130)),              # SIMT fp32, d = 64
         ("tiny_fp32", dict(B=1, H=1, T=70, dk=128, dv=128))]  # SIMT fp32, d = 128


@pytest.mark.parametrize("name,over", CASES, ids=lambda x: str(x))
def test_chunk_fwd_euler_matches_oracle(efla, cuda, name, over):
    w = W[name].replace(**over)
    inp = unit_keys(workloads.make_chunk_inputs(w))
    d = {k: (None if v is None else v.to(cuda)) for k, v in inp.items()}
    o, ST = efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], rule=efla.EFLA_RULE_EULER)
    o_ref, ST_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"], mode=oracle.EULER)
    tol = TOL[w.dtype]
    assert rel_frob(o, o_ref) <= tol, rel_frob(o, o_ref)
    assert rel_frob(ST, ST_ref) <= tol, rel_frob(ST, ST_ref)
    # the rule really switched: the exact flow differs by far more than the tolerance here
    o_x, _ = efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"])
    assert rel_frob(o_x, o_ref) > 3 * tol


@pytest.mark.parametrize("dtype,D", [(torch.float32, 128), (torch.bfloat16, 64)])
def test_decode_euler_matches_oracle(efla, cuda, dtype, D):
    w = workloads.DECODE_WORKLOAD.replace(N=4, H=3, dk=D, dv=D, steps=20)
    S = workloads.make_decode_state(w)
    steps = {k: v.to(dtype) for k, v in workloads.make_decode_steps(w).items()}
    Sd = S.to(cuda)
    So = S.double().numpy().copy()
    os_, orefs = [], []
    for s in range(w.steps):
        o = efla.efla_recurrent_step(steps["q"][s].to(cuda), steps["k"][s].to(cuda), steps["v"][s].to(cuda),
                                     steps["beta"][s].to(cuda), Sd, rule=efla.EFLA_RULE_EULER)
        oref, So = oracle.step(steps["q"][s], steps["k"][s], steps["v"][s], steps["beta"][s], So,
                               mode=oracle.EULER)
        os_.append(o.double().cpu().numpy())
        orefs.append(oref)
    tol = TOL[dtype]
    assert rel_frob(np.stack(os_), np.stack(orefs)) <= tol
    assert rel_frob(Sd, So) <= tol
