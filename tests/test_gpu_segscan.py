"""The segmented scan of long streams (efla_chunk_fwd_segmented) against the fp64 oracle.

Splitting a stream into segments changes only the order of operations (the chunk map is
affine in the state: S_out = Phi S_in + S_loc, O = O_loc + R S_in), so the results must
match the oracle within the usual bf16 tolerance (2e-2, relative Frobenius).
"""
import pytest
import torch

import oracle
import workloads
from helpers import TOL, rel_frob

pytestmark = pytest.mark.gpu

W = workloads.CHUNK_WORKLOADS


def dev(inp, cuda):
    return {k: (None if v is None else v.to(cuda)) for k, v in inp.items()}


@pytest.mark.parametrize("name,over,segments,gated", [
    ("longctx_bf16", {"H": 2, "T": 1000}, 2, False),       # two segments, ragged tail
    ("longctx_bf16", {"H": 2, "T": 2600}, 3, False),       # three
    ("lm1p3b_bf16", {"B": 1, "H": 3, "T": 1537}, 2, False),  # no S0
    ("stiff_bf16", {"B": 1, "H": 2, "T": 1100}, 2, False),
    ("longctx_bf16", {"H": 2, "T": 1500}, 2, True),        # gated flow
], ids=str)
def test_segmented_matches_oracle(efla, cuda, name, over, segments, gated):
    w = W[name].replace(**over)
    inp = workloads.make_chunk_inputs(w)
    if gated:
        inp["g"] = workloads.make_log_decay((w.B, w.H, w.T), w.seed + 7)
    d = dev(inp, cuda)
    o, ST = efla.efla_chunk_fwd_segmented(d["q"], d["k"], d["v"], d["beta"], d["S0"], g=d.get("g"),
                                          segments=segments)
    if gated:
        o_ref, S_ref = oracle.fwd_gated(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["S0"])
    else:
        o_ref, S_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"])
    eo, es = rel_frob(o, o_ref), rel_frob(ST, S_ref)
    assert eo <= TOL[w.dtype] and es <= TOL[w.dtype], (eo, es)


def test_one_segment_is_the_plain_forward_bitwise(efla, cuda):
    w = W["longctx_bf16"].replace(H=2, T=700)
    d = dev(workloads.make_chunk_inputs(w), cuda)
    o1, S1 = efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"])
    o2, S2 = efla.efla_chunk_fwd_segmented(d["q"], d["k"], d["v"], d["beta"], d["S0"], segments=1)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_segmented_long_context_full_size(efla, cuda):
    """B1 H16 T32768 d128 bf16 with S0, the library's segment count, every stream vs the oracle."""
    w = W["longctx_bf16"]
    inp = workloads.make_chunk_inputs(w)
    d = dev(inp, cuda)
    o, ST = efla.efla_chunk_fwd_segmented(d["q"], d["k"], d["v"], d["beta"], d["S0"], segments=0)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"])
    eo, es = rel_frob(o, o_ref), rel_frob(ST, S_ref)
    worst = max(rel_frob(o[0, h], o_ref[0, h]) for h in range(w.H))
    print(f"segmented long context: o {eo:.3e} (worst stream {worst:.3e}), S_T {es:.3e}")
    assert eo <= 2e-2 and es <= 2e-2 and worst <= 2e-2
