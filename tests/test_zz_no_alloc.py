"""The allocation-free chunked forward, efla_chunk_fwd_noalloc (B200 only).

It serves callers that cannot allocate device memory (code embedded in a runtime that
owns every device allocation, or paths where cudaMalloc's device synchronisation is not
acceptable): its scratch is a static device array inside the library.  This file is
collected last so that a stop-at-first-failure run has already run every other test;
it also passes on its own in a fresh process (the first call sets the scratch up).
"""
import ctypes

import pytest
import torch

import oracle
import workloads
from helpers import TOL, rel_frob

pytestmark = pytest.mark.gpu

CASES = [("lm1p3b_bf16", {"B": 1, "H": 3, "T": 333}),
         ("longctx_bf16", {"H": 2, "T": 200}),
         ("tiny_fp32", {"T": 130})]


@pytest.mark.parametrize("name,over", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_entry_point_twice(efla, cuda, name, over):
    w = workloads.CHUNK_WORKLOADS[name].replace(**over)
    inp = workloads.make_chunk_inputs(w)
    d = {k: (None if v is None else v.to(cuda)) for k, v in inp.items()}
    o_ref, S_ref = efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"])
    o_orc, S_orc = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"])
    tol = TOL[w.dtype]
    o = torch.empty_like(o_ref)
    S = torch.empty_like(S_ref)
    for _ in range(2):                       # two calls in a row share the static scratch
        o.fill_(float("nan"))
        S.fill_(float("nan"))
        efla.efla_chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["beta"], d["S0"], o=o, S_T=S)
        torch.cuda.synchronize()
        assert efla.efla_noalloc_status() == efla.EFLA_OK
        assert rel_frob(o, o_ref) <= tol and rel_frob(S, S_ref) <= tol
        # and against the fp64 oracle directly, not only against the other CUDA entry point
        assert rel_frob(o, o_orc) <= tol and rel_frob(S, S_orc) <= tol


def test_noalloc_rejects_bad_arguments(efla, cuda):
    L = efla.lib
    P = [ctypes.c_void_p(0x10000000 * (i + 1)) for i in range(7)]
    assert L.efla_chunk_fwd_noalloc(*P, 1, 1, 64, 96, 96, 64, 1, None) == efla.EFLA_ERR_UNSUPPORTED
    assert L.efla_chunk_fwd_noalloc(*P, 1, 1, -1, 128, 128, 64, 1, None) == efla.EFLA_ERR_INVALID_ARG
