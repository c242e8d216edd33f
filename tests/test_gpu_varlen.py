"""Packed variable-length batches on the GPU against the fp64 oracle, through the C ABI.

Each (sequence, head) of a packed batch is its own recurrence (Section 3.3's chunking per
sequence): the oracle runs every sequence as a one-stream batch from its S0 slice, and the
packed output must match it within the usual tolerances (1e-4 fp32, 2e-2 bf16).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import TOL, rel_frob

pytestmark = pytest.mark.gpu

W = workloads.CHUNK_WORKLOADS
MIX = [1, 63, 64, 65, 200, 0, 517, 130, 3]


def run(efla, inp, cuda, gated=False, rule=0):
    d = {k: (v.to(cuda) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    return efla.efla_chunk_fwd_varlen(d["q"], d["k"], d["v"], d["beta"], d["cu"], S0=d["S0"],
                                      g=d.get("g") if gated else None, rule=rule)


def check_against_oracle(inp, o, ST, tol, gated=False, rule=0):
    cu = inp["cu"]
    worst = 0.0
    for n in range(len(cu) - 1):
        a, b = cu[n], cu[n + 1]
        sl = lambda x: x[:, a:b][None].contiguous()
        S0 = None if inp["S0"] is None else inp["S0"][n][None]
        if gated:
            o_ref, S_ref = oracle.fwd_gated(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["beta"]), sl(inp["g"]),
                                            S0, mode=rule)
        else:
            o_ref, S_ref = oracle.fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["beta"]), S0, mode=rule)
        if b > a:
            e = rel_frob(o[:, a:b], o_ref[0])
            assert e <= tol, (n, b - a, e)
            worst = max(worst, e)
        es = rel_frob(ST[n], S_ref[0])
        assert es <= tol, (n, b - a, es)
        worst = max(worst, es)
    return worst


@pytest.mark.parametrize("name,over,gated", [
    ("longctx_bf16", {"H": 3}, False),                    # bf16, d 128: tensor-core path, S0 given
    ("lm1p3b_bf16", {"H": 2}, True),                     # gated, tensor-core path
    ("tiny_fp32", {"H": 2}, False),                      # fp32, d 64: CUDA-core path
    ("tiny_fp32", {"H": 2, "s0_std": 0.1}, True),        # gated fp32 with S0
    ("lm1p3b_bf16", {"H": 2, "dk": 64, "dv": 64}, False),  # bf16, d 64: CUDA-core path
], ids=str)
def test_varlen_matches_oracle_per_sequence(efla, cuda, name, over, gated):
    w = W[name].replace(**over)
    inp = workloads.make_varlen_inputs(w, MIX, with_g=gated)
    o, ST = run(efla, inp, cuda, gated)
    torch.cuda.synchronize()
    check_against_oracle(inp, o, ST, TOL[w.dtype], gated)


def test_varlen_euler_rule(efla, cuda):
    w = W["lm1p3b_bf16"].replace(H=2)
    inp = workloads.make_varlen_inputs(w, [70, 5, 140])
    o, ST = run(efla, inp, cuda, rule=oracle.EULER)
    check_against_oracle(inp, o, ST, TOL[w.dtype], rule=oracle.EULER)


@pytest.mark.parametrize("name", ["lm1p3b_bf16", "tiny_fp32"])
def test_equal_lengths_packed_equal_the_dense_batch_bitwise(efla, cuda, name):
    """B equal-length sequences packed along T give bit for bit the dense [B,H,T,d] forward."""
    w = W[name].replace(B=3, H=2, T=200)
    dense = {k: (None if v is None else v.to(cuda)) for k, v in workloads.make_chunk_inputs(w).items()}
    o_d, S_d = efla.efla_chunk_fwd(dense["q"], dense["k"], dense["v"], dense["beta"], dense["S0"])
    pack = lambda x: x.permute(1, 0, 2, 3).reshape(w.H, w.B * w.T, -1).contiguous()
    beta_p = dense["beta"].permute(1, 0, 2).reshape(w.H, w.B * w.T).contiguous()
    o_p, S_p = efla.efla_chunk_fwd_varlen(pack(dense["q"]), pack(dense["k"]), pack(dense["v"]), beta_p,
                                          [0, w.T, 2 * w.T, 3 * w.T])
    assert torch.equal(o_p, pack(o_d))
    assert torch.equal(S_p, S_d.reshape(w.B * w.H, w.dk, w.dv).reshape(w.B, w.H, w.dk, w.dv))


def test_varlen_all_empty_passes_state_through(efla, cuda):
    w = W["longctx_bf16"].replace(H=2)
    inp = workloads.make_varlen_inputs(w, [0, 0])
    o, ST = run(efla, inp, cuda)
    assert o.numel() == 0 and torch.equal(ST, inp["S0"].to(cuda))


def test_varlen_length_mix_at_scale(efla, cuda):
    """A 16-head bf16 batch of 24 sequences (log-uniform length mix, 16,384 tokens in all, the
    1.3B-layer distributions): every sequence and head against the oracle."""
    w = W["lm1p3b_bf16"]
    lengths = workloads.varlen_lengths(24, 16384, seed=5)
    inp = workloads.make_varlen_inputs(w.replace(H=16), lengths)
    o, ST = run(efla, inp, cuda)
    torch.cuda.synchronize()
    worst = check_against_oracle(inp, o, ST, 2e-2)
    print(f"varlen mix: {len(lengths)} sequences, lengths {min(lengths)}..{max(lengths)}, worst {worst:.3e}")
