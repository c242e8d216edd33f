"""CUDA path vs the fp64 oracle on the same seeded inputs, through the C ABI (B200 only).

Tolerances (relative Frobenius error, whole tensor): 1e-4 for fp32 inputs, 2e-2 for bf16
inputs with fp32 accumulation and state.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import TOL, rel_frob

pytestmark = pytest.mark.gpu

W = workloads.CHUNK_WORKLOADS


def to_dev(inp, dev):
    return {k: (None if v is None else v.to(dev)) for k, v in inp.items()}


def run_fwd(efla, d, chunk=64):
    return efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=chunk)


# ------------------------------------------------------------------------------ gate
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gate_extremes(efla, cuda, dtype):
    lams = [0.0, 1e-41, 1e-30, 1e-12, 1e-8, 1e-4, 0.5, 1.0, 64.0, 1e3, 1e6]
    betas = [0.01, 0.5, 0.98, 3.0]
    dk = 64
    ks, bs, want = [], [], []
    for lam in lams:
        for b in betas:
            kv = torch.zeros(dk, dtype=torch.float64)
            kv[5] = math.sqrt(lam)
            kv = kv.to(dtype)
            bt = torch.tensor(b, dtype=torch.float64).to(dtype)
            lam_c = float((kv.double() ** 2).sum())
            ks.append(kv); bs.append(bt)
            want.append(oracle.alpha(float(bt.double()), lam_c))
    k = torch.stack(ks).to(cuda)
    beta = torch.stack(bs).to(cuda)
    alpha = efla.efla_gate(k, beta).double().cpu().numpy()
    want = np.array(want)
    err = np.abs(alpha - want) / np.maximum(np.abs(want), 1e-300)
    assert err.max() <= 2e-6, (err.max(), alpha[err.argmax()], want[err.argmax()])
    zero = [i for i, (l, _) in enumerate((l, b) for l in lams for b in betas) if l == 0.0]
    assert all(alpha[i] == float(beta[i].double()) for i in zero)      # exact limit at lambda = 0


# ------------------------------------------------------------------------------ chunk forward
SMALL_CASES = [
    # (workload, overrides): several chunks plus a ragged tail, oracle in seconds
    ("tiny_fp32", {}),
    ("tiny_fp32", {"T": 200, "H": 3}),
    ("tiny_fp32", {"dk": 128, "dv": 128, "T": 130}),
    ("lm1p3b_bf16", {"B": 1, "H": 2, "T": 333}),
    ("lm1p3b_bf16", {"B": 2, "H": 3, "T": 64, "dk": 64, "dv": 64}),
    ("longctx_bf16", {"H": 2, "T": 1000}),
    ("stiff_bf16", {"B": 1, "H": 2, "T": 517}),
    ("stiff_bf16", {"B": 1, "H": 1, "T": 1}),
    ("lm1p3b_bf16", {"B": 1, "H": 1, "T": 63}),
    ("lm1p3b_bf16", {"B": 1, "H": 1, "T": 65}),
]


@pytest.mark.parametrize("name,over", SMALL_CASES, ids=lambda x: str(x))
def test_chunk_fwd_small(efla, cuda, name, over):
    w = W[name].replace(**over)
    inp = workloads.make_chunk_inputs(w)
    o, ST = run_fwd(efla, to_dev(inp, cuda))
    o_ref, ST_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"])
    tol = TOL[w.dtype]
    assert rel_frob(o, o_ref) <= tol, rel_frob(o, o_ref)
    assert rel_frob(ST, ST_ref) <= tol, rel_frob(ST, ST_ref)


FULL = ["tiny_fp32", "lm1p3b_bf16", "longctx_bf16", "stiff_bf16"]


def per_stream_errors(x, ref):
    """Relative Frobenius error of every (b, h) stream: [B, H] float64."""
    x = x.detach().double().cpu().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    axes = tuple(range(2, ref.ndim))
    num = np.sqrt(((x - ref) ** 2).sum(axis=axes))
    den = np.sqrt((ref ** 2).sum(axis=axes))
    return num / np.where(den > 0, den, 1.0)


@pytest.mark.parametrize("name", FULL)
def test_chunk_fwd_full_size(efla, cuda, name):
    """The full workload in the bench's launch configuration, every stream against the oracle:
    whole-tensor error on o and S_T, and the worst single (b, h) stream."""
    w = W[name]
    inp = workloads.make_chunk_inputs(w, with_mask=True)
    o, ST = run_fwd(efla, to_dev(inp, cuda))
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(ST).all()
    tol = TOL[w.dtype]
    o_ref, ST_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"])
    eo, es = rel_frob(o, o_ref), rel_frob(ST, ST_ref)
    po, ps = per_stream_errors(o, o_ref), per_stream_errors(ST, ST_ref)
    print(f"{name}: o {eo:.3e} (worst stream {po.max():.3e}), S_T {es:.3e} (worst stream {ps.max():.3e})")
    assert eo <= tol and es <= tol, (eo, es)
    assert po.max() <= tol and ps.max() <= tol, (np.unravel_index(po.argmax(), po.shape), po.max(),
                                                 np.unravel_index(ps.argmax(), ps.shape), ps.max())
    bad = inp["corrupt"]
    if bad.any():
        # the high-energy tokens dominate ||o||_F: the clean tokens must also agree on their own
        clean = ~bad.numpy()                                         # [B, T]
        og = o.double().cpu().numpy().transpose(0, 2, 1, 3)[clean]   # [n_clean, H, dv]
        orf = o_ref.transpose(0, 2, 1, 3)[clean]
        ec = rel_frob(og, orf)
        print(f"{name}: o over the {int(clean.sum())} clean (b, t) tokens {ec:.3e}")
        assert ec <= tol, ec


def test_state_carry_split_equals_single_run(efla, cuda):
    """Running [0, T1) then [T1, T) with S_T fed back as S0 equals one run of [0, T)."""
    w = W["longctx_bf16"].replace(H=2, T=640)
    d = to_dev(workloads.make_chunk_inputs(w), cuda)
    o, ST = run_fwd(efla, d)
    T1 = 256
    first = {k: (v[:, :, :T1].contiguous() if k in ("q", "k", "v", "beta") else v) for k, v in d.items()}
    o1, S1 = run_fwd(efla, first)
    second = {k: (v[:, :, T1:].contiguous() if k in ("q", "k", "v", "beta") else v) for k, v in d.items()}
    second["S0"] = S1
    o2, S2 = run_fwd(efla, second)
    assert rel_frob(torch.cat([o1, o2], 2), o) <= 1e-2
    assert rel_frob(S2, ST) <= 1e-3


def test_initial_state_aliases_final_state(efla, cuda):
    w = W["longctx_bf16"].replace(H=2, T=192)
    d = to_dev(workloads.make_chunk_inputs(w), cuda)
    o, ST = run_fwd(efla, d)
    S = d["S0"].clone()
    o2, S2 = efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], S, S_T=S)
    assert S2.data_ptr() == S.data_ptr()
    assert torch.equal(o2, o) and torch.equal(S, ST)


@pytest.mark.parametrize("name", ["tiny_fp32", "lm1p3b_bf16"])
def test_streams_are_independent_bitwise(efla, cuda, name):
    w = W[name].replace(B=2, H=3, T=200)
    d = to_dev(workloads.make_chunk_inputs(w), cuda)
    o, ST = run_fwd(efla, d)
    b, h = 1, 2
    one = {k: (None if v is None else v[b:b + 1, h:h + 1].contiguous()) for k, v in d.items()}
    o1, S1 = run_fwd(efla, one)
    assert torch.equal(o1[0, 0], o[b, h]) and torch.equal(S1[0, 0], ST[b, h])


def test_empty_sequence_passes_state_through(efla, cuda):
    w = W["longctx_bf16"].replace(H=2, T=0)
    d = to_dev(workloads.make_chunk_inputs(w), cuda)
    o, ST = run_fwd(efla, d)
    assert o.numel() == 0 and torch.equal(ST, d["S0"])
    d["S0"] = None
    o, ST = run_fwd(efla, d)
    assert torch.count_nonzero(ST) == 0


def test_zero_gate_is_identity_on_state(efla, cuda):
    """beta = 0 gives alpha = 0: the state is untouched and o_t = S0^T q_t."""
    w = W["longctx_bf16"].replace(H=2, T=100)
    inp = workloads.make_chunk_inputs(w)
    inp["beta"] = torch.zeros_like(inp["beta"])
    d = to_dev(inp, cuda)
    o, ST = run_fwd(efla, d)
    assert rel_frob(ST, d["S0"]) <= 1e-6
    ref = torch.einsum("bhtk,bhkv->bhtv", inp["q"].double(), inp["S0"].double())
    assert rel_frob(o, ref) <= 2e-2


def test_workspace_reports_no_timeout(efla, cuda):
    w = W["lm1p3b_bf16"].replace(B=1, H=2, T=256)
    d = to_dev(workloads.make_chunk_inputs(w), cuda)
    ws = efla.new_workspace(1, 2, 256, 128, 128)
    efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], None, workspace=ws)
    assert efla.efla_workspace_status(ws, clear=True) == efla.EFLA_OK


def test_invalid_arguments_raise(efla, cuda):
    w = W["lm1p3b_bf16"].replace(B=1, H=1, T=64, dk=96, dv=96)
    d = to_dev(workloads.make_chunk_inputs(w), cuda)
    with pytest.raises(efla.EflaError) as e:
        run_fwd(efla, d)
    assert e.value.status == efla.EFLA_ERR_UNSUPPORTED


# ------------------------------------------------------------------------------ decode
@pytest.mark.parametrize("dtype,D", [(torch.float32, 128), (torch.float32, 64), (torch.bfloat16, 128)])
def test_decode_small(efla, cuda, dtype, D):
    w = workloads.DECODE_WORKLOAD.replace(N=5, H=3, dk=D, dv=D, steps=40)
    S = workloads.make_decode_state(w)
    steps = workloads.make_decode_steps(w)
    steps = {k: v.to(dtype) for k, v in steps.items()}
    Sd = S.to(cuda)
    So = S.double().numpy().copy()
    os_, orefs = [], []
    for s in range(w.steps):
        o = efla.efla_recurrent_step(steps["q"][s].to(cuda), steps["k"][s].to(cuda),
                                     steps["v"][s].to(cuda), steps["beta"][s].to(cuda), Sd)
        oref, So = oracle.step(steps["q"][s], steps["k"][s], steps["v"][s], steps["beta"][s], So)
        os_.append(o.double().cpu().numpy()); orefs.append(oref)
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    assert rel_frob(np.stack(os_), np.stack(orefs)) <= tol
    assert rel_frob(Sd, So) <= tol


def test_decode_full_size(efla, cuda):
    """1000 in-place steps at N=256, H=16, d=128; the oracle follows every head: o over all
    1000 steps and the final state, whole-tensor relative Frobenius error."""
    w = workloads.DECODE_WORKLOAD
    S = workloads.make_decode_state(w, device=cuda)
    S_o = S.double().cpu().numpy()                                  # oracle state, updated in place
    steps = workloads.make_decode_steps(w, device=cuda)
    outs = torch.empty((w.steps, w.N, w.H, w.dv), device=cuda, dtype=torch.float32)
    for s in range(w.steps):
        efla.efla_recurrent_step(steps["q"][s], steps["k"][s], steps["v"][s], steps["beta"][s], S,
                                 o=outs[s])
    torch.cuda.synchronize()
    err2 = ref2 = 0.0
    for s in range(w.steps):
        oref, S_o = oracle.step(steps["q"][s].cpu(), steps["k"][s].cpu(), steps["v"][s].cpu(),
                                steps["beta"][s].cpu(), S_o)
        d = outs[s].double().cpu().numpy() - oref
        err2 += float((d * d).sum())
        ref2 += float((oref * oref).sum())
    eo = math.sqrt(err2 / ref2)
    es = rel_frob(S, S_o)
    print(f"decode: o {eo:.3e}, S {es:.3e}")
    assert eo <= 1e-4 and es <= 1e-4, (eo, es)


# ------------------------------------------------------------------------------ failure detection
def test_bounded_wait_reports_timeout(efla, cuda):
    """A device wait that nothing completes gives up after its bound and is reported on the host;
    the context stays usable afterwards."""
    ws = efla.new_workspace(1, 1, 64, 128, 128)
    efla.efla_selftest_wait_timeout(ws, limit_ns=2_000_000)
    assert efla.efla_workspace_status(ws, clear=True) == efla.EFLA_ERR_TIMEOUT
    assert efla.efla_workspace_status(ws) == efla.EFLA_OK
    w = W["lm1p3b_bf16"].replace(B=1, H=1, T=64)
    inp = workloads.make_chunk_inputs(w)
    d = to_dev(inp, cuda)
    o, ST = efla.efla_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], None, workspace=ws)
    o_ref, ST_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], None)
    assert rel_frob(o, o_ref) <= 2e-2 and efla.efla_workspace_status(ws) == efla.EFLA_OK
