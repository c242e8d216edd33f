"""Shared test helpers: error metric and oracle runs on a subset of streams."""
from __future__ import annotations

import numpy as np
import torch

import oracle


def rel_frob(x, ref) -> float:
    """||x - ref||_F / ||ref||_F over the whole tensor (float64)."""
    x = x.detach().double().cpu().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = ref.detach().double().cpu().numpy() if hasattr(ref, "detach") else np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def oracle_streams(inp: dict, streams):
    """fp64 oracle over the selected (b, h) streams. Returns o [n,T,dv], S_T [n,dk,dv]."""
    q, k, v, beta, S0 = inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"]
    sel = lambda t: torch.stack([t[b, h] for b, h in streams])[None]
    o, ST = oracle.fwd(sel(q), sel(k), sel(v), sel(beta), None if S0 is None else sel(S0))
    return o[0], ST[0]


TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
