"""Seeded synthetic inputs for the EFLA chunked forward and the decode step.

This module only draws inputs: shapes, value distributions, dtype casts. It holds none
of the method's arithmetic, so the CUDA path and the fp64 oracle can both take their
inputs from it without sharing any of the computation they are compared on.

Layouts (row-major, head-major):
    q, k : [B, H, T, d_k]      v : [B, H, T, d_v]      beta : [B, H, T]
    S0   : [B, H, d_k, d_v] float32 (or None: zero initial state)

Distributions follow the workloads the Exact Flow Linear Attention summary page
describes (1.3B-scale LM layers, Section 4.1 / App. C; "corrupted and high-energy
inputs", Section 4.3).  The standard deviation is the second argument of N(mu, sigma).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

__all__ = ["ChunkWorkload", "DecodeWorkload", "CHUNK_WORKLOADS", "DECODE_WORKLOAD",
           "make_chunk_inputs", "make_decode_state", "make_decode_steps", "make_log_decay",
           "make_varlen_inputs", "varlen_lengths"]


@dataclasses.dataclass(frozen=True)
class ChunkWorkload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    dtype: torch.dtype
    dist: str                 # "gauss" | "lognorm_dir" | "stiff"
    s0_std: Optional[float]   # None: S0 is absent (zero state)
    seed: int

    def replace(self, **kw) -> "ChunkWorkload":
        return dataclasses.replace(self, **kw)

    @property
    def tokens(self) -> int:
        """Tokens per call: B*T (each token spans all H heads)."""
        return self.B * self.T


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    N: int
    H: int
    dk: int
    dv: int
    steps: int
    s_std: float
    seed: int

    def replace(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


# Seeds are 42 + workload index (the pages' training runs used seed 42, App. C).
CHUNK_WORKLOADS = {
    # tiny fp32 case, unnormalised keys (norm ~ 8)
    "tiny_fp32": ChunkWorkload("tiny_fp32", 1, 2, 256, 64, 64, 64, torch.float32,
                               "gauss", None, 43),
    # 1.3B-layer shape: bf16 in, fp32 state
    "lm1p3b_bf16": ChunkWorkload("lm1p3b_bf16", 4, 16, 2048, 128, 128, 64, torch.bfloat16,
                                 "lognorm_dir", None, 44),
    # long context with a given initial state
    "longctx_bf16": ChunkWorkload("longctx_bf16", 1, 16, 32768, 128, 128, 64, torch.bfloat16,
                                  "lognorm_dir", 0.02, 45),
    # stiff / high-energy keys with 1 % corrupted tokens
    "stiff_bf16": ChunkWorkload("stiff_bf16", 2, 16, 4096, 128, 128, 64, torch.bfloat16,
                                "stiff", None, 46),
}

DECODE_WORKLOAD = DecodeWorkload("decode_fp32", 256, 16, 128, 128, 1000, 0.1, 47)


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def make_chunk_inputs(w: ChunkWorkload, with_mask: bool = False) -> dict:
    """Draw q, k, v, beta (in w.dtype) and S0 (float32 or None) on the CPU.

    The draw order is fixed, so the same workload always gives the same tensors.  With
    with_mask, the dict also holds "corrupt" [B, T] bool: the (b, t) tokens replaced by
    high-energy noise (the "stiff" distribution; all False for the others).
    """
    g = torch.Generator().manual_seed(w.seed)
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    f32 = torch.float32
    if w.dist == "gauss":
        q = torch.randn(B, H, T, dk, generator=g, dtype=f32)
        k = torch.randn(B, H, T, dk, generator=g, dtype=f32)
        v = torch.randn(B, H, T, dv, generator=g, dtype=f32)
        beta = torch.sigmoid(torch.randn(B, H, T, generator=g, dtype=f32))
    elif w.dist == "lognorm_dir":
        # direction uniform on the sphere, norm ~ LogNormal(0, 0.5)
        q = _unit_rows(torch.randn(B, H, T, dk, generator=g, dtype=f32))
        q = q * torch.exp(0.5 * torch.randn(B, H, T, 1, generator=g, dtype=f32))
        k = _unit_rows(torch.randn(B, H, T, dk, generator=g, dtype=f32))
        k = k * torch.exp(0.5 * torch.randn(B, H, T, 1, generator=g, dtype=f32))
        v = torch.randn(B, H, T, dv, generator=g, dtype=f32)
        beta = torch.sigmoid(torch.randn(B, H, T, generator=g, dtype=f32))
    elif w.dist == "stiff":
        q = torch.randn(B, H, T, dk, generator=g, dtype=f32)
        scales = torch.tensor([1.0, 10.0, 100.0], dtype=f32)
        s = scales[torch.randint(0, 3, (B, 1, T, 1), generator=g)]       # per (b, t), all heads
        k = torch.randn(B, H, T, dk, generator=g, dtype=f32) * s
        v = torch.randn(B, H, T, dv, generator=g, dtype=f32)
        beta = torch.sigmoid(2.0 + torch.randn(B, H, T, generator=g, dtype=f32))
        corrupt = torch.rand(B, 1, T, 1, generator=g) < 0.01             # 1 % of (b, t) tokens
        cq = 100.0 * torch.randn(B, H, T, dk, generator=g, dtype=f32)
        ck = 100.0 * torch.randn(B, H, T, dk, generator=g, dtype=f32)
        cv = 100.0 * torch.randn(B, H, T, dv, generator=g, dtype=f32)
        q = torch.where(corrupt, cq, q)
        k = torch.where(corrupt, ck, k)
        v = torch.where(corrupt, cv, v)
    else:
        raise ValueError(f"unknown distribution {w.dist!r}")
    if w.dist != "stiff":
        corrupt = torch.zeros(B, 1, T, 1, dtype=torch.bool)
    S0 = None
    if w.s0_std is not None:
        S0 = w.s0_std * torch.randn(B, H, dk, dv, generator=g, dtype=f32)
    out = {
        "q": q.to(w.dtype).contiguous(),
        "k": k.to(w.dtype).contiguous(),
        "v": v.to(w.dtype).contiguous(),
        "beta": beta.to(w.dtype).contiguous(),
        "S0": S0,
    }
    if with_mask:
        out["corrupt"] = corrupt[:, 0, :, 0].clone()
    return out


def varlen_lengths(n: int, total: int, seed: int, min_len: int = 1) -> list:
    """n sequence lengths summing to `total`, a log-uniform mix (short and long sequences
    together, as in packed training batches); at least min_len each."""
    g = torch.Generator().manual_seed(seed)
    w = torch.exp(torch.rand(n, generator=g) * 4.0)            # weights spread over e^0 .. e^4
    raw = (w / w.sum() * (total - n * min_len)).floor().to(torch.int64) + min_len
    raw[-1] += total - int(raw.sum())
    return [int(x) for x in raw]


def make_varlen_inputs(w: ChunkWorkload, lengths, with_g: bool = False) -> dict:
    """A packed batch: sequence n drawn as a one-stream workload of w's distribution with
    length lengths[n], all heads, packed head-major along the token axis.

    Returns q, k [H, total_T, d_k], v [H, total_T, d_v], beta [H, total_T] (w.dtype),
    S0 [N, H, d_k, d_v] float32 or None, cu (list of N + 1 offsets) and, with with_g,
    g [H, total_T] float32 (make_log_decay).
    """
    parts = [make_chunk_inputs(w.replace(B=1, T=int(L), seed=w.seed + 31 * n)) for n, L in enumerate(lengths)]
    cat = lambda key: torch.cat([p[key][0] for p in parts], dim=1).contiguous()
    out = {"q": cat("q"), "k": cat("k"), "v": cat("v"), "beta": cat("beta")}
    out["S0"] = None if w.s0_std is None else torch.cat([p["S0"] for p in parts], dim=0).contiguous()
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    out["cu"] = cu
    if with_g:
        out["g"] = make_log_decay((w.H, cu[-1]), w.seed + 7)
    return out


def make_log_decay(shape, seed: int, device="cpu") -> torch.Tensor:
    """Per-token log-decay g of the gated flow, float32: g = -softplus(N(-3, 1.5)).

    The pages give no gated workload; this draw makes most per-token decays e^g lie in
    (0.9, 1) with a tail down to about 0.3, so a 64-token chunk decays its entry state by
    e^-3 on average and the within-chunk ratios Gam_r / Gam_s span several orders.
    """
    g = torch.Generator(device=device).manual_seed(seed)
    x = -3.0 + 1.5 * torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return -torch.nn.functional.softplus(x)


def make_decode_state(w: DecodeWorkload, device="cpu") -> torch.Tensor:
    """Initial decode state S ~ N(0, s_std) float32, [N, H, d_k, d_v]."""
    g = torch.Generator(device=device).manual_seed(w.seed)
    return w.s_std * torch.randn(w.N, w.H, w.dk, w.dv, generator=g, device=device,
                                 dtype=torch.float32)


def make_decode_steps(w: DecodeWorkload, steps: Optional[int] = None, device="cpu") -> dict:
    """Per-step decode inputs for `steps` consecutive tokens, float32.

    q, v ~ N(0, 1); k ~ N(0, 1) scaled to unit norm; beta = sigmoid(N(0, 1)).
    Shapes: q, k [steps, N, H, d_k]; v [steps, N, H, d_v]; beta [steps, N, H].
    On a CUDA device the draw uses torch's device generator (1000 full-size steps are
    1.5 G normals, a minute of host time); the values then differ from a CPU draw, so
    every consumer must take the same tensors.
    """
    steps = w.steps if steps is None else steps
    g = torch.Generator(device=device).manual_seed(w.seed + 1)
    shp = (steps, w.N, w.H)
    f32 = torch.float32
    q = torch.randn(*shp, w.dk, generator=g, device=device, dtype=f32)
    k = _unit_rows(torch.randn(*shp, w.dk, generator=g, device=device, dtype=f32))
    v = torch.randn(*shp, w.dv, generator=g, device=device, dtype=f32)
    beta = torch.sigmoid(torch.randn(*shp, generator=g, device=device, dtype=f32))
    return {"q": q, "k": k, "v": v, "beta": beta}


def make_cotangents(w: ChunkWorkload, with_state_grad: bool = True) -> dict:
    """The backward pass's seeded inputs: dO [B,H,T,dv] ~ N(0, 1) in w.dtype and
    dS_T [B,H,dk,dv] ~ N(0, 1) float32 (or None), drawn on the CPU from seed w.seed + 1000."""
    g = torch.Generator().manual_seed(w.seed + 1000)
    dO = torch.randn(w.B, w.H, w.T, w.dv, generator=g, dtype=torch.float32).to(w.dtype).contiguous()
    dST = torch.randn(w.B, w.H, w.dk, w.dv, generator=g, dtype=torch.float32) if with_state_grad else None
    return {"dO": dO, "dS_T": dST}
