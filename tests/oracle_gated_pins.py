"""Pins of the oracle's gated flow (efla_oracle_fwd_gated) to facts other than its own code.

The pages give Gated EFLA only by name (Section 3.4) and title (App. F), so the reading is
the oracle's own: a per-token log-decay g added to the zero-order-hold ODE of each token,
    dS/dtau = g S - beta (k k^T S - k v^T),   tau in [0, 1]   (row convention).
Reference values come from:
  * the dense matrix exponential of the whole generator g I - beta k k^T and
    Gauss-Legendre quadrature of the input integral (no rank-1 collapse used);
  * g = 0, which must give the ungated exact flow (itself pinned in oracle_pins.py);
  * beta = 0, a pure decay S_t = e^{g_t} S_{t-1};
  * the small-step limit: with beta and g both scaled by eps, one gated step differs from
    one explicit Euler step of the ODE by O(eps^2);
  * the scalar ODE along a unit key and the pure decay on its orthogonal complement;
  * the Euler mode (the gated delta rule): the ungated Euler step applied to e^g S;
  * the gated chunkwise form (tests/chunk_mirror.py), written independently.
"""
from __future__ import annotations

import math

import numpy as np

import oracle
from oracle_pins import expm, rel, unit


def gated_one_stream(lib, q, k, v, beta, g, S0, mode=oracle.EXACT):
    T, dk = k.shape
    dv = v.shape[1]
    o, ST = oracle.fwd_gated(q[None, None], k[None, None], v[None, None],
                             np.asarray(beta, np.float64).reshape(1, 1, T),
                             np.asarray(g, np.float64).reshape(1, 1, T),
                             None if S0 is None else S0[None, None], mode=mode, threads=1, lib=lib)
    return o[0, 0], ST[0, 0]


def gated_zoh_flow(S0, k, v, beta, g, panels=8, nodes=24):
    """S(1) for dS/dtau = M S + beta k v^T, M = g I - beta k k^T, by dense expm and quadrature."""
    M = g * np.eye(len(k)) - beta * np.outer(k, k)
    S = expm(M) @ S0
    x, w = np.polynomial.legendre.leggauss(nodes)
    b = beta * np.outer(k, v)
    edges = np.linspace(0.0, 1.0, panels + 1)
    acc = np.zeros_like(S0)
    for lo, hi in zip(edges[:-1], edges[1:]):
        half = 0.5 * (hi - lo)
        for xi, wi in zip(x, w):
            tau = lo + half * (xi + 1.0)
            acc += half * wi * (expm((1.0 - tau) * M) @ b)
    return S + acc


def pin_gated_zoh_matrix_exponential(lib):
    """One gated step equals the dense ZOH solution of the gated ODE to 1e-12."""
    rng = np.random.default_rng(2201)
    for (dk, dv) in ((2, 2), (3, 3), (4, 4), (3, 2)):
        for g in (0.0, -1e-3, -0.4, -3.0, 0.2):
            for bl in (1e-6, 1e-2, 0.7, 5.0, 40.0):
                beta = float(rng.uniform(0.05, 1.5))
                k = math.sqrt(bl / beta) * unit(rng, dk)
                S0 = rng.standard_normal((dk, dv))
                v = rng.standard_normal(dv)
                q = rng.standard_normal(dk)
                o, S1 = gated_one_stream(lib, q[None], k[None], v[None], [beta], [g], S0)
                Sref = gated_zoh_flow(S0, k, v, beta, g)
                assert rel(S1, Sref) <= 1e-12, (dk, dv, g, bl, rel(S1, Sref))
                assert rel(o[0], Sref.T @ q) <= 1e-12


def pin_gated_sequence(lib):
    """T gated tokens compose the per-token gated flows in order."""
    rng = np.random.default_rng(2202)
    dk, dv, T = 3, 2, 6
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk)) * rng.uniform(0.2, 3.0, (T, 1))
    v = rng.standard_normal((T, dv))
    beta = rng.uniform(0.1, 1.0, T)
    g = -rng.uniform(0.0, 1.0, T)
    S0 = rng.standard_normal((dk, dv))
    o, ST = gated_one_stream(lib, q, k, v, beta, g, S0)
    S = S0.copy()
    for t in range(T):
        S = gated_zoh_flow(S, k[t], v[t], beta[t], g[t])
        assert rel(o[t], S.T @ q[t]) <= 1e-12, t
    assert rel(ST, S) <= 1e-12


def pin_gated_zero_decay_is_exact_flow(lib):
    """g = 0 gives the ungated exact flow (and, in Euler mode, the ungated delta rule)."""
    rng = np.random.default_rng(2203)
    B, H, T, dk, dv = 1, 2, 23, 5, 4
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk)) * rng.uniform(0.1, 5.0, (B, H, T, 1))
    v = rng.standard_normal((B, H, T, dv))
    beta = rng.uniform(0, 1.5, (B, H, T))
    S0 = rng.standard_normal((B, H, dk, dv))
    for mode in (oracle.EXACT, oracle.EULER):
        o, ST = oracle.fwd(q, k, v, beta, S0, mode=mode, threads=1, lib=lib)
        og, STg = oracle.fwd_gated(q, k, v, beta, np.zeros((B, H, T)), S0, mode=mode, threads=1, lib=lib)
        assert rel(og, o) <= 1e-14 and rel(STg, ST) <= 1e-14, mode


def pin_gated_pure_decay(lib):
    """beta = 0: nothing is written and S_t = e^{g_t} S_{t-1}; o_t = S_t^T q_t."""
    rng = np.random.default_rng(2204)
    dk, dv, T = 4, 3, 9
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    g = -rng.uniform(0.0, 2.0, T)
    S0 = rng.standard_normal((dk, dv))
    o, ST = gated_one_stream(lib, q, k, v, np.zeros(T), g, S0)
    for t in range(T):
        St = math.exp(float(np.sum(g[:t + 1]))) * S0
        assert rel(o[t], St.T @ q[t]) <= 1e-14, t
    assert rel(ST, math.exp(float(np.sum(g))) * S0) <= 1e-14


def pin_gated_small_step_limit(lib):
    """With beta and g scaled by eps, a gated step minus one explicit Euler step of the gated
    ODE shrinks like eps^2 (ratio 4 per halving)."""
    rng = np.random.default_rng(2205)
    dk, dv = 4, 3
    S0 = rng.standard_normal((dk, dv))
    k = 1.7 * unit(rng, dk)
    v = rng.standard_normal(dv)
    q = rng.standard_normal(dk)
    beta0, g0 = 0.8, -0.6
    errs = []
    for eps in (1e-2, 5e-3, 2.5e-3, 1.25e-3):
        beta, g = eps * beta0, eps * g0
        _, S1 = gated_one_stream(lib, q[None], k[None], v[None], [beta], [g], S0)
        Seul = S0 + g * S0 - beta * np.outer(k, k @ S0 - v)
        errs.append(np.linalg.norm(S1 - Seul))
    ratios = [errs[i] / errs[i + 1] for i in range(len(errs) - 1)]
    assert all(3.9 <= r <= 4.1 for r in ratios), ratios


def pin_gated_key_direction(lib):
    """Along a unit key the ODE is scalar: k^T S(1) = e^{g - beta} k^T S0 + beta (1 - e^{g - beta}) / (beta - g) v^T;
    the orthogonal complement only decays: (I - k k^T) S(1) = e^g (I - k k^T) S0."""
    rng = np.random.default_rng(2206)
    for dk, dv in ((4, 4), (5, 3)):
        for g in (-0.01, -0.7, -2.5):
            u = unit(rng, dk)
            S0 = rng.standard_normal((dk, dv))
            v = rng.standard_normal(dv)
            q = rng.standard_normal(dk)
            beta = float(rng.uniform(0.1, 2.0))
            _, S1 = gated_one_stream(lib, q[None], u[None], v[None], [beta], [g], S0)
            c = g - beta
            along = math.exp(c) * (u @ S0) + beta * (1.0 - math.exp(c)) / (beta - g) * v
            assert rel(u @ S1, along) <= 1e-13, (g, rel(u @ S1, along))
            Pp = np.eye(dk) - np.outer(u, u)
            assert rel(Pp @ S1, math.exp(g) * (Pp @ S0)) <= 1e-13


def pin_gated_euler_mode_is_decay_then_delta_rule(lib):
    """Euler mode (the gated delta rule): the ungated delta-rule step applied to e^g S."""
    rng = np.random.default_rng(2207)
    dk, dv, T = 4, 3, 8
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    beta = rng.uniform(0.0, 0.5, T)
    g = -rng.uniform(0.0, 1.0, T)
    S0 = rng.standard_normal((dk, dv))
    o, ST = gated_one_stream(lib, q, k, v, beta, g, S0, mode=oracle.EULER)
    S = S0.copy()
    from oracle_pins import one_stream
    for t in range(T):
        ot, S = one_stream(lib, q[t:t + 1], k[t:t + 1], v[t:t + 1], beta[t:t + 1], math.exp(g[t]) * S,
                           oracle.EULER)
        assert rel(o[t], ot[0]) <= 1e-14, t
    assert rel(ST, S) <= 1e-14


def pin_gated_chunk_identity(lib):
    """The gated chunkwise form, written independently, equals the sequential gated oracle to 1e-12."""
    from chunk_mirror import chunk_fwd_mirror_gated
    rng = np.random.default_rng(2208)
    for (B, H, T, dk, dv, C, s0) in ((1, 2, 40, 8, 6, 16, True), (2, 1, 37, 5, 7, 8, False),
                                     (1, 1, 64, 16, 16, 64, True), (1, 1, 5, 4, 4, 16, True)):
        q = rng.standard_normal((B, H, T, dk))
        k = rng.standard_normal((B, H, T, dk)) * rng.uniform(0.1, 3.0, (B, H, T, 1))
        v = rng.standard_normal((B, H, T, dv))
        beta = rng.uniform(0.0, 1.0, (B, H, T))
        g = -rng.uniform(0.0, 0.5, (B, H, T))
        S0 = rng.standard_normal((B, H, dk, dv)) if s0 else None
        o, ST = oracle.fwd_gated(q, k, v, beta, g, S0, threads=1, lib=lib)
        om, STm = chunk_fwd_mirror_gated(q, k, v, beta, g, S0, C)
        assert rel(o, om) <= 1e-12 and rel(ST, STm) <= 1e-12, (T, C, rel(o, om), rel(ST, STm))


def pin_gated_decode_step_is_forward(lib):
    """A gated decode step is the gated forward over one token."""
    rng = np.random.default_rng(2209)
    N, H, dk, dv, steps = 2, 2, 4, 3, 5
    S = rng.standard_normal((N, H, dk, dv))
    qs, ks = rng.standard_normal((2, steps, N, H, dk))
    vs = rng.standard_normal((steps, N, H, dv))
    bs = rng.uniform(0, 1, (steps, N, H))
    gs = -rng.uniform(0, 1, (steps, N, H))
    mv = lambda x: np.moveaxis(x, 0, 2)
    o_f, S_f = oracle.fwd_gated(mv(qs), mv(ks), mv(vs), mv(bs), mv(gs), S, threads=1, lib=lib)
    Sd = S.copy()
    for s in range(steps):
        o, Sd = oracle.step_gated(qs[s], ks[s], vs[s], bs[s], gs[s], Sd, threads=1, lib=lib)
        assert rel(o, o_f[:, :, s]) <= 1e-15
    assert rel(Sd, S_f) <= 1e-15


GATED_PINS = [pin_gated_zoh_matrix_exponential, pin_gated_sequence, pin_gated_zero_decay_is_exact_flow,
              pin_gated_pure_decay, pin_gated_small_step_limit, pin_gated_key_direction,
              pin_gated_euler_mode_is_decay_then_delta_rule, pin_gated_chunk_identity,
              pin_gated_decode_step_is_forward]
