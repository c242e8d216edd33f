"""Checks that pin the fp64 oracle to facts fixed by the pages and by mathematics.

Each pin takes a loaded oracle library (ctypes handle) and raises AssertionError when the
oracle disagrees.  They are plain functions so that test_oracle_mutants.py can run the
same suite against copies of the oracle with a planted mistake and show each is caught.

None of these re-types the oracle's update formula.  Reference values come from:
  * a dense matrix exponential (own scaling-and-squaring Taylor, cross-checked against
    scipy.linalg.expm) and Gauss-Legendre quadrature of the input integral: the ZOH
    solution of dS/dtau = -A S + k v^T, A = k k^T (summary page Section 3.1, App. E);
  * explicit Euler / RK4 integration of the same ODE with fine substeps (Section 2: the
    delta rule is one Euler step);
  * the contraction of the key direction by exp(-beta*lambda) and the untouched
    orthogonal complement (Section 3.4);
  * the small beta*lambda limit alpha -> beta (Section 3.4);
  * the scalar (d = 1) solution of the ODE in closed form;
  * a block (chunkwise, UT-transform) formulation written independently in tests
    (Section 3.3), which must agree to rounding.
Row convention throughout: S is d_k x d_v, o_t = S_t^T q_t.
"""
from __future__ import annotations

import math

import numpy as np

import oracle


# ----------------------------------------------------------------------------- helpers
def expm_taylor(M: np.ndarray) -> np.ndarray:
    """exp(M) by scaling and squaring with a degree-24 Taylor polynomial (fp64)."""
    nrm = np.linalg.norm(M, 1)
    s = max(0, int(math.ceil(math.log2(nrm))) + 1) if nrm > 0.5 else 0
    X = M / (2.0 ** s)
    E = np.eye(M.shape[0])
    term = np.eye(M.shape[0])
    for j in range(1, 25):
        term = term @ X / j
        E = E + term
    for _ in range(s):
        E = E @ E
    return E


def expm(M: np.ndarray) -> np.ndarray:
    E = expm_taylor(M)
    try:
        import scipy.linalg
        E2 = scipy.linalg.expm(M)
        scale = max(1.0, np.abs(E2).max())
        assert np.abs(E - E2).max() <= 1e-12 * scale, "Taylor expm disagrees with scipy"
    except ImportError:  # pragma: no cover
        pass
    return E


def zoh_flow(S0, k, v, beta, panels=8, nodes=24):
    """S(beta) for dS/dtau = -A S + k v^T, S(0) = S0, A = k k^T (row convention).

    Integrating factor (App. E): S(beta) = e^{-beta A} S0 + int_0^beta e^{-(beta - tau) A} k v^T dtau,
    the integral by composite Gauss-Legendre quadrature.
    """
    A = np.outer(k, k)
    S = expm(-beta * A) @ S0
    x, w = np.polynomial.legendre.leggauss(nodes)
    b = np.outer(k, v)
    edges = np.linspace(0.0, beta, panels + 1)
    acc = np.zeros_like(S0)
    for lo, hi in zip(edges[:-1], edges[1:]):
        half = 0.5 * (hi - lo)
        for xi, wi in zip(x, w):
            tau = lo + half * (xi + 1.0)
            acc += half * wi * (expm(-(beta - tau) * A) @ b)
    return S + acc


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    d = np.linalg.norm(a - b)
    n = np.linalg.norm(b)
    return d / n if n > 0 else d


def one_stream(lib, q, k, v, beta, S0, mode=oracle.EXACT):
    """Run the oracle on a single (b, h) stream: q, k [T, dk], v [T, dv], beta [T]."""
    T, dk = k.shape
    dv = v.shape[1]
    o, ST = oracle.fwd(q[None, None], k[None, None], v[None, None],
                       np.asarray(beta, np.float64).reshape(1, 1, T),
                       None if S0 is None else S0[None, None], mode=mode, threads=1, lib=lib)
    return o[0, 0], ST[0, 0]


def unit(rng, d):
    x = rng.standard_normal(d)
    return x / np.linalg.norm(x)


# ----------------------------------------------------------------------------- pins
def pin_zoh_matrix_exponential(lib):
    """One step equals S0 e^{-beta A} + int b e^{-(beta - tau) A} dtau to 1e-12 (Sections 3.1-3.2, App. D-E)."""
    rng = np.random.default_rng(1201)
    shapes = [(2, 2), (3, 3), (4, 4), (3, 2), (2, 4)]
    for (dk, dv) in shapes:
        for bl in np.logspace(-6, math.log10(50.0), 7):
            beta = float(rng.uniform(0.05, 1.5))
            lam = bl / beta
            k = math.sqrt(lam) * unit(rng, dk)
            S0 = rng.standard_normal((dk, dv))
            v = rng.standard_normal(dv)
            q = rng.standard_normal(dk)
            o, S1 = one_stream(lib, q[None], k[None], v[None], [beta], S0)
            Sref = zoh_flow(S0, k, v, beta)
            assert rel(S1, Sref) <= 1e-12, (dk, dv, bl, rel(S1, Sref))
            # read-out after the write: o_t = S_t^T q_t
            assert rel(o[0], Sref.T @ q) <= 1e-12, (dk, dv, bl)


def pin_zoh_sequence(lib):
    """T tokens compose the per-token flows in order, each output read from its own S_t."""
    rng = np.random.default_rng(1202)
    dk, dv, T = 3, 2, 7
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk)) * rng.uniform(0.2, 3.0, (T, 1))
    v = rng.standard_normal((T, dv))
    beta = rng.uniform(0.1, 1.0, T)
    S0 = rng.standard_normal((dk, dv))
    o, ST = one_stream(lib, q, k, v, beta, S0)
    S = S0.copy()
    for t in range(T):
        S = zoh_flow(S, k[t], v[t], beta[t])
        assert rel(o[t], S.T @ q[t]) <= 1e-12, t
    assert rel(ST, S) <= 1e-12


def pin_small_step_limit(lib):
    """alpha -> beta as ||k|| -> 0 with 0 <= beta - alpha <= beta^2 lambda / 2; alpha = beta at lambda = 0 (Section 3.4)."""
    for beta in (0.3, 0.9, 2.5):
        assert lib.efla_oracle_alpha(beta, 0.0) == beta
        ulp = math.ulp(beta)
        for eps in (1e-2, 1e-3, 1e-4, 1e-6, 1e-8):
            lam = eps * eps
            a = lib.efla_oracle_alpha(beta, lam)
            gap = beta - a
            # 0 <= beta - alpha <= beta^2 lambda / 2, up to the rounding of alpha itself
            assert -4 * ulp <= gap <= 0.5 * beta * beta * lam + 4 * ulp, (beta, eps, a)
            if eps >= 1e-3:
                # leading terms of the expansion: beta^2 lam / 2 - beta^3 lam^2 / 6
                expect = 0.5 * beta ** 2 * lam - beta ** 3 * lam ** 2 / 6.0
                assert abs(gap - expect) <= 1e-6 * expect, (beta, eps, gap, expect)
    # the state difference to the Euler (delta-rule) step shrinks like beta^2 lambda
    rng = np.random.default_rng(1203)
    dk, dv = 4, 3
    S0 = rng.standard_normal((dk, dv))
    v = rng.standard_normal(dv)
    q = rng.standard_normal(dk)
    u = unit(rng, dk)
    beta = 0.7
    for eps in (1e-1, 1e-2, 1e-3):
        k = eps * u
        _, Se = one_stream(lib, q[None], k[None], v[None], [beta], S0, oracle.EXACT)
        _, Sd = one_stream(lib, q[None], k[None], v[None], [beta], S0, oracle.EULER)
        Seul = S0 - beta * np.outer(k, k @ S0 - v)         # one Euler step of the ODE
        assert rel(Sd, Seul) <= 1e-14
        lam = eps * eps
        r = np.linalg.norm(k @ S0 - v)
        bound = 0.5 * beta * beta * lam * eps * r
        diff = np.linalg.norm(Se - Sd)
        assert diff <= bound * (1 + 1e-5)
        assert diff >= bound * (1 - beta * lam) * (1 - 1e-5)


def pin_euler_convergence(lib):
    """n-substep Euler of the ODE converges to the oracle step at first order; RK4 agrees to 1e-10 (Section 2)."""
    rng = np.random.default_rng(1204)
    dk, dv = 4, 3
    S0 = rng.standard_normal((dk, dv))
    k = 1.3 * unit(rng, dk)
    v = rng.standard_normal(dv)
    q = rng.standard_normal(dk)
    beta = 0.8
    _, S1 = one_stream(lib, q[None], k[None], v[None], [beta], S0)

    def f(S):
        return -np.outer(k, k @ S - v)

    errs = []
    for n in (64, 128, 256, 512, 1024):
        S, h = S0.copy(), beta / n
        for _ in range(n):
            S = S + h * f(S)
        errs.append(np.linalg.norm(S - S1))
    ratios = [errs[i] / errs[i + 1] for i in range(len(errs) - 1)]
    assert all(1.9 <= r <= 2.1 for r in ratios), ratios
    S, n = S0.copy(), 2000
    h = beta / n
    for _ in range(n):
        a1 = f(S); a2 = f(S + 0.5 * h * a1); a3 = f(S + 0.5 * h * a2); a4 = f(S + h * a3)
        S = S + h / 6.0 * (a1 + 2 * a2 + 2 * a3 + a4)
    assert rel(S1, S) <= 1e-10, rel(S1, S)


def pin_contraction(lib):
    """The key direction contracts by exp(-beta lambda); the orthogonal complement is unchanged (Section 3.4)."""
    rng = np.random.default_rng(1205)
    for dk, dv in ((4, 4), (5, 3)):
        for nk in (1.0, 0.3, 2.7):
            u = unit(rng, dk)
            k = nk * u
            S0 = rng.standard_normal((dk, dv))
            v = rng.standard_normal(dv)
            q = rng.standard_normal(dk)
            beta = float(rng.uniform(0.1, 2.0))
            _, S1 = one_stream(lib, q[None], k[None], v[None], [beta], S0)
            lam = nk * nk
            # component along the key direction relaxes toward v / ||k||
            lhs = u @ S1 - v / nk
            rhs = math.exp(-beta * lam) * (u @ S0 - v / nk)
            assert rel(lhs, rhs) <= 1e-12, (nk, rel(lhs, rhs))
            Pp = np.eye(dk) - np.outer(u, u)
            assert rel(Pp @ S1, Pp @ S0) <= 1e-13
            if nk == 1.0:
                assert rel(k @ S1, math.exp(-beta) * (k @ S0) + (1 - math.exp(-beta)) * v) <= 1e-13


def pin_stiff_limit(lib):
    """beta lambda >= 40: alpha = 1/lambda to fp64, so k^T S_t = v^T (the key slot is overwritten)."""
    rng = np.random.default_rng(1206)
    for bl in (40.0, 1e3, 1e6):
        beta = 0.9
        lam = bl / beta
        a = lib.efla_oracle_alpha(beta, lam)
        assert abs(a * lam - 1.0) <= 4e-16
        dk, dv = 4, 3
        k = math.sqrt(lam) * unit(rng, dk)
        S0 = rng.standard_normal((dk, dv))
        v = rng.standard_normal(dv)
        q = rng.standard_normal(dk)
        _, S1 = one_stream(lib, q[None], k[None], v[None], [beta], S0)
        assert rel(k @ S1, v) <= 1e-12, bl


def pin_nonexpansive(lib):
    """With v = 0 and beta >= 0 the spectral norm of S never grows; beta < 0 expands along k (Section 3.4)."""
    rng = np.random.default_rng(1207)
    dk, dv, T = 5, 4, 40
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk)) * rng.uniform(0.1, 4.0, (T, 1))
    v = np.zeros((T, dv))
    beta = rng.uniform(0.0, 3.0, T)
    S = rng.standard_normal((dk, dv))
    for t in range(T):
        _, S1 = one_stream(lib, q[t:t + 1], k[t:t + 1], v[t:t + 1], beta[t:t + 1], S)
        assert np.linalg.norm(S1, 2) <= np.linalg.norm(S, 2) * (1 + 1e-13)
        assert np.linalg.norm(S1) <= np.linalg.norm(S) * (1 + 1e-13)
        S = S1
    u = unit(rng, dk)
    S0 = np.outer(u, rng.standard_normal(dv))
    _, S1 = one_stream(lib, q[:1], 1.5 * u[None], v[:1], [-0.5], S0)
    assert np.linalg.norm(S1) > np.linalg.norm(S0) * 1.5


def pin_scalar_closed_form(lib):
    """d_k = d_v = 1: S_t = e^{-beta k^2} S_{t-1} + (1 - e^{-beta k^2}) v / k, o_t = q S_t."""
    rng = np.random.default_rng(1208)
    T = 12
    q = rng.standard_normal((T, 1))
    k = rng.standard_normal((T, 1)) * 2.0
    v = rng.standard_normal((T, 1))
    beta = rng.uniform(0.05, 2.0, T)
    S0 = np.array([[0.37]])
    o, ST = one_stream(lib, q, k, v, beta, S0)
    s = 0.37
    for t in range(T):
        kk = float(k[t, 0])
        e = math.exp(-beta[t] * kk * kk)
        s = e * s + (1.0 - e) * float(v[t, 0]) / kk
        assert abs(o[t, 0] - float(q[t, 0]) * s) <= 1e-13 * max(1.0, abs(s))
    assert abs(ST[0, 0] - s) <= 1e-13 * max(1.0, abs(s))


def pin_chunk_identity(lib):
    """The chunkwise UT form (Section 3.3), written independently, equals the sequential oracle to 1e-12."""
    from chunk_mirror import chunk_fwd_mirror
    rng = np.random.default_rng(1209)
    for (B, H, T, dk, dv, C, s0) in ((1, 2, 40, 8, 6, 16, True), (2, 1, 37, 5, 7, 8, False),
                                     (1, 1, 64, 16, 16, 64, True), (1, 1, 5, 4, 4, 16, True)):
        q = rng.standard_normal((B, H, T, dk))
        k = rng.standard_normal((B, H, T, dk)) * rng.uniform(0.1, 3.0, (B, H, T, 1))
        v = rng.standard_normal((B, H, T, dv))
        beta = rng.uniform(0.0, 1.0, (B, H, T))
        S0 = rng.standard_normal((B, H, dk, dv)) if s0 else None
        o, ST = oracle.fwd(q, k, v, beta, S0, threads=1, lib=lib)
        om, STm = chunk_fwd_mirror(q, k, v, beta, S0, C)
        assert rel(o, om) <= 1e-12 and rel(ST, STm) <= 1e-12, (T, C, rel(o, om), rel(ST, STm))


def pin_streams_independent(lib):
    """Each (b, h) stream depends only on its own slice, and S0 = None means a zero state."""
    rng = np.random.default_rng(1210)
    B, H, T, dk, dv = 2, 3, 9, 4, 5
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    beta = rng.uniform(0, 1, (B, H, T))
    S0 = rng.standard_normal((B, H, dk, dv))
    o, ST = oracle.fwd(q, k, v, beta, S0, threads=2, lib=lib)
    for b in range(B):
        for h in range(H):
            o1, S1 = one_stream(lib, q[b, h], k[b, h], v[b, h], beta[b, h], S0[b, h])
            assert np.array_equal(o1, o[b, h]) and np.array_equal(S1, ST[b, h])
    oz, STz = oracle.fwd(q, k, v, beta, None, threads=2, lib=lib)
    oz2, STz2 = oracle.fwd(q, k, v, beta, np.zeros_like(S0), threads=2, lib=lib)
    assert np.array_equal(oz, oz2) and np.array_equal(STz, STz2)


def pin_decode_step_is_forward(lib):
    """A decode step is the forward recurrence over one token, state carried in place."""
    rng = np.random.default_rng(1211)
    N, H, dk, dv, steps = 2, 2, 4, 3, 5
    S = rng.standard_normal((N, H, dk, dv))
    qs = rng.standard_normal((steps, N, H, dk))
    ks = rng.standard_normal((steps, N, H, dk))
    vs = rng.standard_normal((steps, N, H, dv))
    bs = rng.uniform(0, 1, (steps, N, H))
    o_f, S_f = oracle.fwd(np.moveaxis(qs, 0, 2), np.moveaxis(ks, 0, 2), np.moveaxis(vs, 0, 2),
                          np.moveaxis(bs, 0, 2), S, threads=1, lib=lib)
    Sd = S.copy()
    for s in range(steps):
        o, Sd = oracle.step(qs[s], ks[s], vs[s], bs[s], Sd, threads=1, lib=lib)
        assert rel(o, o_f[:, :, s]) <= 1e-15
    assert rel(Sd, S_f) <= 1e-15


ALL_PINS = [pin_zoh_matrix_exponential, pin_zoh_sequence, pin_small_step_limit,
            pin_euler_convergence, pin_contraction, pin_stiff_limit, pin_nonexpansive,
            pin_scalar_closed_form, pin_chunk_identity, pin_streams_independent,
            pin_decode_step_is_forward]
