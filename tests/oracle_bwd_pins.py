"""Checks that pin the oracle's backward pass to facts that do not come from it.

Each pin takes a loaded oracle library and raises AssertionError on disagreement, so that
test_oracle_bwd.py can run the same suite on copies of the oracle with a planted mistake.

References, none of which re-types the reverse sweep:
  * central finite differences of the oracle's own forward pass (itself pinned by
    oracle_pins.py to the ZOH solution of the pages' ODE, Sections 2, 3.1-3.4): for a loss
    L = sum(dO * o) + sum(dS_T * S_T), the directional derivative of L along a random
    direction of every input must equal the inner product of that direction with the
    returned gradient;
  * the same finite differences, element by element, on a tiny case;
  * the gate's derivatives by finite differences of the gate itself, and the limit
    d alpha / d lambda -> -beta^2 / 2 as lambda -> 0 (from alpha = beta - beta^2 lambda / 2 + ...);
  * a second algorithm for the same numbers (tests/bwd_mirror.py: no stored states, each
    earlier state rebuilt from the later one, column slices summed), to 1e-12.
"""
from __future__ import annotations

import numpy as np

import oracle


def _problem(rng, B=1, H=2, T=6, dk=3, dv=4, with_state=True, stiff=False):
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk)) * (3.0 if stiff else 0.7)
    v = rng.standard_normal((B, H, T, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, T)) - (2.0 if stiff else 0.0)))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.5 if with_state else None
    dO = rng.standard_normal((B, H, T, dv))
    dST = rng.standard_normal((B, H, dk, dv)) if with_state else None
    return q, k, v, beta, S0, dO, dST


def _loss(lib, q, k, v, beta, S0, dO, dST, mode):
    o, ST = oracle.fwd(q, k, v, beta, S0, mode=mode, threads=1, lib=lib)
    L = float(np.sum(dO * o))
    if dST is not None:
        L += float(np.sum(dST * ST))
    return L


def _directional_check(lib, mode, stiff=False, seed=0, h=1e-6, tol=1e-7):
    rng = np.random.default_rng(seed)
    q, k, v, beta, S0, dO, dST = _problem(rng, stiff=stiff)
    grads = oracle.bwd(q, k, v, beta, dO, S0=S0, dS_T=dST, mode=mode, threads=1, lib=lib)
    names = ["q", "k", "v", "beta", "S0"]
    base = [q, k, v, beta, S0]
    for idx, (name, g) in enumerate(zip(names, grads)):
        d = rng.standard_normal(base[idx].shape)
        plus = [x.copy() if x is not None else None for x in base]
        minus = [x.copy() if x is not None else None for x in base]
        plus[idx] = base[idx] + h * d
        minus[idx] = base[idx] - h * d
        fd = (_loss(lib, *plus, dO, dST, mode) - _loss(lib, *minus, dO, dST, mode)) / (2 * h)
        an = float(np.sum(g * d))
        scale = max(1.0, abs(fd))
        assert abs(fd - an) <= tol * scale, (
            f"{name}: finite difference {fd!r} vs reverse sweep {an!r} (mode {mode}, stiff {stiff})")


def pin_bwd_directional_exact(lib):
    _directional_check(lib, oracle.EXACT, seed=1)


def pin_bwd_directional_stiff(lib):
    """beta*lambda up to ~50: the key direction is all but overwritten, dbeta ~ e^{-beta lambda}."""
    _directional_check(lib, oracle.EXACT, stiff=True, seed=2)


def pin_bwd_directional_euler(lib):
    _directional_check(lib, oracle.EULER, seed=3)


def pin_bwd_elementwise(lib):
    """Every element of every gradient on a tiny case (B1 H1 T3 d2) by central differences."""
    rng = np.random.default_rng(4)
    q, k, v, beta, S0, dO, dST = _problem(rng, B=1, H=1, T=3, dk=2, dv=2)
    grads = oracle.bwd(q, k, v, beta, dO, S0=S0, dS_T=dST, threads=1, lib=lib)
    base = [q, k, v, beta, S0]
    h = 1e-6
    for idx, g in enumerate(grads):
        x = base[idx]
        for pos in np.ndindex(x.shape):
            plus = [y.copy() for y in base]
            minus = [y.copy() for y in base]
            plus[idx][pos] += h
            minus[idx][pos] -= h
            fd = (_loss(lib, *plus, dO, dST, oracle.EXACT) - _loss(lib, *minus, dO, dST, oracle.EXACT)) / (2 * h)
            assert abs(fd - g[pos]) <= 1e-7 * max(1.0, abs(fd)), (idx, pos, fd, g[pos])


def pin_bwd_zero_state_and_no_final_gradient(lib):
    """Without S0 and dS_T the gradients equal those of a zero S0 and a zero dS_T."""
    rng = np.random.default_rng(5)
    q, k, v, beta, _, dO, _ = _problem(rng, with_state=False)
    a = oracle.bwd(q, k, v, beta, dO, threads=1, lib=lib)
    z0 = np.zeros(q.shape[:2] + (q.shape[-1], v.shape[-1]))
    b = oracle.bwd(q, k, v, beta, dO, S0=z0, dS_T=z0, threads=1, lib=lib)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def pin_gate_derivatives(lib):
    """d alpha / d lambda against finite differences of alpha, on both sides of the series
    switch at beta*lambda = 1e-3, and its lambda -> 0 limit."""
    for beta in (0.05, 0.7, 3.0):
        for x in (1e-9, 1e-5, 5e-4, 9.99e-4, 1.001e-3, 2e-3, 0.1, 1.0, 7.0, 40.0):
            lam = x / beta
            h = 1e-4 / beta     # alpha is analytic in lambda (also across 0): a fixed step
            fd = (oracle.alpha(beta, lam + h, lib) - oracle.alpha(beta, lam - h, lib)) / (2 * h)
            an = oracle.dalpha_dlambda(beta, lam, lib)
            assert abs(fd - an) <= 1e-6 * max(abs(an), beta * beta * 1e-3), (beta, x, fd, an)
        assert abs(oracle.dalpha_dlambda(beta, 1e-14, lib) + 0.5 * beta * beta) <= 1e-12 * beta * beta


def pin_bwd_state_reversal(lib):
    """The reverse sweep the CUDA kernel uses (residuals stored, earlier states rebuilt from
    later ones, column slices summed; tests/bwd_mirror.py) gives the oracle's gradients to
    1e-12, with and without slicing, in both modes."""
    from bwd_mirror import stream_bwd
    rng = np.random.default_rng(6)
    for mode, cols in ((oracle.EXACT, None), (oracle.EXACT, 2), (oracle.EULER, 3)):
        q, k, v, beta, S0, dO, dST = _problem(rng, B=1, H=2, T=9, dk=4, dv=6)
        got = oracle.bwd(q, k, v, beta, dO, S0=S0, dS_T=dST, mode=mode, threads=1, lib=lib)
        for h in range(2):
            ref = stream_bwd(q[0, h], k[0, h], v[0, h], beta[0, h], dO[0, h], S0[0, h], dST[0, h],
                             euler=(mode == oracle.EULER), slice_cols=cols)
            for x, y in zip((g[0, h] for g in got), ref):
                assert np.allclose(x, y, rtol=1e-12, atol=1e-12), (mode, cols, h)


def pin_bwd_chunkwise_form(lib):
    """The chunkwise (UT-form) reverse mode, derived independently (tests/chunk_bwd_mirror.py),
    equals the oracle's token-by-token reverse sweep to 1e-10, for several chunk lengths
    including ragged tails, stiff keys and the Euler rule."""
    from chunk_bwd_mirror import chunk_bwd_mirror
    for (mode, stiff, C, T, seed) in ((oracle.EXACT, False, 4, 11, 31), (oracle.EXACT, True, 8, 20, 32),
                                      (oracle.EULER, False, 5, 13, 33), (oracle.EXACT, False, 64, 70, 34)):
        rng = np.random.default_rng(seed)
        q, k, v, beta, S0, dO, dST = _problem(rng, B=1, H=2, T=T, dk=4, dv=3, stiff=stiff)
        ref = oracle.bwd(q, k, v, beta, dO, S0, dST, mode=mode, threads=1, lib=lib)
        got = chunk_bwd_mirror(q, k, v, beta, dO, S0, dST, C=C, euler=(mode == oracle.EULER))
        for name, a, b in zip(("dq", "dk", "dv", "dbeta", "dS0"), got, ref):
            e = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)
            assert e <= 1e-10, (mode, stiff, C, name, e)


ALL_PINS = [pin_bwd_directional_exact, pin_bwd_directional_stiff, pin_bwd_directional_euler,
            pin_bwd_elementwise, pin_bwd_zero_state_and_no_final_gradient, pin_gate_derivatives,
            pin_bwd_state_reversal, pin_bwd_chunkwise_form]
