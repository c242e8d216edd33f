"""Chunkwise (UT-transform) form of the EFLA forward in fp64 numpy, for tests only.

An independent restatement of the chunk algebra (Exact Flow Linear Attention, Section 3.3:
tokens stacked into matrices, a lower-triangular causal mask, the UT transform).  Inside a
chunk of n tokens with entering state S (row convention, d_k x d_v):

    delta_r = alpha_r (v_r - S_{r-1}^T k_r),   S_r = S_{r-1} + k_r delta_r^T
 => (I + A) Delta = diag(alpha) (V - K S),      A = strict_tril(diag(alpha) K K^T)
 => Delta = U - W S with T = (I + A)^{-1} diag(alpha), W = T K, U = T V
    O = Q S + (Q K^T masked, diagonal included) Delta,   S <- S + K^T Delta

The sequential oracle and this block form are two different algorithms for the same
numbers; agreement to 1e-12 pins the oracle's time indexing and read-out convention.
The tests also use it to inspect intermediates (alpha, T, W, U).
"""
from __future__ import annotations

import numpy as np


def gate(k: np.ndarray, beta: np.ndarray) -> np.ndarray:
    lam = np.sum(k * k, axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        a = -np.expm1(-beta * lam) / lam
    return np.where(lam == 0.0, beta, a)


def chunk_intermediates(K, V, beta):
    """alpha, T, W, U of one chunk (K [n, dk], V [n, dv], beta [n])."""
    n = K.shape[0]
    a = gate(K, beta)
    A = np.tril(a[:, None] * (K @ K.T), -1)
    Tm = np.linalg.solve(np.eye(n) + A, np.diag(a))
    return a, Tm, Tm @ K, Tm @ V


def chunk_fwd_mirror(q, k, v, beta, S0, C: int):
    q, k, v, beta = (np.asarray(x, np.float64) for x in (q, k, v, beta))
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, T, dv))
    ST = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[b, h], np.float64)
            for c0 in range(0, T, C):
                sl = slice(c0, min(T, c0 + C))
                Q, K, V = q[b, h, sl], k[b, h, sl], v[b, h, sl]
                _, _, W, U = chunk_intermediates(K, V, beta[b, h, sl])
                Delta = U - W @ S
                P = np.tril(Q @ K.T)
                o[b, h, sl] = Q @ S + P @ Delta
                S = S + K.T @ Delta
            ST[b, h] = S
    return o, ST


def chunk_fwd_mirror_gated(q, k, v, beta, g, S0, C: int):
    """The same chunk algebra with a per-token log-decay g (the gated flow).

    Inside a chunk, with G_r = g_0 + ... + g_r and Gam_r = e^{G_r} (cumulative decay from
    the chunk's entry state), the gated writes delta_r = abar_r v_r - alpha_r e^{g_r}
    S_{r-1}^T k_r and S_r = e^{g_r} S_{r-1} + k_r delta_r^T give
        (I + A) Delta = diag(abar) V - diag(alpha Gam) K S,
        A[r, s] = alpha_r (Gam_r / Gam_s) k_r . k_s   (s < r),
        O = diag(Gam) Q S + (Q K^T (.) D, lower incl. diagonal) Delta,  D[r, s] = Gam_r / Gam_s,
        S <- Gam_last S + K^T diag(Gam_last / Gam) Delta.
    alpha = beta phi1(beta lambda), abar = beta phi1(beta lambda - g), phi1(x) = (1 - e^{-x})/x.
    """
    q, k, v, beta, g = (np.asarray(x, np.float64) for x in (q, k, v, beta, g))
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, T, dv))
    ST = np.zeros((B, H, dk, dv))

    def phi1(x):
        with np.errstate(divide="ignore", invalid="ignore"):
            r = -np.expm1(-x) / x
        return np.where(x == 0.0, 1.0, r)

    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[b, h], np.float64)
            for c0 in range(0, T, C):
                sl = slice(c0, min(T, c0 + C))
                Q, K, V, bt, gg = q[b, h, sl], k[b, h, sl], v[b, h, sl], beta[b, h, sl], g[b, h, sl]
                n = K.shape[0]
                lam = np.sum(K * K, axis=1)
                a = bt * phi1(bt * lam)
                ab = bt * phi1(bt * lam - gg)
                Gc = np.cumsum(gg)
                Dm = np.exp(Gc[:, None] - Gc[None, :])
                A = np.tril(a[:, None] * Dm * (K @ K.T), -1)
                R = ab[:, None] * V - (a * np.exp(Gc))[:, None] * (K @ S)
                Delta = np.linalg.solve(np.eye(n) + A, R)
                P = np.tril((Q @ K.T) * Dm)
                o[b, h, sl] = np.exp(Gc)[:, None] * (Q @ S) + P @ Delta
                S = np.exp(Gc[-1]) * S + K.T @ (np.exp(Gc[-1] - Gc)[:, None] * Delta)
            ST[b, h] = S
    return o, ST
