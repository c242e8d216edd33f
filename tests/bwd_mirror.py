"""The backward pass as the CUDA kernel organises it, restated in fp64 numpy (tests only).

The oracle keeps every state of a stream and sweeps back over them.  The kernel keeps none:
a forward sweep stores only the residuals r_t = S_{t-1}^T k_t - v_t, and the reverse sweep
rebuilds each earlier state from the later one by adding the rank-1 write back,
S_{t-1} = S_t + alpha_t k_t r_t^T, with the state split into column slices whose partial
row sums (dq, dk, dalpha) are added up afterwards.  Agreement with the oracle to 1e-12
shows that this reorganisation is exact algebra (no inverse of I - alpha k k^T is taken).
"""
from __future__ import annotations

import numpy as np


def _alpha(beta, lam, euler):
    if euler:
        return beta
    if lam == 0.0:
        return beta
    return -np.expm1(-beta * lam) / lam


def _dalpha(beta, lam, euler):
    """(d alpha / d beta, d alpha / d lambda) by the closed forms, with the series near 0."""
    if euler:
        return 1.0, 0.0
    x = beta * lam
    if abs(x) < 1e-3:
        return np.exp(-x), beta * beta * (-0.5 + x / 3.0 - x * x / 8.0 + x ** 3 / 30.0 - x ** 4 / 144.0)
    a = -np.expm1(-x) / lam
    return np.exp(-x), (beta * np.exp(-x) - a) / lam


def stream_bwd(q, k, v, beta, dO, S0=None, dST=None, euler=False, slice_cols=None):
    """One stream: q, k [T, dk], v, dO [T, dv], beta [T].  Returns dq, dk, dv, dbeta, dS0."""
    T, dk = k.shape
    dv_ = v.shape[1]
    cols = slice_cols or dv_
    S = np.zeros((dk, dv_)) if S0 is None else S0.astype(np.float64).copy()
    R = np.empty((T, dv_))
    alphas = np.empty(T)
    for t in range(T):                          # forward sweep: residuals only
        lam = float(k[t] @ k[t])
        alphas[t] = _alpha(beta[t], lam, euler)
        R[t] = S.T @ k[t] - v[t]
        S -= alphas[t] * np.outer(k[t], R[t])
    G = np.zeros((dk, dv_)) if dST is None else dST.astype(np.float64).copy()
    dq = np.zeros((T, dk)); dkk = np.zeros((T, dk)); dvv = np.zeros((T, dv_)); dalpha = np.zeros(T)
    for t in range(T - 1, -1, -1):              # reverse sweep, slice by slice
        a = alphas[t]
        for j0 in range(0, dv_, cols):
            sl = slice(j0, j0 + cols)
            G[:, sl] += np.outer(q[t], dO[t, sl])
            dq[t] += S[:, sl] @ dO[t, sl]
            g = G[:, sl].T @ k[t]
            dvv[t, sl] = a * g
            dalpha[t] -= g @ R[t, sl]
            S[:, sl] += a * np.outer(k[t], R[t, sl])           # S_{t-1}, rebuilt
            dkk[t] -= a * (G[:, sl] @ R[t, sl] + S[:, sl] @ g)
            G[:, sl] -= a * np.outer(k[t], g)
    dbeta = np.empty(T)
    for t in range(T):                          # the gate's share
        lam = float(k[t] @ k[t])
        dadb, dadl = _dalpha(beta[t], lam, euler)
        if lam == 0.0 and not euler:
            dadb, dadl = 1.0, -0.5 * beta[t] * beta[t]
        dbeta[t] = dalpha[t] * dadb
        dkk[t] += dalpha[t] * dadl * 2.0 * k[t]
    return dq, dkk, dvv, dbeta, G
