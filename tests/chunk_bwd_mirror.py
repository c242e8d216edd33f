"""The backward pass through the chunkwise (UT) form, in fp64 numpy (tests only).

Exact Flow Linear Attention, Section 3.3 computes a chunk as dense products; its reverse
mode differentiates those products instead of the token recurrence.  Per chunk, with S the
entering state (row convention) and dS' the gradient of the leaving state:
    forward:  G = K K^T, A = strict_tril(diag(alpha) G), X = (I + A)^{-1}, T = X diag(alpha),
              R = V - K S, Delta = T R, P = tril_incl(Q K^T), O = Q S + P Delta,
              S' = S + K^T Delta
    reverse:  dDelta = P^T dO + K dS'                  dR = T^T dDelta     dV = dR
              dS = dS' + Q^T dO - K^T dR               (carried to the previous chunk)
              dP = tril_incl(dO Delta^T)               dQ = dO S^T + dP K
              dT = dDelta R^T                          dX = dT diag(alpha)
              dalpha_j += sum_i dT_ij X_ij             dA = strict_tril(-X^T dX X^T)
              dalpha_r += sum_s dA_rs G_rs             dG = diag(alpha) dA
              dK = Delta dS'^T + dP^T Q - dR S^T + (dG + dG^T) K
    gate:     dbeta = dalpha dalpha/dbeta,  dK_r += dalpha_r dalpha/dlambda 2 k_r.
The chain of chunks runs backwards carrying dS (the column slices of dS are independent, as
the forward's state columns are); every other line is local to its chunk once the chunk's
entering state S and leaving-state gradient dS' are known.  Agreement with the pinned oracle
backward to 1e-10 pins this derivation.
"""
from __future__ import annotations

import numpy as np

from bwd_mirror import _alpha, _dalpha


def chunk_bwd_mirror(q, k, v, beta, dO, S0=None, dS_T=None, C: int = 64, euler: bool = False):
    q, k, v, beta, dO = (np.asarray(x, np.float64) for x in (q, k, v, beta, dO))
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    out = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros((B, H, T)), np.zeros((B, H, dk, dv))]
    dq, dkk, dvv, dbeta, dS0 = out
    for b in range(B):
        for h in range(H):
            # forward: entering states of every chunk
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[b, h], np.float64)
            starts = list(range(0, T, C))
            states, cache = [], []
            for c0 in starts:
                sl = slice(c0, min(T, c0 + C))
                Q, K, V, bt = q[b, h, sl], k[b, h, sl], v[b, h, sl], beta[b, h, sl]
                n = K.shape[0]
                lam = np.sum(K * K, axis=1)
                a = np.array([_alpha(bt[i], lam[i], euler) for i in range(n)])
                G = K @ K.T
                A = np.tril(a[:, None] * G, -1)
                X = np.linalg.inv(np.eye(n) + A)
                Tm = X * a[None, :]
                R = V - K @ S
                Delta = Tm @ R
                states.append(S)
                cache.append((sl, Q, K, lam, a, G, X, Tm, R, Delta, bt))
                S = S + K.T @ Delta
            dS = np.zeros((dk, dv)) if dS_T is None else np.array(dS_T[b, h], np.float64)
            for S, (sl, Q, K, lam, a, G, X, Tm, R, Delta, bt) in zip(reversed(states), reversed(cache)):
                dOc = dO[b, h, sl]
                P = np.tril(Q @ K.T)
                dSn = dS                                   # gradient of the leaving state
                dDelta = P.T @ dOc + K @ dSn
                dR = Tm.T @ dDelta
                dS = dSn + Q.T @ dOc - K.T @ dR
                dP = np.tril(dOc @ Delta.T)
                dQ = dOc @ S.T + dP @ K
                dT = dDelta @ R.T
                dX = dT * a[None, :]
                da = np.sum(dT * X, axis=0)
                dA = np.tril(-X.T @ dX @ X.T, -1)
                da += np.sum(dA * G, axis=1)
                dG = a[:, None] * dA
                dK = Delta @ dSn.T + dP.T @ Q - dR @ S.T + (dG + dG.T) @ K
                ab = np.array([_dalpha(bt[i], lam[i], euler) for i in range(len(bt))])
                dK += (da * ab[:, 1] * 2.0)[:, None] * K
                dq[b, h, sl], dkk[b, h, sl], dvv[b, h, sl] = dQ, dK, dR
                dbeta[b, h, sl] = da * ab[:, 0]
            dS0[b, h] = dS
    return tuple(out)
