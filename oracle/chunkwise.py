"""Chunkwise-parallel form of the Gated Delta Rule-2, in float64 numpy.

TEST INFRASTRUCTURE ONLY (see the package docstring).  This is the oracle's
second route to the recurrence's result, used to pin that the chunkwise
decomposition (Gated DeltaNet-2 guide, "Chunkwise Parallel Algorithm for GPU
Training": chunks of C tokens, intra-chunk work as matrix products, the state
handed across chunk boundaries) reproduces the token-by-token update for any
chunk size.  The WY factors with folded channel-wise decay follow the snilld.dk
article ("Hvad betyder det for traening og inferens": WY form as in KDA, the
cumulative channel-wise decay folded into the factors of each rank-one erase).

Derivation, per chunk with entering state S and local positions t = 1..C:
g_t = sum_{r<=t} log alpha_r (per key channel), Gamma_t = exp(g_t).  Writing the
step as S_t = D_t S_{t-1} + k_t u_t^T with u_t = w_t*v_t - S_{t-1}^T D_t (b_t*k_t)
and unrolling gives (I + A) U~ = (w*v) - (K*B*Gamma) S, where
A[t,s] = sum_i b[t,i] k[t,i] k[s,i] exp(g[t,i] - g[s,i]) for s < t.  Hence
U~ = U - W S with T = (I + A)^-1, W = T (K*B*Gamma), U = T (w*v), and

    O       = (Q*Gamma) S + mask_{s<=t}((Q*Gamma)(K/Gamma)^T) U~
    S_next  = Diag(Gamma_C) S + (K * Gamma_C/Gamma)^T U~
"""
from __future__ import annotations

import numpy as np


def _unit(q, k, v, la, b, w, S, C):
    T = q.shape[0]
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        Q, K, V, LA, Bg, Wg = q[sl], k[sl], v[sl], la[sl], b[sl], w[sl]
        n = Q.shape[0]
        g = np.cumsum(LA, axis=0)
        G = np.exp(g)
        A = np.zeros((n, n))
        for t in range(n):
            for s in range(t):
                A[t, s] = np.sum(Bg[t] * K[t] * K[s] * np.exp(g[t] - g[s]))
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ (K * Bg * G)
        U = Tm @ (Wg * V)
        Ut = U - W @ S
        P = np.zeros((n, n))
        for t in range(n):
            for s in range(t + 1):
                P[t, s] = np.sum(Q[t] * K[s] * np.exp(g[t] - g[s]))
        o[sl] = (Q * G) @ S + P @ Ut
        S = np.exp(g[-1])[:, None] * S + (K * np.exp(g[-1] - g)).T @ Ut
    return o, S


def forward(q, k, v, log_alpha, b, w, S0=None, C=64):
    """Chunkwise forward with chunk size C; tokens [B,T,H,D].  Returns (o, S_T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dk, dv))
    for bb in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[bb, h], dtype=np.float64)
            o[bb, :, h], S_T[bb, h] = _unit(q[bb, :, h], k[bb, :, h], v[bb, :, h],
                                            log_alpha[bb, :, h], b[bb, :, h], w[bb, :, h], S, C)
    return o, S_T
