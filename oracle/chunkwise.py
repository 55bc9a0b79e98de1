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


def _unit_backward(q, k, v, la, b, w, S0, do, dS_T, C):
    """Reverse mode of the chunk form above for one (batch, head): the entering state of
    every chunk from a forward sweep, then the chunks in reverse.  Per chunk (rows are its
    tokens; Kb = K*B*Gamma, Qh = Q*Gamma, Kn = K/Gamma, Vw = W*V, A strictly lower and
    P lower parts of Kb Kn^T and Qh Kn^T, T = (I + A)^-1, R = Vw - Kb S, U = T R,
    O = Qh S + P U, St = S + Kn^T U, S_next = Diag(Gamma_C) St), given dO and dS_next:

        dSt = Diag(Gamma_C) dS_next;   dGamma_C = rowsum(dS_next * St)
        dQh = dO S^T;  dS = Qh^T dO + dSt;  dP = lower(dO U^T);  dU = P^T dO + Kn dSt
        dKn = U dSt^T;  dR = T^T dU;  dA = strict_lower(-T^T (dU R^T) T^T)
        dVw = dR;  dKb = -dR S^T + dA Kn;  dS -= Kb^T dR
        dKn += dA^T Kb + dP^T Qh;  dQh += dP Kn
        dK = dKb*B*Gamma + dKn/Gamma;  dB = dKb*K*Gamma;  dQ = dQh*Gamma
        dW = dVw*V;  dV = dVw*W
        dg = dKb*Kb + dQh*Qh - dKn*Kn  (+ dGamma_C*Gamma_C on the last row)
        dlog_alpha = reverse cumsum of dg over the chunk's rows
    """
    T = q.shape[0]
    dk, dv = q.shape[1], v.shape[1]
    starts = list(range(0, T, C))
    S = S0.copy()
    Sin = []
    for c0 in starts:
        sl = slice(c0, min(T, c0 + C))
        Sin.append(S.copy())
        _, S = _unit(q[sl], k[sl], v[sl], la[sl], b[sl], w[sl], S, C)
    grads = {n: np.zeros_like(a) for n, a in (("dq", q), ("dk", k), ("dv", v), ("dlog_alpha", la), ("db", b),
                                              ("dw", w))}
    dS_next = dS_T.copy()
    for ci in range(len(starts) - 1, -1, -1):
        c0 = starts[ci]
        sl = slice(c0, min(T, c0 + C))
        Q, K, V, LA, Bg, Wg, dO = q[sl], k[sl], v[sl], la[sl], b[sl], w[sl], do[sl]
        S = Sin[ci]
        n = Q.shape[0]
        g = np.cumsum(LA, axis=0)
        Gm = np.exp(g)
        Kb, Qh, Kn, Vw = K * Bg * Gm, Q * Gm, K / Gm, Wg * V
        low = np.tril(np.ones((n, n)), -1)
        A = low * (Kb @ Kn.T)
        P = np.tril(Qh @ Kn.T)
        Tm = np.linalg.inv(np.eye(n) + A)
        R = Vw - Kb @ S
        U = Tm @ R
        St = S + Kn.T @ U
        GC = Gm[-1]
        dSt = GC[:, None] * dS_next
        dGC = np.sum(dS_next * St, axis=1)
        dQh = dO @ S.T
        dS = Qh.T @ dO + dSt
        dP = np.tril(dO @ U.T)
        dU = P.T @ dO + Kn @ dSt
        dKn = U @ dSt.T
        dR = Tm.T @ dU
        dA = low * (-Tm.T @ (dU @ R.T) @ Tm.T)
        dVw = dR
        dKb = -dR @ S.T + dA @ Kn
        dS -= Kb.T @ dR
        dKn += dA.T @ Kb + dP.T @ Qh
        dQh += dP @ Kn
        grads["dk"][sl] = dKb * Bg * Gm + dKn / Gm
        grads["db"][sl] = dKb * K * Gm
        grads["dq"][sl] = dQh * Gm
        grads["dw"][sl] = dVw * V
        grads["dv"][sl] = dVw * Wg
        dg = dKb * Kb + dQh * Qh - dKn * Kn
        dg[-1] += dGC * GC
        grads["dlog_alpha"][sl] = np.cumsum(dg[::-1], axis=0)[::-1]
        dS_next = dS
    grads["dS0"] = dS_next
    return grads


def backward(q, k, v, log_alpha, b, w, S0, do, dS_T=None, C=64):
    """Chunkwise gradients with chunk size C; tokens [B,T,H,D].  Returns the same dict as
    the token-level oracle backward (dq, dk, dv, dlog_alpha, db, dw, dS0)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S0 = np.zeros((B, H, dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float64)
    dS_T = np.zeros((B, H, dk, dv)) if dS_T is None else np.asarray(dS_T, dtype=np.float64)
    out = {n: np.zeros((B, T, H, d)) for n, d in (("dq", dk), ("dk", dk), ("dv", dv), ("dlog_alpha", dk),
                                                  ("db", dk), ("dw", dv))}
    out["dS0"] = np.zeros((B, H, dk, dv))
    f = lambda a: np.asarray(a, dtype=np.float64)
    for bb in range(B):
        for h in range(H):
            gu = _unit_backward(f(q[bb, :, h]), f(k[bb, :, h]), f(v[bb, :, h]), f(log_alpha[bb, :, h]),
                                f(b[bb, :, h]), f(w[bb, :, h]), S0[bb, h], f(do[bb, :, h]), dS_T[bb, h], C)
            for n in ("dq", "dk", "dv", "dlog_alpha", "db", "dw"):
                out[n][bb, :, h] = gu[n]
            out["dS0"][bb, h] = gu["dS0"]
    return out
