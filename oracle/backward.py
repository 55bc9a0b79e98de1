"""Gradients of the Gated Delta Rule-2 recurrence, in float64 numpy.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Reverse mode of the token-by-token
definition the oracle's forward follows (snilld.dk, "Hvad Gated DeltaNet-2 aendrer", the
compact update; readout after the update):

    S'  = Diag(alpha_t) S_{t-1},   alpha_t = exp(log_alpha_t)
    e   = S'^T (b_t * k_t)                      (what the erase removes)
    u   = w_t * v_t - e
    S_t = S' + k_t u^T
    o_t = S_t^T q_t

Given dL/do_t for every token and dL/dS_T, one backward sweep over t = T-1 .. 0 carries
G = dL/dS_t and produces the gradients of every input and of S0:

    dq_t = S_t do_t;            G += q_t do_t^T
    dk_t = G u;                 du = G^T k_t
    dw_t = du * v_t;  dv_t = du * w_t;  de = -du
    G'   = G + (b_t * k_t) de^T   (dL/dS')
    dx   = S' de;  db_t = dx * k_t;  dk_t += dx * b_t
    dlog_alpha_t = alpha_t * rowsum(G' * S_{t-1})
    G    = Diag(alpha_t) G'        (dL/dS_{t-1})

Every state S_t of the run is kept (memory grows with T: meant for test sizes).  Pinned
in the tests against central finite differences of the forward.
"""
from __future__ import annotations

import numpy as np


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def backward(q, k, v, log_alpha, b, w, S0, do, dS_T=None):
    """Tokens [B,T,H,D], S0 [B,H,dk,dv] (or None = zeros), do [B,T,H,dv], dS_T
    [B,H,dk,dv] (or None = zero).  Returns dict(dq, dk, dv, dlog_alpha, db, dw, dS0)."""
    q, k, v, la, b, w, S0, do, dS_T = map(_f64, (q, k, v, log_alpha, b, w, S0, do, dS_T))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if S0 is None else S0.copy()
    # forward, keeping every state (S_t for t = -1 .. T-1) and every u
    states = np.empty((T + 1, B, H, dk, dv))
    us = np.empty((T, B, H, dv))
    states[0] = S
    for t in range(T):
        al = np.exp(la[:, t])                                   # [B,H,dk]
        Sp = al[..., None] * S
        x = b[:, t] * k[:, t]
        e = np.einsum("bhij,bhi->bhj", Sp, x)
        u = w[:, t] * v[:, t] - e
        S = Sp + k[:, t][..., None] * u[:, :, None, :]
        states[t + 1] = S
        us[t] = u
    g = {n: np.zeros_like(a) for n, a in (("dq", q), ("dk", k), ("dv", v), ("dlog_alpha", la), ("db", b), ("dw", w))}
    G = np.zeros((B, H, dk, dv)) if dS_T is None else dS_T.copy()
    for t in range(T - 1, -1, -1):
        St, Sprev, u = states[t + 1], states[t], us[t]
        al = np.exp(la[:, t])
        Sp = al[..., None] * Sprev
        dot = do[:, t]                                          # [B,H,dv]
        g["dq"][:, t] = np.einsum("bhij,bhj->bhi", St, dot)
        G = G + q[:, t][..., None] * dot[:, :, None, :]
        g["dk"][:, t] = np.einsum("bhij,bhj->bhi", G, u)
        du = np.einsum("bhij,bhi->bhj", G, k[:, t])
        g["dw"][:, t] = du * v[:, t]
        g["dv"][:, t] = du * w[:, t]
        de = -du
        x = b[:, t] * k[:, t]
        Gp = G + x[..., None] * de[:, :, None, :]
        dx = np.einsum("bhij,bhj->bhi", Sp, de)
        g["db"][:, t] = dx * k[:, t]
        g["dk"][:, t] += dx * b[:, t]
        g["dlog_alpha"][:, t] = al * np.sum(Gp * Sprev, axis=-1)
        G = al[..., None] * Gp
    g["dS0"] = G
    return g
