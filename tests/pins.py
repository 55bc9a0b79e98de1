"""Pins of the CPU oracle: facts the pages and the mathematics fix.

Each ``pin_*`` function takes a loaded oracle library (so that the mutation test
can run the same checks against deliberately broken copies of the oracle) and
raises AssertionError when the oracle disagrees.  None of them re-types the
oracle's own formula: each compares it with a special case stated on the pages,
a closed form, an invariant, or a hand-worked example.
"""
from __future__ import annotations

import json
import os

import numpy as np

import oracle
import oracle.chunkwise as chunkwise

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _l2(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def rand_case(seed, B=2, T=37, H=3, dk=8, dv=6, S0=True, decay=0.25):
    """Random float64 inputs [B,T,H,D]: unit q, k; gates in (0,1); log alpha <= 0."""
    r = np.random.default_rng(seed)
    d = dict(q=_l2(r.standard_normal((B, T, H, dk))), k=_l2(r.standard_normal((B, T, H, dk))),
             v=r.standard_normal((B, T, H, dv)),
             log_alpha=-decay * np.logaddexp(0.0, r.standard_normal((B, T, H, dk))),
             b=_sig(r.standard_normal((B, T, H, dk))), w=_sig(r.standard_normal((B, T, H, dv))))
    d["S0"] = r.standard_normal((B, H, dk, dv)) if S0 else None
    return d


def _fwd(lib, d, **kw):
    return oracle.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], lib=lib, **kw)


def _close(a, b, tol=1e-10, what=""):
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, np.max(np.abs(b)) if b.size else 1.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e}"


# --- hand-worked examples -------------------------------------------------------------

def _golden(lib, name):
    with open(os.path.join(GOLDEN, name)) as f:
        g = json.load(f)
    B, T, H, dk, dv = g["B"], g["T"], g["H"], g["dk"], g["dv"]
    arr = lambda key, D: np.array(g[key], dtype=np.float64).reshape(B, T, H, D)
    d = dict(q=arr("q", dk), k=arr("k", dk), v=arr("v", dv), log_alpha=np.log(arr("alpha", dk)),
             b=arr("b", dk), w=arr("w", dv), S0=np.array(g["S0"]).reshape(B, H, dk, dv))
    o, S = _fwd(lib, d)
    _close(o, arr("o", dv), 1e-12, name + " o")
    _close(S, np.array(g["S_T"]).reshape(B, H, dk, dv), 1e-12, name + " S_T")


def pin_golden_onehot(lib):
    _golden(lib, "onehot_d2.json")


def pin_golden_erase_orientation(lib):
    _golden(lib, "erase_orientation_d2.json")


# --- special cases the pages name -----------------------------------------------------

def pin_kda_reduction(lib):
    """b = w = beta scalar per token: S = (I - beta k k^T) Diag(alpha) S + beta k v^T (KDA)."""
    d = rand_case(11)
    beta = d["b"][..., :1]
    d["b"] = np.broadcast_to(beta, d["b"].shape).copy()
    d["w"] = np.broadcast_to(beta, d["w"].shape).copy()
    o, S = _fwd(lib, d)
    B, T, H, dk = d["q"].shape
    for bb in range(B):
        for h in range(H):
            St = d["S0"][bb, h].copy()
            for t in range(T):
                kk, be = d["k"][bb, t, h], beta[bb, t, h, 0]
                M = (np.eye(dk) - be * np.outer(kk, kk)) @ np.diag(np.exp(d["log_alpha"][bb, t, h]))
                St = M @ St + be * np.outer(kk, d["v"][bb, t, h])
                _close(o[bb, t, h], St.T @ d["q"][bb, t, h], 1e-10, "kda o")
            _close(S[bb, h], St, 1e-10, "kda S")


def pin_gdn_reduction(lib):
    """Additionally alpha scalar: S = alpha (I - beta k k^T) S + beta k v^T (Gated DeltaNet)."""
    d = rand_case(12)
    beta = d["b"][..., :1]
    a = d["log_alpha"][..., :1]
    d["b"] = np.broadcast_to(beta, d["b"].shape).copy()
    d["w"] = np.broadcast_to(beta, d["w"].shape).copy()
    d["log_alpha"] = np.broadcast_to(a, d["log_alpha"].shape).copy()
    o, S = _fwd(lib, d)
    B, T, H, dk = d["q"].shape
    for bb in range(B):
        for h in range(H):
            St = d["S0"][bb, h].copy()
            for t in range(T):
                kk, be, al = d["k"][bb, t, h], beta[bb, t, h, 0], np.exp(a[bb, t, h, 0])
                St = al * (St - be * np.outer(kk, kk @ St)) + be * np.outer(kk, d["v"][bb, t, h])
                _close(o[bb, t, h], St.T @ d["q"][bb, t, h], 1e-10, "gdn o")
            _close(S[bb, h], St, 1e-10, "gdn S")


def pin_deltanet_error_form(lib):
    """alpha = 1, b = w = beta: the classical delta rule in the guide's d_v x d_k
    orientation, S <- S - beta (S k - v) k^T, is our state transposed."""
    d = rand_case(13)
    beta = d["b"][..., :1]
    d["b"] = np.broadcast_to(beta, d["b"].shape).copy()
    d["w"] = np.broadcast_to(beta, d["w"].shape).copy()
    d["log_alpha"] = np.zeros_like(d["log_alpha"])
    o, S = _fwd(lib, d)
    B, T, H, _ = d["q"].shape
    for bb in range(B):
        for h in range(H):
            P = d["S0"][bb, h].T.copy()            # d_v x d_k
            for t in range(T):
                kk, be = d["k"][bb, t, h], beta[bb, t, h, 0]
                P = P - be * np.outer(P @ kk - d["v"][bb, t, h], kk)
                _close(o[bb, t, h], P @ d["q"][bb, t, h], 1e-10, "deltanet o")
            _close(S[bb, h], P.T, 1e-10, "deltanet S")


def pin_decoupled_guide_form(lib):
    """alpha = 1: the guide's decoupled update S <- S (I - (b*k) k^T) + (w*v) k^T on a
    d_v x d_k state, y = S q, equals our d_k x d_v state transposed."""
    d = rand_case(14)
    d["log_alpha"] = np.zeros_like(d["log_alpha"])
    o, S = _fwd(lib, d)
    B, T, H, dk = d["q"].shape
    for bb in range(B):
        for h in range(H):
            P = d["S0"][bb, h].T.copy()
            for t in range(T):
                kk = d["k"][bb, t, h]
                P = P @ (np.eye(dk) - np.outer(d["b"][bb, t, h] * kk, kk)) \
                    + np.outer(d["w"][bb, t, h] * d["v"][bb, t, h], kk)
                _close(o[bb, t, h], P @ d["q"][bb, t, h], 1e-10, "guide o")
            _close(S[bb, h], P.T, 1e-10, "guide S")


# --- closed forms ------------------------------------------------------------------------

def pin_hebbian_closed_form(lib):
    """b = 0, alpha = 1, w = 1: linear attention.  S_T = S0 + K^T V and
    o_t = S0^T q_t + sum_{s<=t} (k_s . q_t) v_s."""
    d = rand_case(15)
    d["b"] = np.zeros_like(d["b"])
    d["w"] = np.ones_like(d["w"])
    d["log_alpha"] = np.zeros_like(d["log_alpha"])
    o, S = _fwd(lib, d)
    B, T, H, _ = d["q"].shape
    mask = np.tril(np.ones((T, T)))
    for bb in range(B):
        for h in range(H):
            Q, K, V = d["q"][bb, :, h], d["k"][bb, :, h], d["v"][bb, :, h]
            _close(S[bb, h], d["S0"][bb, h] + K.T @ V, 1e-10, "hebbian S")
            _close(o[bb, :, h], Q @ d["S0"][bb, h] + ((Q @ K.T) * mask) @ V, 1e-10, "hebbian o")


def pin_gated_linear_attention_closed_form(lib):
    """b = 0 (no erase): channel-decayed linear attention with global cumsum G,
    o_t = (q_t * e^{G_t})^T S0 + sum_{s<=t} ((q_t * e^{G_t - G_s}) . k_s)(w_s * v_s)."""
    d = rand_case(16)
    d["b"] = np.zeros_like(d["b"])
    o, S = _fwd(lib, d)
    B, T, H, _ = d["q"].shape
    for bb in range(B):
        for h in range(H):
            G = np.cumsum(d["log_alpha"][bb, :, h], axis=0)
            Q, K = d["q"][bb, :, h], d["k"][bb, :, h]
            WV = d["w"][bb, :, h] * d["v"][bb, :, h]
            for t in range(T):
                ref = (Q[t] * np.exp(G[t])) @ d["S0"][bb, h]
                for s in range(t + 1):
                    ref = ref + np.sum(Q[t] * np.exp(G[t] - G[s]) * K[s]) * WV[s]
                _close(o[bb, t, h], ref, 1e-10, "gla o")
            ST = np.exp(G[-1])[:, None] * d["S0"][bb, h] + (K * np.exp(G[-1] - G)).T @ WV
            _close(S[bb, h], ST, 1e-10, "gla S")


# --- invariants ---------------------------------------------------------------------------

def pin_retrieval_invariant(lib):
    """||k_t|| = 1 and b_t = 1: S_t^T k_t = w_t * v_t for any alpha and S_{t-1};
    read out with q_t = k_t, o_t is exactly w_t * v_t."""
    d = rand_case(17)
    d["b"] = np.ones_like(d["b"])
    d["q"] = d["k"].copy()
    o, _ = _fwd(lib, d)
    _close(o, d["w"] * d["v"], 1e-12, "retrieval")


def pin_pure_erase(lib):
    """Pure erase (b = 1, w = 0) with unit k: the key is wiped, S_t^T k_t = 0."""
    d = rand_case(18)
    d["b"] = np.ones_like(d["b"])
    d["w"] = np.zeros_like(d["w"])
    d["q"] = d["k"].copy()
    o, _ = _fwd(lib, d)
    _close(o, np.zeros_like(o), 1e-12, "pure erase")


def pin_passive_preservation(lib):
    """Passive preservation (b = 0, w = 0, alpha = 1): the state passes unchanged."""
    d = rand_case(19)
    d["b"] = np.zeros_like(d["b"])
    d["w"] = np.zeros_like(d["w"])
    d["log_alpha"] = np.zeros_like(d["log_alpha"])
    o, S = _fwd(lib, d)
    assert np.array_equal(S, d["S0"]), "passive: state changed"
    _close(o, np.einsum("bthi,bhij->bthj", d["q"], d["S0"]), 1e-12, "passive o")


def pin_transition_spectrum(lib):
    """One step with w = 0 applied to S0 = I gives the transition M = (I - k (b*k)^T) D.
    det M = (1 - sum_i b_i k_i^2) prod_i alpha_i; with alpha = 1 its eigenvalues
    are 1 (d-1 times) and 1 - sum_i b_i k_i^2, inside [0, 1] for unit k (the
    guide's spectral bound, read for eigenvalues)."""
    d = rand_case(20, B=1, T=1, H=4, dk=7, dv=7)
    d["w"] = np.zeros_like(d["w"])
    d["S0"] = np.broadcast_to(np.eye(7), (1, 4, 7, 7)).copy()
    _, M = _fwd(lib, d)
    d1 = dict(d, log_alpha=np.zeros_like(d["log_alpha"]))
    _, M1 = _fwd(lib, d1)
    for h in range(4):
        k, b, la = d["k"][0, 0, h], d["b"][0, 0, h], d["log_alpha"][0, 0, h]
        lam = 1.0 - np.sum(b * k * k)
        assert abs(np.linalg.det(M[0, h]) - lam * np.exp(la.sum())) < 1e-12, "det"
        ev = np.sort(np.linalg.eigvals(M1[0, h]).real)
        assert np.allclose(ev, np.sort(np.r_[np.ones(6), lam]), atol=1e-9), "spectrum"
        assert 0.0 <= lam <= 1.0


def pin_linearity(lib):
    """(o, S_T) is linear in (S0, v) jointly for fixed q, k, alpha, b, w."""
    d1, d2 = rand_case(21), rand_case(22)
    c = -0.7
    mix = dict(d1, v=d1["v"] + c * d2["v"], S0=d1["S0"] + c * d2["S0"])
    o1, S1 = _fwd(lib, d1)
    o2, S2 = _fwd(lib, dict(d1, v=d2["v"], S0=d2["S0"]))
    o3, S3 = _fwd(lib, mix)
    _close(o3, o1 + c * o2, 1e-10, "linear o")
    _close(S3, S1 + c * S2, 1e-10, "linear S")


def pin_chunk_invariance(lib):
    """The chunkwise WY form (separate numpy derivation) equals the recurrence for
    every chunk size, including a partial last chunk."""
    for T in (1, 63, 64, 65, 150):
        d = rand_case(23 + T, B=1, T=T, H=2, dk=8, dv=5)
        o, S = _fwd(lib, d)
        for C in (16, 32, 64, 128):
            o2, S2 = chunkwise.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], C)
            _close(o, o2, 1e-10, f"chunk C={C} T={T} o")
            _close(S, S2, 1e-10, f"chunk C={C} T={T} S")


def pin_split_handoff(lib):
    """Running [0, T1) then [T1, T) from the handed-over state equals one run."""
    d = rand_case(30, T=50)
    o, S = _fwd(lib, d)
    first = {k: (v[:, :20] if k != "S0" else v) for k, v in d.items()}
    oa, Sa = _fwd(lib, first)
    second = {k: (v[:, 20:] if k != "S0" else Sa) for k, v in d.items()}
    ob, Sb = _fwd(lib, second)
    _close(np.concatenate([oa, ob], axis=1), o, 1e-12, "split o")
    _close(Sb, S, 1e-12, "split S")


ALL = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
