"""CPU oracle for the Gated DeltaNet-2 token mixer (double precision).

TEST INFRASTRUCTURE ONLY: the test suite, the package's ``smoke()`` check and the
benchmark's CPU-baseline leg are the only callers.  The CUDA path never imports
this package, and this package imports nothing from the CUDA path.

* ``forward`` / ``decode_step`` call ``gdn2_oracle.c``: the recurrence of the
  Gated Delta Rule-2 written out token by token (snilld.dk article, the compact
  update; readout after the update as in the guide's PyTorch loop).
* ``chunkwise.forward`` re-derives the chunkwise WY form in numpy; it is a
  second, independent route to the same numbers, used to pin chunk invariance.
* ``backward.backward`` is reverse mode of the token-by-token recurrence (fp64, every
  state kept), pinned against central finite differences of ``forward``;
  ``chunkwise.backward`` re-derives it in chunk form (the blueprint of the GPU backward).
* ``short_conv`` is the layer's 4-tap causal depthwise convolution, a plain loop
  over taps.
* ``activations`` maps the raw projections to the mixer's inputs (L2-normalised
  q and k, sigmoid gates, log alpha = -s_h softplus(a)); composed with
  ``forward`` it is what the raw-projection entry point computes.

Every function takes float64 numpy arrays in the layouts of the C ABI:
tokens [B, T, H, D], states [B, H, d_k, d_v].
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_oracle.c")
LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(src: str = _SRC, out: str = LIB_PATH, extra=()) -> str:
    """Compile the C oracle into a shared library with gcc; returns its path."""
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-pthread", *extra, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _bind(lib):
    D = ctypes.POINTER(ctypes.c_double)
    L = ctypes.c_long
    lib.gdn2_oracle_forward.argtypes = [D] * 9 + [L] * 5 + [ctypes.c_int]
    lib.gdn2_oracle_forward.restype = ctypes.c_int
    lib.gdn2_oracle_decode_step.argtypes = [D] * 8 + [L] * 4 + [ctypes.c_int]
    lib.gdn2_oracle_decode_step.restype = ctypes.c_int
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the C oracle.  ``path`` loads another build."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        if not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(_SRC):
            build()
        _lib = _bind(ctypes.CDLL(LIB_PATH))
    return _lib


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def forward(q, k, v, log_alpha, b, w, S0=None, nthreads=None, lib=None):
    """Returns (o [B,T,H,dv], S_T [B,H,dk,dv]) for tokens [B,T,H,D]."""
    q, k, v, log_alpha, b, w, S0 = map(_f64, (q, k, v, log_alpha, b, w, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dk, dv))
    lib = lib or load()
    rc = lib.gdn2_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                 _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv,
                                 nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle forward failed: {rc}")
    return o, S_T


def forward_varlen(q, k, v, log_alpha, b, w, cu_seqlens, S0=None, nthreads=None, lib=None):
    """Packed variable-length sequences: tokens [T,H,D], sequence n = rows
    [cu_seqlens[n], cu_seqlens[n+1]).  Each sequence is an independent run of the
    recurrence from its own entering state (the stateful-serving reading of the
    DeltaNet-2 AI architecture guide: the endpoint accepts and returns the state),
    so this is `forward` on each slice.  Returns (o [T,H,dv], S_T [N,H,dk,dv])."""
    q, k, v, log_alpha, b, w, S0 = map(_f64, (q, k, v, log_alpha, b, w, S0))
    cu = [int(x) for x in np.asarray(cu_seqlens).ravel()]
    N = len(cu) - 1
    T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((T, H, dv))
    S_T = np.zeros((N, H, dk, dv))
    for n in range(N):
        a, e = cu[n], cu[n + 1]
        s0 = None if S0 is None else S0[n:n + 1]
        if e == a:
            if s0 is not None:
                S_T[n] = s0[0]
            continue
        sl = [x[a:e][None] for x in (q, k, v, log_alpha, b, w)]
        o_n, s_n = forward(*sl, S0=s0, nthreads=nthreads, lib=lib)
        o[a:e] = o_n[0]
        S_T[n] = s_n[0]
    return o, S_T


def _sigmoid(x):
    # 1 / (1 + e^-x), evaluated on the side where the exponential cannot overflow
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def activations(q_raw, k_raw, a_raw, b_raw, w_raw, decay_scale=None):
    """The layer's input activations, in float64, for tokens [..., H, D] (H the
    second-to-last axis).

    * q and k are divided by their Euclidean norm per (token, head) (Gated DeltaNet-2
      guide, "Normalization and Short Convolutions"); a zero vector stays zero (the
      norm is floored at 1e-12).
    * b = sigmoid(b_raw), w = sigmoid(w_raw): the erase and write gates take values in
      (0, 1) and come from sigmoid projections (same guide, "Decoupled Erase and Write
      Gates"; snilld.dk, "Hvad Gated DeltaNet-2 aendrer").
    * log alpha = -s_h softplus(a_raw) = -s_h log(1 + e^a), a channel-wise decay in
      (0, 1) with a positive per-head scale s_h (decay_scale [H], default 1).

    Returns dict(q, k, log_alpha, b, w)."""
    q_raw, k_raw, a_raw, b_raw, w_raw = map(_f64, (q_raw, k_raw, a_raw, b_raw, w_raw))

    def l2n(x):
        n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
        return x / np.maximum(n, 1e-12)

    H = q_raw.shape[-2]
    s = np.ones(H) if decay_scale is None else np.asarray(decay_scale, dtype=np.float64).reshape(H)
    softplus = np.logaddexp(0.0, a_raw)
    return dict(q=l2n(q_raw), k=l2n(k_raw), log_alpha=-s[:, None] * softplus, b=_sigmoid(b_raw),
                w=_sigmoid(w_raw))


def short_conv(x, weight, bias=None, hist=None):
    """Causal depthwise convolution with 4 taps over the token axis of one sequence
    (Gated DeltaNet-2 guide, "Normalization and Short Convolutions": the layer convolves
    each channel of q, k and v over tokens t-3 .. t, padding on the left, with a bias):
    y[t, c] = bias[c] + sum_j weight[c, j] x[t - 3 + j, c], tokens before the first taken
    from ``hist`` ([3, C], oldest first) or zero.

    x: [T, C]; weight [C, 4]; bias [C] or None.  Returns (y [T, C], the last three inputs
    [3, C] of the history followed by x)."""
    x = _f64(x)
    T, C = x.shape
    w = _f64(weight).reshape(C, 4)
    ext = np.zeros((T + 3, C))
    if hist is not None:
        ext[:3] = _f64(hist).reshape(3, C)
    ext[3:] = x
    y = np.zeros((T, C)) if bias is None else np.tile(_f64(bias).reshape(1, C), (T, 1))
    for t in range(T):
        for j in range(4):
            y[t] += w[:, j] * ext[t + j]
    return y, ext[T:T + 3].copy()


def decode_step(q, k, v, log_alpha, b, w, S, nthreads=None, lib=None):
    """One token per unit: tokens [B,H,D], S [B,H,dk,dv].  Returns (o, S_new)."""
    q, k, v, log_alpha, b, w = map(_f64, (q, k, v, log_alpha, b, w))
    S = np.array(S, dtype=np.float64, copy=True, order="C")
    B, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, dv))
    lib = lib or load()
    rc = lib.gdn2_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                     _ptr(S), _ptr(o), B, H, dk, dv, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle decode failed: {rc}")
    return o, S
