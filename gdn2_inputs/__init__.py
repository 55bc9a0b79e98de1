"""Seeded synthetic inputs for the Gated DeltaNet-2 token mixer.

This module only draws inputs.  It holds none of the recurrence's arithmetic,
and both the CUDA path and the CPU oracle read their inputs from it.

Recipe (the same for every workload):

* One random stream per tensor and block.  Block ``j`` of tensor ``name`` in a
  workload seeded ``seed`` comes from ``numpy.random.default_rng([seed, tid, j])``,
  where ``tid`` is the tensor's position in the draw order
  ``q, k, v, noise_alpha, noise_b, noise_w, S`` (0..6) and a block is
  ``BLOCK`` consecutive elements of the C-order tensor.  Decode step ``j`` uses
  ``seed = [seed, 1000 + j]`` instead, so every step draws fresh tokens.
* Draws are standard normal in float64; ``N(0, s)`` means standard deviation s.
* q and k are L2-normalised per (token, head) in float64, as the layer does
  before the mixer (Gated DeltaNet-2 guide, "Normalization and Short
  Convolutions").
* log alpha = -softplus(x)/16, or -softplus(2x)/8 for the heavy-tail decay of
  the long-context workload.  The decay gate is stored as log alpha in fp32.
* b = sigmoid(x), w = sigmoid(x): the erase and write gates are sigmoid
  projections (Gated DeltaNet-2 guide, "Decoupled Erase and Write Gates").
* The mixed-gate workload gives head h the regime h mod 3: (0) b = w = beta and
  alpha scalar per (token, head), the Gated DeltaNet case; (1) b = w = beta
  scalar with channel-wise alpha, the KDA case; (2) all gates channel-wise.
  A scalar gate uses the draw at channel 0 broadcast over the channels.
* Values are rounded once to the workload's dtype (round to nearest even);
  the oracle then reads those rounded values widened to float64.

Tensors are [B, T, H, D] (prefill) or [B, H, D] (decode); the state is
[B, H, d_k, d_v] float32.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os

import numpy as np

BLOCK = 1 << 20
_TID = {"q": 0, "k": 1, "v": 2, "alpha": 3, "b": 4, "w": 5, "S": 6}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    B: int
    H: int
    T: int               # tokens per sequence (1 for decode)
    dk: int
    dv: int
    dtype: str           # "f32" or "bf16": dtype of q, k, v, b, w and o
    seed: int
    decay: str = "base"  # "base": -softplus(N(0,1))/16; "heavy": -softplus(N(0,2))/8
    regimes: bool = False
    steps: int = 1       # decode steps
    state_std: float = 0.0  # std of the initial state (0 = zero state)
    C: int = 64


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", "prefill", 1, 1, 256, 64, 64, "f32", seed=0),
    "prefill_b8_h16_t4096": Workload("prefill_b8_h16_t4096", "prefill", 8, 16, 4096, 128, 128, "bf16", seed=1),
    "long_b1_h16_t65536": Workload("long_b1_h16_t65536", "prefill", 1, 16, 65536, 128, 128, "bf16", seed=2,
                                   decay="heavy"),
    "decode_b256_h16": Workload("decode_b256_h16", "decode", 256, 16, 1, 128, 128, "bf16", seed=3,
                                steps=1000, state_std=0.02),
    "mixed_b4_h32_t8192": Workload("mixed_b4_h32_t8192", "prefill", 4, 32, 8192, 128, 128, "bf16", seed=4,
                                   regimes=True),
    # packed serving batch: 64 sequences, lengths log-uniform in [16, 8192] (packed_lengths),
    # each continuing from an entering state N(0, 0.02)
    "packed_n64_h16": Workload("packed_n64_h16", "packed", 64, 16, 8192, 128, 128, "bf16", seed=5,
                               state_std=0.02),
}


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _draw(seed_key, tid: int, shape, transform=None, row: int = 1) -> np.ndarray:
    """Standard normals in float64, block by block, transformed, stored as float32."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    nblk = (n + BLOCK - 1) // BLOCK

    def one(j):
        lo, hi = j * BLOCK, min(n, (j + 1) * BLOCK)
        x = np.random.default_rng(list(seed_key) + [tid, j]).standard_normal(hi - lo)
        if transform is not None:
            x = transform(x.reshape(-1, row)).reshape(-1)
        out[lo:hi] = x

    if nblk == 1:
        one(0)
    else:
        with _cf.ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(one, range(nblk)))
    return out.reshape(shape)


def _l2(x):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True))


def _softplus(x):
    return np.logaddexp(0.0, x)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _log_alpha(decay):
    if decay == "heavy":
        return lambda x: -_softplus(2.0 * x) / 8.0
    return lambda x: -_softplus(x) / 16.0


def _round(x: np.ndarray, dtype: str):
    """Round float32 values to the storage dtype; returns a CPU torch tensor."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.bfloat16) if dtype == "bf16" else t.to(torch.float32)


def _apply_regimes(log_alpha, b, w, H):
    """Head h gets regime h mod 3 (see the module docstring); works in place."""
    heads = np.arange(H)
    scalar_gate = heads % 3 <= 1     # regimes 0 and 1: b = w = beta scalar
    scalar_alpha = heads % 3 == 0    # regime 0: alpha scalar too
    beta = b[:, :, scalar_gate, :1].copy()
    b[:, :, scalar_gate, :] = beta
    w[:, :, scalar_gate, :] = beta
    la = log_alpha[:, :, scalar_alpha, :1].copy()
    log_alpha[:, :, scalar_alpha, :] = la


def prefill_inputs(wl: Workload, B=None, T=None, H=None, seed=None):
    """Inputs of a prefill workload as CPU torch tensors.

    Returns dict(q, k, v, b, w: dtype [B,T,H,D]; log_alpha: float32 [B,T,H,dk];
    S0: float32 [B,H,dk,dv] or None).  B, T, H and seed may be overridden to draw
    a smaller case of the same recipe.
    """
    B = wl.B if B is None else B
    T = wl.T if T is None else T
    H = wl.H if H is None else H
    key = [wl.seed if seed is None else seed]
    sk, sv = (B, T, H, wl.dk), (B, T, H, wl.dv)
    q = _draw(key, _TID["q"], sk, _l2, wl.dk)
    k = _draw(key, _TID["k"], sk, _l2, wl.dk)
    v = _draw(key, _TID["v"], sv)
    la = _draw(key, _TID["alpha"], sk, _log_alpha(wl.decay))
    b = _draw(key, _TID["b"], sk, _sigmoid)
    w = _draw(key, _TID["w"], sv, _sigmoid)
    if wl.regimes:
        _apply_regimes(la, b, w, H)
    S0 = None
    if wl.state_std > 0:
        S0 = _draw(key, _TID["S"], (B, H, wl.dk, wl.dv), lambda x: wl.state_std * x)
    import torch
    out = dict(q=_round(q, wl.dtype), k=_round(k, wl.dtype), v=_round(v, wl.dtype),
               b=_round(b, wl.dtype), w=_round(w, wl.dtype),
               log_alpha=torch.from_numpy(la),
               S0=None if S0 is None else torch.from_numpy(S0))
    return out


def raw_inputs(wl: Workload, B=None, T=None, H=None, seed=None):
    """The raw projections behind a prefill workload: the same draws as
    ``prefill_inputs`` before any activation, for the raw-projection entry point.

    Returns dict(q_raw, k_raw, v, b_raw, w_raw: dtype [B,T,H,D]; a_raw: float32
    [B,T,H,dk]; decay_scale: float32 [H]; S0).  The decay pre-activation and scale
    reproduce the workload's gate: log alpha = -decay_scale * softplus(a_raw), with
    a_raw = x and scale 1/16 ("base"), or a_raw = 2x and scale 1/8 ("heavy")."""
    import torch
    B = wl.B if B is None else B
    T = wl.T if T is None else T
    H = wl.H if H is None else H
    key = [wl.seed if seed is None else seed]
    sk, sv = (B, T, H, wl.dk), (B, T, H, wl.dv)
    heavy = wl.decay == "heavy"
    q = _draw(key, _TID["q"], sk)
    k = _draw(key, _TID["k"], sk)
    v = _draw(key, _TID["v"], sv)
    a = _draw(key, _TID["alpha"], sk, (lambda x: 2.0 * x) if heavy else None)
    b = _draw(key, _TID["b"], sk)
    w = _draw(key, _TID["w"], sv)
    S0 = None
    if wl.state_std > 0:
        S0 = torch.from_numpy(_draw(key, _TID["S"], (B, H, wl.dk, wl.dv), lambda x: wl.state_std * x))
    scale = np.full(H, 1.0 / 8.0 if heavy else 1.0 / 16.0, dtype=np.float32)
    return dict(q_raw=_round(q, wl.dtype), k_raw=_round(k, wl.dtype), v=_round(v, wl.dtype),
                b_raw=_round(b, wl.dtype), w_raw=_round(w, wl.dtype), a_raw=torch.from_numpy(a),
                decay_scale=torch.from_numpy(scale), S0=S0)


def packed_lengths(n: int, lo: int, hi: int, seed: int):
    """A seeded serving-like length mix: n lengths log-uniform in [lo, hi] (integers)."""
    rng = np.random.default_rng([seed, 2000])
    return [int(x) for x in np.exp(rng.uniform(np.log(lo), np.log(hi), size=n)).round()]


def packed_inputs(wl: Workload, lengths, H=None, seed=None, state_std=None):
    """Packed variable-length sequences drawn with a prefill workload's recipe.

    Returns dict(q, k, v, b, w: dtype [T,H,D]; log_alpha: float32 [T,H,dk];
    cu_seqlens: int32 [N+1]; S0: float32 [N,H,dk,dv] or None), T = sum(lengths).
    """
    import torch
    H = wl.H if H is None else H
    T = int(sum(lengths))
    d = prefill_inputs(wl, B=1, T=max(T, 1), H=H, seed=seed)
    out = {k: (None if v is None else v[0, :T]) for k, v in d.items() if k != "S0"}
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    out["cu_seqlens"] = torch.from_numpy(cu)
    std = wl.state_std if state_std is None else state_std
    S0 = None
    if std > 0:
        key = [(wl.seed if seed is None else seed) + 7919]
        S0 = torch.from_numpy(_draw(key, _TID["S"], (len(lengths), H, wl.dk, wl.dv), lambda x: std * x))
    out["S0"] = S0
    return out


def decode_state(wl: Workload, B=None, H=None, seed=None):
    """Initial decode state, float32 [B, H, dk, dv], N(0, state_std)."""
    B = wl.B if B is None else B
    H = wl.H if H is None else H
    key = [wl.seed if seed is None else seed]
    import torch
    S = _draw(key, _TID["S"], (B, H, wl.dk, wl.dv), lambda x: wl.state_std * x)
    return torch.from_numpy(S)


def decode_tokens(wl: Workload, step: int, B=None, H=None, seed=None):
    """Tokens of decode step ``step``: dict(q,k,v,b,w: dtype [B,H,D]; log_alpha fp32 [B,H,dk])."""
    B = wl.B if B is None else B
    H = wl.H if H is None else H
    key = [wl.seed if seed is None else seed, 1000 + step]
    sk, sv = (B, H, wl.dk), (B, H, wl.dv)
    q = _draw(key, _TID["q"], sk, _l2, wl.dk)
    k = _draw(key, _TID["k"], sk, _l2, wl.dk)
    v = _draw(key, _TID["v"], sv)
    la = _draw(key, _TID["alpha"], sk, _log_alpha(wl.decay))
    b = _draw(key, _TID["b"], sk, _sigmoid)
    w = _draw(key, _TID["w"], sv, _sigmoid)
    import torch
    return dict(q=_round(q, wl.dtype), k=_round(k, wl.dtype), v=_round(v, wl.dtype),
                b=_round(b, wl.dtype), w=_round(w, wl.dtype), log_alpha=torch.from_numpy(la))


def decode_tokens_many(wl: Workload, steps, B=None, H=None, seed=None):
    """decode_tokens for many steps, drawn on a thread pool; returns a list."""
    with _cf.ThreadPoolExecutor(_threads()) as ex:
        return list(ex.map(lambda j: decode_tokens(wl, j, B=B, H=H, seed=seed), steps))


def as_f64(t):
    """A CPU torch tensor widened to a float64 numpy array (the values the GPU sees)."""
    import torch
    return t.detach().to("cpu").to(torch.float64).numpy()
