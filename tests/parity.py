"""Shared helpers of the GPU parity tests: the error metric, the tolerances, and
the oracle run on a sample of (batch, head) units."""
from __future__ import annotations

import numpy as np

import gdn2_inputs as gi
import oracle

# max |gpu - oracle| / RMS(oracle), per output tensor
TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    if rms == 0.0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref))) / rms


def unit_inputs(d, bb, h, lo=None, hi=None):
    """float64 inputs of one (batch, head) unit, shaped [1, T, 1, D]."""
    sl = slice(lo, hi)
    out = {}
    for k in ("q", "k", "v", "log_alpha", "b", "w"):
        out[k] = gi.as_f64(d[k][bb:bb + 1, sl, h:h + 1])
    out["S0"] = None if d.get("S0") is None else gi.as_f64(d["S0"][bb:bb + 1, h:h + 1])
    return out


def oracle_units(d, units, S0=None):
    """Oracle (o [T, dv], S_T [dk, dv]) for each unit of ``units``.

    Units are stacked along the batch axis of one oracle call so that its
    threads run them in parallel.
    """
    per = [unit_inputs(d, bb, h) for bb, h in units]
    cat = {k: np.concatenate([p[k] for p in per], axis=0) for k in ("q", "k", "v", "log_alpha", "b", "w")}
    s0 = None
    if S0 is not None:
        s0 = np.concatenate([gi.as_f64(S0[bb:bb + 1, h:h + 1]) for bb, h in units], axis=0)
    elif d.get("S0") is not None:
        s0 = np.concatenate([p["S0"] for p in per], axis=0)
    o, S = oracle.forward(cat["q"], cat["k"], cat["v"], cat["log_alpha"], cat["b"], cat["w"], s0)
    return [(o[n, :, 0], S[n, 0]) for n in range(len(units))]


def check_units(d, o_gpu, S_gpu, tol, units=None, group=32):
    """Element-wise parity of every listed (batch, head) unit (all of them by default):
    o [B,T,H,dv] and S_T [B,H,dk,dv] of the GPU (CPU tensors) against the oracle, unit by
    unit, in groups of ``group`` units per oracle call.  Returns the worst errors."""
    B, H = d["q"].shape[0], d["q"].shape[2]
    if units is None:
        units = [(bb, h) for bb in range(B) for h in range(H)]
    worst_o = worst_s = 0.0
    for i in range(0, len(units), group):
        part = units[i:i + group]
        for (bb, h), (o_ref, S_ref) in zip(part, oracle_units(d, part)):
            eo = rel_err(o_gpu[bb, :, h].double().numpy(), o_ref)
            es = rel_err(S_gpu[bb, h].double().numpy(), S_ref)
            assert eo <= tol and es <= tol, (bb, h, eo, es)
            worst_o, worst_s = max(worst_o, eo), max(worst_s, es)
    return worst_o, worst_s
