"""Decode step on the GPU against the CPU oracle (parity), through the C ABI."""
import dataclasses

import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import gated_delta_rule_95_b200 as g
from tests.parity import TOL, rel_err
import oracle

pytestmark = pytest.mark.gpu
WL = gi.WORKLOADS["decode_b256_h16"]


def _to(d, dev="cuda"):
    return {k: (None if v is None else v.to(dev)) for k, v in d.items()}


def _seq(tokens, key):
    """Stack per-step tokens [B,H,D] into a sequence [B,T,H,D] as float64."""
    return np.stack([gi.as_f64(t[key]) for t in tokens], axis=1)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
def test_decode_small(dtype, dk, dv):
    wl = dataclasses.replace(WL, dk=dk, dv=dv, dtype=dtype)
    B, H, steps = 3, 5, 6
    S = gi.decode_state(wl, B=B, H=H)
    toks = [gi.decode_tokens(wl, j, B=B, H=H) for j in range(steps)]
    Sd = S.cuda()
    outs = []
    for t in toks:
        td = _to(t)
        outs.append(g.gdn2_decode_step(td["q"], td["k"], td["v"], td["log_alpha"], td["b"], td["w"], Sd).float().cpu())
    torch.cuda.synchronize()
    seq = {k: _seq(toks, k) for k in ("q", "k", "v", "log_alpha", "b", "w")}
    o_ref, S_ref = oracle.forward(**seq, S0=gi.as_f64(S))
    o_gpu = torch.stack(outs, dim=1).numpy()
    assert rel_err(o_gpu, o_ref) <= TOL[dtype]
    assert rel_err(Sd.cpu().numpy(), S_ref) <= TOL[dtype]
    assert g.gdn2_device_status() == 0


def test_decode_full_size_1000_steps_sampled():
    """The benchmarked workload: B=256, H=16, d=128, 1000 steps, fresh tokens per
    step; o checked at sampled steps and S after step 1000 on sampled units."""
    steps = WL.steps
    S = gi.decode_state(WL)
    toks = gi.decode_tokens_many(WL, range(steps))
    Sd = S.cuda()
    check_steps = {0, 1, 2, 500, steps - 1}
    o_at = {}
    for j, t in enumerate(toks):
        td = _to(t)
        o = g.gdn2_decode_step(td["q"], td["k"], td["v"], td["log_alpha"], td["b"], td["w"], Sd)
        if j in check_steps:
            o_at[j] = o.float().cpu()
    S_gpu = Sd.cpu()
    assert torch.isfinite(S_gpu).all()
    units = [(0, 0), (17, 3), (128, 8), (255, 15), (200, 11)]
    seq = {k: np.stack([np.stack([gi.as_f64(t[k][b, h]) for t in toks]) for b, h in units])[:, :, None]
           for k in ("q", "k", "v", "log_alpha", "b", "w")}
    S0 = np.stack([gi.as_f64(S[b, h]) for b, h in units])[:, None]
    o_ref, S_ref = oracle.forward(**seq, S0=S0)
    for n, (b, h) in enumerate(units):
        for j in check_steps:
            assert rel_err(o_at[j][b, h].numpy(), o_ref[n, j, 0]) <= TOL["bf16"], (b, h, j)
        assert rel_err(S_gpu[b, h].numpy(), S_ref[n, 0]) <= TOL["bf16"], (b, h)
    assert g.gdn2_device_status() == 0
