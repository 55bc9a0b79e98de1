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


def test_decode_full_size_1000_steps_256_units():
    """The benchmarked workload: B=256, H=16, d=128, 1000 steps, fresh tokens per step.
    o is checked element by element at steps 0, 1, 500 and 999 and S after step 1000, on
    256 (sequence, head) units spread over every sequence block and every head."""
    steps = WL.steps
    S = gi.decode_state(WL)
    toks = gi.decode_tokens_many(WL, range(steps))
    Sd = S.cuda()
    check_steps = (0, 1, 500, steps - 1)
    o_at = {}
    for j, t in enumerate(toks):
        td = _to(t)
        o = g.gdn2_decode_step(td["q"], td["k"], td["v"], td["log_alpha"], td["b"], td["w"], Sd)
        if j in check_steps:
            o_at[j] = o.float().cpu()
    S_gpu = Sd.cpu()
    assert torch.isfinite(S_gpu).all()
    # unit n = (sequence n, head (7 n) mod 16): all 256 sequences, every head 16 times
    bs = np.arange(WL.B)
    hs = (7 * bs) % WL.H
    seq = {k: np.stack([gi.as_f64(t[k][bs, hs]) for t in toks], axis=1)[:, :, None]
           for k in ("q", "k", "v", "log_alpha", "b", "w")}
    S0 = gi.as_f64(S[bs, hs])[:, None]
    o_ref, S_ref = oracle.forward(**seq, S0=S0)
    worst = 0.0
    for n, (b, h) in enumerate(zip(bs, hs)):
        for j in check_steps:
            e = rel_err(o_at[j][b, h].numpy(), o_ref[n, j, 0])
            assert e <= TOL["bf16"], (b, h, j, e)
            worst = max(worst, e)
        e = rel_err(S_gpu[b, h].numpy(), S_ref[n, 0])
        assert e <= TOL["bf16"], (b, h, e)
        worst = max(worst, e)
    print(f"decode 1000 steps, 256 units: worst error {worst:.2e}")
    assert g.gdn2_device_status() == 0
