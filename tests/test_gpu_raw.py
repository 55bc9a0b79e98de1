"""Prefill on the raw projections (normalisation and gate activations inside the kernel)
on the GPU against the CPU oracle's activations followed by its recurrence (parity):
ragged shapes, per-head decay scales, packed sequences, extreme logits and zero
vectors, and the full-size workload on sampled units."""
import dataclasses

import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import gated_delta_rule_95_b200 as g
import oracle
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu
BASE = gi.WORKLOADS["prefill_b8_h16_t4096"]
RAW = ("q_raw", "k_raw", "v", "a_raw", "b_raw", "w_raw")


def _run(d, scale="input", cu=None, **kw):
    x = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    s = x["decay_scale"] if scale == "input" else scale
    o, S = g.gdn2_chunk_fwd_raw(*(x[n] for n in RAW), x["S0"], decay_scale=s,
                                cu_seqlens=None if cu is None else cu.cuda(), **kw)
    torch.cuda.synchronize()
    return o, S


def _act(d, scale):
    f = {n: gi.as_f64(d[n]) for n in RAW}
    a = oracle.activations(f["q_raw"], f["k_raw"], f["a_raw"], f["b_raw"], f["w_raw"], scale)
    return dict(q=a["q"], k=a["k"], v=f["v"], log_alpha=a["log_alpha"], b=a["b"], w=a["w"])


def _oracle(d, scale):
    S0 = None if d["S0"] is None else gi.as_f64(d["S0"])
    return oracle.forward(**_act(d, scale), S0=S0)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
def test_ragged_shapes_with_head_scales(dk, dv):
    wl = dataclasses.replace(BASE, dk=dk, dv=dv, state_std=0.05)
    d = gi.raw_inputs(wl, B=2, T=200, H=3)  # 3 full chunks and a tail of 8
    d["decay_scale"] = torch.tensor([1 / 16, 1 / 8, 1 / 2], dtype=torch.float32)
    o, S = _run(d)
    o_ref, S_ref = _oracle(d, d["decay_scale"].numpy())
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["bf16"]
    assert g.gdn2_device_status() == 0


def test_default_scale_is_one_and_no_state_out():
    d = gi.raw_inputs(BASE, B=1, T=130, H=2)
    d["a_raw"] = d["a_raw"] - 4.0  # softplus(a - 4) keeps the unit-scale decay mild
    o, S = _run(d, scale=None, want_state=False)
    assert S is None
    o_ref, _ = _oracle(d, None)
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]


def test_extreme_logits_and_zero_vectors():
    d = gi.raw_inputs(dataclasses.replace(BASE, state_std=0.05), B=1, T=96, H=2)
    for n in ("b_raw", "w_raw"):
        x = d[n].float()
        x[0, ::3] *= 30.0  # saturated gates, both signs
        d[n] = x.to(torch.bfloat16)
    a = d["a_raw"]
    a[0, 5] = 400.0   # log alpha = -25: a near-total decay
    a[0, 6] = -40.0   # softplus(-40): no decay
    d["q_raw"][0, 10] = 0
    d["k_raw"][0, 11] = 0  # a zero key: no erase, no write
    d["q_raw"][0, 12] *= 1000  # scale does not matter after normalisation
    o, S = _run(d)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    o_ref, S_ref = _oracle(d, d["decay_scale"].numpy())
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["bf16"]
    assert torch.count_nonzero(o[0, 10].cpu()) == 0  # q = 0 reads nothing


def test_packed_sequences():
    wl = dataclasses.replace(BASE, state_std=0.05)
    lengths = [1, 63, 64, 65, 0, 130, 7]
    T = sum(lengths)
    d0 = gi.raw_inputs(wl, B=1, T=T, H=2)
    d = {n: d0[n][0] for n in RAW}
    d["decay_scale"] = d0["decay_scale"]
    d["S0"] = gi.packed_inputs(wl, lengths, H=2)["S0"]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    o, S = _run(d, cu=cu)
    assert g.gdn2_device_status() == 0
    a = _act(d, d["decay_scale"].numpy())
    o_ref, S_ref = oracle.forward_varlen(**a, cu_seqlens=cu.numpy(), S0=gi.as_f64(d["S0"]))
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["bf16"]
    assert torch.equal(S[4].cpu(), d["S0"][4])  # the empty sequence keeps its state


def test_no_tokens_copies_state():
    wl = dataclasses.replace(BASE, state_std=0.05)
    d = gi.raw_inputs(wl, B=2, T=0, H=2)
    o, S = _run(d)
    assert o.numel() == 0 and torch.equal(S.cpu(), d["S0"])


def test_full_prefill_b8_h16_t4096_sampled():
    d = gi.raw_inputs(BASE)
    o, S = _run(d)
    assert g.gdn2_device_status() == 0
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    units = [(0, 0), (4, 9), (7, 15)]
    sub = {n: torch.cat([d[n][bb:bb + 1, :, h:h + 1] for bb, h in units], 0) for n in RAW}
    scale = d["decay_scale"].numpy()
    assert np.all(scale == scale[0])  # every head of the workload has the same scale
    a = _act(sub, scale[:1])
    o_ref, S_ref = oracle.forward(**a)
    o_c, S_c = o.cpu(), S.cpu()
    for n, (bb, h) in enumerate(units):
        assert rel_err(o_c[bb, :, h].numpy(), o_ref[n, :, 0]) <= TOL["bf16"], (bb, h)
        assert rel_err(S_c[bb, h].numpy(), S_ref[n, 0]) <= TOL["bf16"], (bb, h)


# ---- decode on raw projections ---------------------------------------------------------------

@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("bf16", 64, 128), ("f32", 128, 64), ("f32", 64, 64)])
def test_decode_raw_matches_oracle(dtype, dk, dv):
    wl = dataclasses.replace(BASE, dk=dk, dv=dv, dtype=dtype, state_std=0.05)
    d = gi.raw_inputs(wl, B=4, T=1, H=3)
    d["decay_scale"] = torch.tensor([1 / 16, 1 / 4, 1.0], dtype=torch.float32)
    d["q_raw"][1, 0, 2] = 0  # a zero query
    x = {n: d[n][:, 0].contiguous().cuda() for n in RAW}
    S = d["S0"].clone().cuda()
    o = g.gdn2_decode_step_raw(*(x[n] for n in RAW), S, decay_scale=d["decay_scale"].cuda())
    torch.cuda.synchronize()
    a = _act({n: d[n][:, 0] for n in RAW}, d["decay_scale"].numpy())
    o_ref, S_ref = oracle.decode_step(a["q"], a["k"], a["v"], a["log_alpha"], a["b"], a["w"], gi.as_f64(d["S0"]))
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL[dtype]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL[dtype]
    assert torch.count_nonzero(o[1, 2].cpu()) == 0


def test_decode_raw_steps_equal_chunk_forward_raw():
    d = gi.raw_inputs(dataclasses.replace(BASE, state_std=0.05), B=2, T=70, H=2)
    o_c, S_c = _run(d)
    x = {n: d[n].cuda() for n in RAW}
    S = d["S0"].clone().cuda()
    outs = [g.gdn2_decode_step_raw(*(x[n][:, t].contiguous() for n in RAW), S,
                                   decay_scale=d["decay_scale"].cuda()) for t in range(70)]
    od = torch.stack(outs, 1)
    torch.cuda.synchronize()
    assert rel_err(od.cpu().numpy(), o_c.cpu().numpy()) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_c.cpu().numpy()) <= TOL["bf16"]


GDN2_ERR_RANGE = 7


def test_decay_beyond_the_chunk_range_is_flagged():
    """The chunk form scales keys by exp(-g) with g the in-chunk cumulative log decay; below
    g = -80 that leaves the fp32 range.  With s_h = 1 and a_raw shifted by +3 (softplus(3) is
    about 3.05 per token, about -195 over a chunk), the raw entry must report the range
    error through the device status; an in-range call afterwards reports clean again."""
    wl = dataclasses.replace(BASE, seed=31)
    d = gi.raw_inputs(wl, B=1, T=128, H=2)
    d["a_raw"] = (d["a_raw"] + 3.0).contiguous()
    _run(d, scale=None)
    assert g.gdn2_device_status() == GDN2_ERR_RANGE
    d = gi.raw_inputs(wl, B=1, T=128, H=2)
    o, S = _run(d)
    assert g.gdn2_device_status() == 0
    o_ref, S_ref = _oracle(d, gi.as_f64(d["decay_scale"]))
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]


def test_plain_entry_flags_decay_beyond_the_chunk_range():
    """Same bound on the plain entry: log alpha = -2 per token gives -128 over a chunk."""
    wl = dataclasses.replace(BASE, seed=32)
    d = gi.prefill_inputs(wl, B=1, T=64, H=1)
    x = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    la = torch.full_like(x["log_alpha"], -2.0)
    g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], la, x["b"], x["w"], None)
    assert g.gdn2_device_status() == GDN2_ERR_RANGE
    g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], None)
    assert g.gdn2_device_status() == 0
