"""Chunkwise prefill forward on the GPU against the CPU oracle (parity), through
the C ABI, from small ragged shapes to the full workloads on sampled units."""
import dataclasses

import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import gated_delta_rule_95_b200 as g
from tests.parity import TOL, check_units, rel_err
import oracle

pytestmark = pytest.mark.gpu
BASE = gi.WORKLOADS["prefill_b8_h16_t4096"]


def _cuda(d):
    return {k: (None if v is None else v.cuda()) for k, v in d.items()}


def _run(d, S0=None, **kw):
    x = _cuda(d)
    s0 = x["S0"] if S0 is None else S0
    o, S = g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], s0, **kw)
    torch.cuda.synchronize()
    return o, S


def _full_oracle(d):
    f = {k: gi.as_f64(d[k]) for k in ("q", "k", "v", "log_alpha", "b", "w")}
    return oracle.forward(**f, S0=None if d["S0"] is None else gi.as_f64(d["S0"]))


def test_tiny_f32_workload():
    wl = gi.WORKLOADS["tiny_f32"]
    d = gi.prefill_inputs(wl)
    o, S = _run(d)
    o_ref, S_ref = _full_oracle(d)
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["f32"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["f32"]


SHAPES = [  # B, T, H, dk, dv, with initial state
    (1, 64, 1, 128, 128, False), (2, 1, 3, 128, 128, True), (1, 63, 2, 128, 128, True),
    (1, 65, 2, 64, 64, False), (2, 200, 2, 128, 64, True), (1, 130, 1, 64, 128, True),
    (1, 256, 2, 128, 128, True), (3, 129, 1, 128, 128, False),
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,T,H,dk,dv,s0", SHAPES)
def test_shapes(dtype, B, T, H, dk, dv, s0):
    wl = dataclasses.replace(BASE, dk=dk, dv=dv, dtype=dtype, state_std=0.05 if s0 else 0.0, seed=100 + T)
    d = gi.prefill_inputs(wl, B=B, T=T, H=H)
    o, S = _run(d)
    o_ref, S_ref = _full_oracle(d)
    assert rel_err(o.float().cpu().numpy(), o_ref) <= TOL[dtype]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL[dtype]
    assert g.gdn2_device_status() == 0


def test_state_aliasing_and_no_state_out():
    wl = dataclasses.replace(BASE, state_std=0.05, seed=7)
    d = gi.prefill_inputs(wl, B=2, T=100, H=2)
    o1, S1 = _run(d)
    x = _cuda(d)
    S_inout = x["S0"].clone()
    o2, S2 = g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], S_inout, S_T=S_inout)
    o3, S3 = g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], want_state=False)
    torch.cuda.synchronize()
    assert S3 is None
    assert torch.equal(o1, o2) and torch.equal(o1, o3) and torch.equal(S1, S2)


def test_empty_sequence_copies_state():
    wl = dataclasses.replace(BASE, state_std=0.05, seed=8)
    d = gi.prefill_inputs(wl, B=2, T=0, H=3)
    o, S = _run(d)
    assert o.shape == (2, 0, 3, 128) and torch.equal(S.cpu(), d["S0"])
    d["S0"] = None
    o, S = _run(d)
    assert torch.count_nonzero(S) == 0


def test_split_handoff_matches_one_run():
    wl = dataclasses.replace(BASE, seed=9)
    d = gi.prefill_inputs(wl, B=2, T=200, H=2)
    o, S = _run(d)
    first = {k: (v[:, :72].contiguous() if k != "S0" else v) for k, v in d.items()}
    o1, S1 = _run(first)
    second = {k: (v[:, 72:].contiguous() if k != "S0" else None) for k, v in d.items()}
    o2, S2 = _run(second, S0=S1)
    assert rel_err(torch.cat([o1, o2], 1).float().cpu().numpy(), o.float().cpu().numpy()) <= TOL["bf16"]
    assert rel_err(S2.cpu().numpy(), S.cpu().numpy()) <= TOL["bf16"]


def test_decode_steps_match_chunk_forward():
    wl = dataclasses.replace(BASE, state_std=0.05, seed=10)
    d = gi.prefill_inputs(wl, B=2, T=100, H=2)
    o, S = _run(d)
    x = _cuda(d)
    Sd = x["S0"].clone()
    outs = []
    for t in range(100):
        sl = {k: x[k][:, t].contiguous() for k in ("q", "k", "v", "log_alpha", "b", "w")}
        outs.append(g.gdn2_decode_step(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["b"], sl["w"], Sd))
    od = torch.stack(outs, 1)
    torch.cuda.synchronize()
    assert rel_err(od.float().cpu().numpy(), o.float().cpu().numpy()) <= TOL["bf16"]
    assert rel_err(Sd.cpu().numpy(), S.cpu().numpy()) <= TOL["bf16"]


def _full_size(name):
    """The full workload in one launch; every (batch, head) unit checked element by element."""
    wl = gi.WORKLOADS[name]
    d = gi.prefill_inputs(wl)
    o, S = _run(d)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    eo, es = check_units(d, o.cpu(), S.cpu(), TOL["bf16"])
    print(f"{name}: every unit, worst o {eo:.2e}, worst S_T {es:.2e}")
    assert g.gdn2_device_status() == 0
    return d


def test_full_prefill_b8_h16_t4096_all_units():
    _full_size("prefill_b8_h16_t4096")


def test_full_mixed_gates_b4_h32_t8192_all_units():
    # 128 units: every head of every gate regime (head mod 3)
    _full_size("mixed_b4_h32_t8192")


def test_full_long_context_b1_h16_t65536_all_units():
    d = _full_size("long_b1_h16_t65536")
    # the chunk-start decay reference needs the in-chunk cumulative log decay > -80
    la = d["log_alpha"].view(1, -1, 64, 16, 128)
    g_min = float(torch.cumsum(la, dim=2).min())
    print(f"long-context workload: min in-chunk cumulative log decay = {g_min:.2f}")
    assert g_min > -80.0


@pytest.mark.parametrize("B,T,H", [(2, 130, 3), (1, 1, 2), (3, 64, 1), (1, 200, 4)])
def test_f32_d64_tensor_core_kernel(B, T, H):
    # fp32 inputs with d_k = d_v = 64 run on the split-product (3 x tf32) tensor-core kernel:
    # entering states, a single token, an exact chunk, ragged lengths, several heads
    wl = dataclasses.replace(BASE, dk=64, dv=64, dtype="f32", state_std=0.05, seed=400 + T)
    d = gi.prefill_inputs(wl, B=B, T=T, H=H)
    o, S = _run(d)
    o_ref, S_ref = _full_oracle(d)
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["f32"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["f32"]
    assert g.gdn2_device_status() == 0


def test_f32_d64_state_aliasing():
    wl = dataclasses.replace(BASE, dk=64, dv=64, dtype="f32", state_std=0.05, seed=77)
    d = gi.prefill_inputs(wl, B=2, T=100, H=2)
    o1, S1 = _run(d)
    x = _cuda(d)
    S_inout = x["S0"].clone()
    o2, S2 = g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], S_inout, S_T=S_inout)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
