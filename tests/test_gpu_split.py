"""Sequence-split prefill on the GPU against the CPU oracle and the unsplit kernel
(parity): segment counts from 1 to 16 over ragged lengths, both head dimensions, entering
states, and the long-context workload with the library's segment choice."""
import dataclasses

import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import gated_delta_rule_95_b200 as g
import oracle
from tests.parity import TOL, oracle_units, rel_err

pytestmark = pytest.mark.gpu
BASE = gi.WORKLOADS["prefill_b8_h16_t4096"]
NAMES = ("q", "k", "v", "log_alpha", "b", "w")


def _cuda(d):
    return {k: (None if v is None else v.cuda()) for k, v in d.items()}


def _split(x, segments, want_state=True):
    # outputs start as NaN, so that anything the call fails to write shows
    B, T, H, _ = x["q"].shape
    dk, dv = x["q"].shape[-1], x["v"].shape[-1]
    o = torch.full((B, T, H, dv), float("nan"), device="cuda")
    S_T = torch.full((B, H, dk, dv), float("nan"), device="cuda") if want_state else None
    o, S = g.gdn2_chunk_fwd_split(*(x[n] for n in NAMES), x["S0"], segments=segments, o=o, S_T=S_T,
                                  want_state=want_state)
    torch.cuda.synchronize()
    return o, S


@pytest.mark.parametrize("d,T,segments", [(128, 1000, 2), (128, 1000, 3), (128, 1000, 5), (128, 1000, 16),
                                          (64, 777, 4), (128, 100, 4)])
def test_split_matches_oracle(d, T, segments):
    wl = dataclasses.replace(BASE, dk=d, dv=d, state_std=0.05)
    dd = gi.prefill_inputs(wl, B=2, T=T, H=2)
    x = _cuda(dd)
    o, S = _split(x, segments)
    assert g.gdn2_device_status() == 0
    f = {n: gi.as_f64(dd[n]) for n in NAMES}
    o_ref, S_ref = oracle.forward(**f, S0=gi.as_f64(dd["S0"]))
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["bf16"]


def test_one_segment_is_the_plain_forward():
    dd = gi.prefill_inputs(dataclasses.replace(BASE, state_std=0.05), B=2, T=300, H=2)
    x = _cuda(dd)
    o1, S1 = _split(x, 1)
    o2, S2 = g.gdn2_chunk_fwd(*(x[n] for n in NAMES), x["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_split_close_to_unsplit_and_no_state_out():
    dd = gi.prefill_inputs(BASE, B=1, T=4096, H=4)
    x = _cuda(dd)
    o1, _ = _split(x, 8, want_state=False)
    o2, S2 = g.gdn2_chunk_fwd(*(x[n] for n in NAMES), None)
    torch.cuda.synchronize()
    assert rel_err(o1.cpu().numpy(), o2.cpu().numpy()) <= TOL["bf16"]


def test_long_context_b1_h16_t65536_auto_segments():
    wl = gi.WORKLOADS["long_b1_h16_t65536"]
    dd = gi.prefill_inputs(wl)
    x = _cuda(dd)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    P = g.lib().gdn2_chunk_fwd_split_segments(wl.B, wl.T, wl.H, sms)
    assert P > 1
    o, S = _split(x, None)
    assert g.gdn2_device_status() == 0
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    units = [(0, 0), (0, 9)]
    refs = oracle_units(dd, units)
    o_c, S_c = o.cpu(), S.cpu()
    for (bb, h), (o_ref, S_ref) in zip(units, refs):
        assert rel_err(o_c[bb, :, h].numpy(), o_ref) <= TOL["bf16"], (bb, h)
        assert rel_err(S_c[bb, h].numpy(), S_ref) <= TOL["bf16"], (bb, h)
