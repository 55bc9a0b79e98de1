"""Packed variable-length prefill on the GPU against the CPU oracle (parity): ragged
lengths across chunk boundaries, empty sequences, entering states, state aliasing,
out-of-order offsets, and the full packed serving batch on sampled sequences."""
import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import gated_delta_rule_95_b200 as g
import oracle
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu
BASE = gi.WORKLOADS["prefill_b8_h16_t4096"]
GDN2_ERR_SHAPE = 2


def _run(d, S0="input", **kw):
    x = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    s0 = x["S0"] if S0 == "input" else S0
    o, S = g.gdn2_chunk_fwd_varlen(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["cu_seqlens"],
                                   s0, **kw)
    torch.cuda.synchronize()
    return o, S


def _oracle(d, seqs=None):
    f = {k: gi.as_f64(d[k]) for k in ("q", "k", "v", "log_alpha", "b", "w")}
    cu = d["cu_seqlens"].numpy()
    S0 = None if d["S0"] is None else gi.as_f64(d["S0"])
    if seqs is None:
        return oracle.forward_varlen(**f, cu_seqlens=cu, S0=S0)
    # only the sampled sequences: pack them on their own
    lens = [int(cu[n + 1] - cu[n]) for n in seqs]
    sub = {k: np.concatenate([f[k][cu[n]:cu[n + 1]] for n in seqs]) for k in f}
    cs = np.concatenate([[0], np.cumsum(lens)])
    s0 = None if S0 is None else S0[list(seqs)]
    return oracle.forward_varlen(**sub, cu_seqlens=cs, S0=s0), cs


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64)])
def test_ragged_lengths(dk, dv):
    import dataclasses
    wl = dataclasses.replace(BASE, dk=dk, dv=dv, state_std=0.05)
    lengths = [1, 63, 64, 65, 0, 200, 130, 7]
    d = gi.packed_inputs(wl, lengths, H=2)
    o, S = _run(d)
    o_ref, S_ref = _oracle(d)
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["bf16"]
    assert g.gdn2_device_status() == 0


def test_zero_states_and_no_state_out():
    lengths = [100, 3, 64]
    d = gi.packed_inputs(BASE, lengths, H=3, state_std=0.0)
    o, S = _run(d, want_state=False)
    assert S is None
    o_ref, _ = _oracle(d)
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]


def test_state_aliasing():
    lengths = [90, 17, 0, 64]
    d = gi.packed_inputs(BASE, lengths, H=2, state_std=0.05)
    S = d["S0"].clone().cuda()
    o, S_out = _run(d, S0=S, S_T=S)
    assert S_out.data_ptr() == S.data_ptr()
    o_ref, S_ref = _oracle(d)
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["bf16"]
    # the empty sequence keeps its entering state exactly
    assert torch.equal(S[2].cpu(), d["S0"][2])


def test_all_sequences_empty():
    d = gi.packed_inputs(BASE, [0, 0, 0], H=2, state_std=0.05)
    o, S = _run(d)
    assert o.numel() == 0
    assert torch.equal(S.cpu(), d["S0"])


def test_offsets_out_of_order_are_reported():
    d = gi.packed_inputs(BASE, [50, 50], H=1)
    d["cu_seqlens"] = torch.tensor([0, 70, 30], dtype=torch.int32)  # a negative length
    _run(d)
    assert g.gdn2_device_status() == GDN2_ERR_SHAPE
    assert g.gdn2_device_status() == 0  # reported once, then cleared


def test_full_packed_serving_batch_sampled():
    wl = gi.WORKLOADS["packed_n64_h16"]
    lengths = gi.packed_lengths(wl.B, 16, wl.T, wl.seed)
    d = gi.packed_inputs(wl, lengths)
    o, S = _run(d)
    assert g.gdn2_device_status() == 0
    order = np.argsort(lengths)
    seqs = [int(order[0]), int(order[len(order) // 2]), int(order[-1])]  # shortest, median, longest
    (o_ref, S_ref), cs = _oracle(d, seqs)
    cu = d["cu_seqlens"].numpy()
    o_c, S_c = o.cpu().numpy(), S.cpu().numpy()
    for i, n in enumerate(seqs):
        got_o = o_c[cu[n]:cu[n + 1]]
        ref_o = o_ref[cs[i]:cs[i + 1]]
        assert rel_err(got_o, ref_o) <= TOL["bf16"], n
        assert rel_err(S_c[n], S_ref[i]) <= TOL["bf16"], n
