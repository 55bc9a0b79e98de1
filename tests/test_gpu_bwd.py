"""Backward pass on the GPU against the fp64 gradient oracle (parity): fp32 and bf16
inputs, ragged lengths, both head sizes, with and without entering-state and final-state
gradients, and a consistency check against finite differences of the GPU forward."""
import dataclasses

import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import gated_delta_rule_95_b200 as g
from oracle import backward as ob
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu
BASE = gi.WORKLOADS["prefill_b8_h16_t4096"]
NAMES = ("q", "k", "v", "log_alpha", "b", "w")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0")


def _cot(B, T, H, dk, dv, seed):
    rng = np.random.default_rng(seed)
    do = torch.from_numpy(rng.standard_normal((B, T, H, dv)).astype(np.float32))
    dS = torch.from_numpy(rng.standard_normal((B, H, dk, dv)).astype(np.float32))
    return do, dS


def _check(d, do, dS, dtype, with_dS=True):
    x = {k_: (None if v_ is None else v_.cuda()) for k_, v_ in d.items()}
    gg = g.gdn2_chunk_bwd(*(x[n] for n in NAMES), x["S0"], do.cuda(), dS.cuda() if with_dS else None)
    torch.cuda.synchronize()
    assert g.gdn2_device_status() == 0
    ref = ob.backward(**{n: gi.as_f64(d[n]) for n in NAMES}, S0=None if d["S0"] is None else gi.as_f64(d["S0"]),
                      do=do.double().numpy(), dS_T=dS.double().numpy() if with_dS else None)
    for n in GRADS:
        err = rel_err(gg[n].cpu().numpy(), ref[n])
        assert err <= TOL[dtype], (n, err)


@pytest.mark.parametrize("dk,dv,T", [(64, 64, 150), (128, 128, 200), (128, 64, 64), (64, 128, 65)])
def test_bwd_f32(dk, dv, T):
    wl = dataclasses.replace(BASE, dk=dk, dv=dv, dtype="f32", state_std=0.05)
    d = gi.prefill_inputs(wl, B=2, T=T, H=2)
    do, dS = _cot(2, T, 2, dk, dv, 7)
    _check(d, do, dS, "f32")


@pytest.mark.parametrize("with_S0,with_dS", [(True, True), (False, True), (True, False)])
def test_bwd_bf16(with_S0, with_dS):
    wl = dataclasses.replace(BASE, state_std=0.05 if with_S0 else 0.0)
    d = gi.prefill_inputs(wl, B=1, T=300, H=3)
    do, dS = _cot(1, 300, 3, 128, 128, 8)
    _check(d, do, dS, "bf16", with_dS)


def test_bwd_long_sequence_sampled_units():
    # 2048 tokens (32 chunks) of the prefill workload's recipe, all 4 heads against the oracle
    d = gi.prefill_inputs(dataclasses.replace(BASE, state_std=0.02), B=1, T=2048, H=4)
    do, dS = _cot(1, 2048, 4, 128, 128, 9)
    _check(d, do, dS, "bf16")


def test_bwd_no_tokens():
    d = gi.prefill_inputs(dataclasses.replace(BASE, state_std=0.05), B=1, T=0, H=2)
    do, dS = _cot(1, 0, 2, 128, 128, 10)
    x = {k_: (None if v_ is None else v_.cuda()) for k_, v_ in d.items()}
    gg = g.gdn2_chunk_bwd(*(x[n] for n in NAMES), x["S0"], do.cuda(), dS.cuda())
    torch.cuda.synchronize()
    assert torch.equal(gg["dS0"].cpu(), dS)


def test_bwd_full_prefill_b8_h16_t4096_sampled_units():
    # the bench's backward workload; two (batch, head) units against the oracle, whose
    # gradients depend on that unit's inputs and cotangents only
    wl = BASE
    d = gi.prefill_inputs(wl)
    do, dS = _cot(wl.B, wl.T, wl.H, wl.dk, wl.dv, 11)
    x = {k_: (None if v_ is None else v_.cuda()) for k_, v_ in d.items()}
    gg = g.gdn2_chunk_bwd(*(x[n] for n in NAMES), x["S0"], do.cuda(), dS.cuda())
    torch.cuda.synchronize()
    assert g.gdn2_device_status() == 0
    for bb, h in [(0, 0), (6, 11)]:
        sl = {n: gi.as_f64(d[n][bb:bb + 1, :, h:h + 1]) for n in NAMES}
        ref = ob.backward(**sl, S0=None, do=do[bb:bb + 1, :, h:h + 1].double().numpy(),
                          dS_T=dS[bb:bb + 1, h:h + 1].double().numpy())
        for n in GRADS:
            got = gg[n][bb:bb + 1, h:h + 1] if n == "dS0" else gg[n][bb:bb + 1, :, h:h + 1]
            err = rel_err(got.cpu().numpy(), ref[n])
            assert err <= TOL["bf16"], (bb, h, n, err)


@pytest.mark.parametrize("T", [1, 37, 64, 129])
def test_bwd_bf16_short_and_exact_chunks(T):
    # a single partial chunk, exactly one chunk, one chunk and a token
    wl = dataclasses.replace(BASE, state_std=0.05)
    d = gi.prefill_inputs(wl, B=2, T=T, H=2)
    do, dS = _cot(2, T, 2, 128, 128, 20 + T)
    _check(d, do, dS, "bf16")


def test_bwd_bf16_many_units_ragged_sampled():
    # 2016 (batch, head, chunk) units, more than one per SM, the last chunk of every sequence
    # partial; two (batch, head) units against the oracle
    wl = dataclasses.replace(BASE, state_std=0.02)
    B, T, H = 2, 4000, 16
    d = gi.prefill_inputs(wl, B=B, T=T, H=H)
    do, dS = _cot(B, T, H, 128, 128, 21)
    x = {k_: (None if v_ is None else v_.cuda()) for k_, v_ in d.items()}
    gg = g.gdn2_chunk_bwd(*(x[n] for n in NAMES), x["S0"], do.cuda(), dS.cuda())
    torch.cuda.synchronize()
    assert g.gdn2_device_status() == 0
    for bb, h in [(0, 0), (1, 15)]:
        sl = {n: gi.as_f64(d[n][bb:bb + 1, :, h:h + 1]) for n in NAMES}
        ref = ob.backward(**sl, S0=gi.as_f64(d["S0"][bb:bb + 1, h:h + 1]),
                          do=do[bb:bb + 1, :, h:h + 1].double().numpy(),
                          dS_T=dS[bb:bb + 1, h:h + 1].double().numpy())
        for n in GRADS:
            got = gg[n][bb:bb + 1, h:h + 1] if n == "dS0" else gg[n][bb:bb + 1, :, h:h + 1]
            err = rel_err(got.cpu().numpy(), ref[n])
            assert err <= TOL["bf16"], (bb, h, n, err)


def test_bwd_bf16_without_dS0():
    # the entering-state gradient not requested (NULL): the other gradients unchanged
    wl = dataclasses.replace(BASE, state_std=0.05)
    d = gi.prefill_inputs(wl, B=1, T=200, H=2)
    do, dS = _cot(1, 200, 2, 128, 128, 22)
    x = {k_: (None if v_ is None else v_.cuda()) for k_, v_ in d.items()}
    args = [x[n] for n in NAMES]
    full = g.gdn2_chunk_bwd(*args, x["S0"], do.cuda(), dS.cuda())
    part = g.gdn2_chunk_bwd(*args, x["S0"], do.cuda(), dS.cuda(), want_dS0=False)
    torch.cuda.synchronize()
    assert part["dS0"] is None
    for n in GRADS[:-1]:
        assert torch.equal(full[n], part[n]), n
