"""The CPU oracle against what the pages and the mathematics fix (no GPU)."""
import numpy as np
import pytest

import oracle
from tests import pins


@pytest.mark.parametrize("pin", pins.ALL, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.load())


def test_decode_step_is_one_token_forward():
    d = pins.rand_case(40, T=1)
    o, S = oracle.forward(**d)
    sq = {k: v[:, 0] for k, v in d.items() if k != "S0"}
    o2, S2 = oracle.decode_step(S=d["S0"], **sq)
    assert np.array_equal(o[:, 0], o2) and np.array_equal(S, S2)


def test_empty_sequence_keeps_state():
    d = pins.rand_case(41, T=0)
    o, S = oracle.forward(**d)
    assert o.shape[1] == 0 and np.array_equal(S, d["S0"])


def test_zero_state_default():
    d = pins.rand_case(42)
    z = dict(d, S0=np.zeros_like(d["S0"]))
    o1, S1 = oracle.forward(**dict(d, S0=None))
    o2, S2 = oracle.forward(**z)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


def test_thread_count_does_not_change_result():
    d = pins.rand_case(43, B=3, H=5)
    o1, S1 = oracle.forward(**d, nthreads=1)
    o2, S2 = oracle.forward(**d, nthreads=7)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


def test_packed_sequences_are_independent_runs():
    """Packed variable-length sequences: the same tokens as equal-length batch rows give
    the batch result exactly; an empty sequence hands its entering state through; a
    sequence's result does not depend on its neighbours."""
    import numpy as np
    import gdn2_inputs as gi
    import oracle
    wl = gi.WORKLOADS["prefill_b8_h16_t4096"]
    d = gi.prefill_inputs(wl, B=3, T=40, H=2)
    f = {k: gi.as_f64(d[k]) for k in ("q", "k", "v", "log_alpha", "b", "w")}
    S0 = np.random.default_rng(0).normal(0, 0.05, (3, 2, 128, 128))
    o_ref, S_ref = oracle.forward(**f, S0=S0)
    packed = {k: f[k].reshape(120, 2, -1) for k in f}
    o, S = oracle.forward_varlen(**packed, cu_seqlens=np.array([0, 40, 80, 120]), S0=S0)
    assert np.array_equal(o.reshape(3, 40, 2, -1), o_ref) and np.array_equal(S, S_ref)
    # an empty sequence in the middle, and the neighbours unchanged
    S0e = np.concatenate([S0[:1], S0[1:2] * 3, S0[1:]])
    o2, S2 = oracle.forward_varlen(**packed, cu_seqlens=np.array([0, 40, 40, 80, 120]), S0=S0e)
    assert np.array_equal(S2[1], S0e[1]) and np.array_equal(o2, o)
    assert np.array_equal(S2[[0, 2, 3]], S)
