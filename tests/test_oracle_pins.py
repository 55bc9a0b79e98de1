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
