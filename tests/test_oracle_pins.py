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


# ---- the input activations of the raw-projection entry point ------------------------------

def _act(q=None, k=None, a=None, b=None, w=None, scale=None, H=1, D=4):
    z = np.zeros((1, 1, H, D))
    f = lambda x: z if x is None else np.asarray(x, dtype=np.float64).reshape(1, 1, H, D)
    return oracle.activations(f(q), f(k), f(a), f(b), f(w), scale)


def test_activations_closed_forms():
    # a 3-4-5 vector normalises to (0.6, 0.8); a zero vector stays zero
    r = _act(q=[3.0, 4.0, 0.0, 0.0], k=[0.0, 0.0, 0.0, 0.0])
    assert np.allclose(r["q"].ravel(), [0.6, 0.8, 0.0, 0.0], rtol=0, atol=1e-15)
    assert np.array_equal(r["k"].ravel(), np.zeros(4))
    # sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4
    r = _act(b=[0.0, np.log(3.0), -np.log(3.0), 0.0], w=[np.log(3.0), 0.0, 0.0, -np.log(3.0)])
    assert np.allclose(r["b"].ravel(), [0.5, 0.75, 0.25, 0.5], rtol=0, atol=1e-15)
    assert np.allclose(r["w"].ravel(), [0.75, 0.5, 0.5, 0.25], rtol=0, atol=1e-15)
    # softplus(0) = ln 2, softplus(ln(e - 1)) = 1, softplus(50) = 50 (to 2e-22),
    # softplus(-50) = e^-50 (to first order): log alpha = -s softplus(a), s = 0.25
    r = _act(a=[0.0, np.log(np.e - 1.0), 50.0, -50.0], scale=[0.25])
    want = -0.25 * np.array([np.log(2.0), 1.0, 50.0, np.exp(-50.0)])
    assert np.allclose(r["log_alpha"].ravel(), want, rtol=1e-14, atol=0)


def test_activations_identities():
    rng = np.random.default_rng(7)
    x = 6.0 * rng.standard_normal((2, 3, 4, 8))
    H = x.shape[-2]
    p = oracle.activations(x, x, x, x, x, np.full(H, 1.0))
    m = oracle.activations(-x, -x, -x, -x, -x, np.full(H, 1.0))
    # sigmoid(x) + sigmoid(-x) = 1; softplus(x) - softplus(-x) = x; unit norms, directions kept
    assert np.allclose(p["b"] + m["b"], 1.0, rtol=0, atol=1e-15)
    assert np.allclose(-p["log_alpha"] + m["log_alpha"], x, rtol=0, atol=1e-13)
    assert np.allclose(np.linalg.norm(p["q"], axis=-1), 1.0, rtol=0, atol=1e-15)
    assert np.allclose(p["q"] * np.linalg.norm(x, axis=-1, keepdims=True), x, rtol=0, atol=1e-13)
    # the per-head scale multiplies log alpha of its own head only
    s = np.array([1.0, 2.0, 0.5, 3.0])
    q = oracle.activations(x, x, x, x, x, s)
    assert np.allclose(q["log_alpha"], p["log_alpha"] * s[:, None], rtol=1e-15, atol=0)
    # every decay lies in (0, 1) and every gate in (0, 1)
    assert np.all(p["log_alpha"] < 0) and np.all((p["w"] > 0) & (p["w"] < 1))


# ---- the short convolution -----------------------------------------------------------------

def test_short_conv_is_a_truncated_full_convolution():
    # y[:, c] equals numpy's full convolution with the taps reversed, cut to the first T
    rng = np.random.default_rng(11)
    x = rng.standard_normal((37, 6))
    w = rng.standard_normal((6, 4))
    bias = rng.standard_normal(6)
    y, _ = oracle.short_conv(x, w, bias)
    for c in range(6):
        ref = np.convolve(x[:, c], w[c, ::-1])[:37] + bias[c]
        assert np.allclose(y[:, c], ref, rtol=0, atol=1e-13)


def test_short_conv_impulse_and_causality():
    w = np.arange(1.0, 9.0).reshape(2, 4)
    x = np.zeros((8, 2))
    x[2] = 1.0  # an impulse at token 2: y[2 + s] = w[:, 3 - s] for s = 0..3, zero elsewhere
    y, hist = oracle.short_conv(x, w)
    want = np.zeros((8, 2))
    for s in range(4):
        want[2 + s] = w[:, 3 - s]
    assert np.array_equal(y, want)
    assert np.array_equal(hist, x[-3:])
    # a change at token 5 leaves tokens 0..4 alone
    x2 = x.copy()
    x2[5] = 7.0
    y2, _ = oracle.short_conv(x2, w)
    assert np.array_equal(y2[:5], y[:5]) and not np.array_equal(y2[5:], y[5:])


@pytest.mark.parametrize("cut", [1, 2, 3, 10])
def test_short_conv_history_handoff(cut):
    # splitting a sequence and carrying the last three inputs equals one run, also when the
    # first part is shorter than the window
    rng = np.random.default_rng(12)
    x = rng.standard_normal((20, 5))
    w = rng.standard_normal((5, 4))
    h0 = rng.standard_normal((3, 5))
    y, h = oracle.short_conv(x, w, None, h0)
    ya, ha = oracle.short_conv(x[:cut], w, None, h0)
    yb, hb = oracle.short_conv(x[cut:], w, None, ha)
    assert np.allclose(np.concatenate([ya, yb]), y, rtol=0, atol=1e-13)
    assert np.array_equal(hb, h)
    if cut < 3:  # the old history's tail survives in front of the new tokens
        assert np.array_equal(ha[:3 - cut], h0[cut:])
