"""The gradient oracle against the forward oracle (no GPU): central finite differences of
the fp64 recurrence for every input and the entering state, and the chunkwise reverse-mode
re-derivation against the token-level one for several chunk sizes."""
import numpy as np
import pytest

import oracle
from oracle import backward as ob
from oracle import chunkwise as cw


def _case(seed, B=1, T=9, H=2, dk=4, dv=3, decay=0.3):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    d = dict(q=rng.standard_normal((B, T, H, dk)), k=k, v=rng.standard_normal((B, T, H, dv)),
             log_alpha=-decay * rng.random((B, T, H, dk)), b=rng.random((B, T, H, dk)),
             w=rng.random((B, T, H, dv)), S0=rng.standard_normal((B, H, dk, dv)))
    return d, rng.standard_normal((B, T, H, dv)), rng.standard_normal((B, H, dk, dv))


def _loss(d, do, dS):
    o, S = oracle.forward(**d)
    return float(np.sum(o * do) + np.sum(S * dS))


GRAD = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "b": "db", "w": "dw", "S0": "dS0"}


@pytest.mark.parametrize("seed", [1, 2])
def test_gradients_match_finite_differences(seed):
    d, do, dS = _case(seed)
    g = ob.backward(**d, do=do, dS_T=dS)
    eps = 1e-6
    for name, gname in GRAD.items():
        x = d[name]
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            fd = (_loss(dict(d, **{name: xp}), do, dS) - _loss(dict(d, **{name: xm}), do, dS)) / (2 * eps)
            assert abs(fd - g[gname][idx]) <= 1e-7 * max(1.0, abs(fd)), (name, idx, fd, g[gname][idx])


def test_zero_cotangents_give_zero_gradients():
    d, do, dS = _case(3)
    g = ob.backward(**d, do=np.zeros_like(do), dS_T=None)
    assert all(np.array_equal(v, np.zeros_like(v)) for v in g.values())


@pytest.mark.parametrize("C,T", [(1, 5), (4, 13), (5, 13), (16, 13), (64, 70)])
def test_chunkwise_backward_matches_token_backward(C, T):
    d, do, dS = _case(10 + C, T=T, dk=6, dv=5)
    g1 = ob.backward(**d, do=do, dS_T=dS)
    g2 = cw.backward(**d, do=do, dS_T=dS, C=C)
    for n in g1:
        assert np.allclose(g1[n], g2[n], rtol=1e-10, atol=1e-11), n
