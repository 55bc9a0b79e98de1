"""The seeded input generator: determinism and the recipe's value ranges (no GPU)."""
import numpy as np
import torch

import gdn2_inputs as gi


def test_deterministic_and_seed_sensitive():
    wl = gi.WORKLOADS["prefill_b8_h16_t4096"]
    a = gi.prefill_inputs(wl, B=1, T=64, H=2)
    b = gi.prefill_inputs(wl, B=1, T=64, H=2)
    c = gi.prefill_inputs(wl, B=1, T=64, H=2, seed=99)
    for k in ("q", "k", "v", "b", "w", "log_alpha"):
        assert torch.equal(a[k], b[k])
        assert not torch.equal(a[k], c[k])


def test_recipe_ranges():
    wl = gi.WORKLOADS["prefill_b8_h16_t4096"]
    d = gi.prefill_inputs(wl, B=1, T=128, H=2)
    for k in ("q", "k", "v", "b", "w"):
        assert d[k].dtype == torch.bfloat16 and d[k].shape == (1, 128, 2, 128)
    assert d["log_alpha"].dtype == torch.float32
    n = np.linalg.norm(gi.as_f64(d["k"]), axis=-1)
    assert np.all(np.abs(n - 1) < 1e-2)
    la = gi.as_f64(d["log_alpha"])
    assert la.max() < 0 and la.min() > -2
    for k in ("b", "w"):
        x = gi.as_f64(d[k])
        assert x.min() >= 0 and x.max() <= 1


def test_fp32_workload_is_fp32():
    d = gi.prefill_inputs(gi.WORKLOADS["tiny_f32"])
    assert d["q"].dtype == torch.float32 and d["q"].shape == (1, 256, 1, 64)


def test_heavy_decay_tail():
    heavy = gi.prefill_inputs(gi.WORKLOADS["long_b1_h16_t65536"], T=256, H=2)
    base = gi.prefill_inputs(gi.WORKLOADS["prefill_b8_h16_t4096"], B=1, T=256, H=2)
    assert heavy["log_alpha"].min() < 2 * base["log_alpha"].min()
    assert heavy["log_alpha"].mean() < 1.5 * base["log_alpha"].mean()


def test_mixed_gate_regimes():
    wl = gi.WORKLOADS["mixed_b4_h32_t8192"]
    d = gi.prefill_inputs(wl, B=1, T=64, H=6)
    b, w, la = (gi.as_f64(d[k]) for k in ("b", "w", "log_alpha"))
    for h in range(6):
        scalar_gate = np.all(b[0, :, h] == b[0, :, h, :1]) and np.array_equal(b[0, :, h], w[0, :, h])
        scalar_alpha = np.all(la[0, :, h] == la[0, :, h, :1])
        assert scalar_gate == (h % 3 <= 1)
        assert scalar_alpha == (h % 3 == 0)


def test_decode_steps_are_fresh():
    wl = gi.WORKLOADS["decode_b256_h16"]
    t0 = gi.decode_tokens(wl, 0, B=2, H=2)
    t1 = gi.decode_tokens(wl, 1, B=2, H=2)
    assert not torch.equal(t0["q"], t1["q"])
    S = gi.decode_state(wl, B=2, H=2)
    assert S.shape == (2, 2, 128, 128) and abs(float(S.std()) - 0.02) < 2e-3
