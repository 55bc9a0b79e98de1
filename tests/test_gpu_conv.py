"""The short causal convolution on the GPU against the CPU oracle (parity): fixed-length
and packed batches, carried history in and out (in place), streaming one token at a time,
bad offsets, and the full projection-sized tensor on sampled channels.

Tolerance, from the arithmetic: the kernel accumulates the four taps and the bias in fp32
(error at most a few units of 2^-24 of the sum of the terms' magnitudes) and rounds y to
its dtype (half an ulp: 2^-9 relative for bf16, 2^-24 for fp32)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_95_b200 as g
import oracle

pytestmark = pytest.mark.gpu
GDN2_ERR_SHAPE = 2


def _draw(shape, seed, dtype):
    x = torch.from_numpy(np.random.default_rng(seed).standard_normal(shape).astype(np.float32))
    return x.to(dtype)


def _params(C, seed, bias=True):
    rng = np.random.default_rng(seed)
    w = torch.from_numpy((0.5 * rng.standard_normal((C, 4))).astype(np.float32))
    b = torch.from_numpy((0.1 * rng.standard_normal(C)).astype(np.float32)) if bias else None
    return w, b


def _f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


def _check(y_gpu, x, w, b, hist, dtype):
    """y_gpu [T, C] against the oracle on one sequence x [T, C]."""
    xf, wf = _f64(x), _f64(w)
    y_ref, h_ref = oracle.short_conv(xf, wf, None if b is None else _f64(b), None if hist is None else _f64(hist))
    mag, _ = oracle.short_conv(np.abs(xf), np.abs(wf), None if b is None else np.abs(_f64(b)),
                               None if hist is None else np.abs(_f64(hist)))
    rel = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -23
    bound = rel * np.abs(y_ref) + 8 * 2.0 ** -24 * mag + 1e-30
    err = np.abs(_f64(y_gpu) - y_ref)
    assert np.all(err <= bound), float(np.max(err / bound))
    return h_ref


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("with_hist,bias", [(False, True), (True, True), (True, False)])
def test_fixed_length(dtype, with_hist, bias):
    B, T, C = 3, 37, 72
    x = _draw((B, T, C), 1, dtype)
    w, b = _params(C, 2, bias)
    hist = _draw((B, 3, C), 3, dtype) if with_hist else None
    y, h = g.gdn2_short_conv(x.cuda(), w.cuda(), None if b is None else b.cuda(),
                             hist=None if hist is None else hist.cuda(), want_hist=True)
    torch.cuda.synchronize()
    for n in range(B):
        h_ref = _check(y[n], x[n], w, b, None if hist is None else hist[n], dtype)
        assert np.array_equal(_f64(h[n]), h_ref)  # the history is a copy of inputs: exact
    assert g.gdn2_device_status() == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_packed_with_history_in_place(dtype):
    lengths = [0, 1, 2, 5, 40, 0, 17, 3]
    T, C = sum(lengths), 64
    x = _draw((T, C), 4, dtype)
    w, b = _params(C, 5)
    hist = _draw((len(lengths), 3, C), 6, dtype)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    hd = hist.cuda()
    y, h = g.gdn2_short_conv(x.cuda(), w.cuda(), b.cuda(), cu_seqlens=cu.cuda(), hist=hd, hist_out=hd)
    torch.cuda.synchronize()
    assert h.data_ptr() == hd.data_ptr()
    for n in range(len(lengths)):
        a, e = int(cu[n]), int(cu[n + 1])
        h_ref = _check(y[a:e], x[a:e], w, b, hist[n], dtype)
        assert np.array_equal(_f64(h[n]), h_ref), n
    assert g.gdn2_device_status() == 0


def test_streaming_one_token_at_a_time():
    # decode: T = 1 calls with the history updated in place equal one call over the tokens
    B, T, C = 4, 9, 128
    x = _draw((B, T, C), 7, torch.bfloat16).cuda()
    w, b = _params(C, 8)
    w, b = w.cuda(), b.cuda()
    y_all, h_all = g.gdn2_short_conv(x, w, b, want_hist=True)
    h = torch.zeros((B, 3, C), dtype=torch.bfloat16, device="cuda")
    ys = []
    for t in range(T):
        y_t, _ = g.gdn2_short_conv(x[:, t:t + 1].contiguous(), w, b, hist=h, hist_out=h)
        ys.append(y_t)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(ys, 1), y_all) and torch.equal(h, h_all)


def test_offsets_out_of_order_are_reported():
    x = _draw((30, 16), 9, torch.bfloat16).cuda()
    w, _ = _params(16, 10)
    cu = torch.tensor([0, 20, 10, 30], dtype=torch.int32).cuda()
    g.gdn2_short_conv(x, w.cuda(), cu_seqlens=cu, want_hist=True)
    assert g.gdn2_device_status() == GDN2_ERR_SHAPE
    assert g.gdn2_device_status() == 0


def test_full_projection_size_sampled():
    # q, k and v projections of the prefill workload side by side: B8 T4096, 3 x 16 x 128
    # channels; every token of 1024 sampled channels is checked
    B, T, C = 8, 4096, 6144
    x = _draw((B, T, C), 11, torch.bfloat16)
    w, b = _params(C, 12)
    y, h = g.gdn2_short_conv(x.cuda(), w.cuda(), b.cuda(), want_hist=True)
    torch.cuda.synchronize()
    assert g.gdn2_device_status() == 0
    cols = np.r_[0:512, C - 512:C]
    yc, hc = y.cpu(), h.cpu()
    for n in range(B):
        h_ref = _check(yc[n][:, cols], x[n][:, cols], w[cols], b[cols], None, torch.bfloat16)
        assert np.array_equal(_f64(hc[n][:, cols]), h_ref)
