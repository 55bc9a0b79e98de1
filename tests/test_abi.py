"""The C ABI library on the host: it loads, exports every symbol the header
declares, and rejects bad arguments before touching CUDA (no GPU needed)."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_95_b200 as g

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            with open(os.path.join(ROOT, "include", fn)) as f:
                names += re.findall(r"GDN2_API[^;(]*?\b(gdn2_\w+)\s*\(", f.read())
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = header_symbols()
    assert "gdn2_chunk_fwd" in names and "gdn2_decode_step" in names


@pytest.mark.parametrize("name", header_symbols())
def test_library_exports(name):
    assert hasattr(g.lib(), name)


def test_version_and_status_strings():
    L = g.lib()
    assert L.gdn2_version() >= 100
    for s in range(8):
        assert L.gdn2_status_string(s) and L.gdn2_status_string(s) != b"unknown status"
    assert L.gdn2_status_string(8) == b"unknown status"


P = ctypes.c_void_p
A = P(0x10000)   # aligned, never dereferenced: validation fails before any use
M = P(0x10008)   # misaligned


def chunk(q=A, k=A, v=A, la=A, b=A, w=A, S0=None, o=A, ST=None, B=1, T=64, H=1, dk=128, dv=128, dt=1):
    return g.lib().gdn2_chunk_fwd(q, k, v, la, b, w, S0, o, ST, B, T, H, dk, dv, dt, None)


def decode(q=A, k=A, v=A, la=A, b=A, w=A, S=A, o=A, B=1, H=1, dk=128, dv=128, dt=1):
    return g.lib().gdn2_decode_step(q, k, v, la, b, w, S, o, B, H, dk, dv, dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dk=96), 2), (dict(dv=32), 2), (dict(B=-1), 2), (dict(T=-5), 2), (dict(H=-1), 2),
    (dict(dt=7), 3), (dict(q=None), 1), (dict(o=None), 1), (dict(la=None), 1),
    (dict(k=M), 4), (dict(S0=M), 4), (dict(ST=M), 4),
    (dict(B=0), 0), (dict(H=0), 0),
])
def test_chunk_fwd_validation(kw, status):
    assert chunk(**kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(dk=80), 2), (dict(B=-2), 2), (dict(dt=2), 3), (dict(S=None), 1), (dict(w=None), 1),
    (dict(v=M), 4), (dict(S=M), 4), (dict(B=0), 0),
])
def test_decode_step_validation(kw, status):
    assert decode(**kw) == status


def varlen(q=A, k=A, v=A, la=A, b=A, w=A, cu=A, S0=None, o=A, ST=None, N=2, T=100, H=1, dk=128, dv=128, dt=1):
    return g.lib().gdn2_chunk_fwd_varlen(q, k, v, la, b, w, cu, S0, o, ST, N, T, H, dk, dv, dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dk=96), 2), (dict(N=-1), 2), (dict(T=-1), 2), (dict(dt=0), 3), (dict(dt=5), 3),
    (dict(cu=None), 1), (dict(q=None), 1), (dict(o=None), 1),
    (dict(cu=P(0x10002)), 4), (dict(v=M), 4), (dict(ST=M), 4),
    (dict(N=0), 0), (dict(H=0), 0),
])
def test_chunk_fwd_varlen_validation(kw, status):
    assert varlen(**kw) == status


def raw(q=A, k=A, v=A, a=A, b=A, w=A, sc=None, cu=None, S0=None, o=A, ST=None, B=2, T=100, H=1, dk=128, dv=128,
        dt=1):
    return g.lib().gdn2_chunk_fwd_raw(q, k, v, a, b, w, sc, cu, S0, o, ST, B, T, H, dk, dv, dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dk=96), 2), (dict(B=-1), 2), (dict(T=-1), 2), (dict(dt=0), 3), (dict(dt=7), 3),
    (dict(q=None), 1), (dict(a=None), 1), (dict(w=None), 1), (dict(o=None), 1),
    (dict(sc=P(0x10002)), 4), (dict(cu=P(0x10001)), 4), (dict(b=M), 4), (dict(S0=M), 4),
    (dict(B=0), 0), (dict(H=0), 0), (dict(cu=A, B=0), 0),
])
def test_chunk_fwd_raw_validation(kw, status):
    assert raw(**kw) == status


def conv(x=A, w=A, b=None, cu=None, hi=None, y=P(0x20000), ho=None, B=2, T=10, C=64, dt=1):
    return g.lib().gdn2_short_conv(x, w, b, cu, hi, y, ho, B, T, C, dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(C=60), 2), (dict(C=-8), 2), (dict(B=-1), 2), (dict(T=-1), 2), (dict(dt=4), 3),
    (dict(x=None), 1), (dict(w=None), 1), (dict(y=None), 1),
    (dict(y=A), 2),  # y aliasing x
    (dict(b=P(0x10008)), 4), (dict(hi=P(0x10004)), 4), (dict(cu=P(0x10002)), 4),
    (dict(B=0), 0), (dict(C=0), 0),
])
def test_short_conv_validation(kw, status):
    assert conv(**kw) == status


def decode_raw(q=A, k=A, v=A, a=A, b=A, w=A, sc=None, S=A, o=A, B=2, H=1, dk=128, dv=128, dt=1):
    return g.lib().gdn2_decode_step_raw(q, k, v, a, b, w, sc, S, o, B, H, dk, dv, dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dk=80), 2), (dict(B=-2), 2), (dict(dt=2), 3), (dict(S=None), 1), (dict(a=None), 1),
    (dict(v=M), 4), (dict(sc=P(0x10002)), 4), (dict(B=0), 0),
])
def test_decode_step_raw_validation(kw, status):
    assert decode_raw(**kw) == status


def split(q=A, k=A, v=A, la=A, b=A, w=A, S0=None, o=A, ST=None, B=1, T=1000, H=2, dk=128, dv=128, dt=1, seg=4,
          ws=P(0x40000), wsb=1 << 30):
    return g.lib().gdn2_chunk_fwd_split(q, k, v, la, b, w, S0, o, ST, B, T, H, dk, dv, dt, seg, ws, wsb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dk=64), 2), (dict(seg=0), 2), (dict(T=-1), 2), (dict(dt=0), 3), (dict(ws=None), 1),
    (dict(ws=P(0x40008)), 4), (dict(wsb=1000), 2), (dict(q=None), 1), (dict(B=0), 0),
])
def test_chunk_fwd_split_validation(kw, status):
    assert split(**kw) == status


def split_static(q=A, k=A, v=A, la=A, b=A, w=A, S0=None, o=A, ST=None, B=1, T=8192, H=16, dk=128, dv=128, dt=1,
                 seg=5):
    return g.lib().gdn2_chunk_fwd_split_static(q, k, v, la, b, w, S0, o, ST, B, T, H, dk, dv, dt, seg, None)


@pytest.mark.parametrize("kw,status", [
    (dict(seg=6), 2), (dict(dk=64), 2), (dict(seg=0), 2), (dict(dt=0), 3), (dict(q=None), 1),
    (dict(o=M), 4), (dict(B=0), 0),
])
def test_chunk_fwd_split_static_validation(kw, status):
    assert split_static(**kw) == status


def bwd(q=A, k=A, v=A, la=A, b=A, w=A, S0=None, dO=A, dST=None, dq=A, dk_=A, dv_=A, dla=A, db=A, dw=A, dS0=None,
        B=1, T=100, H=2, dk=128, dv=128, dt=1, ws=P(0x40000), wsb=1 << 30):
    return g.lib().gdn2_chunk_bwd(q, k, v, la, b, w, S0, dO, dST, dq, dk_, dv_, dla, db, dw, dS0, B, T, H, dk, dv, dt,
                                  ws, wsb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dk=96), 2), (dict(T=-1), 2), (dict(dt=5), 3), (dict(dO=None), 1), (dict(ws=None), 1), (dict(dw=None), 1),
    (dict(dq=M), 4), (dict(ws=P(0x40008)), 4), (dict(wsb=1000), 2), (dict(B=0), 0), (dict(T=0), 0),
])
def test_chunk_bwd_validation(kw, status):
    assert bwd(**kw) == status


def test_bwd_workspace_size():
    L = g.lib()
    assert L.gdn2_chunk_bwd_workspace_bytes(2, 100, 3, 128, 64) == 4 * 2 * 3 * 2 * (128 * 64 + 128)
    assert L.gdn2_chunk_bwd_workspace_bytes(2, 100, 3, 96, 64) == 0


def test_split_segment_model_and_workspace():
    L = g.lib()
    assert L.gdn2_chunk_fwd_split_segments(8, 4096, 16, 148) == 1  # 128 units already fill the GPU
    assert L.gdn2_chunk_fwd_split_segments(1, 65536, 16, 148) > 1
    assert L.gdn2_chunk_fwd_split_segments(1, 64, 1, 148) == 1  # one chunk cannot be split
    assert L.gdn2_chunk_fwd_split_workspace_bytes(2, 3, 128, 128, 5) == 3 * 2 * 3 * 5 * 128 * 128 * 4
    assert L.gdn2_chunk_fwd_split_workspace_bytes(2, 3, 128, 128, 1) == 0


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16)
    la = torch.zeros(1, 64, 1, 128)
    with pytest.raises(ValueError):
        g.gdn2_chunk_fwd(x, x, x, la, x, x, o=x, S_T=torch.zeros(1, 1, 128, 128))


def csize(q=A, k=A, v=A, la=A, b=A, w=A, S0=None, o=A, ST=None, B=1, T=300, H=2, dk=128, dv=128, dt=1, chunk=32):
    return g.lib().gdn2_chunk_fwd_csize(q, k, v, la, b, w, S0, o, ST, B, T, H, dk, dv, dt, chunk, None)


@pytest.mark.parametrize("kw,status", [
    (dict(chunk=16), 2), (dict(chunk=96), 2), (dict(chunk=256), 2), (dict(chunk=0), 2), (dict(dk=96), 2),
    (dict(dv=32), 2), (dict(T=-1), 2), (dict(dt=0), 3), (dict(dt=4), 3), (dict(q=None), 1), (dict(la=None), 1),
    (dict(o=None), 1), (dict(w=M), 4), (dict(ST=M), 4), (dict(B=0), 0), (dict(H=0, chunk=128), 0),
])
def test_chunk_fwd_csize_validation(kw, status):
    assert csize(**kw) == status


def test_csize_shared_memory_footprint():
    # C = 128: region X (the stacked [-Kb; Qh] tile, 256 rows x 128 fp32 channels, later
    # [P; Kn^T]), region Y (Kn, then A solved into T: 128 x 128 fp32), the solve's 64 x 72
    # fp32 scratch, 1 KB of alignment slack and the barrier / decay block
    L = g.lib()
    n128 = L.gdn2_chunk_fwd_csize_smem_bytes(128, 128)
    assert n128 == 4 * (256 * 128 + 128 * 128 + 64 * 72) + 1024 + 544
    # every size on a tcgen05 kernel: one layout for both head sizes, within one block's
    # 227 KB, the 32-token chunk's tiles the smaller
    for C in (32, 64, 128):
        n = L.gdn2_chunk_fwd_csize_smem_bytes(C, 128)
        assert 0 < n <= 227 * 1024 and L.gdn2_chunk_fwd_csize_smem_bytes(C, 64) == n
    assert L.gdn2_chunk_fwd_csize_smem_bytes(32, 128) < L.gdn2_chunk_fwd_csize_smem_bytes(64, 128)
    assert L.gdn2_chunk_fwd_csize_smem_bytes(16, 128) == 0 and L.gdn2_chunk_fwd_csize_smem_bytes(64, 96) == 0
