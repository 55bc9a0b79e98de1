"""Gated DeltaNet-2 token mixer for NVIDIA B200 (sm_100a).

Python binding of ``libgdn2.so`` (the C ABI declared in ``include/gdn2.h``).
It only marshals arguments: every step of the computation runs in the
library's CUDA kernels.  PyTorch provides device memory and streams.  There is
no CPU fallback: without the built library every call raises.

    o, S_T = gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0=None)   # prefill, C = 64
    o      = gdn2_decode_step(q, k, v, log_alpha, b, w, S)       # S updated in place

Shapes: prefill tokens [B, T, H, D], decode tokens [B, H, D], states
[B, H, d_k, d_v] float32; q, k, v, b, w in bfloat16 or float32 (one dtype);
log_alpha float32 (log of the channel-wise decay, <= 0); o is always float32.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["gdn2_chunk_fwd", "gdn2_chunk_fwd_csize", "gdn2_chunk_bwd", "gdn2_chunk_fwd_split", "gdn2_chunk_fwd_split_static", "gdn2_chunk_fwd_varlen", "gdn2_chunk_fwd_raw", "gdn2_short_conv", "gdn2_decode_step", "gdn2_decode_step_raw", "gdn2_device_status", "GDN2Error", "library_path", "lib"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

GDN2_F32, GDN2_BF16 = 0, 1
_DT = {torch.float32: GDN2_F32, torch.bfloat16: GDN2_BF16}


class GDN2Error(RuntimeError):
    """A gdn2_* call returned a non-zero status."""

    def __init__(self, fn, status):
        msg = lib().gdn2_status_string(status).decode()
        if status == 5:
            msg += " (" + lib().gdn2_last_cuda_error().decode() + ")"
        super().__init__(f"{fn}: status {status}: {msg}")
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, "libgdn2.so")


def lib(path=None):
    """The loaded C library (ctypes).  Raises if it has not been built.  ``path`` loads
    another build of the same library in its place (the instrumented build of the
    profiling driver)."""
    global _LIB
    if path is not None and (_LIB is None or _LIB._name != path):
        _LIB = None
    if _LIB is None:
        path = path or library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m gated_delta_rule_95_b200.build` "
                               "(or __graft_entry__.build()); there is no fallback path")
        L = ctypes.CDLL(path)
        P, I = ctypes.c_void_p, ctypes.c_int
        L.gdn2_chunk_fwd.argtypes = [P] * 9 + [I] * 6 + [P]
        L.gdn2_chunk_fwd.restype = I
        L.gdn2_chunk_bwd.argtypes = [P] * 16 + [I] * 6 + [P, ctypes.c_size_t, P]
        L.gdn2_chunk_bwd.restype = I
        L.gdn2_chunk_bwd_workspace_bytes.argtypes = [I] * 5
        L.gdn2_chunk_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.gdn2_chunk_fwd_split.argtypes = [P] * 9 + [I] * 7 + [P, ctypes.c_size_t, P]
        L.gdn2_chunk_fwd_split.restype = I
        L.gdn2_chunk_fwd_split_static.argtypes = [P] * 9 + [I] * 7 + [P]
        L.gdn2_chunk_fwd_split_static.restype = I
        L.gdn2_chunk_fwd_split_segments.argtypes = [I] * 4
        L.gdn2_chunk_fwd_split_segments.restype = I
        L.gdn2_chunk_fwd_split_workspace_bytes.argtypes = [I] * 5
        L.gdn2_chunk_fwd_split_workspace_bytes.restype = ctypes.c_size_t
        L.gdn2_chunk_fwd_csize.argtypes = [P] * 9 + [I] * 7 + [P]
        L.gdn2_chunk_fwd_csize.restype = I
        L.gdn2_chunk_fwd_csize_smem_bytes.argtypes = [I] * 2
        L.gdn2_chunk_fwd_csize_smem_bytes.restype = ctypes.c_size_t
        L.gdn2_chunk_fwd_varlen.argtypes = [P] * 10 + [I] * 6 + [P]
        L.gdn2_chunk_fwd_varlen.restype = I
        L.gdn2_chunk_fwd_raw.argtypes = [P] * 11 + [I] * 6 + [P]
        L.gdn2_chunk_fwd_raw.restype = I
        L.gdn2_short_conv.argtypes = [P] * 7 + [I] * 4 + [P]
        L.gdn2_short_conv.restype = I
        L.gdn2_decode_step.argtypes = [P] * 8 + [I] * 5 + [P]
        L.gdn2_decode_step.restype = I
        L.gdn2_decode_step_raw.argtypes = [P] * 9 + [I] * 5 + [P]
        L.gdn2_decode_step_raw.restype = I
        L.gdn2_device_status.argtypes = []
        L.gdn2_device_status.restype = I
        L.gdn2_status_string.argtypes = [I]
        L.gdn2_status_string.restype = ctypes.c_char_p
        L.gdn2_last_cuda_error.argtypes = []
        L.gdn2_last_cuda_error.restype = ctypes.c_char_p
        L.gdn2_version.argtypes = []
        L.gdn2_version.restype = I
        _LIB = L
    return _LIB


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev, stream):
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _on(device, fn, *args):
    """Calls ``fn`` with ``device`` current (the library keys its per-device state, the
    error word, scratch address and kernel attributes, by the current device)."""
    with torch.cuda.device(device):
        return fn(*args)


def _check_tokens(name, tensors, dtype, device):
    for n, t in tensors.items():
        if not t.is_cuda or t.device != device:
            raise ValueError(f"{name}: {n} must be a CUDA tensor on {device}")
        if not t.is_contiguous():
            raise ValueError(f"{name}: {n} must be contiguous")
        want = torch.float32 if n in ("log_alpha", "a_raw", "S0", "S", "S_T", "o", "decay_scale", "weight",
                                      "bias") else dtype
        if t.dtype != want:
            raise ValueError(f"{name}: {n} must be {want}, got {t.dtype}")


def gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0=None, *, o=None, S_T=None, want_state=True, stream=None):
    """Chunkwise prefill forward.  Returns (o [B,T,H,d_v], S_T [B,H,d_k,d_v] or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in _DT:
        raise ValueError(f"gdn2_chunk_fwd: unsupported dtype {q.dtype}")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ts = dict(q=q, k=k, v=v, log_alpha=log_alpha, b=b, w=w, o=o)
    if S0 is not None:
        ts["S0"] = S0
    if S_T is not None:
        ts["S_T"] = S_T
    _check_tokens("gdn2_chunk_fwd", ts, q.dtype, q.device)
    rc = _on(q.device, lib().gdn2_chunk_fwd, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(o),
                              _ptr(S_T), B, T, H, dk, dv, _DT[q.dtype], _stream(q.device, stream))
    if rc != 0:
        raise GDN2Error("gdn2_chunk_fwd", rc)
    return o, S_T


def gdn2_chunk_fwd_csize(q, k, v, log_alpha, b, w, S0=None, *, chunk=64, o=None, S_T=None, want_state=True,
                         stream=None):
    """Chunkwise prefill forward at chunk size 32, 64 or 128 (bf16 inputs).  Returns
    (o [B,T,H,d_v], S_T [B,H,d_k,d_v] or None), like gdn2_chunk_fwd."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in _DT:
        raise ValueError(f"gdn2_chunk_fwd_csize: unsupported dtype {q.dtype}")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ts = dict(q=q, k=k, v=v, log_alpha=log_alpha, b=b, w=w, o=o)
    if S0 is not None:
        ts["S0"] = S0
    if S_T is not None:
        ts["S_T"] = S_T
    _check_tokens("gdn2_chunk_fwd_csize", ts, q.dtype, q.device)
    rc = _on(q.device, lib().gdn2_chunk_fwd_csize, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0),
                                    _ptr(o), _ptr(S_T), B, T, H, dk, dv, _DT[q.dtype], int(chunk),
                                    _stream(q.device, stream))
    if rc != 0:
        raise GDN2Error("gdn2_chunk_fwd_csize", rc)
    return o, S_T


def gdn2_chunk_bwd(q, k, v, log_alpha, b, w, S0, dO, dS_T=None, *, workspace=None, want_dS0=True, out=None,
                   stream=None):
    """Backward of gdn2_chunk_fwd: gradients of L given dO = dL/do [B,T,H,d_v] fp32 and
    dS_T = dL/dS_T (or None).  Returns dict(dq, dk, dv, dlog_alpha, db, dw: fp32 like the
    inputs; dS0 [B,H,d_k,d_v] or None).  workspace (uint8 CUDA tensor of at least
    gdn2_chunk_bwd_workspace_bytes) is allocated when not given."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in _DT:
        raise ValueError(f"gdn2_chunk_bwd: unsupported dtype {q.dtype}")
    L = lib()
    need = L.gdn2_chunk_bwd_workspace_bytes(B, T, H, dk, dv)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    g = out if out is not None else dict(
        dq=torch.empty((B, T, H, dk), **f32), dk=torch.empty((B, T, H, dk), **f32),
        dv=torch.empty((B, T, H, dv), **f32), dlog_alpha=torch.empty((B, T, H, dk), **f32),
        db=torch.empty((B, T, H, dk), **f32), dw=torch.empty((B, T, H, dv), **f32),
        dS0=torch.empty((B, H, dk, dv), **f32) if want_dS0 else None)
    ts = dict(q=q, k=k, v=v, log_alpha=log_alpha, b=b, w=w, o=dO)
    for n, t in (("S0", S0), ("S_T", dS_T)):
        if t is not None:
            ts[n] = t
    _check_tokens("gdn2_chunk_bwd", ts, q.dtype, q.device)
    for n, t in g.items():
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or t.device != q.device):
            raise ValueError(f"gdn2_chunk_bwd: {n} must be a contiguous fp32 tensor on {q.device}")
    rc = _on(q.device, L.gdn2_chunk_bwd, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(dO),
                          _ptr(dS_T), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlog_alpha"]),
                          _ptr(g["db"]), _ptr(g["dw"]), _ptr(g["dS0"]), B, T, H, dk, dv, _DT[q.dtype],
                          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(q.device, stream))
    if rc != 0:
        raise GDN2Error("gdn2_chunk_bwd", rc)
    return g


def gdn2_chunk_fwd_split(q, k, v, log_alpha, b, w, S0=None, *, segments=None, workspace=None, o=None, S_T=None,
                         want_state=True, stream=None):
    """Chunkwise prefill forward with each sequence split into ``segments`` parallel segments
    (bf16, d_k = d_v).  segments=None takes the library's choice for this device's SM count;
    workspace (a uint8 CUDA tensor of at least gdn2_chunk_fwd_split_workspace_bytes) is
    allocated when not given.  Returns (o [B,T,H,d_v], S_T [B,H,d_k,d_v] or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype != torch.bfloat16:
        raise ValueError("gdn2_chunk_fwd_split: bf16 inputs only")
    L = lib()
    if segments is None:
        sms = torch.cuda.get_device_properties(q.device).multi_processor_count
        segments = L.gdn2_chunk_fwd_split_segments(B, T, H, sms)
    need = L.gdn2_chunk_fwd_split_workspace_bytes(B, H, dk, dv, segments)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ts = dict(q=q, k=k, v=v, log_alpha=log_alpha, b=b, w=w, o=o)
    if S0 is not None:
        ts["S0"] = S0
    if S_T is not None:
        ts["S_T"] = S_T
    _check_tokens("gdn2_chunk_fwd_split", ts, q.dtype, q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _on(q.device, L.gdn2_chunk_fwd_split, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(o),
                                _ptr(S_T), B, T, H, dk, dv, _DT[q.dtype], segments, _ptr(workspace), wbytes,
                                _stream(q.device, stream))
    if rc != 0:
        raise GDN2Error("gdn2_chunk_fwd_split", rc)
    return o, S_T


def gdn2_chunk_fwd_split_static(q, k, v, log_alpha, b, w, S0=None, *, segments, o=None, S_T=None, want_state=True,
                                stream=None):
    """gdn2_chunk_fwd_split with the library's fixed 16 MiB device scratch instead of a
    workspace (the call allocates nothing when o and S_T are given)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype != torch.bfloat16:
        raise ValueError("gdn2_chunk_fwd_split_static: bf16 inputs only")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ts = dict(q=q, k=k, v=v, log_alpha=log_alpha, b=b, w=w, o=o)
    if S0 is not None:
        ts["S0"] = S0
    if S_T is not None:
        ts["S_T"] = S_T
    _check_tokens("gdn2_chunk_fwd_split_static", ts, q.dtype, q.device)
    rc = _on(q.device, lib().gdn2_chunk_fwd_split_static, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0),
                                           _ptr(o), _ptr(S_T), B, T, H, dk, dv, _DT[q.dtype], segments,
                                           _stream(q.device, stream))
    if rc != 0:
        raise GDN2Error("gdn2_chunk_fwd_split_static", rc)
    return o, S_T


def gdn2_chunk_fwd_varlen(q, k, v, log_alpha, b, w, cu_seqlens, S0=None, *, o=None, S_T=None, want_state=True,
                          stream=None):
    """Chunkwise prefill forward over packed variable-length sequences.

    q, k, b: [T, H, d_k]; v, w: [T, H, d_v]; log_alpha: [T, H, d_k]; cu_seqlens: int32 [N + 1]
    on the device.  Returns (o [T, H, d_v], S_T [N, H, d_k, d_v] or None)."""
    T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype != torch.bfloat16:
        raise ValueError("gdn2_chunk_fwd_varlen: bf16 inputs only")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous():
        raise ValueError("gdn2_chunk_fwd_varlen: cu_seqlens must be a contiguous int32 vector")
    if cu_seqlens.device != q.device:
        raise ValueError("gdn2_chunk_fwd_varlen: cu_seqlens must be on the inputs' device")
    N = cu_seqlens.numel() - 1
    if o is None:
        o = torch.empty((T, H, dv), dtype=torch.float32, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    ts = dict(q=q, k=k, v=v, log_alpha=log_alpha, b=b, w=w, o=o)
    if S0 is not None:
        ts["S0"] = S0
    if S_T is not None:
        ts["S_T"] = S_T
    _check_tokens("gdn2_chunk_fwd_varlen", ts, q.dtype, q.device)
    rc = _on(q.device, lib().gdn2_chunk_fwd_varlen, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(cu_seqlens),
                                     _ptr(S0), _ptr(o), _ptr(S_T), N, T, H, dk, dv, _DT[q.dtype],
                                     _stream(q.device, stream))
    if rc != 0:
        raise GDN2Error("gdn2_chunk_fwd_varlen", rc)
    return o, S_T


def gdn2_chunk_fwd_raw(q_raw, k_raw, v, a_raw, b_raw, w_raw, S0=None, *, decay_scale=None, cu_seqlens=None,
                       o=None, S_T=None, want_state=True, stream=None):
    """Chunkwise prefill forward on the raw projections (q, k normalised, sigmoid gates and
    log alpha = -decay_scale[h] * softplus(a_raw) inside the kernel).

    Without cu_seqlens: q_raw, k_raw, b_raw [B, T, H, d_k], v, w_raw [B, T, H, d_v], a_raw fp32
    [B, T, H, d_k]; returns (o [B, T, H, d_v], S_T [B, H, d_k, d_v] or None).  With cu_seqlens
    (int32 [N + 1] on the device) the tensors are packed, [T, H, D], and S0 / S_T are
    [N, H, d_k, d_v].  decay_scale: fp32 [H] on the device, or None for 1."""
    if q_raw.dtype != torch.bfloat16:
        raise ValueError("gdn2_chunk_fwd_raw: bf16 inputs only")
    if cu_seqlens is None:
        B, T, H, dk = q_raw.shape
        o_shape = (B, T, H, v.shape[-1])
    else:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous():
            raise ValueError("gdn2_chunk_fwd_raw: cu_seqlens must be a contiguous int32 vector")
        if cu_seqlens.device != q_raw.device:
            raise ValueError("gdn2_chunk_fwd_raw: cu_seqlens must be on the inputs' device")
        T, H, dk = q_raw.shape
        B = cu_seqlens.numel() - 1
        o_shape = (T, H, v.shape[-1])
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(o_shape, dtype=torch.float32, device=q_raw.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q_raw.device)
    ts = dict(q_raw=q_raw, k_raw=k_raw, v=v, a_raw=a_raw, b_raw=b_raw, w_raw=w_raw, o=o)
    for n, t in (("S0", S0), ("S_T", S_T), ("decay_scale", decay_scale)):
        if t is not None:
            ts[n] = t
    if decay_scale is not None and decay_scale.numel() != H:
        raise ValueError("gdn2_chunk_fwd_raw: decay_scale must hold one value per head")
    _check_tokens("gdn2_chunk_fwd_raw", ts, q_raw.dtype, q_raw.device)
    rc = _on(q_raw.device, lib().gdn2_chunk_fwd_raw, _ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(a_raw), _ptr(b_raw), _ptr(w_raw),
                                  _ptr(decay_scale), _ptr(cu_seqlens), _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk,
                                  dv, _DT[q_raw.dtype], _stream(q_raw.device, stream))
    if rc != 0:
        raise GDN2Error("gdn2_chunk_fwd_raw", rc)
    return o, S_T


def gdn2_short_conv(x, weight, bias=None, *, cu_seqlens=None, hist=None, y=None, hist_out=None, want_hist=False,
                    stream=None):
    """Short causal depthwise convolution (4 taps) over the token axis.

    x: [B, T, C] (or packed [T, C] with cu_seqlens int32 [N + 1] on the device); weight fp32
    [C, 4] (or [C, 1, 4]); bias fp32 [C] or None; hist: [B, 3, C] carried history or None.
    Returns (y like x, hist_out [B, 3, C] or None); hist_out may be hist (in-place update)."""
    if x.dtype not in _DT:
        raise ValueError(f"gdn2_short_conv: unsupported dtype {x.dtype}")
    if cu_seqlens is None:
        B, T, C = x.shape
    else:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous():
            raise ValueError("gdn2_short_conv: cu_seqlens must be a contiguous int32 vector")
        if cu_seqlens.device != x.device:
            raise ValueError("gdn2_short_conv: cu_seqlens must be on the inputs' device")
        T, C = x.shape
        B = cu_seqlens.numel() - 1
    if weight.numel() != 4 * C:
        raise ValueError("gdn2_short_conv: weight must hold 4 taps per channel")
    if y is None:
        y = torch.empty_like(x)
    if hist_out is None and want_hist:
        hist_out = torch.empty((B, 3, C), dtype=x.dtype, device=x.device)
    ts = dict(x=x, weight=weight, y=y)
    for n, t in (("bias", bias), ("hist", hist), ("hist_out", hist_out)):
        if t is not None:
            ts[n] = t
    _check_tokens("gdn2_short_conv", ts, x.dtype, x.device)
    rc = _on(x.device, lib().gdn2_short_conv, _ptr(x), _ptr(weight), _ptr(bias), _ptr(cu_seqlens), _ptr(hist), _ptr(y),
                               _ptr(hist_out), B, T, C, _DT[x.dtype], _stream(x.device, stream))
    if rc != 0:
        raise GDN2Error("gdn2_short_conv", rc)
    return y, hist_out


def gdn2_decode_step(q, k, v, log_alpha, b, w, S, *, o=None, stream=None):
    """One decode step; S [B,H,d_k,d_v] fp32 is updated in place.  Returns o [B,H,d_v]."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in _DT:
        raise ValueError(f"gdn2_decode_step: unsupported dtype {q.dtype}")
    if o is None:
        o = torch.empty((B, H, dv), dtype=torch.float32, device=q.device)
    _check_tokens("gdn2_decode_step", dict(q=q, k=k, v=v, log_alpha=log_alpha, b=b, w=w, S=S, o=o), q.dtype,
                  q.device)
    rc = _on(q.device, lib().gdn2_decode_step, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S), _ptr(o),
                                B, H, dk, dv, _DT[q.dtype], _stream(q.device, stream))
    if rc != 0:
        raise GDN2Error("gdn2_decode_step", rc)
    return o


def gdn2_decode_step_raw(q_raw, k_raw, v, a_raw, b_raw, w_raw, S, *, decay_scale=None, o=None, stream=None):
    """One decode step on the raw projections (q, k normalised, sigmoid gates, log alpha =
    -decay_scale[h] * softplus(a_raw) inside the step); S [B,H,d_k,d_v] fp32 is updated in
    place.  Returns o [B,H,d_v]."""
    B, H, dk = q_raw.shape
    dv = v.shape[-1]
    if q_raw.dtype not in _DT:
        raise ValueError(f"gdn2_decode_step_raw: unsupported dtype {q_raw.dtype}")
    if decay_scale is not None and decay_scale.numel() != H:
        raise ValueError("gdn2_decode_step_raw: decay_scale must hold one value per head")
    if o is None:
        o = torch.empty((B, H, dv), dtype=torch.float32, device=q_raw.device)
    ts = dict(q_raw=q_raw, k_raw=k_raw, v=v, a_raw=a_raw, b_raw=b_raw, w_raw=w_raw, S=S, o=o)
    if decay_scale is not None:
        ts["decay_scale"] = decay_scale
    _check_tokens("gdn2_decode_step_raw", ts, q_raw.dtype, q_raw.device)
    rc = _on(q_raw.device, lib().gdn2_decode_step_raw, _ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(a_raw), _ptr(b_raw), _ptr(w_raw),
                                    _ptr(decay_scale), _ptr(S), _ptr(o), B, H, dk, dv, _DT[q_raw.dtype],
                                    _stream(q_raw.device, stream))
    if rc != 0:
        raise GDN2Error("gdn2_decode_step_raw", rc)
    return o


def gdn2_device_status() -> int:
    """Synchronises the device and returns (then clears) the library's device status."""
    return lib().gdn2_device_status()
