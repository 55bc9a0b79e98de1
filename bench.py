"""Benchmark of the Gated DeltaNet-2 token mixer on B200.

Primary line: prefill tokens/s per layer of the chunkwise forward on the 1.3B
layer shape (B=8, H=16, T=4096, d_k=d_v=128, bf16 q/k/v/b/w, fp32 log-alpha,
state and output).  Alongside it, in the same JSON line: decode steps/s on
B=256 sequences x H=16 heads (1000 steps, fresh tokens per step), each with its
roofline against the measured HBM copy bandwidth.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun, one process per GPU): every rank runs its own copy of the
workload (independent (batch, head) units need no exchange), the timed region is
bracketed by barriers, and the slowest rank's time is reported.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gdn2_inputs as gi  # noqa: E402

PREFILL = gi.WORKLOADS["prefill_b8_h16_t4096"]
DECODE = gi.WORKLOADS["decode_b256_h16"]
PACKED = gi.WORKLOADS["packed_n64_h16"]
METRIC = "GDN-2 prefill tokens/s per layer"
UNIT = "tokens/s"
# algorithmic HBM bytes per token-head: q,k,v,b,w bf16 + log-alpha fp32 in, o out (bf16 in
# the algorithmic figure of the hot path; the library writes o in fp32, 256 B more)
PREFILL_BYTES_PER_TOKEN_HEAD = 5 * 128 * 2 + 128 * 4 + 128 * 2
PREFILL_BYTES_FP32_O = PREFILL_BYTES_PER_TOKEN_HEAD + 128 * 2
# dense-tile tensor FLOPs per token-head at C=64, d=128: 2C(3dk + 2dv) + 6 dk dv
PREFILL_FLOP_PER_TOKEN_HEAD = 2 * 64 * (3 * 128 + 2 * 128) + 6 * 128 * 128
# state read + write per (sequence, head) and step, fp32 128x128
DECODE_STATE_BYTES = 2 * 128 * 128 * 4
# nominal dense tf32 : bf16 tensor throughput on B200 (1.1 : 2.25 PFLOP/s); the products run in tf32
TF32_PER_BF16 = 1.1 / 2.25
# backward: dense matrix-product FLOPs per chunk-head (C = 64, d = 128) of the chunkwise
# reverse mode including its forward recomputation: 7 products of C^2 d_k, 10 of C d_k d_v,
# 6 of C^2 d_v and 2 of C^3 multiply-adds
BWD_FLOP_PER_CHUNK_HEAD = 2 * (7 * 64 * 64 * 128 + 10 * 64 * 128 * 128 + 6 * 64 * 64 * 128 + 2 * 64 ** 3)
# CUDA-core fp32 peak: 148 SMs x 128 FMA lanes x 2 FLOP x 1.965 GHz
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"], "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "src": "fallback"}


def profile_traffic(kernel):
    """DRAM bytes per launch recorded from an ncu capture (profiles/traffic.md), or None."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) >= 3 and cells[0] == kernel:
                try:
                    return float(cells[2])
                except ValueError:
                    return None
    return None


class Clocks:
    """Samples SM clock and clock-event (throttle) reasons through NVML on a
    background thread while the timed region runs (reading only)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, index, period_s=0.002):
        self.index, self.period = index, period_s
        self.sm, self.reasons, self.mx = [], set(), None

    def _handle(self):
        """NVML handle of the CUDA device (matched by UUID: NVML and CUDA indices can differ)."""
        import pynvml as N
        import torch
        try:
            u = str(torch.cuda.get_device_properties(self.index).uuid)
            return N.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ids = [x for x in vis.split(",") if x.strip()]
            idx = int(ids[self.index]) if ids and ids[self.index].strip().isdigit() else self.index
            return N.nvmlDeviceGetHandleByIndex(idx)

    def _sample(self, N):
        self.sm.append(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM))
        r = self.getr(self.h)
        for name, bit in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        import pynvml as N
        while not self.stop:
            self._sample(N)
            time.sleep(self.period)

    def __enter__(self):
        import threading
        self.stop = False
        self.thread = None
        try:
            import pynvml as N
            N.nvmlInit()
            self.h = self._handle()
            self.mx = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
            self.getr = getattr(N, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                N.nvmlDeviceGetCurrentClocksThrottleReasons
            self._sample(N)
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception:
            self.thread = None
        return self

    def __exit__(self, *a):
        self.stop = True
        if self.thread is not None:
            self.thread.join(timeout=2)
            try:
                import pynvml as N
                self._sample(N)
            except Exception:
                pass

    def summary(self):
        if not self.sm:
            return {"sm_mhz": None, "sm_max_mhz": self.mx, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(self.sm)), "sm_max_mhz": self.mx, "reasons": sorted(self.reasons),
                "samples": len(self.sm), "source": "NVML during the timed region"}


def dist_init(n, backend="nccl"):
    """One process per GPU: reads RANK / WORLD_SIZE / LOCAL_RANK from the environment."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != n:
        raise SystemExit(f"--gpus {n} but WORLD_SIZE={world}")
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, int(os.environ.get("LOCAL_RANK", "0"))


def job_throughput(world, units_per_rank, ms_max):
    """Whole-job rate: every rank processes units_per_rank in the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


def max_over_ranks(x, world, device):
    """Largest value of x over all ranks (x on every rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def time_prefill(args, rank, world, dev):
    import torch
    import gated_delta_rule_95_b200 as g
    d = gi.prefill_inputs(PREFILL)
    x = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
    B, T, H = PREFILL.B, PREFILL.T, PREFILL.H
    o = torch.empty((B, T, H, PREFILL.dv), dtype=torch.float32, device=dev)
    S_T = torch.empty((B, H, PREFILL.dk, PREFILL.dv), dtype=torch.float32, device=dev)

    def step():
        g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], None, o=o, S_T=S_T)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with Clocks(dev.index if dev.index is not None else 0) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(st)
        for i in range(args.steps):
            ev[i][0].record(st)
            step()
            ev[i][1].record(st)
        t1.record(st)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    kernel_ms = [a.elapsed_time(b) for a, b in ev]
    ok = g.gdn2_device_status() == 0
    return dict(total_ms=total_ms, kernel_ms=float(np.mean(kernel_ms)), clocks=clk.summary(), ok=ok,
                tokens=B * T, token_heads=B * T * H)


def time_packed(args, dev):
    """The packed serving batch (variable-length sequences with entering states)."""
    import torch
    import gated_delta_rule_95_b200 as g
    lengths = gi.packed_lengths(PACKED.B, 16, PACKED.T, PACKED.seed)
    d = gi.packed_inputs(PACKED, lengths)
    x = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
    T, H = x["q"].shape[0], PACKED.H
    o = torch.empty((T, H, PACKED.dv), dtype=torch.float32, device=dev)
    S_T = torch.empty((PACKED.B, H, PACKED.dk, PACKED.dv), dtype=torch.float32, device=dev)

    def step():
        g.gdn2_chunk_fwd_varlen(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["cu_seqlens"], x["S0"],
                                o=o, S_T=S_T)

    ms = _time_loop(step, args.steps, args.warmup)
    return dict(ms=ms, tokens=T, token_heads=T * H, units=PACKED.B * H, n_seq=PACKED.B,
                ok=g.gdn2_device_status() == 0)


def _time_loop(step, steps, warmup):
    """Mean device time of one call of ``step`` (ms): CUDA events on the current stream
    around ``steps`` back-to-back calls, after ``warmup`` untimed ones."""
    import torch
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(st)
    for _ in range(steps):
        step()
    t1.record(st)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


def time_conv(args, dev):
    """The short convolution over the q, k, v projections of the prefill workload, side by
    side: [B, T, 3 H d] bf16 (each element read once and written once)."""
    import torch
    import gated_delta_rule_95_b200 as g
    B, T, C = PREFILL.B, PREFILL.T, PREFILL.H * (2 * PREFILL.dk + PREFILL.dv)
    gen = torch.Generator(device=dev)
    gen.manual_seed(PREFILL.seed)
    x = torch.randn((B, T, C), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    w = 0.5 * torch.randn((C, 4), generator=gen, device=dev, dtype=torch.float32)
    b = 0.1 * torch.randn((C,), generator=gen, device=dev, dtype=torch.float32)
    y = torch.empty_like(x)

    def step():
        g.gdn2_short_conv(x, w, b, y=y)

    ms = _time_loop(step, args.steps, args.warmup)
    return dict(ms=ms, bytes=2 * x.numel() * x.element_size(), tokens=B * T, C=C,
                ok=g.gdn2_device_status() == 0)


def time_long(args, dev):
    """The long-context workload (B1 H16 T65536: 16 (batch, head) units for 148 SMs), plain
    and with the sequence split at the library's segment count."""
    import torch
    import gated_delta_rule_95_b200 as g
    wl = gi.WORKLOADS["long_b1_h16_t65536"]
    d = gi.prefill_inputs(wl)
    x = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
    o = torch.empty((wl.B, wl.T, wl.H, wl.dv), dtype=torch.float32, device=dev)
    S_T = torch.empty((wl.B, wl.H, wl.dk, wl.dv), dtype=torch.float32, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    P = g.lib().gdn2_chunk_fwd_split_segments(wl.B, wl.T, wl.H, sms)
    ws = torch.empty(max(1, g.lib().gdn2_chunk_fwd_split_workspace_bytes(wl.B, wl.H, wl.dk, wl.dv, P)),
                     dtype=torch.uint8, device=dev)
    args_t = [x[n] for n in ("q", "k", "v", "log_alpha", "b", "w")]

    def plain():
        g.gdn2_chunk_fwd(*args_t, None, o=o, S_T=S_T)

    def split():
        g.gdn2_chunk_fwd_split(*args_t, None, segments=P, workspace=ws, o=o, S_T=S_T)

    ms_plain = _time_loop(plain, max(3, args.steps // 4), args.warmup)
    ms_split = _time_loop(split, max(3, args.steps // 4), args.warmup)
    return dict(ms_plain=ms_plain, ms_split=ms_split, P=P, tokens=wl.B * wl.T, token_heads=wl.B * wl.T * wl.H,
                ok=g.gdn2_device_status() == 0)


def time_bwd(args, dev):
    """The backward of the prefill workload (gradients of all inputs and S0 given dO, dS_T)."""
    import torch
    import gated_delta_rule_95_b200 as g
    d = gi.prefill_inputs(PREFILL)
    x = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
    B, T, H, dk, dv = PREFILL.B, PREFILL.T, PREFILL.H, PREFILL.dk, PREFILL.dv
    gen = torch.Generator(device=dev)
    gen.manual_seed(PREFILL.seed)
    dO = torch.randn((B, T, H, dv), generator=gen, device=dev)
    dS = torch.randn((B, H, dk, dv), generator=gen, device=dev)
    ws = torch.empty(g.lib().gdn2_chunk_bwd_workspace_bytes(B, T, H, dk, dv), dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = dict(dq=torch.empty((B, T, H, dk), **f32), dk=torch.empty((B, T, H, dk), **f32),
               dv=torch.empty((B, T, H, dv), **f32), dlog_alpha=torch.empty((B, T, H, dk), **f32),
               db=torch.empty((B, T, H, dk), **f32), dw=torch.empty((B, T, H, dv), **f32),
               dS0=torch.empty((B, H, dk, dv), **f32))
    args_t = [x[n] for n in ("q", "k", "v", "log_alpha", "b", "w")]

    def step():
        g.gdn2_chunk_bwd(*args_t, None, dO, dS, workspace=ws, out=out)

    ms = _time_loop(step, max(3, args.steps // 4), args.warmup)
    return dict(ms=ms, tokens=B * T, token_heads=B * T * H, chunk_heads=B * H * (T // 64),
                ok=g.gdn2_device_status() == 0)


def time_csize(args, dev):
    """The prefill workload at chunk sizes 32, 64 and 128 through gdn2_chunk_fwd_csize (each on
    a tcgen05 kernel): latency, and the on-chip footprint that sets how many CTAs share an SM
    (the call needs no device memory besides its tensors)."""
    import torch
    import gated_delta_rule_95_b200 as g
    d = gi.prefill_inputs(PREFILL)
    x = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
    B, T, H, dk, dv = PREFILL.B, PREFILL.T, PREFILL.H, PREFILL.dk, PREFILL.dv
    o = torch.empty((B, T, H, dv), dtype=torch.float32, device=dev)
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    args_t = [x[n] for n in ("q", "k", "v", "log_alpha", "b", "w")]
    sm_total = 228 * 1024  # shared memory of one SM, 1 KB of it reserved per resident CTA
    out = {}
    for C in (32, 64, 128):
        def step(C=C):
            g.gdn2_chunk_fwd_csize(*args_t, None, chunk=C, o=o, S_T=S_T)

        ms = _time_loop(step, args.steps, args.warmup)
        smem = g.lib().gdn2_chunk_fwd_csize_smem_bytes(C, dk)
        out[C] = dict(ms=ms, smem=smem, ctas_per_sm=sm_total // (smem + 1024),
                      kernel={32: "chunk_fwd_tc32_kernel (tcgen05)", 64: "chunk_fwd_tc_kernel (tcgen05)",
                              128: "chunk_fwd_tc128_kernel (tcgen05, phases in sequence)"}[C],
                      tmem_cols=512, ctas=B * H)
    arg_bytes = sum(t.numel() * t.element_size() for t in args_t + [o, S_T])
    return dict(sizes=out, tokens=B * T, token_heads=B * T * H, arg_bytes=arg_bytes, ok=g.gdn2_device_status() == 0)


def time_raw(args, dev):
    """The prefill workload fed with raw projections (activations inside the kernel)."""
    import torch
    import gated_delta_rule_95_b200 as g
    d = gi.raw_inputs(PREFILL)
    x = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
    B, T, H = PREFILL.B, PREFILL.T, PREFILL.H
    o = torch.empty((B, T, H, PREFILL.dv), dtype=torch.float32, device=dev)
    S_T = torch.empty((B, H, PREFILL.dk, PREFILL.dv), dtype=torch.float32, device=dev)

    def step():
        g.gdn2_chunk_fwd_raw(x["q_raw"], x["k_raw"], x["v"], x["a_raw"], x["b_raw"], x["w_raw"], None,
                             decay_scale=x["decay_scale"], o=o, S_T=S_T)

    ms = _time_loop(step, args.steps, args.warmup)
    return dict(ms=ms, tokens=B * T, token_heads=B * T * H, ok=g.gdn2_device_status() == 0)


def time_tiny_f32(args, dev):
    """The tiny fp32 workload (B1 H1 T256, d_k = d_v = 64, fp32 inputs: the 1e-4 parity bar)
    through gdn2_chunk_fwd, which runs it on the split-product tensor-core kernel."""
    import torch
    import gated_delta_rule_95_b200 as g
    wl = gi.WORKLOADS["tiny_f32"]
    d = gi.prefill_inputs(wl)
    x = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
    o = torch.empty((wl.B, wl.T, wl.H, wl.dv), dtype=torch.float32, device=dev)
    S_T = torch.empty((wl.B, wl.H, wl.dk, wl.dv), dtype=torch.float32, device=dev)

    def step():
        g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], None, o=o, S_T=S_T)

    ms = _time_loop(step, max(args.steps, 100), args.warmup)
    return dict(ms=ms, tokens=wl.B * wl.T, ok=g.gdn2_device_status() == 0)


def time_prefill_e2e(args, dev):
    """Same step through the public API with pinned host buffers, copies included: every
    step copies its inputs host->device, runs the forward and copies o and S_T back.  Steps
    are pipelined the way a serving loop would run them, on two streams and two sets of
    device buffers: step i's device->host copy overlaps step i+1's host->device copy (the
    two directions of the link are independent)."""
    import torch
    import gated_delta_rule_95_b200 as g
    d = gi.prefill_inputs(PREFILL)
    host = {k: v.pin_memory() for k, v in d.items() if v is not None}
    B, T, H = PREFILL.B, PREFILL.T, PREFILL.H
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    o_host = torch.empty((B, T, H, PREFILL.dv), dtype=torch.float32).pin_memory()
    s_host = torch.empty((B, H, PREFILL.dk, PREFILL.dv), dtype=torch.float32).pin_memory()
    d2h = o_host.numel() * 4 + s_host.numel() * 4
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dx = [{k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in host.items()} for _ in range(2)]
    do = [torch.empty(o_host.shape, dtype=torch.float32, device=dev) for _ in range(2)]
    ds = [torch.empty(s_host.shape, dtype=torch.float32, device=dev) for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]  # buffer set j: forward done
    drained = [torch.cuda.Event() for _ in range(2)]   # buffer set j: outputs copied back

    def step(i):
        j = i % 2
        x = dx[j]
        for k, v in host.items():
            x[k].copy_(v, non_blocking=True)  # on s_in: after the forward that last read x
        s_in.wait_event(drained[j])  # the outputs of step i - 2 have left the device
        g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], None, o=do[j], S_T=ds[j],
                         stream=s_in)
        computed[j].record(s_in)
        s_out.wait_event(computed[j])
        with torch.cuda.stream(s_out):
            o_host.copy_(do[j], non_blocking=True)
            s_host.copy_(ds[j], non_blocking=True)
        drained[j].record(s_out)

    with torch.cuda.stream(s_in):
        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize()
        n = args.steps
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(n):
            step(i)
        s_in.wait_stream(s_out)
        t1.record(s_in)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / n
    return {"value": B * T / (ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "steps": n, "warmup": args.warmup,
            "pipelining": "two streams: step i's device->host copy overlaps step i+1's host->device copy"}


def time_decode(dev, n_steps, world=1, raw=False, flush=False):
    """Decode steps on the decode workload; raw=True runs the raw-projection step on the same
    token draws read as raw projections (the timing does not depend on the values).

    flush=False: one event pair around the 1000-step loop (steps back to back; the tail of a
    step's state writes may still sit in L2 when the next step reads it).  flush=True: every
    step timed by its own event pair, with a 256 MiB buffer (twice the L2) written between
    steps outside the pairs, so that every step reads its state from HBM."""
    import torch
    import gated_delta_rule_95_b200 as g
    S = gi.decode_state(DECODE).to(dev)
    toks = gi.decode_tokens_many(DECODE, range(n_steps))
    td = [{k: v.to(dev) for k, v in t.items()} for t in toks]
    del toks
    o = torch.empty((DECODE.B, DECODE.H, DECODE.dv), dtype=torch.float32, device=dev)
    scale = torch.full((DECODE.H,), 1.0 / 16.0, dtype=torch.float32, device=dev)
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None

    def run(j):
        t = td[j]
        if raw:
            g.gdn2_decode_step_raw(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], S, decay_scale=scale, o=o)
        else:
            g.gdn2_decode_step(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], S, o=o)

    for j in range(3):
        run(j)
    torch.cuda.synchronize()
    barrier(world)
    st = torch.cuda.current_stream()
    with Clocks(dev.index if dev.index is not None else 0) as clk:
        if flush:
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_steps)]
            for j in range(n_steps):
                scratch.fill_(j & 0xFF)
                ev[j][0].record(st)
                run(j)
                ev[j][1].record(st)
            torch.cuda.synchronize()
            total = sum(a.elapsed_time(b) for a, b in ev)
        else:
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(st)
            for j in range(n_steps):
                run(j)
            t1.record(st)
            torch.cuda.synchronize()
            total = t0.elapsed_time(t1)
    ms = max_over_ranks(total, world, dev) / n_steps
    return dict(ms_per_step=ms, clocks=clk.summary(), ok=g.gdn2_device_status() == 0)


def cpu_baseline(seconds_target=15.0):
    """The oracle, as it stands, on a bounded sample of the prefill workload:
    whole (batch, head) units over the full sequence, as many as fit in about
    seconds_target of wall time on the host's cores."""
    import oracle
    cores = os.cpu_count() or 1
    d = gi.prefill_inputs(PREFILL)
    f = {k: gi.as_f64(d[k]) for k in ("q", "k", "v", "log_alpha", "b", "w")}
    del d
    one = {k: v[:1, :, :1] for k, v in f.items()}
    t = time.perf_counter()
    oracle.forward(**one, nthreads=1)
    per_unit = time.perf_counter() - t
    total = PREFILL.B * PREFILL.H
    units = int(max(1, min(total, seconds_target * cores / max(per_unit, 1e-3))))
    nb = max(1, min(PREFILL.B, units // PREFILL.H)) if units >= PREFILL.H else 1
    nh = PREFILL.H if units >= PREFILL.H else units
    units = nb * nh
    sample = {k: np.ascontiguousarray(v[:nb, :, :nh]) for k, v in f.items()}
    del f
    threads = min(cores, units)
    t = time.perf_counter()
    oracle.forward(**sample, nthreads=threads)
    dt = time.perf_counter() - t
    value = units * PREFILL.T / PREFILL.H / dt
    return {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{units} of the {total} (batch, head) units ({nb} sequences x {nh} heads), full T="
                      f"{PREFILL.T}, fp64 token-by-token recurrence, {dt:.1f} s wall on {threads} threads; "
                      f"value = units x T / H / time (tokens/s per layer)"}


def config_dict():
    return {"workload": "prefill_b8_h16_t4096: B=8 H=16 T=4096 d_k=d_v=128 C=64, bf16 q,k,v,b,w; "
                        "fp32 log-alpha, state and output",
            "global_batch": PREFILL.B, "seq_len": PREFILL.T, "heads": PREFILL.H, "d_k": 128, "d_v": 128,
            "chunk": 64, "l2": "inputs larger than L2 (1.2 GB read per step)", "parallelism": "replicas"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    vals = []
    cb = None
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(seconds_target=8.0)
        if i >= args.warmup:
            vals.append(cb["value"])
    value = float(np.mean(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": PREFILL.B * PREFILL.T / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(),
            "cpu_baseline": dict(cb, value=value),
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=DECODE.steps)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    import torch
    rank, world, local = dist_init(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pk = peaks()

    pre = time_prefill(args, rank, world, dev)
    ms = pre["total_ms"] / args.steps
    value = job_throughput(world, pre["tokens"], ms)
    achieved = pre["token_heads"] * PREFILL_BYTES_PER_TOKEN_HEAD / (pre["kernel_ms"] * 1e-3) / 1e9
    tflops = pre["token_heads"] * PREFILL_FLOP_PER_TOKEN_HEAD / (pre["kernel_ms"] * 1e-3) / 1e12
    traffic = profile_traffic("chunk_fwd_tc_kernel")

    dec = time_decode(dev, args.decode_steps, world, flush=True)
    dec_b2b = time_decode(dev, args.decode_steps, world)
    dec_raw = time_decode(dev, args.decode_steps, world, raw=True)
    pak = time_packed(args, dev)
    raw = time_raw(args, dev)
    cv = time_conv(args, dev)
    lg = time_long(args, dev)
    bw = time_bwd(args, dev)
    cs = time_csize(args, dev)
    tf = time_tiny_f32(args, dev)
    bw_tflops = bw["chunk_heads"] * BWD_FLOP_PER_CHUNK_HEAD / (bw["ms"] * 1e-3) / 1e12
    lg_gbs = lg["token_heads"] * PREFILL_BYTES_PER_TOKEN_HEAD / (lg["ms_split"] * 1e-3) / 1e9
    cv_gbs = cv["bytes"] / (cv["ms"] * 1e-3) / 1e9
    raw_gbs = raw["token_heads"] * PREFILL_BYTES_PER_TOKEN_HEAD / (raw["ms"] * 1e-3) / 1e9
    # algorithmic bytes: the token streams plus each sequence's entering and final state
    pak_bytes = pak["token_heads"] * PREFILL_BYTES_PER_TOKEN_HEAD + pak["units"] * DECODE_STATE_BYTES
    pak_gbs = pak_bytes / (pak["ms"] * 1e-3) / 1e9
    dec_units = DECODE.B * DECODE.H
    dec_gbs = dec_units * DECODE_STATE_BYTES / (dec["ms_per_step"] * 1e-3) / 1e9
    decr_gbs = dec_units * DECODE_STATE_BYTES / (dec_raw["ms_per_step"] * 1e-3) / 1e9
    barrier(world)
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    def hbm(kernel, gbs, traffic=None):
        return {"bound": "hbm", "kernel": kernel, "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / pk["hbm_gbs"], "traffic": traffic}

    # secondary legs: one JSON line of their own, printed before the result line
    legs = {
        "legs": "secondary workloads (the result line follows)",
        "decode_raw": {"metric": "GDN-2 decode steps/s, raw projections", "value": 1e3 / dec_raw["ms_per_step"],
                       "unit": "steps/s", "ms_per_step": dec_raw["ms_per_step"], "steps": args.decode_steps,
                       "workload": "decode_b256_h16 through gdn2_decode_step_raw (q, k normalised, sigmoid gates "
                                   "and softplus decay inside the step)",
                       "roofline": hbm("decode_step_kernel (raw)", decr_gbs)},
        "packed": {"metric": "GDN-2 packed prefill tokens/s per layer", "value": pak["tokens"] / (pak["ms"] * 1e-3),
                   "unit": "tokens/s", "ms_per_step": pak["ms"], "steps": args.steps,
                   "workload": f"packed_n64_h16: {pak['n_seq']} sequences, lengths log-uniform in [16, 8192] "
                               f"({pak['tokens']} tokens), H=16 d_k=d_v=128, bf16, entering states N(0, 0.02)",
                   "roofline": hbm("chunk_fwd_tc_kernel (packed)", pak_gbs)},
        "raw": {"metric": "GDN-2 prefill tokens/s per layer, raw projections",
                "value": raw["tokens"] / (raw["ms"] * 1e-3), "unit": "tokens/s", "ms_per_step": raw["ms"],
                "steps": args.steps,
                "workload": "prefill_b8_h16_t4096 fed with the raw projections: q, k L2-normalised, sigmoid "
                            "gates and log alpha = -softplus(a)/16 applied inside the kernel",
                "roofline": hbm("chunk_fwd_tc_kernel (raw)", raw_gbs)},
        "long": {"metric": "GDN-2 prefill tokens/s per layer, long context",
                 "value": lg["tokens"] / (lg["ms_split"] * 1e-3), "unit": "tokens/s", "ms_per_step": lg["ms_split"],
                 "segments": lg["P"], "unsplit_ms_per_step": lg["ms_plain"],
                 "workload": "long_b1_h16_t65536 (B=1 H=16 T=65536, heavy decay tail) through "
                             "gdn2_chunk_fwd_split at the library's segment count",
                 "roofline": hbm("chunk_fwd_tc_kernel (split)", lg_gbs)},
        "bwd": {"metric": "GDN-2 backward tokens/s per layer", "value": bw["tokens"] / (bw["ms"] * 1e-3),
                "unit": "tokens/s", "ms_per_step": bw["ms"],
                "workload": "prefill_b8_h16_t4096 backward: dq, dk, dv, dlog_alpha, db, dw, dS0 from dO and dS_T",
                "kernels": "chunk_fwd_tc_kernel checkpoint pass (states, U, T^T, P^T), bwd_chain_kernel (reverse dS "
                           "sweep, tcgen05), bwd_grad_kernel (per-chunk gradients, tcgen05)",
                "roofline": {"bound": "tensor", "kernel": "the three launches together", "achieved": bw_tflops,
                             "peak": pk["bf16_tflops"] * TF32_PER_BF16, "unit": "TFLOP/s",
                             "frac": bw_tflops / (pk["bf16_tflops"] * TF32_PER_BF16),
                             "peak_src": "measured bf16 x nominal tf32/bf16 ratio",
                             "frac_of_fp32_cuda_core_peak": bw_tflops / FP32_FMA_TFLOPS,
                             "flop_per_chunk_head": BWD_FLOP_PER_CHUNK_HEAD, "traffic": None}},
        "csize": {"metric": "GDN-2 prefill tokens/s per layer by chunk size",
                  "workload": "prefill_b8_h16_t4096 through gdn2_chunk_fwd_csize",
                  "device_bytes": {"arguments": cs["arg_bytes"], "scratch": 0},
                  "sizes": {str(C): {"value": cs["tokens"] / (r["ms"] * 1e-3), "unit": "tokens/s",
                                     "ms_per_step": r["ms"], "kernel": r["kernel"], "ctas": r["ctas"],
                                     "smem_bytes_per_cta": r["smem"], "tmem_columns_per_cta": r["tmem_cols"],
                                     "ctas_per_sm_by_smem": r["ctas_per_sm"],
                                     "roofline": hbm(r["kernel"],
                                                     cs["token_heads"] * PREFILL_BYTES_PER_TOKEN_HEAD
                                                     / (r["ms"] * 1e-3) / 1e9)}
                            for C, r in cs["sizes"].items()}},
        "tiny_f32": {"metric": "GDN-2 prefill tokens/s per layer, fp32 inputs", "value": tf["tokens"] / (tf["ms"] * 1e-3),
                     "unit": "tokens/s", "ms_per_step": tf["ms"],
                     "workload": "tiny_f32: B=1 H=1 T=256 d_k=d_v=64, fp32 inputs (chunk_fwd_f32_tc_kernel: split "
                                 "tf32 products on tcgen05, one CTA: latency-bound)"},
        "conv": {"metric": "short convolution GB/s", "value": cv_gbs, "unit": "GB/s", "ms_per_step": cv["ms"],
                 "steps": args.steps,
                 "workload": f"q, k, v projections of prefill_b8_h16_t4096 side by side: [8, 4096, {cv['C']}] bf16, "
                             "4 taps + bias, zero history",
                 "roofline": hbm("short_conv_kernel", cv_gbs)},
    }
    print(json.dumps(legs), flush=True)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "tf32", "data": "synthetic (seeded normal draws, layer shape)",
        "config": config_dict(),
        "roofline": dict(hbm("chunk_fwd_tc_kernel", achieved, traffic), peak_src=pk["src"],
                         bytes_per_token_head=PREFILL_BYTES_PER_TOKEN_HEAD,
                         frac_fp32_o=achieved * PREFILL_BYTES_FP32_O / PREFILL_BYTES_PER_TOKEN_HEAD / pk["hbm_gbs"],
                         tensor={"achieved_tflops": tflops, "frac_bf16": tflops / pk["bf16_tflops"],
                                 "frac_tf32": tflops / (pk["bf16_tflops"] * TF32_PER_BF16)}),
        "decode": {"value": 1e3 / dec["ms_per_step"], "unit": "steps/s", "ms_per_step": dec["ms_per_step"],
                   "steps": args.decode_steps, "workload": "decode_b256_h16",
                   "timing": "each step its own event pair, L2 flushed (256 MiB written) between steps",
                   "back_to_back_ms_per_step": dec_b2b["ms_per_step"],
                   "roofline": hbm("decode_step_kernel", dec_gbs, profile_traffic("decode_step_kernel")),
                   "clocks": {k: dec["clocks"].get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons")}},
        "gpu_launches": args.steps,
        "clocks": {k: pre["clocks"].get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons", "samples")},
        "device_status_ok": bool(pre["ok"] and dec["ok"] and dec_b2b["ok"] and dec_raw["ok"] and pak["ok"] and raw["ok"] and cv["ok"]
                                 and lg["ok"] and bw["ok"] and cs["ok"] and tf["ok"]),
    }
    if not args.no_e2e:
        line["e2e"] = time_prefill_e2e(args, dev)
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
