"""Runs one kernel of the library on a seeded workload a few times, for profilers.

    python -m gated_delta_rule_95_b200.profile_case --kind prefill --B 8 --H 16 --T 1024 --reps 2
    python -m gated_delta_rule_95_b200.profile_case --kind decode --B 256 --H 16 --reps 4
    python -m gated_delta_rule_95_b200.profile_case --kind bwd --B 2 --H 16 --T 1024 --reps 2
    python -m gated_delta_rule_95_b200.profile_case --kind csize --chunk 128 --B 8 --H 16 --T 1024 --reps 2
    python -m gated_delta_rule_95_b200.profile_case --kind prefill --stamps
    python -m gated_delta_rule_95_b200.profile_case --kind bwd --stamps
    python -m gated_delta_rule_95_b200.profile_case --kind csize --chunk 128 --stamps

Inputs follow the recipe of the named workload (gdn2_inputs) with the given
sizes; it exits 0 after a device synchronisation and a clean device status.

--stamps runs the prefill (the backward, the chunk-size 128 forward) on the instrumented library
(libgdn2_stamps.so, built with GDN2_STAMPS: the kernel's first CTA records clock64 at the
points of its per-chunk schedule) and prints, per chunk, each point's cycle count relative to the
point where the chunk's raw input tiles have landed, and the period between consecutive
chunks.
"""
from __future__ import annotations

import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kind", choices=["prefill", "decode", "bwd", "csize"], required=True)
    ap.add_argument("--workload", default=None)
    ap.add_argument("--B", type=int, default=None)
    ap.add_argument("--H", type=int, default=None)
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--chunk", type=int, default=64)
    ap.add_argument("--stamps", action="store_true")
    a = ap.parse_args()

    import torch

    import gdn2_inputs as gi
    import gated_delta_rule_95_b200 as g

    if a.stamps:
        return stamps(a)

    dev = torch.device("cuda", 0)
    if a.kind == "prefill":
        wl = gi.WORKLOADS[a.workload or "prefill_b8_h16_t4096"]
        d = gi.prefill_inputs(wl, B=a.B, T=a.T, H=a.H)
        x = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
        for _ in range(a.reps):
            g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    elif a.kind == "csize":
        wl = gi.WORKLOADS[a.workload or "prefill_b8_h16_t4096"]
        d = gi.prefill_inputs(wl, B=a.B, T=a.T, H=a.H)
        x = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
        for _ in range(a.reps):
            g.gdn2_chunk_fwd_csize(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], chunk=a.chunk)
    elif a.kind == "bwd":
        wl = gi.WORKLOADS[a.workload or "prefill_b8_h16_t4096"]
        d = gi.prefill_inputs(wl, B=a.B, T=a.T, H=a.H)
        x = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
        B, T, H = x["q"].shape[:3]
        gen = torch.Generator(device=dev)
        gen.manual_seed(wl.seed)
        dO = torch.randn((B, T, H, wl.dv), generator=gen, device=dev)
        dS = torch.randn((B, H, wl.dk, wl.dv), generator=gen, device=dev)
        for _ in range(a.reps):
            g.gdn2_chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], dO, dS)
    else:
        wl = gi.WORKLOADS[a.workload or "decode_b256_h16"]
        S = gi.decode_state(wl, B=a.B, H=a.H).to(dev)
        for j in range(a.reps):
            t = {k: v.to(dev) for k, v in gi.decode_tokens(wl, j, B=a.B, H=a.H).items()}
            g.gdn2_decode_step(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], S)
    torch.cuda.synchronize()
    status = g.gdn2_device_status()
    if status != 0:
        raise SystemExit(f"device status {status}")
    print("ok")


# stamp slots of the chunk kernel (its STAMP points), by role
STAMP_SLOTS = 32
BWD_SLOT_NAMES = {0: "chunk start", 1: "copies landed", 2: "inputs read", 3: "operand tiles written",
                  4: "dSn out, dSt formed", 5: "dU issued", 6: "dU done", 7: "dU rounded, dR issued",
                  8: "dR done", 9: "-dR staged, dS issued, stores issued", 10: "dS done"}
GRAD_SLOT_NAMES = {16: "unit start", 17: "copies landed, S in", 18: "operands built", 19: "first products done",
                   20: "dP, dA, dSt written", 21: "second products done", 22: "gradients written"}
TC128_SLOT_NAMES = {0: "chunk start", 1: "log decay read", 2: "operands built", 3: "[-A; P] done",
                    4: "A read out", 5: "solve done", 6: "state product done", 7: "last operands written",
                    8: "U~ done", 9: "U~ rounded", 10: "output/state product done", 11: "o stored",
                    12: "P written", 13: "Kn Gamma_C written", 14: "Vw added", 15: "state decayed",
                    16: "T rounded", 17: "offsets summed", 18: "prefetch issued"}
SLOT_NAMES = {0: "AP issued", 1: "SP issued", 2: "U diag issued", 3: "U T21 issued", 4: "OP issued",
              5: "raw landed", 6: "operands built", 7: "AP done", 8: "A/P read out", 9: "8x8 inverses",
              10: "32-level done", 11: "64-level done", 12: "U rounded", 13: "R rounded",
              14: "next decay ready", 15: "chunk end", 16: "o stored"}


def stamps(a):
    import ctypes

    import numpy as np
    import torch

    import gdn2_inputs as gi
    import gated_delta_rule_95_b200 as g
    from gated_delta_rule_95_b200 import build as cuda_build

    path = cuda_build.build(stamps=True)
    lib = g.lib(path)  # the instrumented library in place of the product one
    wl = gi.WORKLOADS[a.workload or "prefill_b8_h16_t4096"]
    d = gi.prefill_inputs(wl, B=a.B, T=a.T, H=a.H)
    x = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    names, first, csz = SLOT_NAMES, 5, 64
    if a.kind == "csize":
        if a.chunk != 128:
            raise SystemExit("--stamps with --kind csize: the chunk-size 128 kernel only")
        names, first, csz = TC128_SLOT_NAMES, 0, 128
    if a.kind == "bwd":
        B, T, H = x["q"].shape[:3]
        gen = torch.Generator(device="cuda")
        gen.manual_seed(wl.seed)
        dO = torch.randn((B, T, H, wl.dv), generator=gen, device="cuda")
        dS = torch.randn((B, H, wl.dk, wl.dv), generator=gen, device="cuda")
        names, first = BWD_SLOT_NAMES, 0
    for _ in range(max(2, a.reps)):
        if a.kind == "bwd":
            g.gdn2_chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], dO, dS)
        elif a.kind == "csize":
            g.gdn2_chunk_fwd_csize(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], chunk=128)
        else:
            g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    torch.cuda.synchronize()
    buf = (ctypes.c_ulonglong * (64 * STAMP_SLOTS))()
    lib.gdn2_stamps_read.argtypes = [ctypes.c_void_p, ctypes.c_int]
    n = lib.gdn2_stamps_read(buf, 64 * STAMP_SLOTS)
    st = np.frombuffer(buf, dtype=np.uint64)[:n].astype(np.int64).reshape(-1, STAMP_SLOTS)
    nch = min(64, (x["q"].shape[1] + csz - 1) // csz)
    base = st[:nch, first]
    print("cycles relative to the chunk's first point (clock64 of the first CTA's SM); the "
          "backward visits the chunks in reverse")
    for c in range(nch):
        prev = c + 1 if a.kind == "bwd" else c - 1
        per = base[c] - base[prev] if 0 <= prev < nch else 0
        row = sorted(((int(st[c, s] - base[c]), names[s]) for s in names if st[c, s]))
        print(f"chunk {c} (period {per}): " + ", ".join(f"{n} {v}" for v, n in row))
    per = np.abs(np.diff(base[1:nch]))
    if len(per):
        print(f"median period {int(np.median(per))} cycles")
    if a.kind == "bwd":
        # the per-chunk pass: one CTA per (batch, head, chunk), rows = its first 64 CTAs
        g0 = st[:nch, 16]
        ok_rows = [c for c in range(nch) if g0[c]]
        print("per-chunk pass, cycles from the start of a unit (each CTA's second), median over the first CTAs:")
        print(", ".join(f"{GRAD_SLOT_NAMES[s]} {int(np.median([st[c, s] - g0[c] for c in ok_rows]))}"
                        for s in sorted(GRAD_SLOT_NAMES) if all(st[c, s] for c in ok_rows)))
    status = g.gdn2_device_status()
    if status != 0:
        raise SystemExit(f"device status {status}")
    print("ok")


if __name__ == "__main__":
    main()
