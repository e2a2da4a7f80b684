"""Run hot-path kernels a fixed number of times, for profilers.

    python -m linear_attention_rnn_wkv6_b200.profile_cases [--case NAME[:B:T]] ... [--rounds R] [--library L]

Each case is one of the benchmark's workloads (``synth.WORKLOADS``),
optionally with its batch B and length T replaced, so that a profiler can
capture a smaller instance of the same kernel.  Every round calls each case
once, in the order given, through the C ABI (the backward adds its du
reduction launch).  Inputs are the seeded synthetic ones of ``synth``; nothing
here computes any part of the operator.
"""
from __future__ import annotations

import argparse

import numpy as np

from . import synth


def _dev(a):
    import torch
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def make_case(spec: str):
    """Parse NAME[:B:T] and return (label, callable that launches the case once)."""
    import torch
    import linear_attention_rnn_wkv6_b200 as wkv

    parts = spec.split(":")
    name = parts[0]
    kind, kw = synth.WORKLOADS[name]
    kw = dict(kw)
    if len(parts) == 3:
        kw["B"], kw["T"] = int(parts[1]), int(parts[2])
    if kind in ("wkv4_fwd", "wkv4_bwd"):
        x = synth.make_wkv4(kw["B"], kw["T"], kw["C"], seed=0, with_dy=kind == "wkv4_bwd")
        label = f"{name} B={x.B} T={x.T}"
        if kind == "wkv4_fwd":
            ins = [_dev(getattr(x, n)) for n in ("k", "v", "w", "u")]
            y = torch.empty(x.B, x.T, x.C, device="cuda")
            return label, lambda: wkv.wkv4_fwd(x.B, x.T, x.C, *ins, y)
        ins = [_dev(getattr(x, n)) for n in ("k", "v", "w", "u", "dy")]
        outs = [torch.empty(x.B, x.T, x.C, device="cuda") for _ in range(2)] + \
               [torch.empty(x.C, device="cuda") for _ in range(2)]
        nb = wkv.wkv4_bwd_workspace_bytes(x.B, x.T, x.C)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        return label, lambda: wkv.wkv4_bwd(x.B, x.T, x.C, *ins, *outs, ws, nb)
    if kind == "wkv6_fwd_fused":
        x = synth.make_fused(kw["B"], kw["T"], kw["H"], seed=0, bidir=kw.get("bidir", False))
        label = f"{name} B={x.B} T={x.T} H={x.H}"
        ins = [_dev(getattr(x, n)) for n in ("r", "k", "v", "ww", "w_base", "u", "g", "gn_w", "gn_b")]
        y = torch.empty(x.B, x.T, x.C, device="cuda")
        return label, lambda: wkv.wkv6_fwd_fused(x.B, x.T, x.C, x.H, x.bidir, *ins, x.eps, y)
    args = {k: v for k, v in kw.items() if k not in ("B", "T", "H")}
    make = synth.make_wkv5 if kind.startswith("wkv5") else synth.make_wkv6
    x = make(kw["B"], kw["T"], kw["H"], seed=0, **args)
    label = f"{name} B={x.B} T={x.T} H={x.H}"
    if kind.startswith("wkv6_bwd"):
        bidir = kind == "wkv6_bwd_bidir"
        ins = [_dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u")]
        outs = [torch.empty(x.B, x.T, x.C, device="cuda") for _ in range(4)] + [torch.empty(x.C, device="cuda")]
        nb = wkv.wkv6_bwd_workspace_bytes(x.B, x.T, x.C, x.H, bidir)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        if x.dtype == "bf16":   # the bf16 backward takes dy in bf16 too
            dy = _dev(synth.to_bf16_bits(x.dy))
            return label, lambda: wkv.wkv6_bwd_bf16(x.B, x.T, x.C, x.H, bidir, *ins, dy, *outs, ws, nb)
        dy = _dev(x.dy)
        return label, lambda: wkv.wkv6_bwd(x.B, x.T, x.C, x.H, bidir, *ins, dy, *outs, ws, nb)
    if kind == "wkv5_bwd":
        ins = [_dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u", "dy")]
        outs = [torch.empty(x.B, x.T, x.C, device="cuda") for _ in range(3)] + \
               [torch.empty(x.C, device="cuda") for _ in range(2)]
        nb = wkv.wkv5_bwd_workspace_bytes(x.B, x.T, x.C, x.H)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        return label, lambda: wkv.wkv5_bwd(x.B, x.T, x.C, x.H, *ins, *outs, ws, nb)
    ins = [_dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u")]
    y = torch.empty(x.B, x.T, x.C, device="cuda")
    if kind == "wkv6_decode":
        state = _dev(synth.make_state(x.B, x.H, seed=0))
        return label, lambda: wkv.wkv6_decode(x.B, x.C, x.H, *ins, state, y)
    if kind == "wkv6_fwd_state":
        s0 = _dev(synth.make_state(x.B, x.H, seed=0))
        sT = torch.empty(x.B, x.H, 64, 64, device="cuda")
        return label, lambda: wkv.wkv6_fwd_state(x.B, x.T, x.C, x.H, *ins, s0, y, sT)
    fn = getattr(wkv, kind)
    return label, lambda: fn(x.B, x.T, x.C, x.H, *ins, y)


def main(argv=None) -> int:
    import torch
    import linear_attention_rnn_wkv6_b200 as wkv

    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--case", action="append", required=True,
                    help="workload name from synth.WORKLOADS, optionally NAME:B:T")
    ap.add_argument("--rounds", type=int, default=2)
    ap.add_argument("--library", choices=sorted(wkv.LIBRARY_FILES), default="default",
                    help="the library build whose kernels run (recurrence: the test build)")
    a = ap.parse_args(argv)
    with wkv.use_library(a.library):
        cases = [make_case(c) for c in a.case]
        for _ in range(a.rounds):
            for _, run in cases:
                run()
        torch.cuda.synchronize()
        faults = wkv.wkv_take_device_faults()
    for label, _ in cases:
        print(label)
    if faults:
        print(f"device fault word {faults:#x}")
        return 1
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
