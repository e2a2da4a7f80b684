#!/usr/bin/env python
"""Benchmark of the B200 WKV operator.

One step = one pass of the whole hot path over one batch of each workload:
    RWKV-4 forward            B=8,  T=1024, C=768            fp32
    RWKV-6 bidirectional fwd  B=32, T=196,  H=12, N=64       fp32
    RWKV-6 causal fwd         B=8,  T=4096, H=32, N=64       bf16 r/k/v/w, fp32 state/y
    RWKV-6 bidirectional bwd  B=32, T=196,  H=12, N=64       fp32 (dr, dk, dv, dw, du)
Metric: WKV tokens per second (sum of B*T over the four launches per step),
whole job (all ranks).  Inputs are seeded synthetic data resident in HBM when
the timed region starts; the step's working set (~1.2 GB) is far larger than
the 126 MB L2, so every kernel starts cold.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

For N > 1 launch under torchrun (NCCL): the step runs on one seeded problem of
N x B batches, rank r generating and computing its window [rB, (r+1)B) of it
(weak scaling: B per GPU fixed); the backward's du is all-reduced over the
ranks inside every step (C floats), the one exchange the batch split needs; the
step time is the maximum over ranks.  `--only NAME` times single workloads
(also the ones outside the step), `--library recurrence` the test build of the
library, and `--impl reference` the double-precision CPU oracle (the only
reference this operator has) on a bounded sample.  SM clocks, power and
throttle reasons are sampled through NVML every 2 ms during the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "WKV tokens/sec/GPU and % of roofline (HBM GB/s or FP32/TC util) vs CPU oracle"
UNIT = "tokens/s"
WORKLOAD_NAME = ("wkv-hot-path step: wkv4_fwd B8xT1024xC768 f32 + wkv6_bidir_fwd B32xT196xH12 f32 + "
                 "wkv6_fwd_bf16 B8xT4096xH32 + wkv6_bwd(bidir) B32xT196xH12 f32, N=64")
# Workloads outside the step, measured on their own with --only: the small causal fp32
# forward (B1 T196 H4: four (b, h) units, bound by latency and launch, not by a roof),
# the causal fp32 forward at the bidirectional workload's shape, and the NEXT rows.
EXTRA_WORKLOADS = ["wkv6_causal_f32_b1t196h4", "wkv6_causal_f32_b32t196h12", "wkv6_decode_f32_b512h32",
                   "wkv6_bidir_bwd_bf16_b32t196h12", "wkv4_bwd_f32_b8t1024c768", "wkv5_causal_bf16_b8t4096h32",
                   "wkv5_bwd_f32_b32t196h12", "wkv6_bidir_fused_f32_b32t196h12", "wkv6_state_f32_b32t196h12",
                   "wkv5_causal_f32_b32t196h12"]
STEP_WORKLOADS = ["wkv4_f32_b8t1024c768", "wkv6_bidir_f32_b32t196h12", "wkv6_causal_bf16_b8t4096h32",
                  "wkv6_bidir_bwd_f32_b32t196h12"]
N = 64
L2_BYTES = 126 * 1024 * 1024
FP32_LANES_PER_SM, SMS, SM_MAX_MHZ = 128, 148, 1965.0
FP32_PEAK_TFLOPS = SMS * FP32_LANES_PER_SM * 2 * SM_MAX_MHZ * 1e6 / 1e12   # 74.4 (FMA = 2 flop)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# Algorithmic work per unit (a unit is one token of one head for RWKV-6, one
# (token, channel) for RWKV-4).  Bytes: inputs read once + outputs written once.
# Flops: RWKV-6 forward 5 N^2 per direction (state update 3 N^2 + readout 2 N^2),
# backward 14 N^2 per direction; RWKV-4 ~4 exp + 12 flop.  Each kernel's roofline
# time is the slower of its bytes at HBM bandwidth and its flops at the peak of the
# pipe it computes on (uses_tensor_cores): for the chunked tensor-core forms the
# bytes bind, for the recurrence kernels of the test build the FP32 FMA pipe; both
# fractions are reported per kernel.
ALG = {
    "wkv4_f32_b8t1024c768": dict(bytes_per_unit=3 * 4, flops_per_unit=16),
    "wkv6_causal_f32_b1t196h4": dict(bytes_per_unit=5 * N * 4, flops_per_unit=5 * N * N),
    "wkv6_causal_f32_b32t196h12": dict(bytes_per_unit=5 * N * 4, flops_per_unit=5 * N * N),
    "wkv6_bidir_f32_b32t196h12": dict(bytes_per_unit=5 * N * 4, flops_per_unit=10 * N * N),
    "wkv6_causal_bf16_b8t4096h32": dict(bytes_per_unit=4 * N * 2 + N * 4, flops_per_unit=5 * N * N),
    # the fp32 backward's default path runs on the tensor cores (two-term split bf16 operands)
    "wkv6_bidir_bwd_f32_b32t196h12": dict(bytes_per_unit=9 * N * 4, flops_per_unit=28 * N * N),
    "wkv6_bidir_bwd_bf16_b32t196h12": dict(bytes_per_unit=5 * N * 2 + 4 * N * 4, flops_per_unit=28 * N * N),
    # RWKV-4 backward: k, v, dy in and dk, dv out per (token, channel)
    "wkv4_bwd_f32_b8t1024c768": dict(bytes_per_unit=5 * 4, flops_per_unit=40),
    # decode: the state is read and written once per step (2 N^2 floats) next to 5 N floats of token data
    "wkv6_decode_f32_b512h32": dict(bytes_per_unit=2 * N * N * 4 + 5 * N * 4, flops_per_unit=5 * N * N),
    # RWKV-5: no per-token w; the forward and the causal backward run the tensor-core
    # chunked forms, so both are bound by their bytes: the forward reads bf16 r, k, v and
    # writes fp32 y; the backward reads r, k, v, dy and writes dr, dk, dv (w, dw, u, du
    # are per channel)
    "wkv5_causal_bf16_b8t4096h32": dict(bytes_per_unit=3 * N * 2 + N * 4, flops_per_unit=5 * N * N),
    "wkv5_bwd_f32_b32t196h12": dict(bytes_per_unit=7 * N * 4, flops_per_unit=14 * N * N),
    # fused forward (tensor-core kernel): r, k, v, ww and the gate in, the normalised and gated output out
    "wkv6_bidir_fused_f32_b32t196h12": dict(bytes_per_unit=6 * N * 4, flops_per_unit=10 * N * N),
    # state in/out: the two N x N states of a (b, h) spread over its T = 196 tokens
    "wkv6_state_f32_b32t196h12": dict(bytes_per_unit=5 * N * 4 + 2 * N * N * 4 / 196, flops_per_unit=5 * N * N),
    # RWKV-5 fp32: r, k, v in, y out (w is [C])
    "wkv5_causal_f32_b32t196h12": dict(bytes_per_unit=4 * N * 4, flops_per_unit=5 * N * N),
}
ENTRY = {"wkv6_causal_f32_b1t196h4": "wkv6_fwd", "wkv6_causal_f32_b32t196h12": "wkv6_fwd",
         "wkv4_f32_b8t1024c768": "wkv4_fwd", "wkv6_bidir_f32_b32t196h12": "wkv6_bidir_fwd",
         "wkv6_causal_bf16_b8t4096h32": "wkv6_fwd_bf16", "wkv6_bidir_bwd_f32_b32t196h12": "wkv6_bwd",
         "wkv6_decode_f32_b512h32": "wkv6_decode", "wkv6_bidir_bwd_bf16_b32t196h12": "wkv6_bwd_bf16",
         "wkv4_bwd_f32_b8t1024c768": "wkv4_bwd", "wkv5_causal_bf16_b8t4096h32": "wkv5_fwd_bf16",
         "wkv5_bwd_f32_b32t196h12": "wkv5_bwd", "wkv6_bidir_fused_f32_b32t196h12": "wkv6_fwd_fused",
         "wkv6_state_f32_b32t196h12": "wkv6_fwd_state", "wkv5_causal_f32_b32t196h12": "wkv5_fwd"}
FLUSH_BYTES = 512 << 20   # an L2 flush write; working sets below this get one before every step

LAUNCHES = {"wkv6_causal_f32_b1t196h4": 1, "wkv6_causal_f32_b32t196h12": 1, "wkv4_f32_b8t1024c768": 1, "wkv6_bidir_f32_b32t196h12": 1, "wkv6_causal_bf16_b8t4096h32": 1,
            "wkv6_bidir_bwd_f32_b32t196h12": 3,   # S-kind and G-kind tensor-core kernels and the deterministic du reduction
            "wkv6_decode_f32_b512h32": 1, "wkv6_bidir_bwd_bf16_b32t196h12": 3,
            "wkv4_bwd_f32_b8t1024c768": 2, "wkv5_causal_bf16_b8t4096h32": 1,
            "wkv5_bwd_f32_b32t196h12": 4,   # S and G kinds with the static decay, du reduction, dw total
            "wkv6_bidir_fused_f32_b32t196h12": 1, "wkv6_state_f32_b32t196h12": 1, "wkv5_causal_f32_b32t196h12": 1}


def units_of(name: str, x) -> int:
    if name.startswith("wkv4"):
        return x.B * x.T * x.C
    return x.B * x.T * x.H


def tokens_of(x) -> int:
    return x.B * x.T


# ----------------------------------------------------------------------------- distributed plumbing

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init_group(backend: str, world: int):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity for one rank)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, dist=None, device=None) -> float:
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(dist=None):
    if dist is not None:
        dist.barrier()


# ----------------------------------------------------------------------------- peaks, clocks, traffic

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def load_tensor_peak():
    """Dense bf16 tensor throughput (TFLOP/s): the measured burst figure, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def uses_tensor_cores(name: str, library: str = "default") -> bool:
    """Whether the workload's entry point runs a chunked tensor-core form in that build
    (RWKV-4 and the decode step run on the CUDA cores in every build; the test build
    runs every RWKV-6 and RWKV-5 entry point on its recurrence kernels)."""
    return library == "default" and not name.startswith("wkv4") and "decode" not in name


def kernel_source_hash() -> str:
    import glob
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "linear_attention_rnn_wkv6_b200", "csrc", "*"))):
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(name: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernels have not changed since."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_source_sha") != kernel_source_hash():
        return None
    e = d.get("kernels", {}).get(name)
    return None if e is None else float(e["dram_bytes_per_launch"])


class ClockSampler:
    """Samples the GPU's SM clock, power and throttle reasons every `period_s` during the
    timed region, through NVML from a background thread (a timed region of a few ms
    still gets samples); falls back to an `nvidia-smi -lms 50` child process when NVML
    cannot be loaded."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.dev = device_index
        self.period = period_s
        self.samples = []     # (sm_mhz, sm_max_mhz, power_w, reason names)
        self.source = None
        self.proc = None
        self.thread = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            p = torch.cuda.get_device_properties(self.dev)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop = threading.Event()

            def poll():
                while True:
                    try:
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((sm, sm_max, pw, tuple(n for n, bit in bits.items() if rs & bit)))
                    except Exception:
                        pass
                    if self.stop.wait(self.period):
                        return

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.source = f"NVML every {self.period * 1e3:.0f} ms"
        except Exception:
            try:
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                              "--format=csv,noheader,nounits", "-lms", "50"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi -lms 50"
            except Exception:
                self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            for ln in out.splitlines():
                f = [x.strip() for x in ln.split(",")]
                if len(f) < 8:
                    continue
                try:
                    sm, mx = float(f[0]), float(f[1])
                    pw = float(f[2]) if f[2].replace(".", "", 1).isdigit() else 0.0
                except ValueError:
                    continue
                self.samples.append((sm, mx, pw, tuple(n for n, v in zip(self.NAMES, f[4:8])
                                                      if v.lower().startswith("active"))))

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        sm = [x[0] for x in self.samples]
        reasons = sorted({n for x in self.samples for n in x[3]})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.samples[-1][1], "reasons": reasons,
                "samples": len(sm), "power_w_max": round(max(x[2] for x in self.samples), 1),
                "source": self.source}


# ----------------------------------------------------------------------------- native (CUDA) arm

class DeviceWorkload:
    """Inputs resident in HBM, outputs and workspace preallocated; run() enqueues the ABI call."""

    def __init__(self, name: str, rank: int = 0, world: int = 1):
        import numpy as np
        import torch
        from linear_attention_rnn_wkv6_b200 import synth
        from linear_attention_rnn_wkv6_b200.shard import batch_range
        self.name = name
        # One seeded problem of world x B batches; this rank holds its window of
        # batches.  Workloads without batch windows (static decay, fused, decode) run
        # independent replicas with a rank-dependent seed instead.
        self.split = world > 1 and synth.WORKLOADS[name][0] in (
            "wkv4_fwd", "wkv4_bwd", "wkv6_fwd", "wkv6_fwd_bf16", "wkv6_bidir_fwd", "wkv6_bwd_bidir")
        if self.split:
            Bw = synth.WORKLOADS[name][1]["B"]
            self.kind, self.x = synth.make_workload(name, seed=0, batch_scale=world,
                                                    batches=batch_range(Bw * world, rank, world))
        else:
            self.kind, self.x = synth.make_workload(name, seed=1000 * rank)
        x = self.x

        def dev(a):
            a = np.ascontiguousarray(a)
            if a.dtype == np.uint16:
                a = a.view(np.int16)
            return torch.from_numpy(a).cuda()

        self.host_inputs = {}
        if self.kind.startswith("wkv4"):
            names = ("k", "v", "w", "u") + (("dy",) if self.kind == "wkv4_bwd" else ())
        elif self.kind == "wkv6_fwd_fused":
            names = ("r", "k", "v", "ww", "w_base", "u", "g", "gn_w", "gn_b")
        else:
            names = ("r", "k", "v", "w", "u") + (("dy",) if self.kind in ("wkv6_bwd_bidir", "wkv5_bwd") else ())
        self.inputs = {n: dev(getattr(x, n)) for n in names}
        if getattr(x, "dtype", "f32") == "bf16" and "dy" in names:
            self.inputs["dy"] = dev(synth.to_bf16_bits(x.dy))   # the bf16 backward takes dy in bf16 too
        shape = (x.B, x.T, x.C)
        if self.kind == "wkv6_bwd_bidir":
            self.outputs = [torch.empty(shape, device="cuda") for _ in range(4)] + [torch.empty(x.C, device="cuda")]
            import linear_attention_rnn_wkv6_b200 as wkv
            self.ws_bytes = wkv.wkv6_bwd_workspace_bytes(x.B, x.T, x.C, x.H, 1)
            self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        elif self.kind == "wkv5_bwd":
            import linear_attention_rnn_wkv6_b200 as wkv
            self.outputs = [torch.empty(shape, device="cuda") for _ in range(3)] + \
                           [torch.empty(x.C, device="cuda") for _ in range(2)]
            self.ws_bytes = wkv.wkv5_bwd_workspace_bytes(x.B, x.T, x.C, x.H)
            self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        elif self.kind == "wkv4_bwd":
            import linear_attention_rnn_wkv6_b200 as wkv
            self.outputs = [torch.empty(shape, device="cuda") for _ in range(2)] + \
                           [torch.empty(x.C, device="cuda") for _ in range(2)]
            self.ws_bytes = wkv.wkv4_bwd_workspace_bytes(x.B, x.T, x.C)
            self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        else:
            self.outputs = [torch.empty(shape, device="cuda")]
        if self.kind == "wkv6_decode":
            # the recurrent state stays resident on the device (updated in place every step)
            self.state = dev(synth.make_state(x.B, x.H, seed=1000 * rank + 1))
        if self.kind == "wkv6_fwd_state":
            # the initial state is an input resident on the device; the final state an output
            self.state = dev(synth.make_state(x.B, x.H, seed=1000 * rank + 1))
            self.outputs.append(torch.empty((x.B, x.H, 64, 64), device="cuda"))
        self.units = units_of(name, x)
        self.tokens = tokens_of(x)

    def footprint(self) -> int:
        """Bytes of device memory one call touches: inputs, outputs and workspace."""
        ts = list(self.inputs.values()) + list(self.outputs)
        ts += [t for t in (getattr(self, "ws", None), getattr(self, "state", None)) if t is not None]
        return sum(t.numel() * t.element_size() for t in ts)

    def run(self, stream, inputs=None, outputs=None):
        import linear_attention_rnn_wkv6_b200 as wkv
        x, i = self.x, (inputs or self.inputs)
        o = outputs or self.outputs
        s = stream.cuda_stream
        if self.kind == "wkv4_fwd":
            wkv.wkv4_fwd(x.B, x.T, x.C, i["k"], i["v"], i["w"], i["u"], o[0], s)
        elif self.kind == "wkv6_fwd":
            wkv.wkv6_fwd(x.B, x.T, x.C, x.H, i["r"], i["k"], i["v"], i["w"], i["u"], o[0], s)
        elif self.kind == "wkv4_bwd":
            wkv.wkv4_bwd(x.B, x.T, x.C, i["k"], i["v"], i["w"], i["u"], i["dy"], *o, self.ws, self.ws_bytes, s)
        elif self.kind == "wkv6_bidir_fwd":
            wkv.wkv6_bidir_fwd(x.B, x.T, x.C, x.H, i["r"], i["k"], i["v"], i["w"], i["u"], o[0], s)
        elif self.kind == "wkv6_fwd_bf16":
            wkv.wkv6_fwd_bf16(x.B, x.T, x.C, x.H, i["r"], i["k"], i["v"], i["w"], i["u"], o[0], s)
        elif self.kind == "wkv6_bwd_bidir" and x.dtype == "bf16":
            wkv.wkv6_bwd_bf16(x.B, x.T, x.C, x.H, 1, i["r"], i["k"], i["v"], i["w"], i["u"], i["dy"], *o,
                              self.ws, self.ws_bytes, s)
        elif self.kind == "wkv6_bwd_bidir":
            wkv.wkv6_bwd(x.B, x.T, x.C, x.H, 1, i["r"], i["k"], i["v"], i["w"], i["u"], i["dy"], *o,
                         self.ws, self.ws_bytes, s)
        elif self.kind == "wkv6_fwd_fused":
            wkv.wkv6_fwd_fused(x.B, x.T, x.C, x.H, x.bidir, *(i[n] for n in ("r", "k", "v", "ww", "w_base", "u", "g",
                                                                            "gn_w", "gn_b")), x.eps, o[0], s)
        elif self.kind == "wkv5_fwd_bf16":
            wkv.wkv5_fwd_bf16(x.B, x.T, x.C, x.H, i["r"], i["k"], i["v"], i["w"], i["u"], o[0], s)
        elif self.kind == "wkv5_bwd":
            wkv.wkv5_bwd(x.B, x.T, x.C, x.H, i["r"], i["k"], i["v"], i["w"], i["u"], i["dy"], *o,
                         self.ws, self.ws_bytes, s)
        elif self.kind == "wkv6_decode":
            # [B,1,C] token tensors are the [B,C] arrays the step reads
            wkv.wkv6_decode(x.B, x.C, x.H, i["r"], i["k"], i["v"], i["w"], i["u"], self.state, o[0], s)
        elif self.kind == "wkv6_fwd_state":
            wkv.wkv6_fwd_state(x.B, x.T, x.C, x.H, i["r"], i["k"], i["v"], i["w"], i["u"], self.state, o[0], o[1], s)
        elif self.kind == "wkv5_fwd":
            wkv.wkv5_fwd(x.B, x.T, x.C, x.H, i["r"], i["k"], i["v"], i["w"], i["u"], o[0], s)
        else:
            raise ValueError(self.kind)
        if self.split and self.kind in ("wkv6_bwd_bidir", "wkv4_bwd"):
            # the batch-split backward's one exchange: the per-channel gradients summed
            # over the batch (du; RWKV-4 also dw) are all-reduced over the ranks
            import torch
            from linear_attention_rnn_wkv6_b200.shard import allreduce_du
            with torch.cuda.stream(stream):
                for t in (o[4],) if self.kind == "wkv6_bwd_bidir" else (o[2], o[3]):
                    allreduce_du(t)


class HostSide:
    """Pinned host copies of one workload's inputs and outputs for the end-to-end measurement."""

    def __init__(self, dw: DeviceWorkload):
        import torch
        self.dw = dw
        self.h_in = {n: t.cpu().pin_memory() for n, t in dw.inputs.items()}
        self.d_in = {n: torch.empty_like(t) for n, t in dw.inputs.items()}
        self.d_out = [torch.empty_like(t) for t in dw.outputs]
        self.h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dw.outputs]
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values())
        self.d2h = sum(t.numel() * t.element_size() for t in self.h_out)

        self.comp_done = None   # the last call on d_in / d_out
        self.out_done = None    # the last copy out of d_out

    def run(self, s_in, s_comp, s_out):
        """Copy this workload's inputs in (s_in), call it (s_comp), copy its outputs out
        (s_out).  Events keep the order copy-in -> call -> copy-out, keep the next
        copy-in behind the previous call (which reads d_in) and the next call behind
        the previous copy-out (which reads d_out); the transfers of one workload then
        overlap the calls and transfers of the others, in both directions of the link."""
        import torch
        if self.comp_done is not None:
            s_in.wait_event(self.comp_done)
        with torch.cuda.stream(s_in):
            for n, t in self.h_in.items():
                self.d_in[n].copy_(t, non_blocking=True)
        in_done = torch.cuda.Event()
        in_done.record(s_in)
        s_comp.wait_event(in_done)
        if self.out_done is not None:
            s_comp.wait_event(self.out_done)
        self.dw.run(s_comp, inputs=self.d_in, outputs=self.d_out)
        self.comp_done = torch.cuda.Event()
        self.comp_done.record(s_comp)
        s_out.wait_event(self.comp_done)
        with torch.cuda.stream(s_out):
            for h, d in zip(self.h_out, self.d_out):
                h.copy_(d, non_blocking=True)
        self.out_done = torch.cuda.Event()
        self.out_done.record(s_out)


def run_native(args, rank, world, local):
    import torch
    import linear_attention_rnn_wkv6_b200 as wkv
    torch.cuda.set_device(local)
    dist = init_group("nccl", world)
    dev = torch.device("cuda", local)
    # the selected build for the rest of this process (the context manager is kept
    # referenced: a generator context dropped after __enter__ would be closed, and its
    # exit would restore the default build)
    library_ctx = wkv.use_library(args.library)
    library_ctx.__enter__()
    wkv.load()
    if os.path.basename(wkv.lib_path()) != wkv.LIBRARY_FILES[args.library]:
        raise RuntimeError(f"library {args.library!r} not selected")
    wls = [DeviceWorkload(n, rank, world) for n in (args.only or STEP_WORKLOADS)]
    stream = torch.cuda.Stream()
    tokens_per_step = sum(w.tokens for w in wls)
    # A working set that fits in L2 several times over would stay cached from one step
    # to the next: then every step starts after a write of FLUSH_BYTES (evicting L2),
    # outside the kernels' events, and the step time is the sum of those events.
    ws_bytes = sum(w.footprint() for w in wls)
    flush = ws_bytes < FLUSH_BYTES
    scratch = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev) if flush else None

    def step(evs=None):
        if flush:
            with torch.cuda.stream(stream):
                scratch.fill_(1.0)
        for j, w in enumerate(wls):
            if evs is not None:
                evs[j][0].record(stream)
            w.run(stream)
            if evs is not None:
                evs[j][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if wkv.wkv_take_device_faults() != 0:
        raise RuntimeError("device fault word set during warm-up")

    K = args.steps
    kev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in wls]
           for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0.record(stream)
        for k in range(K):
            step(kev[k])
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(dist)
    elapsed_ms = t0.elapsed_time(t1)
    per_kernel_ms = [sum(kev[k][j][0].elapsed_time(kev[k][j][1]) for k in range(K)) / K for j in range(len(wls))]
    if wkv.wkv_take_device_faults() != 0:
        raise RuntimeError("device fault word set during the timed region")
    elapsed_ms = max_over_ranks(elapsed_ms, dist, dev)
    ms_per_step = elapsed_ms / K
    if flush:
        ms_per_step = max_over_ranks(sum(per_kernel_ms), dist, dev)
    value = tokens_per_step * world / (ms_per_step / 1e3)

    # end-to-end through the public API with host buffers (pinned), copies inside the timed region
    # on three streams (copies in, calls, copies out): see HostSide.run
    hs = [HostSide(w) for w in wls] if not args.no_e2e else []
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    for _ in range(max(1, min(args.warmup, 2))):
        for h in hs:
            h.run(s_in, stream, s_out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    Ke = max(1, min(K, 5))
    barrier(dist)
    torch.cuda.synchronize()
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for _ in range(Ke):
        for h in hs:
            h.run(s_in, stream, s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    # the kernels are deterministic: what came back through the host must equal, bit for
    # bit, what the device-timed calls on the same inputs left in their outputs
    for h in hs:
        for ho, do in zip(h.h_out, h.dw.outputs):
            if not torch.equal(ho, do.cpu()):
                raise RuntimeError(f"{h.dw.name}: end-to-end outputs differ from the device run's")
    barrier(dist)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    e2e_value = tokens_per_step * world * Ke / (e2e_ms / 1e3) if hs else None
    h2d = sum(h.h2d for h in hs)
    d2h = sum(h.d2h for h in hs)

    if rank == 0:
        hbm, hbm_src = load_peaks()
        tc_peak, tc_src = load_tensor_peak()
        kernels = {}
        for j, w in enumerate(wls):
            a = ALG[w.name]
            t_s = per_kernel_ms[j] / 1e3
            alg_bytes = a["bytes_per_unit"] * w.units
            alg_flops = a["flops_per_unit"] * w.units
            # roofline time = the slower of the bytes at HBM bandwidth and the flops at the
            # peak of the pipe the kernel computes on (the tensor pipe for the chunked forms,
            # the FP32 FMA pipe for the recurrences); frac = roofline time / measured time
            pipe = "tensor" if uses_tensor_cores(w.name, args.library) else "fp32"
            t_bytes = alg_bytes / (hbm * 1e9)
            t_flops = alg_flops / ((tc_peak if pipe == "tensor" else FP32_PEAK_TFLOPS) * 1e12)
            if t_bytes >= t_flops:
                bound, achieved, peak, unit = "hbm", alg_bytes / t_s / 1e9, hbm, "GB/s"
                peak_src = f"{hbm_src} HBM copy bandwidth"
            elif pipe == "tensor":
                bound, achieved, peak, unit = "tensor", alg_flops / t_s / 1e12, tc_peak, "TFLOP/s"
                peak_src = f"{tc_src} bf16 tensor throughput"
            else:
                bound, achieved, peak, unit = "alu", alg_flops / t_s / 1e12, FP32_PEAK_TFLOPS, "TFLOP/s"
                peak_src = "derived FP32 FMA peak: 148 SMs x 128 lanes x 2 flop x 1965 MHz"
            kernels[w.name] = {
                "entry": ENTRY[w.name], "launches": LAUNCHES[w.name], "ms": round(per_kernel_ms[j], 4),
                "tokens_per_s": round(w.tokens / t_s, 1), "units": w.units,
                "alg_bytes": alg_bytes, "alg_flops": alg_flops, "pipe": pipe,
                "hbm_gbs": round(alg_bytes / t_s / 1e9, 1), "fp32_tflops": round(alg_flops / t_s / 1e12, 2),
                "hbm_frac": round(alg_bytes / t_s / 1e9 / hbm, 4),
                "fp32_frac": round(alg_flops / t_s / 1e12 / FP32_PEAK_TFLOPS, 4),
                "bound": bound, "achieved": round(achieved, 3), "peak": round(peak, 2), "unit": unit,
                "frac": round(max(t_bytes, t_flops) / t_s, 4), "peak_source": peak_src,
                "share": round(per_kernel_ms[j] / sum(per_kernel_ms), 4),
            }
        dom = max(kernels, key=lambda n: kernels[n]["ms"])
        d = kernels[dom]
        traffic = recorded_traffic(dom)
        clocks = clk.summary()
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 (bf16 inputs on the causal workload)",
            "data": ("synthetic (seeded splitmix64 + Box-Muller): one problem of N x B batches, each rank "
                     "generating its own window of batches" if world > 1 else "synthetic (seeded splitmix64 + "
                     "Box-Muller, seed 0)"),
            "config": {"workload": WORKLOAD_NAME if not args.only else " + ".join(args.only),
                       "tokens_per_step_per_gpu": tokens_per_step,
                       "l2": (f"working set {ws_bytes / 1e6:.0f} MB: L2 (126 MB) flushed before every step by a "
                              f"{FLUSH_BYTES >> 20} MB write outside the kernels' events; ms_per_step is the sum "
                              "of the kernels' event times") if flush else
                             f"inputs larger than L2: step working set {ws_bytes / 1e9:.2f} GB > 126 MB L2, "
                             "no explicit flush",
                       "parallelism": (f"batch split x{world}: one problem of {world} x B batches, rank r "
                                       "owning batches [rB, (r+1)B) (weak scaling: B per GPU fixed); the backward's "
                                       "du all-reduced over the ranks (NCCL, C floats) inside every step"
                                       if world > 1 else "single GPU"),
                       "library": os.path.basename(wkv.lib_path())},
            "roofline": {"kernel": dom, "bound": d["bound"],
                         "achieved": d["achieved"], "peak": d["peak"], "unit": d["unit"], "frac": d["frac"],
                         "traffic": traffic, "peak_source": d["peak_source"]},
            "kernels": kernels,
            "e2e": {"value": round(e2e_value, 1) if e2e_value else None, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": Ke,
                    "note": "public C-ABI calls; every step copies all inputs in from pinned host memory and all "
                            "outputs out, on copy streams of their own, overlapped with the other workloads' "
                            "calls and copies"},
            "gpu_launches": K * sum(LAUNCHES[w.name] for w in wls),
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline and not args.only:
            line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- CPU oracle (baseline / reference arm)

def _oracle_jobs(name: str, x, max_units: int):
    """The oracle calls of a bounded sample of workload `name`, as (prepare, run, units):
    prepare() builds the call's float64 arguments, run(args) is the oracle call.  A unit
    is one (b, channel) series (RWKV-4) or one (b, h) slice, T tokens each."""
    import numpy as np
    import oracle
    oracle.build()
    jobs = []
    if name.startswith("wkv4"):
        blk = 16   # contiguous channel blocks
        for i in range(max_units // blk):
            b, c0 = i % x.B, (i * blk) % x.C
            jobs.append((lambda b=b, c0=c0: (x.k[b:b + 1, :, c0:c0 + blk], x.v[b:b + 1, :, c0:c0 + blk],
                                             x.w[c0:c0 + blk], x.u[c0:c0 + blk]),
                         lambda a: oracle.wkv4_fwd(*a), blk))
        return jobs
    bwd = name == "wkv6_bidir_bwd_f32_b32t196h12"
    for i in range(max_units):
        b, h = (i * 7 + 3) % x.B, (i * 5 + 1) % x.H
        sl = slice(h * N, (h + 1) * N)

        def prepare(b=b, sl=sl):
            a = tuple(x.as_f64(n, slice(b, b + 1), sl) for n in ("r", "k", "v", "w")) + (x.u[sl].astype(np.float64),)
            return a + (x.dy[b:b + 1, :, sl].astype(np.float64),) if bwd else a

        if bwd:
            run = lambda a: oracle.wkv6_bwd(*a, H=1, bidirectional=True)
        else:
            run = lambda a: oracle.wkv6_fwd(*a, H=1, bidirectional="bidir" in name)
        jobs.append((prepare, run, 1))
    return jobs


def _oracle_unit_seconds(name: str, x, max_units: int, budget_s: float):
    """Time the oracle, one call after another (arguments prepared outside the clock),
    on up to max_units units of workload `name` within ~budget_s.
    Returns (seconds per token-unit, jobs run, description)."""
    jobs = _oracle_jobs(name, x, max_units)
    done, units, spent = 0, 0, 0.0
    for prepare, run, n in jobs:
        a = prepare()
        t = time.perf_counter()
        run(a)
        spent += time.perf_counter() - t
        done += 1
        units += n
        if spent > budget_s:
            break
    what = f"{units} channels" if name.startswith("wkv4") else f"{units} (b,h) slices"
    return spent / (units * x.T), done, f"{what} x T={x.T}"


def _oracle_all_cores_seconds(name: str, x, jobs_done: int, threads: int):
    """The same first `jobs_done` oracle calls spread over `threads` threads (the oracle
    runs in C with the interpreter lock released, and keeps no state between calls);
    each thread prepares its calls' arguments inside the timed wall.
    Returns wall seconds per token-unit."""
    from concurrent.futures import ThreadPoolExecutor
    jobs = _oracle_jobs(name, x, 4096)[:jobs_done]
    units = sum(n for _, _, n in jobs)
    work = lambda j: j[1](j[0]())
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(work, jobs[:threads]))   # start the threads
        t = time.perf_counter()
        list(ex.map(work, jobs))
        wall = time.perf_counter() - t
    return wall / (units * x.T)


def cpu_baseline(seconds_total: float = 12.0, all_cores: bool = True):
    """The oracle on a bounded sample of each workload, scaled to the full step:
    single-threaded (the value), and the same calls over every host core."""
    import os
    from linear_attention_rnn_wkv6_b200 import synth
    est_step_s, est_all_s, samples = 0.0, 0.0, []
    tokens = 0
    threads = os.cpu_count() or 1
    for name in STEP_WORKLOADS:
        kind, x = synth.make_workload(name, seed=0)
        per_unit_s, done, desc = _oracle_unit_seconds(name, x, max_units=4096, budget_s=seconds_total / 4)
        units = units_of(name, x)
        est_step_s += per_unit_s * units
        if all_cores:
            est_all_s += _oracle_all_cores_seconds(name, x, done, threads) * units
        tokens += tokens_of(x)
        samples.append(f"{name}: {desc}")
    out = {"value": round(tokens / est_step_s, 2), "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": "; ".join(samples) + "; time per unit scaled to the full step",
           "est_step_s": round(est_step_s, 3)}
    if all_cores:
        out["all_cores"] = {"value": round(tokens / est_all_s, 2), "unit": UNIT, "cores": threads,
                            "note": "the same oracle calls on independent units over a thread per host core"}
    return out


def run_reference(args, rank, world):
    if rank != 0:
        return
    t_start = time.perf_counter()
    from linear_attention_rnn_wkv6_b200 import synth
    budget = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    per_step = []
    tokens = sum(tokens_of(synth.make_workload(n, 0)[1]) for n in STEP_WORKLOADS)
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(budget, all_cores=False)
        if i >= args.warmup:
            per_step.append(cb["est_step_s"])
    est = statistics.median(per_step)
    value = tokens / est
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(est * 1e3, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs)",
        "config": {"workload": WORKLOAD_NAME,
                   "note": "double-precision CPU oracle, single thread; each step times a bounded sample and "
                           "scales it to the full workload"},
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": cb["sample"]},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(time.perf_counter() - t_start, 1),
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle time budget of the cpu_baseline leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--only", action="append", choices=STEP_WORKLOADS + EXTRA_WORKLOADS,
                    help="run only these workloads (profiling); the default step runs all four")
    ap.add_argument("--library", choices=["default", "recurrence"], default="default",
                    help="the library build to time: the product (default) or the test build whose "
                         "chunked-form entry points run the recurrence kernels (for comparison)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_env()
    if world != args.gpus and world == 1 and args.gpus > 1:
        ap.error("for --gpus > 1 launch under torchrun (one process per GPU)")
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_native(args, rank, world, local)


if __name__ == "__main__":
    main()
