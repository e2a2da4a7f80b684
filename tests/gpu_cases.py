"""Helpers for the GPU parity tests: run the C-ABI entry points on synthetic
inputs and compute oracle references on the same (exact) input values."""
from __future__ import annotations

import math

import numpy as np

import linear_attention_rnn_wkv6_b200 as wkv
from linear_attention_rnn_wkv6_b200 import synth

TOL_F32_FWD = 1e-5     # relative L2, fp32 forward
TOL_BF16_FWD = 2e-2    # relative L2, bf16 inputs, fp32 state and output
TOL_F32_GRAD = 1e-4    # relative L2 per gradient tensor


def torch():
    import torch as _t
    return _t


def dev(a: np.ndarray):
    t = torch()
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return t.from_numpy(a).cuda()


def empty_nan(shape):
    t = torch()
    return t.full(shape, float("nan"), dtype=t.float32, device="cuda")


def run_wkv6_fwd(x: synth.Wkv6Inputs, bidir: bool = False, sync: bool = True) -> np.ndarray:
    r, k, v, w, u = (dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u"))
    y = empty_nan((x.B, x.T, x.C))
    if x.dtype == "bf16":
        assert not bidir
        wkv.wkv6_fwd_bf16(x.B, x.T, x.C, x.H, r, k, v, w, u, y)
    elif bidir:
        wkv.wkv6_bidir_fwd(x.B, x.T, x.C, x.H, r, k, v, w, u, y)
    else:
        wkv.wkv6_fwd(x.B, x.T, x.C, x.H, r, k, v, w, u, y)
    assert wkv.wkv_take_device_faults() == 0
    return y.cpu().numpy()


def run_wkv6_bwd(x: synth.Wkv6Inputs, bidir: bool):
    t = torch()
    r, k, v, w, u, dy = (dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u", "dy"))
    outs = [empty_nan((x.B, x.T, x.C)) for _ in range(4)] + [empty_nan((x.C,))]
    nbytes = wkv.wkv6_bwd_workspace_bytes(x.B, x.T, x.C, x.H, bidir)
    ws = t.empty(max(nbytes, 16), dtype=t.uint8, device="cuda")
    wkv.wkv6_bwd(x.B, x.T, x.C, x.H, bidir, r, k, v, w, u, dy, *outs, ws, nbytes)
    assert wkv.wkv_take_device_faults() == 0
    return tuple(o.cpu().numpy() for o in outs)


def run_wkv4(x: synth.Wkv4Inputs) -> np.ndarray:
    k, v, w, u = (dev(getattr(x, n)) for n in ("k", "v", "w", "u"))
    y = empty_nan((x.B, x.T, x.C))
    wkv.wkv4_fwd(x.B, x.T, x.C, k, v, w, u, y)
    assert wkv.wkv_take_device_faults() == 0
    return y.cpu().numpy()


def f64(x: synth.Wkv6Inputs):
    return [x.as_f64(n) for n in ("r", "k", "v", "w")] + [x.u.astype(np.float64)]


def unit_slice(x: synth.Wkv6Inputs, b: int, h: int):
    """The oracle's inputs for one (b, h) unit, as a B=1, H=1 problem."""
    N = x.C // x.H
    sl = slice(h * N, (h + 1) * N)
    out = [x.as_f64(n, slice(b, b + 1), sl) for n in ("r", "k", "v", "w")] + [x.u[sl].astype(np.float64)]
    dy = x.dy[b:b + 1, :, sl].astype(np.float64) if x.dy is not None else None
    return out, dy, sl


def sample_units(B: int, H: int, n: int):
    """min(n, B*H) distinct (b, h) units spread over batch and heads, deterministic.

    Walks the B*H units with a stride coprime to B*H, so it always terminates."""
    total = B * H
    n = min(n, total)
    start = max(1, total // max(n, 1))
    stride = next(s for s in range(start, start + total + 1) if math.gcd(s, total) == 1)
    return [divmod((i * stride + 3) % total, H) for i in range(n)]


def run_wkv6_bwd_bf16(x: synth.Wkv6Inputs, bidir: bool):
    """wkv6_bwd_bf16 on bf16 inputs (x.dtype == "bf16"); dy is rounded to bf16 the same way.
    Returns the fp32 gradients and the float64 dy the oracle must see."""
    t = torch()
    assert x.dtype == "bf16"
    dy_bits = synth.to_bf16_bits(x.dy)
    r, k, v, w, dy = (dev(a) for a in (x.r, x.k, x.v, x.w, dy_bits))
    u = dev(x.u)
    outs = [empty_nan((x.B, x.T, x.C)) for _ in range(4)] + [empty_nan((x.C,))]
    nbytes = wkv.wkv6_bwd_workspace_bytes(x.B, x.T, x.C, x.H, bidir)
    ws = t.empty(max(nbytes, 16), dtype=t.uint8, device="cuda")
    wkv.wkv6_bwd_bf16(x.B, x.T, x.C, x.H, bidir, r, k, v, w, u, dy, *outs, ws, nbytes)
    assert wkv.wkv_take_device_faults() == 0
    return tuple(o.cpu().numpy() for o in outs), synth.bf16_bits_to_f32(dy_bits).astype(np.float64)
