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


def library_for(path: str):
    """The library build whose entry points run `path`'s kernels: the product
    (chunked tensor-core forms, "tensor"/"tensor_cores") or the test build
    ("recurrence": the token-by-token recurrence kernels)."""
    return wkv.use_library("recurrence" if path == "recurrence" else "default")


# ---------------------------------------------------------------- guard bands
# compute-sanitizer is not available here, so every device buffer a GPU test hands
# the library sits between two 4 KiB margins filled with a sentinel byte.  After
# each test (and wherever a test calls check_guards) the margins must be intact:
# a store past either end of an output, a workspace or a state buffer, or into an
# input, shows up as a changed margin byte.
GUARD_BYTES = 4096
SENTINEL = 0xA5
_GUARDS: list = []


def _guarded(nbytes: int, dtype, shape):
    """A device tensor of `shape` (`nbytes` bytes, dtype `dtype`) at a 4 KiB offset into
    a larger buffer whose margins hold SENTINEL; registered for check_guards()."""
    t = torch()
    buf = t.full((nbytes + 2 * GUARD_BYTES,), SENTINEL, dtype=t.uint8, device="cuda")
    inner = buf[GUARD_BYTES:GUARD_BYTES + nbytes].view(dtype).view(shape)
    assert inner.data_ptr() % 16 == 0 and inner.is_contiguous()
    _GUARDS.append(buf)
    return inner


def check_guards() -> None:
    """Synchronise, then assert that every registered buffer's margins are intact."""
    t = torch()
    if not _GUARDS:
        return
    t.cuda.synchronize()
    for buf in _GUARDS:
        head = buf[:GUARD_BYTES]
        tail = buf[buf.numel() - GUARD_BYTES:]
        for name, m in (("before", head), ("after", tail)):
            bad = (m != SENTINEL).nonzero()
            assert bad.numel() == 0, f"guard band {name} a device buffer was written at byte {int(bad[0])}"
    _GUARDS.clear()


def dev(a: np.ndarray):
    """A copy of `a` on the device, inside guard bands."""
    t = torch()
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    src = t.from_numpy(a)
    out = _guarded(src.numel() * src.element_size(), src.dtype, tuple(src.shape))
    out.copy_(src)
    return out


def empty_nan(shape):
    """A float32 output on the device, filled with NaN (so an element the kernel leaves
    unwritten shows), inside guard bands."""
    t = torch()
    n = int(np.prod(shape)) if len(shape) else 1
    out = _guarded(4 * n, t.float32, tuple(shape))
    out.fill_(float("nan"))
    return out


def workspace(nbytes: int):
    """A device workspace of `nbytes` (at least 16) bytes inside guard bands."""
    t = torch()
    n = max(int(nbytes), 16)
    return _guarded(n, t.uint8, (n,))


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
    check_guards()
    return y.cpu().numpy()


def run_wkv6_bwd(x: synth.Wkv6Inputs, bidir: bool):
    t = torch()
    r, k, v, w, u, dy = (dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u", "dy"))
    outs = [empty_nan((x.B, x.T, x.C)) for _ in range(4)] + [empty_nan((x.C,))]
    nbytes = wkv.wkv6_bwd_workspace_bytes(x.B, x.T, x.C, x.H, bidir)
    ws = workspace(nbytes)
    wkv.wkv6_bwd(x.B, x.T, x.C, x.H, bidir, r, k, v, w, u, dy, *outs, ws, nbytes)
    assert wkv.wkv_take_device_faults() == 0
    check_guards()
    return tuple(o.cpu().numpy() for o in outs)


def run_wkv4(x: synth.Wkv4Inputs) -> np.ndarray:
    k, v, w, u = (dev(getattr(x, n)) for n in ("k", "v", "w", "u"))
    y = empty_nan((x.B, x.T, x.C))
    wkv.wkv4_fwd(x.B, x.T, x.C, k, v, w, u, y)
    assert wkv.wkv_take_device_faults() == 0
    check_guards()
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
    ws = workspace(nbytes)
    wkv.wkv6_bwd_bf16(x.B, x.T, x.C, x.H, bidir, r, k, v, w, u, dy, *outs, ws, nbytes)
    assert wkv.wkv_take_device_faults() == 0
    check_guards()
    return tuple(o.cpu().numpy() for o in outs), synth.bf16_bits_to_f32(dy_bits).astype(np.float64)


# ---------------------------------------------------------------- whole-tensor oracle references
# Every batch of a WKV problem is an independent problem, so the oracle runs one
# batch per host thread (it is C called through ctypes, which releases the
# interpreter lock, and keeps no state between calls).

def _map_batches(fn, B: int):
    import os
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=min(B, os.cpu_count() or 4)) as ex:
        return list(ex.map(fn, range(B)))


def _batch_f64(x: synth.Wkv6Inputs, b: int):
    bs = slice(b, b + 1)
    return [x.as_f64(n, bs) for n in ("r", "k", "v", "w")] + [x.u.astype(np.float64)]


def oracle_fwd_full(x: synth.Wkv6Inputs, bidir: bool) -> np.ndarray:
    """The oracle's RWKV-6 forward over the whole [B,T,C] problem."""
    import oracle
    ys = _map_batches(lambda b: oracle.wkv6_fwd(*_batch_f64(x, b), H=x.H, bidirectional=bidir)[0], x.B)
    return np.stack(ys)


def oracle_bwd_full(x: synth.Wkv6Inputs, bidir: bool, dy64: np.ndarray | None = None):
    """The oracle's RWKV-6 backward over the whole problem: dr, dk, dv, dw [B,T,C] and du [C]
    (the per-batch du summed in increasing b).  dy64: the float64 upstream gradient the
    kernels saw (default: x.dy)."""
    import oracle
    dy64 = x.dy.astype(np.float64) if dy64 is None else dy64

    def one(b):
        return oracle.wkv6_bwd(*_batch_f64(x, b), dy64[b:b + 1], H=x.H, bidirectional=bidir)

    parts = _map_batches(one, x.B)
    outs = [np.concatenate([p[i] for p in parts]) for i in range(4)]
    du = np.zeros(x.C)
    for p in parts:
        du += p[4]
    return (*outs, du)
