"""Seeded synthetic inputs for the WKV operator (shared by the CUDA path and the oracle).

This module only draws random numbers and lays them out; it holds none of the
operator's arithmetic.  Both the CUDA path and the double-precision oracle
consume the arrays it returns, so parity compares the two on identical bits.

Generator (counter based, independent of numpy/torch RNG versions):

* splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): ``z = seed + (i + 1) * 0x9E3779B97F4A7C15`` followed
  by the published 64-bit finaliser.  Element ``i`` of a stream is a pure
  function of ``(seed, stream, i)``, so any slice can be regenerated alone.
* uniform in [0, 1): top 53 bits of a draw times 2^-53.
* normal: Box-Muller, one normal per pair of draws (2i, 2i+1), cosine branch.
* every array has its own stream id (draw order r, k, v, w_raw, u, dy, then
  the initial recurrent state s0).

The log-decay handed to the WKV6 entry points is ``ew = -exp(w_raw)``, computed
here in float64 and then rounded to the input dtype: it is the input recipe of
the workloads (decay ``exp(-exp(w_raw))``), not part of the operator.
bf16 inputs are float64 -> float32 -> bfloat16 with round-to-nearest-even.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os
import threading

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_R, STREAM_K, STREAM_V, STREAM_WRAW, STREAM_U, STREAM_DY, STREAM_S0, STREAM_WW, STREAM_G, STREAM_GN = range(10)

_CHUNK = 1 << 16  # elements per block: scratch stays cache resident and is reused in place
_SCALE53 = 1.0 / 9007199254740992.0
_tls = threading.local()


def _mix_inplace(z: np.ndarray, tmp: np.ndarray) -> None:
    """splitmix64 finaliser, in place (no fresh temporaries: first-touch page faults dominate)."""
    np.right_shift(z, np.uint64(30), out=tmp)
    np.bitwise_xor(z, tmp, out=z)
    np.multiply(z, _M1, out=z)
    np.right_shift(z, np.uint64(27), out=tmp)
    np.bitwise_xor(z, tmp, out=z)
    np.multiply(z, _M2, out=z)
    np.right_shift(z, np.uint64(31), out=tmp)
    np.bitwise_xor(z, tmp, out=z)


def _stream_seed(seed: int, stream: int) -> np.uint64:
    z = np.array([(seed * 0x100000001B3 + 0x5851F42D4C957F2D * (stream + 1)) & 0xFFFFFFFFFFFFFFFF],
                 dtype=np.uint64)
    with np.errstate(over="ignore"):
        _mix_inplace(z, np.empty_like(z))
    return z[0]


def _scratch():
    sc = getattr(_tls, "sc", None)
    if sc is None:
        n2 = 2 * _CHUNK
        sc = dict(ramp=np.arange(n2, dtype=np.uint64), z=np.empty(n2, np.uint64),
                  tmp=np.empty(n2, np.uint64), f=np.empty(n2, np.float64), g=np.empty(_CHUNK, np.float64))
        _tls.sc = sc
    return sc


def _uniform01_into(s: np.uint64, start: int, count: int, sc) -> np.ndarray:
    """Uniforms in [0,1) for counters [start, start+count) of the stream seeded s (count <= 2*_CHUNK)."""
    z, tmp, f = sc["z"][:count], sc["tmp"][:count], sc["f"][:count]
    with np.errstate(over="ignore"):
        np.add(sc["ramp"][:count], np.uint64(start + 1), out=z)
        np.multiply(z, _GOLDEN, out=z)
        np.add(z, s, out=z)
        _mix_inplace(z, tmp)
    np.right_shift(z, np.uint64(11), out=tmp)
    np.multiply(tmp, _SCALE53, out=f, casting="unsafe")
    return f


def _blocks(n: int, fill) -> None:
    """Run fill(a, m) over [0, n) in blocks, on a thread pool (numpy releases the GIL)."""
    starts = list(range(0, n, _CHUNK))
    if len(starts) <= 4:
        for a in starts:
            fill(a, min(_CHUNK, n - a))
        return
    workers = min(len(starts), max(1, (os.cpu_count() or 1)))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        list(ex.map(lambda a: fill(a, min(_CHUNK, n - a)), starts))


def uniform(seed: int, stream: int, n: int, lo: float, hi: float, offset: int = 0) -> np.ndarray:
    """n float64 uniforms in [lo, hi) for flat indices [offset, offset+n)."""
    out = np.empty(n, dtype=np.float64)
    s = _stream_seed(seed, stream)

    def fill(a, m):
        f = _uniform01_into(s, offset + a, m, _scratch())
        o = out[a:a + m]
        np.multiply(f, hi - lo, out=o)
        np.add(o, lo, out=o)

    _blocks(n, fill)
    return out


def normal(seed: int, stream: int, n: int, std: float, offset: int = 0) -> np.ndarray:
    """n float64 N(0, std^2) draws for flat indices [offset, offset+n)."""
    out = np.empty(n, dtype=np.float64)
    s = _stream_seed(seed, stream)
    two_pi = 2.0 * math.pi

    def fill(a, m):
        sc = _scratch()
        f = _uniform01_into(s, 2 * (offset + a), 2 * m, sc)
        u1, u2, g = f[0::2], f[1::2], sc["g"][:m]
        o = out[a:a + m]
        np.negative(u1, out=g)
        np.log1p(g, out=g)                 # ln(1 - u1)
        np.multiply(g, -2.0, out=g)
        np.sqrt(g, out=g)                  # sqrt(-2 ln(1 - u1))
        np.multiply(u2, two_pi, out=o)
        np.cos(o, out=o)
        np.multiply(o, g, out=o)
        if std != 1.0:
            np.multiply(o, std, out=o)

    _blocks(n, fill)
    return out


def to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    rnd = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + rnd) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Wkv6Inputs:
    B: int
    T: int
    C: int
    H: int
    r: np.ndarray      # [B,T,C] float32 (or bf16 bits, uint16)
    k: np.ndarray
    v: np.ndarray
    w: np.ndarray      # log-decay ew = -exp(w_raw), [B,T,C]; RWKV-5: decay rate [C] float32 (decay exp(-w))
    u: np.ndarray      # [C] float32
    dy: np.ndarray | None = None  # [B,T,C] float32 upstream gradient
    dtype: str = "f32"

    def as_f64(self, name: str, b=slice(None), c=slice(None)) -> np.ndarray:
        """Exact float64 copy of one input (optionally only batch slice b, channel slice c)."""
        a = getattr(self, name)
        if name in ("u",) or a.ndim == 1:
            return a[c].astype(np.float64)
        a = a[b, :, c] if a.ndim == 3 else a
        if self.dtype == "bf16" and name in ("r", "k", "v", "w"):
            return bf16_bits_to_f32(np.ascontiguousarray(a)).astype(np.float64)
        return a.astype(np.float64)


@dataclasses.dataclass
class Wkv4Inputs:
    B: int
    T: int
    C: int
    k: np.ndarray      # [B,T,C] float32
    v: np.ndarray      # [B,T,C] float32
    w: np.ndarray      # [C] float32, > 0 (decay exp(-w) per step)
    u: np.ndarray      # [C] float32
    dy: np.ndarray | None = None  # [B,T,C] float32 upstream gradient


def _batch_window(B: int, batches, T: int, C: int):
    """(first batch, number of batches, flat offset) of the window `batches` = (lo, hi)
    of a B-batch problem (None: all of it)."""
    lo, hi = (0, B) if batches is None else batches
    if not 0 <= lo <= hi <= B:
        raise ValueError(f"batch window {batches} outside [0, {B}]")
    return lo, hi - lo, lo * T * C


def make_wkv6(B: int, T: int, H: int, N: int = 64, *, seed: int = 0, rkv_std: float = 0.5,
              wraw_lo: float = -6.0, wraw_hi: float = -0.5, u_std: float = 0.5,
              with_dy: bool = False, dy_std: float = 1.0, dtype: str = "f32", batches=None) -> Wkv6Inputs:
    """RWKV-6 inputs: r,k,v ~ N(0, rkv_std^2), w_raw ~ U(wraw_lo, wraw_hi) per (t, channel),
    ew = -exp(w_raw), u ~ N(0, u_std^2) per channel, dy ~ N(0, dy_std^2).
    batches=(lo, hi): only batches lo..hi-1 of the B-batch problem (bit-identical to the
    same slice of the whole problem; B of the result is hi - lo)."""
    C = H * N
    _, Bl, off = _batch_window(B, batches, T, C)
    n = Bl * T * C
    shape = (Bl, T, C)

    def cast(x64: np.ndarray) -> np.ndarray:
        x32 = x64.astype(np.float32).reshape(shape)
        return to_bf16_bits(x32).reshape(shape) if dtype == "bf16" else x32

    r = cast(normal(seed, STREAM_R, n, rkv_std, offset=off))
    k = cast(normal(seed, STREAM_K, n, rkv_std, offset=off))
    v = cast(normal(seed, STREAM_V, n, rkv_std, offset=off))
    w = cast(-np.exp(uniform(seed, STREAM_WRAW, n, wraw_lo, wraw_hi, offset=off)))
    u = normal(seed, STREAM_U, C, u_std).astype(np.float32)
    dy = normal(seed, STREAM_DY, n, dy_std, offset=off).astype(np.float32).reshape(shape) if with_dy else None
    return Wkv6Inputs(Bl, T, C, H, r, k, v, w, u, dy, dtype)


def make_wkv5(B: int, T: int, H: int, N: int = 64, *, seed: int = 0, rkv_std: float = 0.5,
              wraw_lo: float = -6.0, wraw_hi: float = -0.5, u_std: float = 0.5,
              with_dy: bool = False, dy_std: float = 1.0, dtype: str = "f32") -> Wkv6Inputs:
    """RWKV-5 inputs: r, k, v, u, dy as make_wkv6 (same streams); the static decay rate
    w = exp(w_raw) >= 0 per channel, w_raw ~ U(wraw_lo, wraw_hi) (the first C draws of the
    w_raw stream), float32 also for bf16 r, k, v."""
    x = make_wkv6(B, T, H, N, seed=seed, rkv_std=rkv_std, wraw_lo=wraw_lo, wraw_hi=wraw_hi, u_std=u_std,
                  with_dy=with_dy, dy_std=dy_std, dtype=dtype)
    x.w = np.exp(uniform(seed, STREAM_WRAW, H * N, wraw_lo, wraw_hi)).astype(np.float32)
    return x


@dataclasses.dataclass
class FusedInputs:
    """Inputs of the RWKV-6 forward with the decay prologue and the norm/gate epilogue (fp32)."""
    B: int
    T: int
    C: int
    H: int
    bidir: bool
    r: np.ndarray      # [B,T,C]
    k: np.ndarray
    v: np.ndarray
    ww: np.ndarray     # [B,T,C] low-rank decay term tanh(x W1) W2
    w_base: np.ndarray # [C]
    u: np.ndarray      # [C]
    g: np.ndarray      # [B,T,C] gate
    gn_w: np.ndarray   # [C]
    gn_b: np.ndarray   # [C]
    eps: float = 64e-5


def make_fused(B: int, T: int, H: int, N: int = 64, *, seed: int = 0, bidir: bool = False,
               rkv_std: float = 0.5, base_lo: float = -6.0, base_hi: float = -1.0, ww_std: float = 0.5,
               u_std: float = 0.5, eps: float = 64e-5) -> FusedInputs:
    """r, k, v, u as make_wkv6 (same streams); w_base ~ U(base_lo, base_hi) per channel (the
    first C draws of the w_raw stream), ww ~ N(0, ww_std^2), so that the decay pre-activation
    w_base + ww spans the same range as make_wkv6's w_raw; the gate g ~ N(0, 1); the group
    norm's weight ~ N(1, 0.1^2) and bias ~ N(0, 0.1^2) per channel."""
    C = H * N
    n = B * T * C
    shape = (B, T, C)
    f32 = lambda a: a.astype(np.float32)
    r = f32(normal(seed, STREAM_R, n, rkv_std)).reshape(shape)
    k = f32(normal(seed, STREAM_K, n, rkv_std)).reshape(shape)
    v = f32(normal(seed, STREAM_V, n, rkv_std)).reshape(shape)
    w_base = f32(uniform(seed, STREAM_WRAW, C, base_lo, base_hi))
    u = f32(normal(seed, STREAM_U, C, u_std))
    ww = f32(normal(seed, STREAM_WW, n, ww_std)).reshape(shape)
    g = f32(normal(seed, STREAM_G, n, 1.0)).reshape(shape)
    gn_w = f32(1.0 + normal(seed, STREAM_GN, C, 0.1))
    gn_b = f32(normal(seed, STREAM_GN, C, 0.1, offset=C))
    return FusedInputs(B, T, C, H, bidir, r, k, v, ww, w_base, u, g, gn_w, gn_b, eps)


def make_state(B: int, H: int, N: int = 64, *, seed: int = 0, std: float = 1.0) -> np.ndarray:
    """An RWKV-6 recurrent state per (b, h): [B,H,N,N] float32 ~ N(0, std^2) (its own stream)."""
    return normal(seed, STREAM_S0, B * H * N * N, std).astype(np.float32).reshape(B, H, N, N)


def make_wkv4(B: int, T: int, C: int, *, seed: int = 0, kv_std: float = 1.0,
              logw_lo: float = -3.0, logw_hi: float = 1.0, u_std: float = 0.5,
              with_dy: bool = False, dy_std: float = 1.0, batches=None) -> Wkv4Inputs:
    """RWKV-4 inputs: k, v ~ N(0, kv_std^2); w = exp(U(logw_lo, logw_hi)) > 0 per channel;
    u ~ N(0, u_std^2) per channel; dy ~ N(0, dy_std^2).  batches: as make_wkv6."""
    _, Bl, off = _batch_window(B, batches, T, C)
    n = Bl * T * C
    k = normal(seed, STREAM_K, n, kv_std, offset=off).astype(np.float32).reshape(Bl, T, C)
    v = normal(seed, STREAM_V, n, kv_std, offset=off).astype(np.float32).reshape(Bl, T, C)
    w = np.exp(uniform(seed, STREAM_WRAW, C, logw_lo, logw_hi)).astype(np.float32)
    u = normal(seed, STREAM_U, C, u_std).astype(np.float32)
    dy = normal(seed, STREAM_DY, n, dy_std, offset=off).astype(np.float32).reshape(Bl, T, C) if with_dy else None
    return Wkv4Inputs(Bl, T, C, k, v, w, u, dy)


# The workloads: name -> (kind, constructor kwargs).
WORKLOADS = {
    # causal RWKV-6 forward, fp32, small (oracle finishes in seconds)
    "wkv6_causal_f32_b1t196h4": ("wkv6_fwd", dict(B=1, T=196, H=4)),
    # causal RWKV-6 forward, fp32, on the patch-sequence shape of the bidirectional workload
    "wkv6_causal_f32_b32t196h12": ("wkv6_fwd", dict(B=32, T=196, H=12)),
    # RWKV-4 scalar-state forward, fp32
    "wkv4_f32_b8t1024c768": ("wkv4_fwd", dict(B=8, T=1024, C=768)),
    # bidirectional RWKV-6 forward on 224px/16px patch sequences, fp32
    "wkv6_bidir_f32_b32t196h12": ("wkv6_bidir_fwd", dict(B=32, T=196, H=12)),
    # causal RWKV-6 forward, long text-shaped sequences, bf16 inputs, fp32 state/output
    "wkv6_causal_bf16_b8t4096h32": ("wkv6_fwd_bf16", dict(B=8, T=4096, H=32, wraw_lo=-8.0, dtype="bf16")),
    # bidirectional RWKV-6 backward, fp32
    "wkv6_bidir_bwd_f32_b32t196h12": ("wkv6_bwd_bidir", dict(B=32, T=196, H=12, with_dy=True)),
    # bidirectional RWKV-6 backward with bf16 inputs (fp32 gradients)
    "wkv6_bidir_bwd_bf16_b32t196h12": ("wkv6_bwd_bidir", dict(B=32, T=196, H=12, with_dy=True, dtype="bf16")),
    # RWKV-4 backward on the RWKV-4 forward's shape
    "wkv4_bwd_f32_b8t1024c768": ("wkv4_bwd", dict(B=8, T=1024, C=768, with_dy=True)),
    # one recurrent decode step for 512 sequences of the long-text head layout (state from make_state)
    "wkv6_decode_f32_b512h32": ("wkv6_decode", dict(B=512, T=1, H=32)),
    # RWKV-5 (static per-channel decay) forward on the long-text shape, bf16 r, k, v
    "wkv5_causal_bf16_b8t4096h32": ("wkv5_fwd_bf16", dict(B=8, T=4096, H=32, wraw_lo=-8.0, dtype="bf16")),
    # RWKV-5 backward, fp32, on the patch-sequence shape
    "wkv5_bwd_f32_b32t196h12": ("wkv5_bwd", dict(B=32, T=196, H=12, with_dy=True)),
    # bidirectional RWKV-6 forward with the decay prologue and the group-norm/gate epilogue, fp32
    "wkv6_bidir_fused_f32_b32t196h12": ("wkv6_fwd_fused", dict(B=32, T=196, H=12, bidir=True)),
    # causal RWKV-6 forward from an initial state (make_state), final state out, fp32
    "wkv6_state_f32_b32t196h12": ("wkv6_fwd_state", dict(B=32, T=196, H=12)),
    # RWKV-5 (static per-channel decay) forward, fp32, on the patch-sequence shape
    "wkv5_causal_f32_b32t196h12": ("wkv5_fwd", dict(B=32, T=196, H=12)),
}


def make_workload(name: str, seed: int = 0, batch_scale: int = 1, batches=None):
    """The named workload's inputs.  batch_scale: a problem of batch_scale times the
    workload's batch; batches=(lo, hi): only those batches of it (see make_wkv6)."""
    kind, kw = WORKLOADS[name]
    kw = dict(kw, B=kw["B"] * batch_scale)
    if batches is not None:
        if kind in ("wkv4_fwd", "wkv4_bwd") or kind == "wkv6_fwd" or kind == "wkv6_fwd_bf16" or \
                kind in ("wkv6_bidir_fwd", "wkv6_bwd_bidir"):
            kw["batches"] = batches
        else:
            raise ValueError(f"{name}: no batch window for this workload kind")
    if kind in ("wkv4_fwd", "wkv4_bwd"):
        return kind, make_wkv4(seed=seed, **kw)
    if kind.startswith("wkv5"):
        return kind, make_wkv5(seed=seed, **kw)
    if kind == "wkv6_fwd_fused":
        return kind, make_fused(seed=seed, **kw)
    return kind, make_wkv6(seed=seed, **kw)
