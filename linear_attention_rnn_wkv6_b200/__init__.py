"""B200-native RWKV WKV operator: thin Python binding of libwkv.so.

Every function here has the name and argument order of the C entry point it
wraps (include/wkv.h) and only marshals arguments: torch tensors (or raw
integer device addresses) become pointers, ``stream=None`` becomes the current
torch CUDA stream, and a non-zero status raises :class:`WkvError`.  All of the
operator's arithmetic runs in the CUDA kernels of libwkv.so; there is no CPU
fallback.  If the library has not been built, importing the binding's entry
points raises immediately.

Build the library with ``python -m linear_attention_rnn_wkv6_b200.build``.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

__all__ = [
    "WkvError", "lib_path", "load", "wkv6_fwd", "wkv6_fwd_bf16", "wkv6_bidir_fwd", "wkv6_bwd",
    "wkv6_bwd_workspace_bytes", "wkv4_fwd", "wkv_status_string", "wkv_take_device_faults", "wkv_version",
    "wkv6_bwd_noalloc", "wkv6_fwd_state", "wkv6_decode", "wkv6_bwd_bf16", "wkv4_bwd", "wkv4_bwd_workspace_bytes",
    "wkv5_fwd", "wkv5_fwd_bf16", "wkv5_bwd", "wkv5_bwd_workspace_bytes", "wkv6_fwd_fused",
    "wkv_selftest_wait_timeout", "wkv_selftest_index_check", "WKV_FAULT_TIMEOUT", "WKV_FAULT_INDEX",
    "EXPORTED_SYMBOLS",
    "HEAD_SIZE", "LIBRARY_FILES", "use_library",
]

HEAD_SIZE = 64
_HERE = os.path.dirname(os.path.abspath(__file__))
# The builds of the library (same C ABI): the product, the test build whose
# chunked-form entry points run the token-by-token recurrence kernels, and the debug
# build that checks every store index of every kernel.
LIBRARY_FILES = {"default": "libwkv.so", "recurrence": "libwkv_recurrence.so", "debug": "libwkv_debug.so"}
_LIBS: dict = {}
_ACTIVE = ["default"]

# Every extern "C" symbol declared in include/wkv.h.
EXPORTED_SYMBOLS = (
    "wkv6_fwd", "wkv6_fwd_bf16", "wkv6_bidir_fwd", "wkv6_bwd", "wkv6_bwd_workspace_bytes", "wkv4_fwd",
    "wkv_status_string", "wkv_take_device_faults", "wkv_version", "wkv6_bwd_noalloc", "wkv6_fwd_state",
    "wkv6_decode", "wkv6_bwd_bf16", "wkv4_bwd", "wkv4_bwd_workspace_bytes", "wkv5_fwd", "wkv5_fwd_bf16",
    "wkv5_bwd", "wkv5_bwd_workspace_bytes", "wkv6_fwd_fused", "wkv_selftest_wait_timeout",
    "wkv_selftest_index_check",
)
WKV_FAULT_TIMEOUT = 0x1   # fault-word bit: a bounded device-side wait ran out
WKV_FAULT_INDEX = 0x2     # fault-word bit: a kernel's store index was out of range (debug build)

_I = ctypes.c_int
_P = ctypes.c_void_p
_SZ = ctypes.c_size_t

_SIGS = {
    "wkv6_fwd": ([_I] * 4 + [_P] * 6 + [_P], _I),
    "wkv6_fwd_bf16": ([_I] * 4 + [_P] * 6 + [_P], _I),
    "wkv6_bidir_fwd": ([_I] * 4 + [_P] * 6 + [_P], _I),
    "wkv6_bwd": ([_I] * 5 + [_P] * 11 + [_P, _SZ, _P], _I),
    "wkv6_bwd_workspace_bytes": ([_I] * 5, _SZ),
    "wkv4_fwd": ([_I] * 3 + [_P] * 5 + [_P], _I),
    "wkv_status_string": ([_I], ctypes.c_char_p),
    "wkv_take_device_faults": ([ctypes.POINTER(ctypes.c_uint)], _I),
    "wkv_version": ([], _I),
    "wkv_selftest_wait_timeout": ([_P], _I),
    "wkv_selftest_index_check": ([_P], _I),
    "wkv6_bwd_noalloc": ([_I] * 5 + [_P] * 11 + [_P], _I),
    "wkv6_fwd_state": ([_I] * 4 + [_P] * 8 + [_P], _I),
    "wkv6_decode": ([_I] * 3 + [_P] * 7 + [_P], _I),
    "wkv6_bwd_bf16": ([_I] * 5 + [_P] * 11 + [_P, _SZ, _P], _I),
    "wkv4_bwd": ([_I] * 3 + [_P] * 9 + [_P, _SZ, _P], _I),
    "wkv4_bwd_workspace_bytes": ([_I] * 3, _SZ),
    "wkv5_fwd": ([_I] * 4 + [_P] * 6 + [_P], _I),
    "wkv5_fwd_bf16": ([_I] * 4 + [_P] * 6 + [_P], _I),
    "wkv5_bwd": ([_I] * 4 + [_P] * 11 + [_P, _SZ, _P], _I),
    "wkv5_bwd_workspace_bytes": ([_I] * 4, _SZ),
    "wkv6_fwd_fused": ([_I] * 5 + [_P] * 9 + [ctypes.c_float, _P, _P], _I),
}


class WkvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed with status {status}: {wkv_status_string(status)}")


def lib_path(variant: str | None = None) -> str:
    return os.path.join(_HERE, LIBRARY_FILES[variant or _ACTIVE[0]])


def load(variant: str | None = None):
    """Load a build of the library (default: the one selected by use_library, normally
    libwkv.so); raises if it has not been built."""
    variant = variant or _ACTIVE[0]
    lib = _LIBS.get(variant)
    if lib is None:
        path = lib_path(variant)
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m linear_attention_rnn_wkv6_b200.build` "
                               "(the WKV operator has no fallback implementation)")
        lib = ctypes.CDLL(path)
        for name, (args, res) in _SIGS.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _LIBS[variant] = lib
    return lib


@contextlib.contextmanager
def use_library(variant: str):
    """Route the wrappers below to another build of the library inside the block
    ("recurrence": libwkv_recurrence.so, for tests and comparison timings)."""
    if variant not in LIBRARY_FILES:
        raise ValueError(f"unknown library build {variant!r}")
    prev = _ACTIVE[0]
    _ACTIVE[0] = variant
    try:
        yield load(variant)
    finally:
        _ACTIVE[0] = prev


def _ptr(x) -> int | None:
    """Device address of a torch tensor (must be contiguous) or an integer address."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_contiguous():
        raise ValueError("WKV tensors must be contiguous")
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise WkvError(fn, status)


def wkv6_fwd(B, T, C, H, r, k, v, w, u, y, stream=None) -> None:
    """Causal RWKV-6 WKV forward (fp32).  See include/wkv.h."""
    _check("wkv6_fwd", load().wkv6_fwd(B, T, C, H, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(y),
                                       _stream(stream)))


def wkv6_fwd_bf16(B, T, C, H, r, k, v, w, u, y, stream=None) -> None:
    """Causal RWKV-6 WKV forward with bf16 r, k, v, w; fp32 u, state and y."""
    _check("wkv6_fwd_bf16", load().wkv6_fwd_bf16(B, T, C, H, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u),
                                                 _ptr(y), _stream(stream)))


def wkv6_bidir_fwd(B, T, C, H, r, k, v, w, u, y, stream=None) -> None:
    """Bidirectional RWKV-6 WKV forward (fp32)."""
    _check("wkv6_bidir_fwd", load().wkv6_bidir_fwd(B, T, C, H, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u),
                                                   _ptr(y), _stream(stream)))


def wkv6_fwd_state(B, T, C, H, r, k, v, w, u, s0, y, sT, stream=None) -> None:
    """Causal RWKV-6 forward (fp32) from the initial state s0 ([B,H,N,N] or None for zero);
    writes the final state into sT ([B,H,N,N] or None)."""
    _check("wkv6_fwd_state", load().wkv6_fwd_state(B, T, C, H, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u),
                                                   _ptr(s0), _ptr(y), _ptr(sT), _stream(stream)))


def wkv6_decode(B, C, H, r, k, v, w, u, state, y, stream=None) -> None:
    """One recurrent step: r, k, v, w [B,C]; state [B,H,N,N] updated in place; y [B,C]."""
    _check("wkv6_decode", load().wkv6_decode(B, C, H, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(state),
                                             _ptr(y), _stream(stream)))


def wkv6_bwd_workspace_bytes(B, T, C, H, bidirectional) -> int:
    return int(load().wkv6_bwd_workspace_bytes(B, T, C, H, int(bool(bidirectional))))


def wkv6_bwd(B, T, C, H, bidirectional, r, k, v, w, u, dy, dr, dk, dv, dw, du, workspace, workspace_bytes,
             stream=None) -> None:
    """RWKV-6 WKV backward (fp32): dr, dk, dv, dw [B,T,C] and du [C]."""
    _check("wkv6_bwd", load().wkv6_bwd(B, T, C, H, int(bool(bidirectional)), _ptr(r), _ptr(k), _ptr(v), _ptr(w),
                                       _ptr(u), _ptr(dy), _ptr(dr), _ptr(dk), _ptr(dv), _ptr(dw), _ptr(du),
                                       _ptr(workspace), int(workspace_bytes), _stream(stream)))


def wkv6_bwd_bf16(B, T, C, H, bidirectional, r, k, v, w, u, dy, dr, dk, dv, dw, du, workspace, workspace_bytes,
                  stream=None) -> None:
    """wkv6_bwd with bf16 r, k, v, w, dy (bit patterns); u and all gradients fp32."""
    _check("wkv6_bwd_bf16", load().wkv6_bwd_bf16(B, T, C, H, int(bool(bidirectional)), _ptr(r), _ptr(k), _ptr(v),
                                                 _ptr(w), _ptr(u), _ptr(dy), _ptr(dr), _ptr(dk), _ptr(dv),
                                                 _ptr(dw), _ptr(du), _ptr(workspace), int(workspace_bytes),
                                                 _stream(stream)))


def wkv6_bwd_noalloc(B, T, C, H, bidirectional, r, k, v, w, u, dy, dr, dk, dv, dw, du, stream=None) -> None:
    """wkv6_bwd without a workspace, for callers that cannot allocate device memory
    (its scratch is a fixed array inside the library; B*C <= 262144)."""
    _check("wkv6_bwd_noalloc", load().wkv6_bwd_noalloc(B, T, C, H, int(bool(bidirectional)), _ptr(r), _ptr(k), _ptr(v),
                                                       _ptr(w), _ptr(u), _ptr(dy), _ptr(dr), _ptr(dk), _ptr(dv),
                                                       _ptr(dw), _ptr(du), _stream(stream)))


def wkv4_fwd(B, T, C, k, v, w, u, y, stream=None) -> None:
    """RWKV-4 WKV forward (fp32)."""
    _check("wkv4_fwd", load().wkv4_fwd(B, T, C, _ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(y), _stream(stream)))


def wkv4_bwd_workspace_bytes(B, T, C) -> int:
    return int(load().wkv4_bwd_workspace_bytes(B, T, C))


def wkv4_bwd(B, T, C, k, v, w, u, dy, dk, dv, dw, du, workspace, workspace_bytes, stream=None) -> None:
    """RWKV-4 WKV backward (fp32): dk, dv [B,T,C]; dw, du [C]."""
    _check("wkv4_bwd", load().wkv4_bwd(B, T, C, _ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(dy), _ptr(dk), _ptr(dv),
                                       _ptr(dw), _ptr(du), _ptr(workspace), int(workspace_bytes), _stream(stream)))


def wkv6_fwd_fused(B, T, C, H, bidirectional, r, k, v, ww, w_base, u, g, gn_weight, gn_bias, eps, out,
                   stream=None) -> None:
    """RWKV-6 forward at ew = -exp(w_base + ww), then per-head group norm and the gate g (fp32)."""
    _check("wkv6_fwd_fused", load().wkv6_fwd_fused(B, T, C, H, int(bool(bidirectional)), _ptr(r), _ptr(k), _ptr(v),
                                                   _ptr(ww), _ptr(w_base), _ptr(u), _ptr(g), _ptr(gn_weight),
                                                   _ptr(gn_bias), float(eps), _ptr(out), _stream(stream)))


def wkv5_fwd(B, T, C, H, r, k, v, w, u, y, stream=None) -> None:
    """RWKV-5 WKV forward (fp32): static per-channel decay exp(-w), w and u [C]."""
    _check("wkv5_fwd", load().wkv5_fwd(B, T, C, H, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(y),
                                       _stream(stream)))


def wkv5_fwd_bf16(B, T, C, H, r, k, v, w, u, y, stream=None) -> None:
    """RWKV-5 WKV forward with bf16 r, k, v (raw bf16 bits); w, u and y fp32."""
    _check("wkv5_fwd_bf16", load().wkv5_fwd_bf16(B, T, C, H, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(y),
                                                 _stream(stream)))


def wkv5_bwd_workspace_bytes(B, T, C, H) -> int:
    return int(load().wkv5_bwd_workspace_bytes(B, T, C, H))


def wkv5_bwd(B, T, C, H, r, k, v, w, u, dy, dr, dk, dv, dw, du, workspace, workspace_bytes, stream=None) -> None:
    """RWKV-5 WKV backward (fp32): dr, dk, dv [B,T,C]; dw, du [C]."""
    _check("wkv5_bwd", load().wkv5_bwd(B, T, C, H, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(dy), _ptr(dr),
                                       _ptr(dk), _ptr(dv), _ptr(dw), _ptr(du), _ptr(workspace), int(workspace_bytes),
                                       _stream(stream)))


def wkv_status_string(status: int) -> str:
    return load().wkv_status_string(int(status)).decode()


def wkv_take_device_faults() -> int:
    """Synchronise the device and return (and clear) the WKV_FAULT_* bits."""
    out = ctypes.c_uint(0)
    _check("wkv_take_device_faults", load().wkv_take_device_faults(ctypes.byref(out)))
    return int(out.value)


def wkv_selftest_wait_timeout(stream=None) -> None:
    """Launch the one-CTA kernel whose bounded wait runs out (about a second); the fault
    word then holds WKV_FAULT_TIMEOUT (read it with wkv_take_device_faults)."""
    _check("wkv_selftest_wait_timeout", load().wkv_selftest_wait_timeout(_stream(stream)))


def wkv_selftest_index_check(stream=None) -> None:
    """Launch the one-thread kernel whose store index equals its array's size: the check
    skips the store and records WKV_FAULT_INDEX (the debug build raises WkvError with
    WKV_ERR_DEVICE_CHECK, having waited for the kernel)."""
    _check("wkv_selftest_index_check", load().wkv_selftest_index_check(_stream(stream)))


def wkv_version() -> int:
    return int(load().wkv_version())
