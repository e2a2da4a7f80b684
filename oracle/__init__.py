"""Double-precision CPU oracle for the RWKV WKV operator.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / reference leg may import this package; the
product package never does.  It shares no code with the CUDA library.

The arithmetic lives in ``wkv_oracle.c`` (plain C, double precision, the
recurrences exactly as the pages state them); this module compiles it with gcc
and marshals numpy arrays.  Every function takes and returns float64 arrays:
the caller upcasts the exact fp32 / bf16 input values first.

Pinning (what makes this oracle trustworthy) lives in ``tests/test_oracle_pins.py``:
brute-force O(T^2) sum forms, textbook matmul reductions, closed forms,
invariants, finite differences and hand-derived fixtures under ``tests/golden``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_DP = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE double, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _configure(lib):
    I = ctypes.c_int
    lib.oracle_wkv6_fwd.argtypes = [I, I, I, I, I] + [_DP] * 6
    lib.oracle_wkv6_fwd_state.argtypes = [I, I, I, I] + [_DP] * 8
    lib.oracle_wkv6_bwd.argtypes = [I, I, I, I, I] + [_DP] * 11
    lib.oracle_wkv4_fwd.argtypes = [I, I, I] + [_DP] * 5
    lib.oracle_wkv4_bwd.argtypes = [I, I, I] + [_DP] * 9
    lib.oracle_wkv5_fwd.argtypes = [I, I, I, I] + [_DP] * 6
    lib.oracle_wkv5_bwd.argtypes = [I, I, I, I] + [_DP] * 11
    lib.oracle_wkv6_fwd_fused.argtypes = [I, I, I, I, I] + [_DP] * 9 + [ctypes.c_double, _DP]
    for f in (lib.oracle_wkv6_fwd, lib.oracle_wkv6_fwd_state, lib.oracle_wkv6_bwd, lib.oracle_wkv4_fwd,
              lib.oracle_wkv4_bwd, lib.oracle_wkv5_fwd, lib.oracle_wkv5_bwd, lib.oracle_wkv6_fwd_fused):
        f.restype = ctypes.c_int
    return lib


def _d(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(_DP)


class Oracle:
    """The oracle's entry points bound to one compiled copy of ``wkv_oracle.c``."""

    def __init__(self, lib):
        self._lib = _configure(lib)

    def wkv6_fwd(self, r, k, v, w, u, H: int, bidirectional: bool = False) -> np.ndarray:
        """RWKV-6 WKV forward.  r,k,v,w: [B,T,C] (w = log-decay ew <= 0), u: [C] -> y [B,T,C]."""
        r, k, v, w, u = map(_d, (r, k, v, w, u))
        B, T, C = r.shape
        y = np.zeros((B, T, C), dtype=np.float64)
        rc = self._lib.oracle_wkv6_fwd(B, T, C, H, int(bidirectional), _p(r), _p(k), _p(v), _p(w),
                                       _p(u), _p(y))
        if rc != 0:
            raise ValueError(f"oracle_wkv6_fwd failed ({rc})")
        return y

    def wkv6_fwd_state(self, r, k, v, w, u, H: int, s0=None):
        """Causal RWKV-6 forward from the initial state s0 ([B,H,N,N], None = zero).
        Returns (y [B,T,C], sT [B,H,N,N] = the state after the last token)."""
        r, k, v, w, u = map(_d, (r, k, v, w, u))
        B, T, C = r.shape
        N = C // H
        y = np.zeros((B, T, C), dtype=np.float64)
        sT = np.zeros((B, H, N, N), dtype=np.float64)
        s0p = None
        if s0 is not None:
            s0 = _d(s0)
            if s0.shape != (B, H, N, N):
                raise ValueError(f"s0 must have shape {(B, H, N, N)}")
            s0p = _p(s0)
        rc = self._lib.oracle_wkv6_fwd_state(B, T, C, H, _p(r), _p(k), _p(v), _p(w), _p(u), s0p, _p(y), _p(sT))
        if rc != 0:
            raise ValueError(f"oracle_wkv6_fwd_state failed ({rc})")
        return y, sT

    def wkv6_bwd(self, r, k, v, w, u, dy, H: int, bidirectional: bool = False):
        """RWKV-6 WKV backward -> (dr, dk, dv, dw, du); dw is w.r.t. the log-decay ew."""
        r, k, v, w, u, dy = map(_d, (r, k, v, w, u, dy))
        B, T, C = r.shape
        outs = [np.zeros((B, T, C), dtype=np.float64) for _ in range(4)] + [np.zeros(C, dtype=np.float64)]
        rc = self._lib.oracle_wkv6_bwd(B, T, C, H, int(bidirectional), _p(r), _p(k), _p(v), _p(w),
                                       _p(u), _p(dy), *[_p(o) for o in outs])
        if rc != 0:
            raise ValueError(f"oracle_wkv6_bwd failed ({rc})")
        return tuple(outs)

    def wkv4_fwd(self, k, v, w, u) -> np.ndarray:
        """RWKV-4 WKV forward.  k,v: [B,T,C]; w (> 0, decay e^-w), u: [C] -> y [B,T,C]."""
        k, v, w, u = map(_d, (k, v, w, u))
        B, T, C = k.shape
        y = np.zeros((B, T, C), dtype=np.float64)
        rc = self._lib.oracle_wkv4_fwd(B, T, C, _p(k), _p(v), _p(w), _p(u), _p(y))
        if rc != 0:
            raise ValueError(f"oracle_wkv4_fwd failed ({rc})")
        return y

    def wkv4_bwd(self, k, v, w, u, dy):
        """RWKV-4 backward -> (dk, dv [B,T,C], dw, du [C] summed over B and T)."""
        k, v, w, u, dy = map(_d, (k, v, w, u, dy))
        B, T, C = k.shape
        dk = np.zeros((B, T, C), dtype=np.float64)
        dv = np.zeros((B, T, C), dtype=np.float64)
        dw = np.zeros(C, dtype=np.float64)
        du = np.zeros(C, dtype=np.float64)
        rc = self._lib.oracle_wkv4_bwd(B, T, C, _p(k), _p(v), _p(w), _p(u), _p(dy), _p(dk), _p(dv), _p(dw),
                                       _p(du))
        if rc != 0:
            raise ValueError(f"oracle_wkv4_bwd failed ({rc})")
        return dk, dv, dw, du

    def wkv5_fwd(self, r, k, v, w, u, H: int) -> np.ndarray:
        """RWKV-5 forward.  r,k,v: [B,T,C]; w (>= 0, static decay exp(-w)), u: [C] -> y [B,T,C]."""
        r, k, v, w, u = map(_d, (r, k, v, w, u))
        B, T, C = r.shape
        y = np.zeros((B, T, C), dtype=np.float64)
        rc = self._lib.oracle_wkv5_fwd(B, T, C, H, _p(r), _p(k), _p(v), _p(w), _p(u), _p(y))
        if rc != 0:
            raise ValueError(f"oracle_wkv5_fwd failed ({rc})")
        return y

    def wkv5_bwd(self, r, k, v, w, u, dy, H: int):
        """RWKV-5 backward -> (dr, dk, dv [B,T,C], dw, du [C] summed over B and T)."""
        r, k, v, w, u, dy = map(_d, (r, k, v, w, u, dy))
        B, T, C = r.shape
        outs = [np.zeros((B, T, C), dtype=np.float64) for _ in range(3)] + [np.zeros(C, dtype=np.float64)
                                                                               for _ in range(2)]
        rc = self._lib.oracle_wkv5_bwd(B, T, C, H, _p(r), _p(k), _p(v), _p(w), _p(u), _p(dy),
                                       *[_p(o) for o in outs])
        if rc != 0:
            raise ValueError(f"oracle_wkv5_bwd failed ({rc})")
        return tuple(outs)

    def wkv6_fwd_fused(self, r, k, v, ww, w_base, u, g, gn_w, gn_b, eps: float, H: int,
                       bidirectional: bool = False) -> np.ndarray:
        """RWKV-6 forward at ew = -exp(w_base + ww), then per-head group norm (gn_w, gn_b, eps)
        times the gate g.  r,k,v,ww,g: [B,T,C]; w_base,u,gn_w,gn_b: [C] -> out [B,T,C]."""
        r, k, v, ww, w_base, u, g, gn_w, gn_b = map(_d, (r, k, v, ww, w_base, u, g, gn_w, gn_b))
        B, T, C = r.shape
        out = np.zeros((B, T, C), dtype=np.float64)
        rc = self._lib.oracle_wkv6_fwd_fused(B, T, C, H, int(bidirectional), _p(r), _p(k), _p(v), _p(ww),
                                             _p(w_base), _p(u), _p(g), _p(gn_w), _p(gn_b), float(eps), _p(out))
        if rc != 0:
            raise ValueError(f"oracle_wkv6_fwd_fused failed ({rc})")
        return out


def _default() -> Oracle:
    global _lib
    if _lib is None:
        _lib = Oracle(ctypes.CDLL(build()))
    return _lib


def wkv6_fwd(r, k, v, w, u, H: int, bidirectional: bool = False) -> np.ndarray:
    return _default().wkv6_fwd(r, k, v, w, u, H, bidirectional)


def wkv6_fwd_state(r, k, v, w, u, H: int, s0=None):
    return _default().wkv6_fwd_state(r, k, v, w, u, H, s0)


def wkv6_bwd(r, k, v, w, u, dy, H: int, bidirectional: bool = False):
    return _default().wkv6_bwd(r, k, v, w, u, dy, H, bidirectional)


def wkv4_fwd(k, v, w, u) -> np.ndarray:
    return _default().wkv4_fwd(k, v, w, u)


def wkv4_bwd(k, v, w, u, dy):
    return _default().wkv4_bwd(k, v, w, u, dy)


def wkv5_fwd(r, k, v, w, u, H: int) -> np.ndarray:
    return _default().wkv5_fwd(r, k, v, w, u, H)


def wkv5_bwd(r, k, v, w, u, dy, H: int):
    return _default().wkv5_bwd(r, k, v, w, u, dy, H)


def wkv6_fwd_fused(r, k, v, ww, w_base, u, g, gn_w, gn_b, eps: float, H: int, bidirectional: bool = False):
    return _default().wkv6_fwd_fused(r, k, v, ww, w_base, u, g, gn_w, gn_b, eps, H, bidirectional)


def source() -> str:
    with open(_SRC) as f:
        return f.read()


def compile_variant(src: str, path: str) -> Oracle:
    """Compile a modified copy of the oracle source (used by the tests that plant
    mistakes in the oracle to show that the pins catch them)."""
    c_path = path + ".c"
    with open(c_path, "w") as f:
        f.write(src)
    subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11", "-shared",
                           "-fPIC", "-o", path, c_path, "-lm"])
    return Oracle(ctypes.CDLL(path))


def rel_l2(x, ref) -> float:
    """||x - ref||_2 / ||ref||_2 over the whole tensor (0 when both vanish)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.linalg.norm(ref.ravel()))
    num = float(np.linalg.norm((x - ref).ravel()))
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den
