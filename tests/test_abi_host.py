"""Host-side checks of libwkv.so and its test build libwkv_recurrence.so (no GPU
needed, no kernel launched).

The library must load, export every function include/wkv.h declares, and reject
bad arguments on the host with the documented status codes before touching
the device.
"""
import ctypes
import os
import re
import subprocess

import pytest

import linear_attention_rnn_wkv6_b200 as wkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wkv.h")

WKV_OK, WKV_ERR_ARG, WKV_ERR_HEADSIZE, WKV_ERR_ALIGN, WKV_ERR_WORKSPACE = 0, -1, -2, -3, -4


@pytest.fixture(scope="module", params=["default", "recurrence", "debug"])
def lib(request):
    """Every build of the library (the product, the test build, the debug build) carries the same ABI."""
    from linear_attention_rnn_wkv6_b200 import build
    build.build()
    with wkv.use_library(request.param) as handle:
        yield handle


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n.startswith("wkv")))


def test_header_matches_binding():
    assert _declared_functions() == sorted(wkv.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", wkv.lib_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (\w+)$", out, flags=re.M))
    for name in _declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        s = wkv.wkv_status_string(code)
        assert s and s != "unknown status"
    assert wkv.wkv_status_string(12345) == "unknown status"
    assert wkv.wkv_version() >= 100


FAKE = 0x10000000  # a 16-byte aligned non-null address; never dereferenced on these paths


@pytest.mark.parametrize("fn", ["wkv6_fwd", "wkv6_fwd_bf16", "wkv6_bidir_fwd"])
def test_wkv6_forward_argument_errors(lib, fn):
    f = getattr(lib, fn)
    p = [FAKE + 256 * i for i in range(6)]
    assert f(-1, 4, 64, 1, *p, None) == WKV_ERR_ARG
    assert f(1, -4, 64, 1, *p, None) == WKV_ERR_ARG
    assert f(1, 4, 0, 1, *p, None) == WKV_ERR_ARG
    assert f(1, 4, 64, 0, *p, None) == WKV_ERR_ARG
    assert f(1, 4, 100, 3, *p, None) == WKV_ERR_ARG            # C not divisible by H
    assert f(1, 4, 64, 1, *(p[:2] + [None] + p[3:]), None) == WKV_ERR_ARG
    assert f(1, 4, 64, 2, *p, None) == WKV_ERR_HEADSIZE        # N = 32
    assert f(1, 4, 256, 2, *p, None) == WKV_ERR_HEADSIZE       # N = 128
    q = list(p)
    q[3] += 4                                                  # w misaligned
    assert f(1, 4, 64, 1, *q, None) == WKV_ERR_ALIGN
    assert f(1 << 16, 1 << 10, 64 * 64, 64, *p, None) == -7    # B*T*C >= 2^31
    assert f(0, 4, 64, 1, *p, None) == WKV_OK                  # empty problems launch nothing
    assert f(2, 0, 64, 1, *p, None) == WKV_OK


def test_wkv6_backward_argument_errors(lib):
    p = [FAKE + 256 * i for i in range(11)]
    ws = wkv.wkv6_bwd_workspace_bytes(2, 8, 128, 2, 1)
    assert ws == 2 * 2 * 128 * 4                               # du partials and z totals, B*C floats each
    assert lib.wkv6_bwd(-1, 8, 128, 2, 1, *p, FAKE, ws, None) == WKV_ERR_ARG
    assert lib.wkv6_bwd(2, 8, 128, 4, 1, *p, FAKE, ws, None) == WKV_ERR_HEADSIZE
    q = list(p)
    q[7] = None                                                # dk missing
    assert lib.wkv6_bwd(2, 8, 128, 2, 1, *q, FAKE, ws, None) == WKV_ERR_ARG
    assert lib.wkv6_bwd(2, 8, 128, 2, 1, *p, None, ws, None) == WKV_ERR_WORKSPACE
    assert lib.wkv6_bwd(2, 8, 128, 2, 1, *p, FAKE, ws - 4, None) == WKV_ERR_WORKSPACE
    assert lib.wkv6_bwd(2, 8, 128, 2, 1, *p, FAKE + 8, ws, None) == WKV_ERR_ALIGN
    q = list(p)
    q[10] += 8                                                 # du misaligned
    assert lib.wkv6_bwd(2, 8, 128, 2, 0, *q, FAKE, ws, None) == WKV_ERR_ALIGN


def test_wkv6_bwd_bf16_argument_errors(lib):
    p = [FAKE + 256 * i for i in range(11)]
    ws = wkv.wkv6_bwd_workspace_bytes(2, 8, 128, 2, 1)
    f = lib.wkv6_bwd_bf16
    assert f(-1, 8, 128, 2, 1, *p, FAKE, ws, None) == WKV_ERR_ARG
    assert f(2, 8, 128, 4, 1, *p, FAKE, ws, None) == WKV_ERR_HEADSIZE
    assert f(2, 8, 128, 2, 1, *p, None, ws, None) == WKV_ERR_WORKSPACE
    q = list(p)
    q[5] += 8                                                  # dy misaligned
    assert f(2, 8, 128, 2, 1, *q, FAKE, ws, None) == WKV_ERR_ALIGN


def test_wkv6_state_argument_errors(lib):
    f = lib.wkv6_fwd_state
    p = [FAKE + 256 * i for i in range(5)]                     # r, k, v, w, u
    s0, y, sT = FAKE + 4096, FAKE + 8192, FAKE + 12288
    assert f(-1, 4, 64, 1, *p, s0, y, sT, None) == WKV_ERR_ARG
    assert f(1, 4, 64, 2, *p, s0, y, sT, None) == WKV_ERR_HEADSIZE
    assert f(1, 4, 64, 1, *p, s0, None, sT, None) == WKV_ERR_ARG    # y is required
    assert f(1, 4, 64, 1, *p, s0 + 4, y, sT, None) == WKV_ERR_ALIGN
    assert f(1, 4, 64, 1, *p, s0, y, sT + 8, None) == WKV_ERR_ALIGN
    assert f(1 << 20, 1, 64 * 64, 64, *p, s0, y, sT, None) == -7    # too large
    assert f(0, 4, 64, 1, *p, None, y, None, None) == WKV_OK        # states are optional


def test_wkv6_decode_argument_errors(lib):
    f = lib.wkv6_decode
    p = [FAKE + 256 * i for i in range(5)]                     # r, k, v, w, u
    st, y = FAKE + 4096, FAKE + 8192
    assert f(-1, 64, 1, *p, st, y, None) == WKV_ERR_ARG
    assert f(1, 100, 3, *p, st, y, None) == WKV_ERR_ARG               # C not divisible by H
    assert f(1, 64, 2, *p, st, y, None) == WKV_ERR_HEADSIZE
    assert f(1, 64, 1, *p, None, y, None) == WKV_ERR_ARG              # state is required
    assert f(1, 64, 1, *p, st + 4, y, None) == WKV_ERR_ALIGN
    assert f(1 << 20, 64 * 64, 64, *p, st, y, None) == -7             # B*H*N*N >= 2^31
    assert f(0, 64, 1, *p, st, y, None) == WKV_OK


def test_wkv4_bwd_argument_errors(lib):
    p = [FAKE + 256 * i for i in range(9)]                     # k, v, w, u, dy, dk, dv, dw, du
    ws = wkv.wkv4_bwd_workspace_bytes(2, 8, 32)
    assert ws == 4 * (2 * 8 * 32 + 2 * 2 * 32)
    f = lib.wkv4_bwd
    assert f(-1, 8, 32, *p, FAKE, ws, None) == WKV_ERR_ARG
    assert f(2, 8, 0, *p, FAKE, ws, None) == WKV_ERR_ARG
    assert f(2, 8, 32, *(p[:4] + [None] + p[5:]), FAKE, ws, None) == WKV_ERR_ARG      # dy missing
    assert f(2, 8, 32, *p, None, ws, None) == WKV_ERR_WORKSPACE
    assert f(2, 8, 32, *p, FAKE, ws - 4, None) == WKV_ERR_WORKSPACE
    q = list(p)
    q[6] += 4                                                  # dv misaligned
    assert f(2, 8, 32, *q, FAKE, ws, None) == WKV_ERR_ALIGN


def test_wkv5_argument_errors(lib):
    p = [FAKE + 256 * i for i in range(6)]                     # r, k, v, w, u, y
    for f in (lib.wkv5_fwd, lib.wkv5_fwd_bf16):
        assert f(-1, 4, 64, 1, *p, None) == WKV_ERR_ARG
        assert f(1, 4, 64, 2, *p, None) == WKV_ERR_HEADSIZE
        assert f(1, 4, 64, 1, *(p[:3] + [None] + p[4:]), None) == WKV_ERR_ARG   # w missing
        q = list(p)
        q[3] += 4                                              # w misaligned
        assert f(1, 4, 64, 1, *q, None) == WKV_ERR_ALIGN
        assert f(0, 4, 64, 1, *p, None) == WKV_OK
    g = [FAKE + 256 * i for i in range(11)]                    # r, k, v, w, u, dy, dr, dk, dv, dw, du
    ws = wkv.wkv5_bwd_workspace_bytes(2, 8, 128, 2)
    if wkv.lib_path().endswith("libwkv_recurrence.so"):
        assert ws == 4 * (2 * 2 * 8 * 128 + 2 * 2 * 128)      # log-decay and per-token dw [B][T][C], 2 [B][C]
    else:
        assert ws == (2 * 4 + 2 * 8) * 2 * 128               # 2 [B][C] floats, 2 [B][C] doubles
    f = lib.wkv5_bwd
    assert f(-1, 8, 128, 2, *g, FAKE, ws, None) == WKV_ERR_ARG
    assert f(2, 8, 128, 4, *g, FAKE, ws, None) == WKV_ERR_HEADSIZE
    assert f(2, 8, 128, 2, *(g[:9] + [None] + g[10:]), FAKE, ws, None) == WKV_ERR_ARG   # dw missing
    assert f(2, 8, 128, 2, *g, None, ws, None) == WKV_ERR_WORKSPACE
    assert f(2, 8, 128, 2, *g, FAKE, ws - 4, None) == WKV_ERR_WORKSPACE
    assert f(2, 8, 128, 2, *g, FAKE + 4, ws, None) == WKV_ERR_ALIGN


def test_wkv6_fwd_fused_argument_errors(lib):
    p = [FAKE + 256 * i for i in range(9)]                     # r, k, v, ww, w_base, u, g, gn_w, gn_b
    out = FAKE + 4096
    f = lib.wkv6_fwd_fused
    assert f(-1, 4, 64, 1, 0, *p, 1e-5, out, None) == WKV_ERR_ARG
    assert f(1, 4, 64, 2, 0, *p, 1e-5, out, None) == WKV_ERR_HEADSIZE
    assert f(1, 4, 64, 1, 1, *(p[:6] + [None] + p[7:]), 1e-5, out, None) == WKV_ERR_ARG   # gate missing
    assert f(1, 4, 64, 1, 0, *p, 0.0, out, None) == WKV_ERR_ARG                          # eps must be > 0
    assert f(1, 4, 64, 1, 0, *p, float("nan"), out, None) == WKV_ERR_ARG
    q = list(p)
    q[8] += 4                                                  # gn_b misaligned
    assert f(1, 4, 64, 1, 0, *q, 1e-5, out, None) == WKV_ERR_ALIGN
    assert f(0, 4, 64, 1, 0, *p, 1e-5, out, None) == WKV_OK


def test_wkv4_argument_errors(lib):
    p = [FAKE + 256 * i for i in range(5)]
    assert lib.wkv4_fwd(-1, 4, 32, *p, None) == WKV_ERR_ARG
    assert lib.wkv4_fwd(1, 4, 0, *p, None) == WKV_ERR_ARG
    assert lib.wkv4_fwd(1, 4, 32, None, *p[1:], None) == WKV_ERR_ARG
    q = list(p)
    q[4] += 4
    assert lib.wkv4_fwd(1, 4, 32, *q, None) == WKV_ERR_ALIGN
    assert lib.wkv4_fwd(0, 4, 32, *p, None) == WKV_OK


def test_binding_raises_on_error(lib):
    with pytest.raises(wkv.WkvError) as ei:
        wkv.wkv6_fwd(1, 4, 64, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, stream=0)
    assert ei.value.status == WKV_ERR_HEADSIZE


def test_binding_is_marshalling_only():
    """The product package must not reach the oracle or carry a CPU fallback."""
    pkg = os.path.dirname(wkv.__file__)
    for name in os.listdir(pkg):
        if name.endswith(".py"):
            src = open(os.path.join(pkg, name)).read()
            assert "import oracle" not in src and "from oracle" not in src, name
