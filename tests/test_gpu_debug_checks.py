"""The debug build (libwkv_debug.so, -DWKV_DEVICE_CHECKS=1): every global store of
every kernel (and every L2 prefetch of an output row) checks its index against the
size of the array it writes, and every
entry point waits for its kernels and returns WKV_ERR_DEVICE_CHECK when a check
failed (the store is skipped; nothing traps).  compute-sanitizer is not available
on this pool; these checks and the tests' guard bands take its place.

The failure path is exercised by a self-test kernel whose one store has an index
equal to its array's size; every other test here runs small problems of every
entry point through the debug build and requires no check to fail and the results
to match the oracle.
"""
import numpy as np
import pytest

import linear_attention_rnn_wkv6_b200 as wkv
import oracle
from linear_attention_rnn_wkv6_b200 import synth
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu

WKV_ERR_DEVICE_CHECK = -8


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_rnn_wkv6_b200 import build
    build.build()
    oracle.build()


@pytest.fixture
def debug_build():
    with wkv.use_library("debug"):
        yield


def test_index_check_failure_path_product_build():
    """The product build does not wait: the self-test's skipped store shows in the fault word."""
    wkv.wkv_selftest_index_check()
    assert wkv.wkv_take_device_faults() == wkv.WKV_FAULT_INDEX
    assert wkv.wkv_take_device_faults() == 0


def test_index_check_failure_path_debug_build(debug_build):
    with pytest.raises(wkv.WkvError) as ei:
        wkv.wkv_selftest_index_check()
    assert ei.value.status == WKV_ERR_DEVICE_CHECK
    assert wkv.wkv_take_device_faults() == 0      # reported once, then cleared


@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (2, 33, 2), (1, 197, 1)])
@pytest.mark.parametrize("bidir", [False, True])
def test_debug_build_forward(B, T, H, bidir, debug_build):
    x = synth.make_wkv6(B, T, H, seed=500 + T)
    y = gc.run_wkv6_fwd(x, bidir=bidir)
    r, k, v, w, u = gc.f64(x)
    assert oracle.rel_l2(y, oracle.wkv6_fwd(r, k, v, w, u, H=H, bidirectional=bidir)) <= gc.TOL_F32_FWD


@pytest.mark.parametrize("B,T,H", [(1, 65, 1), (2, 130, 2)])
def test_debug_build_forward_bf16(B, T, H, debug_build):
    x = synth.make_wkv6(B, T, H, seed=510 + T, wraw_lo=-8.0, dtype="bf16")
    y = gc.run_wkv6_fwd(x)
    r, k, v, w, u = gc.f64(x)
    assert oracle.rel_l2(y, oracle.wkv6_fwd(r, k, v, w, u, H=H)) <= gc.TOL_BF16_FWD


@pytest.mark.parametrize("B,T,H", [(1, 2, 1), (2, 33, 2), (1, 100, 1)])
@pytest.mark.parametrize("bidir", [False, True])
def test_debug_build_backward(B, T, H, bidir, debug_build):
    x = synth.make_wkv6(B, T, H, seed=520 + T, with_dy=True)
    got = gc.run_wkv6_bwd(x, bidir)
    ref = gc.oracle_bwd_full(x, bidir)
    for name, g, e in zip(("dr", "dk", "dv", "dw", "du"), got, ref):
        assert np.all(np.isfinite(g)), name
        if name == "dw" and T <= 2:
            continue
        assert oracle.rel_l2(g, e) <= gc.TOL_F32_GRAD, name


@pytest.mark.parametrize("bidir", [False, True])
def test_debug_build_backward_bf16_and_noalloc(bidir, debug_build):
    x = synth.make_wkv6(2, 45, 2, seed=530, with_dy=True, dtype="bf16")
    got, dy64 = gc.run_wkv6_bwd_bf16(x, bidir)
    ref = gc.oracle_bwd_full(x, bidir, dy64)
    for name, g, e in zip(("dr", "dk", "dv", "dw", "du"), got, ref):
        assert oracle.rel_l2(g, e) <= gc.TOL_F32_GRAD, name
    x = synth.make_wkv6(3, 40, 1, seed=531, with_dy=True)
    ins = [gc.dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u", "dy")]
    outs = [gc.empty_nan((x.B, x.T, x.C)) for _ in range(4)] + [gc.empty_nan((x.C,))]
    wkv.wkv6_bwd_noalloc(x.B, x.T, x.C, x.H, bidir, *ins, *outs)
    ref = gc.oracle_bwd_full(x, bidir)
    for name, g, e in zip(("dr", "dk", "dv", "dw", "du"), outs, ref):
        assert oracle.rel_l2(g.cpu().numpy(), e) <= gc.TOL_F32_GRAD, name


@pytest.mark.parametrize("B,T,C", [(2, 100, 64), (1, 1100, 32), (2, 30, 20)])   # four channels a thread, and one
def test_debug_build_wkv4(B, T, C, debug_build):
    x = synth.make_wkv4(B, T, C, seed=540 + T, with_dy=True)
    y = gc.run_wkv4(x)
    assert oracle.rel_l2(y, oracle.wkv4_fwd(x.k, x.v, x.w, x.u)) <= gc.TOL_F32_FWD
    ins = [gc.dev(getattr(x, n)) for n in ("k", "v", "w", "u", "dy")]
    outs = [gc.empty_nan((B, T, C)) for _ in range(2)] + [gc.empty_nan((C,)) for _ in range(2)]
    nb = wkv.wkv4_bwd_workspace_bytes(B, T, C)
    wkv.wkv4_bwd(B, T, C, *ins, *outs, gc.workspace(nb), nb)
    ref = oracle.wkv4_bwd(x.k, x.v, x.w, x.u, x.dy)
    for name, g, e in zip(("dk", "dv", "dw", "du"), outs, ref):
        assert oracle.rel_l2(g.cpu().numpy(), e) <= gc.TOL_F32_GRAD, name


def test_debug_build_wkv5_state_decode_fused(debug_build):
    x5 = synth.make_wkv5(2, 70, 2, seed=550, with_dy=True)
    in5 = [gc.dev(getattr(x5, n)) for n in ("r", "k", "v", "w", "u")]
    f5 = [x5.as_f64(n) for n in ("r", "k", "v", "w", "u")]
    y5 = gc.empty_nan((x5.B, x5.T, x5.C))
    wkv.wkv5_fwd(x5.B, x5.T, x5.C, x5.H, *in5, y5)
    assert oracle.rel_l2(y5.cpu().numpy(), oracle.wkv5_fwd(*f5, H=x5.H)) <= gc.TOL_F32_FWD
    g5 = [gc.empty_nan((x5.B, x5.T, x5.C)) for _ in range(3)] + [gc.empty_nan((x5.C,)) for _ in range(2)]
    nb = wkv.wkv5_bwd_workspace_bytes(x5.B, x5.T, x5.C, x5.H)
    wkv.wkv5_bwd(x5.B, x5.T, x5.C, x5.H, *in5, gc.dev(x5.dy), *g5, gc.workspace(nb), nb)
    ref5 = oracle.wkv5_bwd(*f5, x5.dy.astype(np.float64), H=x5.H)
    for name, g, e in zip(("dr", "dk", "dv", "dw", "du"), g5, ref5):
        assert oracle.rel_l2(g.cpu().numpy(), e) <= gc.TOL_F32_GRAD, name
    # state in and out, then a decode step
    x = synth.make_wkv6(2, 50, 2, seed=551)
    f = gc.f64(x)
    s0 = synth.make_state(2, 2, seed=552)
    y, sT = gc.empty_nan((2, 50, x.C)), gc.empty_nan((2, 2, 64, 64))
    wkv.wkv6_fwd_state(2, 50, x.C, 2, *(gc.dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u")), gc.dev(s0), y, sT)
    yo, so = oracle.wkv6_fwd_state(*f, H=2, s0=s0.astype(np.float64))
    assert oracle.rel_l2(y.cpu().numpy(), yo) <= gc.TOL_F32_FWD and oracle.rel_l2(sT.cpu().numpy(), so) <= gc.TOL_F32_FWD
    x1 = synth.make_wkv6(2, 1, 2, seed=553)
    y1 = gc.empty_nan((2, x1.C))
    wkv.wkv6_decode(2, x1.C, 2, *(gc.dev(getattr(x1, n)[:, 0]) for n in ("r", "k", "v", "w")), gc.dev(x1.u), sT, y1)
    yo1, so1 = oracle.wkv6_fwd_state(*gc.f64(x1), H=2, s0=so)
    assert oracle.rel_l2(y1.cpu().numpy(), yo1[:, 0]) <= gc.TOL_F32_FWD
    assert oracle.rel_l2(sT.cpu().numpy(), so1) <= gc.TOL_F32_FWD
    # fused prologue and epilogue, bidirectional
    xf = synth.make_fused(2, 45, 2, seed=554, bidir=True)
    names = ("r", "k", "v", "ww", "w_base", "u", "g", "gn_w", "gn_b")
    yf = gc.empty_nan((2, 45, xf.C))
    wkv.wkv6_fwd_fused(2, 45, xf.C, 2, True, *(gc.dev(getattr(xf, n)) for n in names), xf.eps, yf)
    ref = oracle.wkv6_fwd_fused(*(getattr(xf, n) for n in names), xf.eps, H=2, bidirectional=True)
    assert oracle.rel_l2(yf.cpu().numpy(), ref) <= gc.TOL_F32_FWD
