"""Parity of the CUDA path (called through the C ABI) with the fp64 oracle.

Small problems and the full-size workloads (in the launch configuration the
benchmark times) are compared element by element over the whole tensor; the
oracle runs one batch per host thread for the large ones.
"""
import numpy as np
import pytest

import oracle
from linear_attention_rnn_wkv6_b200 import synth
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.build()


def _rel(a, b):
    return oracle.rel_l2(a, b)


# ------------------------------------------------------------------ forward, small and ragged

F32_PATHS = ["tensor", "recurrence"]


@pytest.fixture(params=F32_PATHS)
def f32_path(request):
    """Run the fp32 forward (causal and bidirectional) through the chunked
    tensor-core kernel with split-bf16 operands (libwkv.so) or the token-by-token
    recurrence (the test build libwkv_recurrence.so)."""
    with gc.library_for(request.param):
        yield request.param


FWD_SHAPES = [  # (B, T, H): several 32-token chunks, ragged tails, T < chunk, single token; 16, 17
    # and 48 sit on the register recurrence's 16-token stage boundaries
    (1, 1, 1), (1, 2, 1), (1, 16, 1), (2, 17, 2), (2, 31, 2), (1, 32, 1), (1, 33, 3), (1, 48, 1), (2, 65, 2),
    (3, 100, 1), (1, 196, 4),
]


@pytest.mark.parametrize("B,T,H", FWD_SHAPES)
@pytest.mark.parametrize("bidir", [False, True])
def test_wkv6_fwd_f32_small(B, T, H, bidir, f32_path):
    x = synth.make_wkv6(B, T, H, seed=T * 10 + H)
    y = gc.run_wkv6_fwd(x, bidir=bidir)
    r, k, v, w, u = gc.f64(x)
    ref = oracle.wkv6_fwd(r, k, v, w, u, H=H, bidirectional=bidir)
    assert np.all(np.isfinite(y))
    assert _rel(y, ref) <= gc.TOL_F32_FWD


# The product build runs problems with T <= 256 and at most 24 (causal) or 36
# (bidirectional) (b, h) units on the cluster kernel (every chunk at once) and the rest
# on the chunk-chain kernel; these shapes keep the chain kernel's small and ragged
# cases covered as well, and the cluster kernel's largest unit counts.
CHAIN_SHAPES = [(5, 33, 7), (6, 100, 6), (1, 257, 2), (3, 31, 11), (6, 196, 4), (9, 70, 4)]


@pytest.mark.parametrize("B,T,H", CHAIN_SHAPES)
@pytest.mark.parametrize("bidir", [False, True])
def test_wkv6_fwd_f32_chain_kernel_shapes(B, T, H, bidir, f32_path):
    x = synth.make_wkv6(B, T, H, seed=T * 10 + H + 1)
    y = gc.run_wkv6_fwd(x, bidir=bidir)
    ref = gc.oracle_fwd_full(x, bidir)
    assert np.all(np.isfinite(y))
    assert _rel(y, ref) <= gc.TOL_F32_FWD


BF16_PATHS = ["tensor", "recurrence"]


@pytest.fixture(params=BF16_PATHS)
def bf16_path(request):
    """Run the bf16 causal forward through the chunked tensor-core kernel or the
    token-by-token recurrence kernel (the test build)."""
    with gc.library_for(request.param):
        yield request.param


def _bf16_bound(path):
    # the oracle sees the same rounded inputs: the recurrence differs only by fp32
    # rounding; the tensor-core path rounds its chunk operands (decay-scaled r and k,
    # the masked chunk matrix and the carried state) to bf16 for the MMAs, about
    # 3e-3 relative L2, inside the 2e-2 tolerance of bf16 inputs
    return 1e-5 if path == "recurrence" else 6e-3


@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (2, 33, 2), (1, 64, 1), (1, 65, 2), (1, 97, 3), (2, 256, 2)])
def test_wkv6_fwd_bf16_small(B, T, H, bf16_path):
    x = synth.make_wkv6(B, T, H, seed=T + 7, wraw_lo=-8.0, dtype="bf16")
    y = gc.run_wkv6_fwd(x)
    r, k, v, w, u = gc.f64(x)
    ref = oracle.wkv6_fwd(r, k, v, w, u, H=H)
    err = _rel(y, ref)
    assert np.all(np.isfinite(y))
    assert err <= gc.TOL_BF16_FWD
    assert err <= _bf16_bound(bf16_path), err


@pytest.mark.parametrize("case", ["strong", "mixed", "zero_decay", "unit_decay"])
def test_wkv6_fwd_bf16_decay_edge_cases(case, bf16_path):
    """Strong decays push the chunk's cumulative log-decay past the tensor-core
    range: those chunks take the exact fallback; the rest stay on tensor cores."""
    B, T, H = 2, 200, 2
    x = synth.make_wkv6(B, T, H, seed=21, dtype="bf16")
    w = synth.bf16_bits_to_f32(x.w).astype(np.float64)
    g = np.random.default_rng(8)
    if case == "strong":
        w = -np.exp(g.uniform(-1.0, 3.0, w.shape))
    elif case == "mixed":
        w[:, 70:75, :] = -40.0            # one chunk leaves the range, its neighbours do not
        w[0, 150, 5] = -np.inf
    elif case == "zero_decay":
        w[:] = -np.inf
    else:
        w[:] = 0.0
    x.w = synth.to_bf16_bits(w.astype(np.float32))
    y = gc.run_wkv6_fwd(x)
    r, k, v, ww, u = gc.f64(x)
    ref = oracle.wkv6_fwd(r, k, v, ww, u, H=H)
    assert np.all(np.isfinite(y))
    assert _rel(y, ref) <= _bf16_bound(bf16_path), _rel(y, ref)


def _with_w(x, w):
    x.w = w.astype(np.float32)
    return x


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("case", ["strong", "mixed", "zero_decay", "unit_decay", "long_memory"])
def test_wkv6_fwd_decay_edge_cases(case, bidir, f32_path):
    B, T, H = 2, 70, 2
    x = synth.make_wkv6(B, T, H, seed=11)
    g = np.random.default_rng(5)
    if case == "strong":          # every token forces a renorm step (|ew| up to e^3)
        w = -np.exp(g.uniform(-1.0, 3.0, x.w.shape))
    elif case == "mixed":         # a few tokens with huge or exactly-zero decay
        w = x.w.astype(np.float64).copy()
        w[:, 5, :] = -60.0
        w[:, 40, 3] = -np.inf
        w[1, 17, :] = -3.0
    elif case == "zero_decay":    # decay exactly 0 everywhere: only the previous token survives
        w = np.full(x.w.shape, -np.inf)
    elif case == "unit_decay":    # decay exactly 1: plain causal / full linear attention
        w = np.zeros(x.w.shape)
    else:                         # very slow decay over a long sequence
        x = synth.make_wkv6(1, 700, 2, seed=12)
        w = -np.exp(np.random.default_rng(6).uniform(-9.0, -6.0, x.w.shape))
    x = _with_w(x, w)
    y = gc.run_wkv6_fwd(x, bidir=bidir)
    r, k, v, ww, u = gc.f64(x)
    ref = oracle.wkv6_fwd(r, k, v, ww, u, H=x.H, bidirectional=bidir)
    assert np.all(np.isfinite(y))
    assert _rel(y, ref) <= gc.TOL_F32_FWD


def test_wkv6_fwd_output_fully_overwritten_and_deterministic(f32_path):
    x = synth.make_wkv6(2, 77, 3, seed=3)
    y1 = gc.run_wkv6_fwd(x, bidir=True)   # outputs start as NaN inside run_wkv6_fwd
    y2 = gc.run_wkv6_fwd(x, bidir=True)
    assert np.all(np.isfinite(y1))
    assert np.array_equal(y1, y2)


def test_wkv6_fwd_slices_match_single_head_calls(f32_path):
    x = synth.make_wkv6(2, 50, 3, seed=4)
    y = gc.run_wkv6_fwd(x)
    for b in range(2):
        for h in range(3):
            sl = slice(64 * h, 64 * h + 64)
            xs = synth.Wkv6Inputs(1, 50, 64, 1, *(np.ascontiguousarray(getattr(x, n)[b:b + 1, :, sl])
                                                 for n in ("r", "k", "v", "w")), x.u[sl].copy())
            assert np.array_equal(gc.run_wkv6_fwd(xs), y[b:b + 1, :, sl])


# ------------------------------------------------------------------ backward, small and ragged

@pytest.fixture(params=["tensor", "recurrence"])
def bwd_path(request):
    """Run the fp32 backward through the chunked tensor-core kernels (split-bf16
    operands) or the two-sweep recurrence kernel (the test build)."""
    with gc.library_for(request.param):
        yield request.param


@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (1, 2, 1), (2, 15, 2), (1, 16, 1), (2, 17, 1), (1, 32, 1), (1, 33, 2),
                                   (2, 65, 1), (1, 130, 2), (1, 50, 3),
                                   (2, 96, 2)])
@pytest.mark.parametrize("bidir", [False, True])
def test_wkv6_bwd_small(B, T, H, bidir, bwd_path):
    x = synth.make_wkv6(B, T, H, seed=100 + T, with_dy=True)
    got = gc.run_wkv6_bwd(x, bidir)
    r, k, v, w, u = gc.f64(x)
    ref = oracle.wkv6_bwd(r, k, v, w, u, x.dy.astype(np.float64), H=H, bidirectional=bidir)
    for name, g, e in zip(("dr", "dk", "dv", "dw", "du"), got, ref):
        assert np.all(np.isfinite(g)), name
        if name == "dw" and T <= 2:
            # exactly zero in exact arithmetic (every token is the first or the last).
            # The tensor-core kernels evaluate the first token's dw in prefix form and
            # the last token's in suffix form, where each term is an exact zero: exact
            # zeros.  The recurrence's pair terms cancel to a residue of ~1e-7.
            bound = 1e-6 if bwd_path == "recurrence" else 0.0
            assert np.max(np.abs(g)) <= bound, (name, np.max(np.abs(g)), bound)
            continue
        assert _rel(g, e) <= gc.TOL_F32_GRAD, (name, _rel(g, e))


@pytest.mark.parametrize("B,T,H", [(2, 3, 1), (1, 31, 2), (2, 33, 1), (1, 65, 2), (2, 197, 2)])
@pytest.mark.parametrize("bidir", [False, True])
def test_wkv6_bwd_decay_gradient_vanishes_at_both_ends(B, T, H, bidir, bwd_path):
    """The first token's decay scales the empty state and the last token's decay scales a
    state no token reads (in both sweep directions), so dw[:, 0, :] and dw[:, T-1, :] are
    exactly zero in exact arithmetic.  The chunked tensor-core backward evaluates the first
    token's dw in prefix form and the last token's in suffix form, where every term is an
    exact zero, so it returns exact zeros; the recurrence's ends are bounded by 1e-6 of the
    largest |dw|."""
    x = synth.make_wkv6(B, T, H, seed=900 + T, with_dy=True)
    dr, dk, dv, dw, du = gc.run_wkv6_bwd(x, bidir)
    ends = np.abs(dw[:, [0, T - 1], :])
    if bwd_path == "recurrence":
        assert ends.max() <= 1e-6 * np.abs(dw).max(), ends.max()
    else:
        assert np.all(ends == 0.0), ends.max()
    r, k, v, w, u = gc.f64(x)
    ref = oracle.wkv6_bwd(r, k, v, w, u, x.dy.astype(np.float64), H=H, bidirectional=bidir)
    assert _rel(dw, ref[3]) <= gc.TOL_F32_GRAD


@pytest.mark.parametrize("bidir", [False, True])
def test_wkv6_bwd_strong_decay_and_determinism(bidir, bwd_path):
    x = synth.make_wkv6(2, 45, 2, seed=7, with_dy=True)
    w = -np.exp(np.random.default_rng(9).uniform(-2.0, 3.5, x.w.shape))
    w[:, 10, :] = -np.inf
    x = _with_w(x, w)
    g1 = gc.run_wkv6_bwd(x, bidir)
    g2 = gc.run_wkv6_bwd(x, bidir)
    for a, b in zip(g1, g2):
        assert np.array_equal(a, b)
    r, k, v, ww, u = gc.f64(x)
    ref = oracle.wkv6_bwd(r, k, v, ww, u, x.dy.astype(np.float64), H=2, bidirectional=bidir)
    for name, g, e in zip(("dr", "dk", "dv", "dw", "du"), g1, ref):
        assert _rel(g, e) <= gc.TOL_F32_GRAD, (name, _rel(g, e))


# ------------------------------------------------------------------ RWKV-4

@pytest.mark.parametrize("B,T,C", [(1, 1, 32), (2, 7, 40), (1, 100, 64), (2, 333, 96), (1, 1024, 32),
                                   (3, 9, 8), (1, 129, 36), (2, 1000, 100), (1, 1025, 32), (2, 2049, 48),
                                   (2, 50, 30), (1, 65, 36), (3, 31, 20)])   # C % 4 != 0: per-channel kernel
def test_wkv4_small(B, T, C):
    x = synth.make_wkv4(B, T, C, seed=T)
    y = gc.run_wkv4(x)
    ref = oracle.wkv4_fwd(x.k, x.v, x.w, x.u)
    assert np.all(np.isfinite(y))
    assert _rel(y, ref) <= gc.TOL_F32_FWD


def test_wkv4_large_keys():
    x = synth.make_wkv4(2, 300, 64, seed=3, kv_std=1.0)
    x.k = (x.k * 30.0).astype(np.float32)     # e^k overflows fp32 without the log-space state
    y = gc.run_wkv4(x)
    ref = oracle.wkv4_fwd(x.k, x.v, x.w, x.u)
    assert np.all(np.isfinite(y))
    assert _rel(y, ref) <= gc.TOL_F32_FWD


# ------------------------------------------------------------------ full-size workloads

def test_workload_causal_f32_small_config_full_tensor(f32_path):
    kind, x = synth.make_workload("wkv6_causal_f32_b1t196h4")
    y = gc.run_wkv6_fwd(x)
    r, k, v, w, u = gc.f64(x)
    assert _rel(y, oracle.wkv6_fwd(r, k, v, w, u, H=x.H)) <= gc.TOL_F32_FWD


def test_workload_wkv4_full_tensor():
    kind, x = synth.make_workload("wkv4_f32_b8t1024c768")
    y = gc.run_wkv4(x)
    assert _rel(y, oracle.wkv4_fwd(x.k, x.v, x.w, x.u)) <= gc.TOL_F32_FWD


def test_workload_bidir_f32_full_tensor(f32_path):
    kind, x = synth.make_workload("wkv6_bidir_f32_b32t196h12")
    y = gc.run_wkv6_fwd(x, bidir=True)
    assert np.all(np.isfinite(y))
    err = _rel(y, gc.oracle_fwd_full(x, True))
    assert err <= gc.TOL_F32_FWD, err


def test_workload_causal_bf16_long_full_tensor(bf16_path):
    kind, x = synth.make_workload("wkv6_causal_bf16_b8t4096h32")
    y = gc.run_wkv6_fwd(x)
    assert np.all(np.isfinite(y))
    err = _rel(y, gc.oracle_fwd_full(x, False))
    assert err <= gc.TOL_BF16_FWD, err
    assert err <= _bf16_bound(bf16_path), err


def test_workload_bidir_bwd_full_tensor(bwd_path):
    kind, x = synth.make_workload("wkv6_bidir_bwd_f32_b32t196h12")
    got = gc.run_wkv6_bwd(x, True)
    ref = gc.oracle_bwd_full(x, True)
    for n, g, e in zip(("dr", "dk", "dv", "dw", "du"), got, ref):
        assert np.all(np.isfinite(g)), n
        err = _rel(g, e)
        assert err <= gc.TOL_F32_GRAD, (n, err)
