"""GPU parity of wkv6_bwd_bf16 (bf16 r, k, v, w, dy; fp32 u and gradients) against
the oracle's backward on the same bf16-rounded input values.

The kernels compute in fp32 from exactly the values the oracle sees, so the fp32
gradient tolerance applies (relative L2 per tensor).  Both algorithms run: the
chunked tensor-core kernels (the default) and the two-sweep recurrence.
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
    from linear_attention_rnn_wkv6_b200 import build
    build.build()


@pytest.fixture(params=["tensor", "recurrence"], autouse=True)
def bwd_path(request):
    with gc.library_for(request.param):
        yield request.param


def _check(x, bidir, got, dy64, H, path):
    r, k, v, w, u = gc.f64(x)
    ref = oracle.wkv6_bwd(r, k, v, w, u, dy64, H=H, bidirectional=bidir)
    for name, g, e in zip(("dr", "dk", "dv", "dw", "du"), got, ref):
        assert np.all(np.isfinite(g)), name
        if name == "dw" and x.T <= 2:
            # exactly zero in exact arithmetic; the tensor-core kernels return exact
            # zeros (prefix form at the first token, suffix form at the last)
            assert np.max(np.abs(g)) <= (1e-6 if path == "recurrence" else 0.0), name
            continue
        err = oracle.rel_l2(g, e)
        assert err <= gc.TOL_F32_GRAD, (name, err)


@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (2, 15, 2), (1, 16, 1), (2, 17, 1), (1, 33, 2), (1, 50, 3), (2, 96, 2)])
@pytest.mark.parametrize("bidir", [False, True])
def test_bwd_bf16_small(B, T, H, bidir, bwd_path):
    x = synth.make_wkv6(B, T, H, seed=400 + T, with_dy=True, dtype="bf16")
    got, dy64 = gc.run_wkv6_bwd_bf16(x, bidir)
    _check(x, bidir, got, dy64, H, bwd_path)


@pytest.mark.parametrize("bidir", [False, True])
def test_bwd_bf16_strong_decay(bidir, bwd_path):
    x = synth.make_wkv6(2, 45, 2, seed=410, with_dy=True, dtype="bf16")
    w = -np.exp(np.random.default_rng(411).uniform(-2.0, 3.5, x.w.shape)).astype(np.float32)
    w[:, 10, :] = -np.inf
    x.w = synth.to_bf16_bits(w)
    got, dy64 = gc.run_wkv6_bwd_bf16(x, bidir)
    _check(x, bidir, got, dy64, 2, bwd_path)


def test_bwd_bf16_workload_full_tensor():
    """The bidirectional backward workload's shape (B32 T196 H12) in bf16, every element."""
    x = synth.make_wkv6(32, 196, 12, seed=0, with_dy=True, dtype="bf16")
    got, dy64 = gc.run_wkv6_bwd_bf16(x, True)
    ref = gc.oracle_bwd_full(x, True, dy64)
    for n, g, e in zip(("dr", "dk", "dv", "dw", "du"), got, ref):
        assert np.all(np.isfinite(g)), n
        err = oracle.rel_l2(g, e)
        assert err <= gc.TOL_F32_GRAD, (n, err)
