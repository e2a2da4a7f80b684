"""GPU parity of wkv6_fwd_fused (decay prologue ew = -exp(w_base + ww), per-head
group norm and gate epilogue) against the oracle, through the C ABI on seeded
inputs; fp32 forward tolerance (relative L2 <= 1e-5)."""
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
def f32_path(request):
    """Both fp32 forward kernels: the chunked tensor-core one (split-bf16 operands; the norm
    and gate in its epilogue) and the token-by-token recurrence (the test build)."""
    with gc.library_for(request.param):
        yield request.param


_NAMES = ("r", "k", "v", "ww", "w_base", "u", "g", "gn_w", "gn_b")


def _run(x):
    import linear_attention_rnn_wkv6_b200 as wkv
    ins = [gc.dev(getattr(x, n)) for n in _NAMES]
    out = gc.empty_nan((x.B, x.T, x.C))
    wkv.wkv6_fwd_fused(x.B, x.T, x.C, x.H, x.bidir, *ins, x.eps, out)
    assert wkv.wkv_take_device_faults() == 0
    return out.cpu().numpy()


def _ref(x, b=slice(None), h=None):
    sl = slice(None) if h is None else slice(64 * h, 64 * h + 64)
    a = {n: getattr(x, n) for n in _NAMES}
    args = [a[n][b, :, sl] if a[n].ndim == 3 else a[n][sl] for n in _NAMES]
    return oracle.wkv6_fwd_fused(*args, x.eps, H=x.H if h is None else 1, bidirectional=x.bidir)


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (2, 17, 2), (1, 196, 3), (2, 77, 1)])
def test_fused_matches_oracle(B, T, H, bidir):
    x = synth.make_fused(B, T, H, seed=800 + T, bidir=bidir)
    out = _run(x)
    assert np.all(np.isfinite(out))
    assert oracle.rel_l2(out, _ref(x)) <= gc.TOL_F32_FWD


@pytest.mark.parametrize("bidir", [False, True])
def test_fused_strong_decay_and_large_eps(bidir):
    """Decay pre-activations up to 3 (per-token decay exp(-e^3), renormalised at every token)
    and a variance offset comparable to the row variances."""
    x = synth.make_fused(2, 90, 2, seed=810, bidir=bidir, base_lo=-8.0, base_hi=2.0, ww_std=1.0, eps=0.05)
    assert oracle.rel_l2(_run(x), _ref(x)) <= gc.TOL_F32_FWD


@pytest.mark.parametrize("bidir", [False, True])
def test_fused_one_fast_forgetting_token(bidir):
    """One token whose decay pre-activation is about 5 in a few channels (log-decay below -80):
    the chunk holding it takes the exact token-by-token path, its neighbours the chunked one."""
    x = synth.make_fused(2, 130, 2, seed=830, bidir=bidir)
    x.ww[:, 40, 3:7] = 6.0
    out = _run(x)
    assert np.all(np.isfinite(out))
    assert oracle.rel_l2(out, _ref(x)) <= gc.TOL_F32_FWD


def test_fused_workload_full_tensor():
    """The patch-sequence shape (B32 T196 H12, bidirectional), every element (the oracle
    runs one batch per host thread)."""
    x = synth.make_fused(32, 196, 12, seed=0, bidir=True)
    out = _run(x)
    ref = np.concatenate(gc._map_batches(lambda b: _ref(x, slice(b, b + 1), None), x.B))
    assert oracle.rel_l2(out, ref) <= gc.TOL_F32_FWD


def test_fused_unit_epilogue_equals_normalised_plain_forward():
    """With unit weight, zero bias and unit gate, the fused output is the plain forward at
    w = -exp(w_base + ww) normalised per head (both computed on the GPU)."""
    import linear_attention_rnn_wkv6_b200 as wkv
    x = synth.make_fused(2, 60, 2, seed=820)
    x.gn_w[:] = 1.0
    x.gn_b[:] = 0.0
    x.g[:] = 1.0
    out = _run(x)
    ew = (-np.exp(x.w_base.astype(np.float64) + x.ww)).astype(np.float32)
    y = gc.empty_nan((x.B, x.T, x.C))
    wkv.wkv6_fwd(x.B, x.T, x.C, x.H, *(gc.dev(a) for a in (x.r, x.k, x.v, ew, x.u)), y)
    yh = y.cpu().numpy().astype(np.float64).reshape(x.B, x.T, x.H, 64)
    norm = (yh - yh.mean(-1, keepdims=True)) / np.sqrt(yh.var(-1, keepdims=True) + x.eps)
    assert oracle.rel_l2(out, norm.reshape(out.shape)) <= gc.TOL_F32_FWD
