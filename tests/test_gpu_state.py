"""GPU parity of the state-carrying entry points (wkv6_fwd_state, wkv6_decode)
against the oracle's causal forward from an initial state.

All calls go through the C ABI on synthetic seeded inputs; expected values come
from the double-precision oracle on the same input bits.  Tolerances are those
of the fp32 forward (relative L2 per tensor).
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


def _rel(a, b):
    return oracle.rel_l2(a, b)


def _run_state(x, s0, T_slice=slice(None)):
    """wkv6_fwd_state on tokens T_slice of x from s0 (numpy or None) -> (y, sT) numpy."""
    import linear_attention_rnn_wkv6_b200 as wkv
    t = gc.torch()
    r, k, v, w = (gc.dev(np.ascontiguousarray(getattr(x, n)[:, T_slice])) for n in ("r", "k", "v", "w"))
    T = r.shape[1]
    u = gc.dev(x.u)
    y = gc.empty_nan((x.B, T, x.C))
    sT = gc.empty_nan((x.B, x.H, 64, 64))
    s0d = gc.dev(s0) if s0 is not None else None
    wkv.wkv6_fwd_state(x.B, T, x.C, x.H, r, k, v, w, u, s0d, y, sT)
    assert wkv.wkv_take_device_faults() == 0
    return y.cpu().numpy(), sT.cpu().numpy()


def _oracle_state(x, s0, T_slice=slice(None)):
    r, k, v, w, u = gc.f64(x)
    return oracle.wkv6_fwd_state(r[:, T_slice], k[:, T_slice], v[:, T_slice], w[:, T_slice], u, x.H,
                                 None if s0 is None else s0.astype(np.float64))


@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (2, 17, 3), (3, 64, 2), (1, 200, 4), (2, 333, 2)])
@pytest.mark.parametrize("with_s0", [False, True])
def test_fwd_state_matches_oracle(B, T, H, with_s0):
    x = synth.make_wkv6(B, T, H, seed=300 + T + H)
    s0 = synth.make_state(B, H, seed=301 + T) if with_s0 else None
    y, sT = _run_state(x, s0)
    yo, so = _oracle_state(x, s0)
    assert _rel(y, yo) <= gc.TOL_F32_FWD, _rel(y, yo)
    assert _rel(sT, so) <= gc.TOL_F32_FWD, _rel(sT, so)


@pytest.mark.parametrize("library", ["default", "recurrence"])
def test_fwd_state_without_s0_is_the_zero_state(library):
    """No initial state is the zero state: the same bits as an explicit zero s0 (both
    builds run the state form on the register recurrence)."""
    x = synth.make_wkv6(2, 150, 3, seed=310)
    with gc.library_for(library):
        y, sT = _run_state(x, None)
        yz, sTz = _run_state(x, np.zeros((x.B, x.H, 64, 64), np.float32))
    assert np.array_equal(y, yz) and np.array_equal(sT, sTz)


def test_fwd_state_without_s0_equals_plain_forward_on_the_same_kernel():
    """In the test build the plain forward runs the same register recurrence as the
    state form: bit-identical outputs."""
    x = synth.make_wkv6(2, 300, 3, seed=311)
    with gc.library_for("recurrence"):
        y, _ = _run_state(x, None)
        assert np.array_equal(y, gc.run_wkv6_fwd(x))


@pytest.mark.parametrize("T", [150, 300])
def test_fwd_state_without_s0_near_chunked_forward(T):
    """Product build: the plain forward takes a chunked form (the cluster form at
    T = 150, the chunk chain at T = 300), the state form the register recurrence;
    both within the fp32 tolerance of each other."""
    x = synth.make_wkv6(2, T, 3, seed=312)
    y, _ = _run_state(x, None)
    assert _rel(y, gc.run_wkv6_fwd(x)) <= gc.TOL_F32_FWD
@pytest.mark.parametrize("cut", [1, 16, 77, 199])
def test_fwd_state_split_sequence(cut):
    """Two calls over [0, cut) and [cut, T) with the carried state match one call and the oracle."""
    x = synth.make_wkv6(2, 200, 2, seed=320)
    s0 = synth.make_state(2, 2, seed=321)
    y1, s1 = _run_state(x, s0, slice(0, cut))
    y2, s2 = _run_state(x, s1, slice(cut, None))
    yo, so = _oracle_state(x, s0)
    y = np.concatenate([y1, y2], axis=1)
    assert _rel(y, yo) <= gc.TOL_F32_FWD, _rel(y, yo)
    assert _rel(s2, so) <= gc.TOL_F32_FWD, _rel(s2, so)


def test_fwd_state_in_place_and_empty():
    import linear_attention_rnn_wkv6_b200 as wkv
    x = synth.make_wkv6(2, 40, 2, seed=330)
    s0 = synth.make_state(2, 2, seed=331)
    r, k, v, w, u = (gc.dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u"))
    st = gc.dev(s0.copy())
    y = gc.empty_nan((x.B, x.T, x.C))
    wkv.wkv6_fwd_state(x.B, x.T, x.C, x.H, r, k, v, w, u, st, y, st)        # s0 and sT the same buffer
    yo, so = _oracle_state(x, s0)
    assert _rel(y.cpu().numpy(), yo) <= gc.TOL_F32_FWD
    assert _rel(st.cpu().numpy(), so) <= gc.TOL_F32_FWD
    # T = 0: the final state is the initial one, or zero without one
    out = gc.empty_nan((x.B, x.H, 64, 64))
    wkv.wkv6_fwd_state(x.B, 0, x.C, x.H, r, k, v, w, u, gc.dev(s0), y, out)
    assert np.array_equal(out.cpu().numpy(), s0)
    wkv.wkv6_fwd_state(x.B, 0, x.C, x.H, r, k, v, w, u, None, y, out)
    assert not np.any(out.cpu().numpy())
    assert wkv.wkv_take_device_faults() == 0


@pytest.mark.parametrize("kind", ["zero", "strong", "mixed"])
def test_fwd_state_decay_edge_cases(kind):
    """Decays down to exactly 0 and fast-forgetting rows (renorm steps) with a nonzero start state."""
    x = synth.make_wkv6(1, 70, 2, seed=340)
    w = x.w.copy()
    if kind == "zero":
        w[:, 5:9, :] = -np.inf
    elif kind == "strong":
        w[:] = -60.0
    else:
        w[:, :, ::3] = -80.0
        w[:, 30:33, 7] = -np.inf
    x.w = w.astype(np.float32)
    s0 = synth.make_state(1, 2, seed=341)
    y, sT = _run_state(x, s0)
    yo, so = _oracle_state(x, s0)
    assert _rel(y, yo) <= gc.TOL_F32_FWD, _rel(y, yo)
    assert _rel(sT, so) <= gc.TOL_F32_FWD, _rel(sT, so)


@pytest.mark.parametrize("B,H,steps", [(1, 1, 1), (3, 2, 20), (64, 4, 6)])
def test_decode_steps_match_oracle(B, H, steps):
    """Repeated wkv6_decode calls reproduce the causal forward token by token from s0."""
    import linear_attention_rnn_wkv6_b200 as wkv
    x = synth.make_wkv6(B, steps, H, seed=350 + B)
    s0 = synth.make_state(B, H, seed=351)
    yo, so = _oracle_state(x, s0)
    st = gc.dev(s0.copy())
    u = gc.dev(x.u)
    ys = []
    for t in range(steps):
        r, k, v, w = (gc.dev(np.ascontiguousarray(getattr(x, n)[:, t])) for n in ("r", "k", "v", "w"))
        y = gc.empty_nan((B, x.C))
        wkv.wkv6_decode(B, x.C, x.H, r, k, v, w, u, st, y)
        ys.append(y.cpu().numpy())
    assert wkv.wkv_take_device_faults() == 0
    y = np.stack(ys, axis=1)
    assert _rel(y, yo) <= gc.TOL_F32_FWD, _rel(y, yo)
    assert _rel(st.cpu().numpy(), so) <= gc.TOL_F32_FWD


def test_decode_at_serving_size_sampled():
    """One decode step for B=256 sequences of H=32 heads, checked on sampled (b, h) units."""
    import linear_attention_rnn_wkv6_b200 as wkv
    B, H = 256, 32
    x = synth.make_wkv6(B, 1, H, seed=360)
    s0 = synth.make_state(B, H, seed=361)
    st = gc.dev(s0.copy())
    y = gc.empty_nan((B, x.C))
    r, k, v, w = (gc.dev(np.ascontiguousarray(getattr(x, n)[:, 0])) for n in ("r", "k", "v", "w"))
    wkv.wkv6_decode(B, x.C, x.H, r, k, v, w, gc.dev(x.u), st, y)
    assert wkv.wkv_take_device_faults() == 0
    y, st = y.cpu().numpy(), st.cpu().numpy()
    for b, h in gc.sample_units(B, H, 24):
        (ru, ku, vu, wu, uu), _, sl = gc.unit_slice(x, b, h)
        yo, so = oracle.wkv6_fwd_state(ru, ku, vu, wu, uu, 1, s0[b:b + 1, h:h + 1].astype(np.float64))
        assert _rel(y[b, sl], yo[0, 0]) <= gc.TOL_F32_FWD
        assert _rel(st[b, h], so[0, 0]) <= gc.TOL_F32_FWD
