"""The bounded waits' failure path on the GPU, without a fault: a wait that nothing
completes gives up after its limit, sets WKV_FAULT_TIMEOUT in the device fault word
and returns; the context stays usable and the next calls run clean."""
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


def test_wait_that_runs_out_is_reported_and_the_context_survives():
    import linear_attention_rnn_wkv6_b200 as wkv
    assert wkv.wkv_take_device_faults() == 0
    wkv.wkv_selftest_wait_timeout()
    assert wkv.wkv_take_device_faults() == wkv.WKV_FAULT_TIMEOUT   # read and cleared
    assert wkv.wkv_take_device_faults() == 0
    # the same context still computes correctly
    x = synth.make_wkv6(2, 40, 2, seed=77)
    y = gc.empty_nan((x.B, x.T, x.C))
    wkv.wkv6_fwd(x.B, x.T, x.C, x.H, *(gc.dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u")), y)
    assert wkv.wkv_take_device_faults() == 0
    ref = oracle.wkv6_fwd(*(x.as_f64(n) for n in ("r", "k", "v", "w")), x.u.astype(np.float64), H=x.H)
    assert oracle.rel_l2(y.cpu().numpy(), ref) <= gc.TOL_F32_FWD
