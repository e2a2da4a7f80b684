"""wkv6_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: code running inside another
framework's plugin or callback that offers no scratch buffer, or a serving
process that reserves its device memory at start-up and may not call cudaMalloc
later.  wkv6_bwd_noalloc keeps its scratch in a fixed array inside libwkv.so
instead.  These tests check, through the C ABI, that its gradients match the
double-precision oracle within the gradient tolerance, call after call (the
shared array keeps the previous call's contents, so each case runs twice with
different upstream gradients, and the cases run from the largest to the
smallest so that every entry a call reads was left non-zero by the one before),
including a problem exactly at the array's size limit, and that it refuses
sizes past that limit.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

import linear_attention_rnn_wkv6_b200 as wkv
from linear_attention_rnn_wkv6_b200 import synth

NOALLOC_LIMIT = 262144  # B*C floats of scratch inside the library
TOL_F32_GRAD = 1e-4     # relative L2 per gradient tensor, as in the other parity tests


def test_noalloc_symbol_and_limit_on_host():
    """Oversized problems are refused on the host before anything touches a GPU."""
    from linear_attention_rnn_wkv6_b200 import build
    build.build()
    lib = wkv.load()
    assert hasattr(lib, "wkv6_bwd_noalloc")
    fake = [0x10000000 + 256 * i for i in range(11)]
    B, C = NOALLOC_LIMIT // 64 + 1, 64          # B*C one batch past the limit
    assert lib.wkv6_bwd_noalloc(B, 4, C, 1, 1, *fake, None) == -7     # WKV_ERR_TOO_LARGE
    assert lib.wkv6_bwd_noalloc(2, 4, 64, 2, 1, *fake, None) == -2    # head size 32 rejected as in wkv6_bwd


@pytest.mark.gpu
@pytest.mark.parametrize("bidir", [False, True])
def test_noalloc_matches_oracle_on_repeated_calls(bidir):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_rnn_wkv6_b200 import build
    build.build()
    import oracle
    oracle.build()
    from tests import gpu_cases as gc

    # (B, T, H): B*C = 262144 exactly (the limit), then two smaller problems
    shapes = [(NOALLOC_LIMIT // 64, 3, 1), (5, 33, 3), (3, 70, 2)]
    assert shapes[0][0] * 64 * shapes[0][2] == NOALLOC_LIMIT
    for i, (B, T, H) in enumerate(shapes):
        x = synth.make_wkv6(B, T, H, seed=41 + i, with_dy=True)
        ins = [gc.dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u")]
        for call in range(2):
            # a different upstream gradient on each call: what the previous call left in
            # the shared array is never the right answer for this one
            dy = x.dy if call == 0 else synth.make_wkv6(B, T, H, seed=141 + i, with_dy=True).dy
            got = [gc.empty_nan((B, T, x.C)) for _ in range(4)] + [gc.empty_nan((x.C,))]
            wkv.wkv6_bwd_noalloc(B, T, x.C, H, bidir, *ins, gc.dev(dy), *got)
            assert wkv.wkv_take_device_faults() == 0
            gc.check_guards()
            ref = gc.oracle_bwd_full(x, bidir, dy.astype(np.float64))
            for name, g, e in zip(("dr", "dk", "dv", "dw", "du"), got, ref):
                g = g.cpu().numpy()
                assert np.all(np.isfinite(g)), (name, B, call)
                if name == "dw" and T <= 2:
                    continue
                rel = oracle.rel_l2(g, e)
                assert rel <= TOL_F32_GRAD, (name, B, call, rel)
