"""wkv6_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: code running inside another
framework's plugin or callback that offers no scratch buffer, or a serving
process that reserves its device memory at start-up and may not call cudaMalloc
later.  wkv6_bwd_noalloc keeps its scratch in a fixed array inside libwkv.so
instead.  These tests check, through the C ABI, that it returns the gradients
the workspace-taking wkv6_bwd returns (within the gradient tolerance: it runs
the recurrence kernel, wkv6_bwd the tensor-core kernels by default), call after
call (the shared array keeps the previous call's contents), and that it
refuses sizes past its fixed limit.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

import linear_attention_rnn_wkv6_b200 as wkv
from linear_attention_rnn_wkv6_b200 import synth

NOALLOC_LIMIT = 262144  # B*C floats of scratch inside the library


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
def test_noalloc_matches_workspace_backward_on_repeated_calls(bidir):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_rnn_wkv6_b200 import build
    build.build()

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()

    # two different problems in a row: the second call must not see the first one's scratch
    cases = [synth.make_wkv6(3, 70, 2, seed=41, with_dy=True), synth.make_wkv6(5, 33, 3, seed=42, with_dy=True)]
    for x in cases:
        ins = [dev(getattr(x, n)) for n in ("r", "k", "v", "w", "u", "dy")]
        shape = (x.B, x.T, x.C)
        ref = [torch.empty(shape, device="cuda") for _ in range(4)] + [torch.empty(x.C, device="cuda")]
        nbytes = wkv.wkv6_bwd_workspace_bytes(x.B, x.T, x.C, x.H, bidir)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        wkv.wkv6_bwd(x.B, x.T, x.C, x.H, bidir, *ins, *ref, ws, nbytes)
        for _ in range(2):
            got = [torch.full(shape, float("nan"), device="cuda") for _ in range(4)] + \
                  [torch.full((x.C,), float("nan"), device="cuda")]
            wkv.wkv6_bwd_noalloc(x.B, x.T, x.C, x.H, bidir, *ins, *got)
            torch.cuda.synchronize()
            for name, g, e in zip(("dr", "dk", "dv", "dw", "du"), got, ref):
                g, e = g.cpu().numpy(), e.cpu().numpy()
                assert np.all(np.isfinite(g)), name
                rel = np.linalg.norm(g - e) / max(np.linalg.norm(e), 1e-30)
                assert rel <= 1e-4, (name, rel)     # the gradient tolerance of the parity tests
    assert wkv.wkv_take_device_faults() == 0
