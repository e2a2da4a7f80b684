"""Host-side rules of bench.py that need no GPU: what a workload's footprint
counts, and when a run flushes L2 between steps."""
import types

import torch

import bench
from linear_attention_rnn_wkv6_b200 import synth

L2_BYTES = 126 * 2**20


def _fake(inputs, outputs, ws=None, state=None):
    w = types.SimpleNamespace(inputs=inputs, outputs=outputs)
    if ws is not None:
        w.ws = ws
    if state is not None:
        w.state = state
    return w


def test_footprint_counts_inputs_outputs_workspace_and_state():
    f = _fake({"k": torch.zeros(10, dtype=torch.float32), "v": torch.zeros(6, dtype=torch.int16)},
              [torch.zeros(4, dtype=torch.float32)], ws=torch.zeros(100, dtype=torch.uint8),
              state=torch.zeros(8, dtype=torch.float32))
    assert bench.DeviceWorkload.footprint(f) == 10 * 4 + 6 * 2 + 4 * 4 + 100 + 8 * 4
    assert bench.DeviceWorkload.footprint(_fake({}, [])) == 0


def test_flush_buffer_exceeds_l2():
    assert bench.FLUSH_BYTES >= 4 * L2_BYTES


def _bytes_of(name):
    """Inputs + outputs of a workload from its shapes (no allocation)."""
    kind, kw = synth.WORKLOADS[name]
    if kind == "wkv4_fwd":
        n = kw["B"] * kw["T"] * kw["C"]
        return 3 * 4 * n
    n = kw["B"] * kw["T"] * kw["H"] * 64
    el = 2 if kw.get("dtype") == "bf16" else 4
    if kind.startswith("wkv6_bwd"):
        return 5 * el * n + 4 * 4 * n
    return 4 * el * n + 4 * n


def test_default_step_is_not_flushed_and_small_workloads_are():
    step = sum(_bytes_of(n) for n in bench.STEP_WORKLOADS)
    assert step > bench.FLUSH_BYTES          # the step's kernels start cold without a flush
    assert _bytes_of("wkv4_f32_b8t1024c768") < bench.FLUSH_BYTES       # alone it would stay in L2
    assert _bytes_of("wkv6_bidir_f32_b32t196h12") < bench.FLUSH_BYTES


def test_every_workload_constructs_on_the_host(monkeypatch):
    """Each workload bench.py can time builds its inputs, outputs, workspace and state
    (device copies redirected to host tensors), alone and as rank 1 of 2; the batch
    window of a split workload has the rank's share of the units."""
    monkeypatch.setattr(torch.Tensor, "cuda", lambda self, *a, **k: self)
    empty = torch.empty

    def host_empty(*a, **k):
        k.pop("device", None)
        return empty(*a, **k)

    monkeypatch.setattr(torch, "empty", host_empty)
    for name in bench.STEP_WORKLOADS + bench.EXTRA_WORKLOADS:
        one = bench.DeviceWorkload(name, 0, 1)
        two = bench.DeviceWorkload(name, 1, 2)
        assert one.units > 0 and one.tokens > 0 and one.footprint() > 0, name
        assert two.units == one.units and two.tokens == one.tokens, name   # weak scaling: B per rank fixed


def test_every_workload_has_its_tables():
    """Each workload bench.py can time has its algorithmic work, entry point and
    launch count, and a synthetic recipe."""
    for name in bench.STEP_WORKLOADS + bench.EXTRA_WORKLOADS:
        assert name in bench.ALG and name in bench.ENTRY and name in bench.LAUNCHES, name
        assert name in synth.WORKLOADS, name
