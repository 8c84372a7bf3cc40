"""Graph replay of a run (SPECTRE_OPT_GRAPH): the replayed step must give the
bytes the directly enqueued launches give, follow pointer and option changes
(which capture again), see new input contents in the same buffers, and hand a
caller that captures its own graph the plain launches."""
from __future__ import annotations

import pytest
import torch

from sub_quadratic_attention_b200.workloads import WORKLOADS, custom, make_inputs

pytestmark = pytest.mark.gpu


def _run(mix, d, y, q=None):
    mix(d["q"] if q is None else q, d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y=y)


@pytest.mark.parametrize("case", ["bf16_long", "fp32_mid", (2, 12288, 2, 64, 6145)])
def test_graph_replay_is_bitwise_equal_to_direct_launches(case):
    from sub_quadratic_attention_b200 import binding
    from sub_quadratic_attention_b200.binding import SpectreMix

    w = WORKLOADS[case] if isinstance(case, str) else custom(*case, dtype="bf16")
    d = {k: v.cuda() for k, v in make_inputs(w).items()}
    q2 = torch.flip(d["q"], dims=[1]).contiguous()
    with SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps, graph=False) as direct, \
            SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps, graph=True) as g:
        y_ref = torch.empty_like(d["x"])
        _run(direct, d, y_ref)
        y_ref2 = torch.empty_like(d["x"])
        _run(direct, d, y_ref2, q=q2)
        # capture, then replay
        ya = torch.full_like(d["x"], float("nan"))
        for _ in range(2):
            _run(g, d, ya)
            torch.cuda.synchronize()
            assert torch.equal(ya, y_ref)
        # another output buffer: captured again
        yb = torch.full_like(d["x"], float("nan"))
        _run(g, d, yb)
        torch.cuda.synchronize()
        assert torch.equal(yb, y_ref)
        # the same buffers with new contents: the replay reads them
        qa = d["q"].clone()
        _run(g, d, ya, q=qa)
        qa.copy_(q2)
        _run(g, d, ya, q=qa)
        torch.cuda.synchronize()
        assert torch.equal(ya, y_ref2)
        # an option change captures again with the new plan
        for m in (direct, g):
            binding.spectre_mix_set_option(m.handle, binding.SPECTRE_OPT_NORM, binding.SPECTRE_NORM["pre_ln"])
        _run(direct, d, y_ref)
        _run(g, d, ya)
        torch.cuda.synchronize()
        assert torch.equal(ya, y_ref)
        for m in (direct, g):
            assert binding.spectre_mix_device_status(m.handle) == binding.SPECTRE_OK


def test_caller_capture_gets_plain_launches():
    """A run enqueued on a stream that the caller is capturing goes into the
    caller's graph (no nested capture); replaying that graph gives the direct
    result."""
    from sub_quadratic_attention_b200.binding import SpectreMix

    w = WORKLOADS["bf16_long"]
    d = {k: v.cuda() for k, v in make_inputs(w).items()}
    with SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps, graph=False) as direct, \
            SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps, graph=True) as g:
        y_ref = torch.empty_like(d["x"])
        _run(direct, d, y_ref)
        y = torch.full_like(d["x"], float("nan"))
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(cg, stream=s):
                g(d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y=y, stream=s)
        torch.cuda.synchronize()
        cg.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref)
        del cg
