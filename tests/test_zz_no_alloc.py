"""The entry point that allocates nothing, checked against the regular one.

spectre_mix_run_noalloc is for callers that may not call cudaMalloc -- code
inside a framework whose caching allocator owns the device memory, or a
latency-critical loop that cannot afford the synchronisation an allocation can
imply.  It runs the same kernels, on the same twiddle tables (both paths build
them with one device kernel), in the library's fixed 64 MiB device scratch.
So two calls in a row must each reproduce spectre_mix_run's y bit for bit,
including a plan that takes the tensor-core slice pass (L = 65536, whose DFT-64
operand and inter-pass twiddles the no-allocation path builds in the scratch).
A shape that does not fit must be refused with SPECTRE_ERR_SCRATCH.  This file
is named so that pytest collects it last.
"""
import pytest
import torch

from sub_quadratic_attention_b200 import binding as b
from sub_quadratic_attention_b200.workloads import WORKLOADS, custom, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    (WORKLOADS["tiny_fp32"], "cuda_cores"),
    (custom(1, 4096, 4, 16, 1000, dtype="bf16", name="noalloc_bf16"), "cuda_cores"),
    (custom(3, 768, 3, 5, 200, dtype="f32", name="noalloc_mixed_radix_odd_c"), "cuda_cores"),
    (custom(1, 65536, 1, 16, 8192, dtype="bf16", name="noalloc_tensor_cores"), "tensor_cores"),
]


@pytest.mark.parametrize("w,slice_pass", CASES, ids=lambda c: getattr(c, "name", c))
def test_noalloc_matches_regular_entry_point_twice(w, slice_pass):
    d = {k: v.cuda() for k, v in make_inputs(w).items()}
    code = b.SPECTRE_F32 if w.dtype == "f32" else b.SPECTRE_BF16
    y_ref = torch.empty_like(d["x"])
    with b.SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps) as mix:
        # the no-allocation path runs the plan's default slice pass too
        assert mix.slice_pass == slice_pass
        mix(d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y=y_ref)
        torch.cuda.synchronize()
        assert b.spectre_mix_device_status(mix.handle) == b.SPECTRE_OK
    assert not torch.isnan(y_ref.float()).any()
    for _ in range(2):
        y = torch.full_like(d["x"], float("nan"))
        st = b.spectre_mix_run_noalloc_status(w.B, w.L, w.H, w.D, w.F, code, w.eps, d["q"], d["k"],
                                              d["v"], d["x"], d["G"], d["gamma"], d["beta"], y)
        assert st == b.SPECTRE_OK, b.spectre_mix_error_string(st)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), float((y.double() - y_ref.double()).abs().max())


def test_noalloc_refuses_shapes_beyond_the_scratch():
    w = WORKLOADS["bf16_long"]   # about 600 MB of workspace
    q = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    G = torch.zeros(16, dtype=torch.float32, device="cuda")
    st = b.spectre_mix_run_noalloc_status(w.B, w.L, w.H, w.D, w.F, b.SPECTRE_BF16, w.eps,
                                          q, q, q, q, G, G, G, q)
    assert st == b.SPECTRE_ERR_SCRATCH
    assert "scratch" in b.spectre_mix_error_string(st)
