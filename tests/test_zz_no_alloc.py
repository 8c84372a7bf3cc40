"""The entry point that allocates nothing, checked against the regular one.

spectre_mix_run_noalloc is for callers that may not call cudaMalloc -- code
inside a framework whose caching allocator owns the device memory, or a
latency-critical loop that cannot afford the synchronisation an allocation can
imply.  It runs the same kernels on the library's fixed 64 MiB device scratch.
Two calls in a row must each match spectre_mix_run within the parity
tolerances, and a shape that does not fit must be refused with
SPECTRE_ERR_SCRATCH.  This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from helpers import TOL
from sub_quadratic_attention_b200 import binding as b
from sub_quadratic_attention_b200.workloads import WORKLOADS, custom, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    WORKLOADS["tiny_fp32"],
    custom(1, 4096, 4, 16, 1000, dtype="bf16", name="noalloc_bf16"),
    custom(3, 768, 3, 5, 200, dtype="f32", name="noalloc_mixed_radix_odd_c"),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_regular_entry_point_twice(w):
    d = {k: v.cuda() for k, v in make_inputs(w).items()}
    code = b.SPECTRE_F32 if w.dtype == "f32" else b.SPECTRE_BF16
    y_ref = torch.empty_like(d["x"])
    with b.SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps) as mix:
        mix(d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y=y_ref)
    torch.cuda.synchronize()
    _, tol_y = TOL[w.dtype]
    for _ in range(2):
        y = torch.full_like(d["x"], float("nan"))
        st = b.spectre_mix_run_noalloc_status(w.B, w.L, w.H, w.D, w.F, code, w.eps, d["q"], d["k"],
                                              d["v"], d["x"], d["G"], d["gamma"], d["beta"], y)
        assert st == b.SPECTRE_OK, b.spectre_mix_error_string(st)
        torch.cuda.synchronize()
        err = float((y.double() - y_ref.double()).abs().max())
        assert np.isfinite(err) and err <= tol_y, err


def test_noalloc_refuses_shapes_beyond_the_scratch():
    w = WORKLOADS["bf16_long"]   # about 600 MB of workspace
    q = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    G = torch.zeros(16, dtype=torch.float32, device="cuda")
    st = b.spectre_mix_run_noalloc_status(w.B, w.L, w.H, w.D, w.F, b.SPECTRE_BF16, w.eps,
                                          q, q, q, q, G, G, G, q)
    assert st == b.SPECTRE_ERR_SCRATCH
    assert "scratch" in b.spectre_mix_error_string(st)
