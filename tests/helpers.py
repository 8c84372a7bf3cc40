"""Shared helpers of the GPU tests: run the library on a workload and compare
with the CPU oracle under the parity tolerances.

Tolerances (the stated bar of the path): fp32 inputs -- relative L2 error of
the pre-LayerNorm output out <= 1e-5 and max |y - y_ref| <= 1e-4; bf16 inputs --
relative L2 error of out <= 1e-2 and max |y - y_ref| <= 2e-2, with y_ref the
unrounded fp64 oracle value.
"""
from __future__ import annotations

import numpy as np
import torch

TOL = {"f32": (1e-5, 1e-4), "bf16": (1e-2, 2e-2)}


def to_device(inputs):
    return {k: v.cuda() for k, v in inputs.items()}


def run_library(w, inputs_cpu, debug=True, stream=None, tensor_cores=None, norm=None,
                complex_gate=False, row_tensor_cores=False):
    """Run the CUDA path through the C ABI.  Returns (out_f32 or None, y) on CPU.
    tensor_cores: None keeps the plan's default slice pass, True/False sets it."""
    from sub_quadratic_attention_b200 import binding
    from sub_quadratic_attention_b200.binding import SpectreMix

    d = to_device(inputs_cpu)
    with SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps, tensor_cores=tensor_cores,
                    norm=norm, complex_gate=complex_gate,
                    row_tensor_cores=row_tensor_cores) as mix:
        y = torch.empty_like(d["x"])
        out = torch.empty((w.B, w.L, w.C), dtype=torch.float32, device="cuda") if debug else None
        mix(d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y=y, out=out,
            stream=stream)
        torch.cuda.synchronize()
        assert binding.spectre_mix_device_status(mix.handle) == binding.SPECTRE_OK
    return (out.cpu() if debug else None), y.cpu()


def oracle_full(w, inputs_cpu, norm="post_ln"):
    import oracle

    return oracle.spectre_mix(inputs_cpu["q"], inputs_cpu["k"], inputs_cpu["v"], inputs_cpu["x"],
                              inputs_cpu["G"], inputs_cpu["gamma"], inputs_cpu["beta"],
                              H=w.H, F=w.F, eps=w.eps, norm=norm)


def rel_l2(a: np.ndarray, ref: np.ndarray) -> float:
    num = 0.0
    den = 0.0
    # chunked to bound temporaries on the largest workloads
    a2 = a.reshape(-1)
    r2 = ref.reshape(-1)
    step = 1 << 24
    for i in range(0, a2.shape[0], step):
        d = a2[i:i + step].astype(np.float64) - r2[i:i + step]
        num += float(np.dot(d, d))
        den += float(np.dot(r2[i:i + step], r2[i:i + step]))
    return (num ** 0.5) / max(den ** 0.5, 1e-300)


def max_abs(a: np.ndarray, ref: np.ndarray) -> float:
    a2 = a.reshape(-1)
    r2 = ref.reshape(-1)
    step = 1 << 24
    m = 0.0
    for i in range(0, a2.shape[0], step):
        m = max(m, float(np.max(np.abs(a2[i:i + step].astype(np.float64) - r2[i:i + step]))))
    return m


def y_numpy(y: torch.Tensor) -> np.ndarray:
    return y.float().numpy()


def check_parity(w, out_gpu, y_gpu, out_ref, y_ref):
    tol_out, tol_y = TOL[w.dtype]
    e_out = rel_l2(out_gpu.numpy(), out_ref) if out_gpu is not None else 0.0
    e_y = max_abs(y_numpy(y_gpu), y_ref)
    assert np.isfinite(e_out) and np.isfinite(e_y)
    assert e_out <= tol_out, f"rel-L2(out) {e_out:.3e} > {tol_out:.0e}"
    assert e_y <= tol_y, f"max|dy| {e_y:.3e} > {tol_y:.0e}"
    return e_out, e_y
