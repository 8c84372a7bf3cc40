"""Parity of the DCT mix (through the C ABI) with the fp64 CPU oracle.

Element by element on small shapes (every supported d, odd token counts, both
dtypes); on sampled tokens of the two full-size workloads in the launch
configuration the benchmark times; and the degenerate rows (all zero, constant,
a single cosine).  Tolerances, from the fp32 arithmetic:
  mix (before the residual): rel-L2 <= 1e-5;
  y: max abs error <= 1e-4 (fp32 y) or 2e-2 (bf16 y, which includes the
     final rounding's half ulp);
  H: abs error <= 1e-4;
  route: exactly (H_gpu <= tau), the decision taken in the kernel's fp32, and
     equal to the oracle's wherever the oracle's H is more than 1e-4 from tau.
"""
import numpy as np
import pytest
import torch

import oracle
from sub_quadratic_attention_b200.workloads import (DCT_WORKLOADS, dct_custom,
                                                     make_dct_inputs)

pytestmark = pytest.mark.gpu

TOL_Y = {"f32": 1e-4, "bf16": 2e-2}
TOL_MIX = 1e-5
TOL_H = 1e-4


def _run(w, inp, debug=True, tau=None):
    from sub_quadratic_attention_b200 import binding

    tau = w.tau if tau is None else tau
    d = {k: v.cuda() for k, v in inp.items()}
    with binding.DctMix(w.d, w.dtype, w.eps) as m:
        mix = torch.empty(d["x"].shape, dtype=torch.float32, device="cuda") if debug else None
        y, H, route = m(d["x"], d["w"], d["gamma"], d["beta"], tau, mix_out=mix)
        torch.cuda.synchronize()
    return {"y": y.cpu(), "H": H.cpu(), "route": route.cpu(),
            "mix": mix.cpu() if debug else None}


def _check(w, got, ref, tau=None, sel=None):
    tau = w.tau if tau is None else tau
    sel = slice(None) if sel is None else sel
    y = got["y"].float().reshape(-1, w.d)[sel].numpy().astype(np.float64)
    ey = np.abs(y - ref["y"].reshape(-1, w.d)).max() if y.size else 0.0
    assert ey <= TOL_Y[w.dtype], f"max|dy| {ey:.3e}"
    Hg = got["H"].reshape(-1)[sel].numpy()
    Hr = ref["H"].reshape(-1)
    eh = np.abs(Hg.astype(np.float64) - Hr).max() if Hg.size else 0.0
    assert eh <= TOL_H, f"max|dH| {eh:.3e}"
    rg = got["route"].reshape(-1)[sel].numpy()
    assert np.array_equal(rg, (Hg <= np.float32(tau)).astype(np.uint8))
    far = np.abs(Hr - tau) > TOL_H
    assert np.array_equal(rg[far], ref["route"].reshape(-1)[far])
    em = 0.0
    if got["mix"] is not None:
        mg = got["mix"].reshape(-1, w.d)[sel].numpy().astype(np.float64)
        mr = ref["mix"].reshape(-1, w.d)
        em = np.linalg.norm(mg - mr) / max(np.linalg.norm(mr), 1e-300)
        assert em <= TOL_MIX, f"rel-L2(mix) {em:.3e}"
    return ey, eh, em


def _oracle(w, inp, tau=None, rows=None):
    x = inp["x"].reshape(-1, w.d)
    if rows is not None:
        x = x[rows]
    return oracle.dct_mix(x, inp["w"], inp["gamma"], inp["beta"], eps=w.eps,
                          tau=w.tau if tau is None else tau)


@pytest.mark.parametrize("B,L,d,dtype", [
    (1, 37, 64, "f32"), (1, 1, 128, "f32"), (2, 33, 256, "f32"), (1, 64, 512, "f32"),
    (1, 9, 1024, "f32"), (3, 50, 256, "bf16"), (1, 31, 1024, "bf16"), (2, 20, 64, "bf16"),
    (1, 300, 128, "bf16"), (1, 4097, 256, "f32"),
])
def test_dct_parity_small(B, L, d, dtype):
    w = dct_custom(B, L, d, dtype, tau=0.75 if d < 1024 else 0.8954)
    inp = make_dct_inputs(w)
    got = _run(w, inp)
    ey, eh, em = _check(w, got, _oracle(w, inp))
    print(f"dct {B}x{L} d={d} {dtype}: max|dy|={ey:.2e} max|dH|={eh:.2e} rel-L2(mix)={em:.2e}")


@pytest.mark.parametrize("name", ["dct_tiny_fp32", "dct_d256", "dct_d1024"])
def test_dct_workload_full_size_sampled(name):
    """The whole workload on the GPU in the benchmark's launch configuration
    (no debug output); the oracle on 768 sampled tokens, the first and the
    last included."""
    w = DCT_WORKLOADS[name]
    inp = make_dct_inputs(w)
    got = _run(w, inp, debug=False)
    g = torch.Generator().manual_seed(7)
    rows = torch.unique(torch.cat([torch.tensor([0, w.T - 1]),
                                   torch.randint(0, w.T, (766,), generator=g)])).numpy()
    ey, eh, _ = _check(w, got, _oracle(w, inp, rows=rows), sel=rows)
    frac = got["route"].float().mean().item()
    print(f"{name}: max|dy|={ey:.2e} max|dH|={eh:.2e} routed={frac:.3f}")


@pytest.mark.parametrize("d", [64, 256, 1024])
def test_dct_degenerate_rows(d):
    """Zero rows (H = 0, route 1, y = beta), constant rows (DC only: H = 0),
    and a single cosine (one coefficient), in an odd number of rows."""
    w = dct_custom(1, 5, d, "f32", tau=0.0)
    inp = make_dct_inputs(w)
    n = torch.arange(d, dtype=torch.float64)
    x = torch.zeros(1, 5, d)
    x[0, 1] = 0.5
    x[0, 2] = torch.cos(torch.pi * (2 * n + 1) * 3 / (2 * d)).float()
    x[0, 3] = torch.randn(d, generator=torch.Generator().manual_seed(d))
    inp["x"] = x
    got = _run(w, inp)
    ref = _oracle(w, inp)
    _check(w, got, ref)
    assert got["H"][0, 0].item() == 0.0 and got["route"][0, 0].item() == 1
    assert torch.allclose(got["y"][0, 0], inp["beta"], atol=1e-6)
    assert got["route"][0, 4].item() == 1                      # the last (odd) row is zero too
    assert abs(got["H"][0, 1].item()) < 1e-4 and abs(got["H"][0, 2].item()) < 1e-4


def test_dct_empty_input_is_a_no_op():
    from sub_quadratic_attention_b200 import binding

    with binding.DctMix(256, "bf16") as m:
        x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
        y, H, route = m(x, torch.ones(256, device="cuda"), torch.ones(256, device="cuda"),
                        torch.zeros(256, device="cuda"), 0.5)
        torch.cuda.synchronize()
    assert y.numel() == 0 and H.numel() == 0 and route.numel() == 0


def test_dct_host_entry_point_matches_device_entry_point():
    from sub_quadratic_attention_b200 import binding

    w = dct_custom(2, 77, 512, "bf16")
    inp = make_dct_inputs(w)
    dev = _run(w, inp, debug=False)
    pinned = {k: v.pin_memory() for k, v in inp.items()}
    y = torch.empty_like(pinned["x"]).pin_memory()
    H = torch.empty(w.B, w.L).pin_memory()
    route = torch.empty(w.B, w.L, dtype=torch.uint8).pin_memory()
    with binding.DctMix(w.d, w.dtype, w.eps) as m:
        m.run_host(pinned["x"], pinned["w"], pinned["gamma"], pinned["beta"], w.tau, y, H, route)
        torch.cuda.synchronize()
    assert torch.equal(y, dev["y"]) and torch.equal(H, dev["H"]) and torch.equal(route, dev["route"])
