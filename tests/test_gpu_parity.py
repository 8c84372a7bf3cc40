"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Element-by-element comparisons on the same seeded inputs: every workload at its
full size (in the launch configuration the benchmark times), a sweep of small
shapes spanning several tiles with ragged tails, and the degenerate cases of the
method (F = 1, zero gate, no truncation, odd channel counts, one token block).
"""
import numpy as np
import pytest
import torch

from helpers import TOL, check_parity, oracle_full, run_library
from sub_quadratic_attention_b200.workloads import WORKLOADS, custom, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny_fp32", "fp32_mid", "bf16_long", "bf16_mixed_radix",
                                  "bf16_very_long"])
def test_workload_full_size(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    out, y = run_library(w, inp)
    out_ref, y_ref = oracle_full(w, inp)
    e_out, e_y = check_parity(w, out, y, out_ref, y_ref)
    print(f"{name}: rel-L2(out)={e_out:.3e} max|dy|={e_y:.3e}")


SWEEP = [
    # (B, L, H, D, F)
    (1, 8, 1, 2, 5), (2, 12, 1, 3, 7), (1, 16, 2, 2, 9), (3, 24, 1, 5, 4), (1, 32, 1, 4, 17),
    (1, 48, 3, 5, 25), (2, 64, 2, 3, 1), (1, 96, 1, 7, 30), (1, 128, 4, 4, 65), (2, 192, 2, 8, 50),
    (1, 256, 1, 16, 129), (1, 384, 3, 3, 100), (1, 512, 2, 32, 257), (1, 768, 1, 24, 385),
    (2, 1024, 2, 16, 200), (1, 1536, 3, 10, 769), (1, 2048, 1, 64, 1025), (1, 3072, 2, 6, 1000),
    (1, 4096, 4, 16, 2049), (1, 6144, 1, 40, 3073), (1, 8192, 2, 8, 1024), (1, 12288, 1, 66, 6145),
    (1, 16384, 1, 32, 8193), (1, 32768, 1, 16, 4000), (1, 65536, 1, 8, 32769),
    (1, 3 * 2 ** 16, 1, 4, 1234), (1, 2 ** 18, 1, 4, 2 ** 17 + 1), (1, 2 ** 19, 1, 2, 5000),
    (1, 3 * 2 ** 17, 1, 2, 3 * 2 ** 16 + 1),
]


@pytest.mark.parametrize("B,L,H,D,F", SWEEP)
def test_shape_sweep_fp32(B, L, H, D, F):
    w = custom(B, L, H, D, F, dtype="f32")
    inp = make_inputs(w)
    out, y = run_library(w, inp)
    out_ref, y_ref = oracle_full(w, inp)
    check_parity(w, out, y, out_ref, y_ref)


@pytest.mark.parametrize("B,L,H,D,F", [(1, 256, 1, 16, 40), (2, 12288, 2, 8, 6145),
                                       (1, 65536, 2, 8, 8192), (1, 3072, 3, 5, 1),
                                       (1, 4096, 7, 72, 1000), (3, 4096, 4, 128, 2049),
                                       (1, 65536, 7, 72, 8192)])
def test_shape_sweep_bf16(B, L, H, D, F):
    """bf16 shapes across the kernel variants: C = 504 (dead lanes in the
    prefetching inverse pass; at L = 65536 channel chunks of 128, 128, 128 and
    120, the last not a multiple of 64, so the prefetching and the plain row
    pass both run in one step, beside the tensor-core slice pass) and C = 512
    with B = 3 (the persistent passes crossing batch boundaries)."""
    w = custom(B, L, H, D, F, dtype="bf16")
    inp = make_inputs(w)
    out, y = run_library(w, inp)
    out_ref, y_ref = oracle_full(w, inp)
    check_parity(w, out, y, out_ref, y_ref)


def _expected_slice_pass(w):
    """The documented range of the tensor-core slice pass: bf16 I/O, L = 65536
    (R = 16, M = 4096 = 64 x 64), and no slice f1 with more than two live k2
    groups, group g covering bins f = f1 + 16 (k1 + 64 k2), k2 in [8g, 8g + 8)."""
    if w.dtype != "bf16" or w.L != 65536:
        return "cuda_cores"
    R = 16

    def live(g, f1):
        return f1 + R * 512 * g < w.F or f1 + R * (63 + 64 * (8 * g + 7)) > w.L - w.F

    worst = max(sum(live(g, f1) for g in range(8)) for f1 in range(R // 2 + 1))
    return "tensor_cores" if worst <= 2 else "cuda_cores"


@pytest.mark.parametrize("case", ["bf16_long", (1, 65536, 2, 8, 8192), (2, 65536, 3, 5, 1000),
                                  (1, 65536, 3, 5, 1), (1, 65536, 1, 64, 4000),
                                  (1, 65536, 7, 72, 8192), (2, 65536, 3, 5, 32769)])
def test_tensor_core_variant(case):
    """The slice pass on the tensor cores (two DFT-64 MMA passes per 4096-point
    transform, fp16 operands, fp32 accumulation) meets the bf16 bar as well:
    odd channel counts (a dead half block), F = 1 (slices with no live bin),
    and a shape outside its range (no truncation) that keeps the CUDA-core
    slice pass."""
    from sub_quadratic_attention_b200.binding import SpectreMix

    w = WORKLOADS[case] if isinstance(case, str) else custom(*case, dtype="bf16")
    with SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps, tensor_cores=True) as mix:
        assert mix.slice_pass == _expected_slice_pass(w)
    inp = make_inputs(w)
    out, y = run_library(w, inp, tensor_cores=True)
    out_ref, y_ref = oracle_full(w, inp)
    e_out, e_y = check_parity(w, out, y, out_ref, y_ref)
    print(f"tensor cores {w.name}: rel-L2(out)={e_out:.3e} max|dy|={e_y:.3e}")


@pytest.mark.parametrize("name", ["bf16_long", "bf16_mixed_radix"])
def test_cuda_core_slice_pass_bf16(name):
    """The CUDA-core slice pass (the option switched off) on the bf16 workloads."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    out, y = run_library(w, inp, tensor_cores=False)
    out_ref, y_ref = oracle_full(w, inp)
    e_out, e_y = check_parity(w, out, y, out_ref, y_ref)
    print(f"cuda cores {name}: rel-L2(out)={e_out:.3e} max|dy|={e_y:.3e}")


def test_zero_gate_gives_layernorm_of_x():
    w = custom(2, 4096, 4, 16, 2049, dtype="f32")
    inp = make_inputs(w)
    inp["G"].zero_()
    out, y = run_library(w, inp)
    assert torch.count_nonzero(out) == 0
    ref = torch.nn.functional.layer_norm(inp["x"].double(), (w.C,), inp["gamma"].double(),
                                         inp["beta"].double(), eps=float(np.float32(w.eps)))
    assert float((y.double() - ref).abs().max()) < 1e-5


def test_repeat_runs_are_bitwise_identical():
    w = WORKLOADS["bf16_long"]
    inp = make_inputs(w)
    out1, y1 = run_library(w, inp)
    out2, y2 = run_library(w, inp)
    assert torch.equal(out1, out2) and torch.equal(y1, y2)


def test_host_buffer_entry_point_matches_device_entry_point():
    from sub_quadratic_attention_b200.binding import SpectreMix

    w = WORKLOADS["fp32_mid"]
    inp = make_inputs(w)
    _, y_dev = run_library(w, inp, debug=False)
    pinned = {k: v.pin_memory() for k, v in inp.items()}
    y_host = torch.empty_like(pinned["x"]).pin_memory()
    with SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps) as mix:
        for _ in range(2):
            mix.run_host(pinned["q"], pinned["k"], pinned["v"], pinned["x"], pinned["G"],
                         pinned["gamma"], pinned["beta"], y_host)
            torch.cuda.synchronize()
            assert torch.equal(y_host, y_dev)


def test_run_rejects_misaligned_and_null_pointers():
    from sub_quadratic_attention_b200 import binding as b

    w = WORKLOADS["tiny_fp32"]
    d = {k: v.cuda() for k, v in make_inputs(w).items()}
    y = torch.empty_like(d["x"])
    h = b.spectre_mix_create(w.B, w.L, w.H, w.D, w.F, b.SPECTRE_F32, w.eps)
    try:
        args = [d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y]
        assert b.spectre_mix_run_status(h, *args) == b.SPECTRE_OK
        bad = list(args)
        bad[0] = d["q"].data_ptr() + 4
        assert b.spectre_mix_run_status(h, *bad) == b.SPECTRE_ERR_ALIGN
        bad = list(args)
        bad[7] = 0
        assert b.spectre_mix_run_status(h, *bad) == b.SPECTRE_ERR_ARG
        torch.cuda.synchronize()
    finally:
        b.spectre_mix_destroy(h)


@pytest.mark.parametrize("norm", ["pre_ln", "post_rms", "pre_rms"])
@pytest.mark.parametrize("case", ["bf16_long", "fp32_mid", (2, 4096, 3, 5, 700),
                                  (1, 524288, 1, 4, 5000)])
def test_norm_variants(norm, case):
    """The norm-order and RMSNorm variants (walk-through §3.3) in every inverse
    kernel: the prefetching one (bf16_long, with the tensor-core slice pass),
    the register-resident one (fp32_mid; an odd channel count in bf16) and
    the shared-memory one (R = 64, fp32)."""
    if isinstance(case, str):
        w = WORKLOADS[case]
    else:
        w = custom(*case, dtype="bf16" if case[1] == 4096 else "f32")
    inp = make_inputs(w)
    out, y = run_library(w, inp, norm=norm)
    out_ref, y_ref = oracle_full(w, inp, norm=norm)
    e_out, e_y = check_parity(w, out, y, out_ref, y_ref)
    print(f"{norm} {w.name}: rel-L2(out)={e_out:.3e} max|dy|={e_y:.3e}")


def _complex_gate(G, seed):
    """G with a seeded phase in (-pi, pi] per bin: a complex64 gate."""
    th = (torch.rand(G.shape, generator=torch.Generator().manual_seed(seed)) * 2 - 1) * np.pi
    return torch.polar(G.float(), th.float())


@pytest.mark.parametrize("case", ["bf16_long", "fp32_mid", (2, 12288, 2, 8, 6145),
                                  (1, 524288, 1, 4, 5000)])
def test_complex_gate(case):
    """A complex gate (relative-position phase) in both slice passes: the
    tensor-core one (bf16_long), the CUDA-core one in fp32 and in bf16 with a
    mixed-radix length, and R = 64."""
    if isinstance(case, str):
        w = WORKLOADS[case]
    else:
        w = custom(*case, dtype="bf16" if case[1] == 12288 else "f32")
    inp = make_inputs(w)
    inp["G"] = _complex_gate(inp["G"], seed=w.L)
    out, y = run_library(w, inp, complex_gate=True)
    out_ref, y_ref = oracle_full(w, inp)
    e_out, e_y = check_parity(w, out, y, out_ref, y_ref)
    print(f"complex gate {w.name}: rel-L2(out)={e_out:.3e} max|dy|={e_y:.3e}")


@pytest.mark.parametrize("B,L,H,D,n,F,dtype", [
    (2, 16384, 4, 32, 4096, 1000, "bf16"),
    (1, 131072, 2, 32, 65536, 8192, "bf16"),     # tensor-core slice pass inside each block
    (1, 3 * 12288, 2, 8, 12288, 6145, "f32"),    # mixed-radix blocks
    (3, 1024, 1, 16, 256, 129, "f32"),
    (1, 4096, 2, 16, 4096, 2049, "f32"),         # one block: the plain mix
])
def test_blockwise_mode(B, L, H, D, n, F, dtype):
    """Blockwise mode: the library, planned on [B, L, C] with block_len = n,
    against the oracle run on the same values as B L / n sequences of n
    tokens with the block's gate [H, n/2 + 1]."""
    from sub_quadratic_attention_b200 import binding
    from sub_quadratic_attention_b200.binding import SpectreMix

    wb = custom(B * (L // n), n, H, D, F, dtype=dtype)
    inp = make_inputs(wb)
    C = H * D
    d = {k: t.cuda() for k, t in inp.items()}
    with SpectreMix(B, L, H, D, F, dtype, wb.eps, block_len=n) as mix:
        y = torch.empty((B, L, C), dtype=d["x"].dtype, device="cuda")
        out = torch.empty((B, L, C), dtype=torch.float32, device="cuda")
        mix(d["q"].view(B, L, C), d["k"].view(B, L, C), d["v"].view(B, L, C),
            d["x"].view(B, L, C), d["G"], d["gamma"], d["beta"], y=y, out=out)
        torch.cuda.synchronize()
        assert binding.spectre_mix_device_status(mix.handle) == binding.SPECTRE_OK
        assert mix.slice_pass == _expected_slice_pass(wb)
    out_ref, y_ref = oracle_full(wb, inp)
    e_out, e_y = check_parity(wb, out.cpu().view(wb.B, n, C), y.cpu().view(wb.B, n, C),
                              out_ref, y_ref)
    print(f"block mode {B}x{L} n={n}: rel-L2(out)={e_out:.3e} max|dy|={e_y:.3e}")


@pytest.mark.parametrize("case", ["bf16_long", "mixed_radix_c128", "batch3_c192"])
def test_row_pass_on_tensor_cores(case):
    """SPECTRE_OPT_ROW_TENSOR_CORES: the row pass as TMA-fed bf16 MMAs (DFT-16
    matrix split into two bf16 terms) gives the oracle's result within the bf16
    bar, at full size and on a mixed-radix plan with B > 1."""
    w = {"bf16_long": WORKLOADS["bf16_long"],
         "mixed_radix_c128": custom(2, 12288, 2, 64, 6145, dtype="bf16"),
         "batch3_c192": custom(3, 4096, 3, 64, 1000, dtype="bf16")}[case]
    inp = make_inputs(w)
    out, y = run_library(w, inp, row_tensor_cores=True)
    out_ref, y_ref = oracle_full(w, inp)
    e_out, e_y = check_parity(w, out, y, out_ref, y_ref)
    print(f"{case}: rel-L2(out)={e_out:.3e} max|dy|={e_y:.3e}")


@pytest.mark.parametrize("case,dtype", [((1, 2 ** 20, 1, 8, 65536), "bf16"), ((1, 2 ** 20, 1, 4, 100000), "f32"),
                                        ((1, 786432, 1, 4, 50000), "bf16"), ((1, 2 ** 20, 1, 2, 2 ** 19 + 1), "f32")])
def test_longest_slices_parked_product(case, dtype):
    """Slices of 16384 and 12288 points (R = 64), whose running product is
    parked in the q row of fp32 A: truncations whose edge falls on a row of
    bins (F = 65536) or inside one (F = 100000), a 12288-point slice, and
    every bin kept (F = L/2 + 1)."""
    w = custom(*case, dtype=dtype)
    inp = make_inputs(w)
    out, y = run_library(w, inp)
    out_ref, y_ref = oracle_full(w, inp)
    e_out, e_y = check_parity(w, out, y, out_ref, y_ref)
    print(f"longest slices {w.name} {dtype}: rel-L2(out)={e_out:.3e} max|dy|={e_y:.3e}")


def test_widest_channels_r16():
    """C = 3616, the widest plan with R = 16 (the inverse pass's shared-memory
    variant holds 16 token rows of all channels: 227 KiB), against the oracle."""
    w = custom(1, 4096, 4, 904, 2049, dtype="bf16")
    inp = make_inputs(w)
    out, y = run_library(w, inp)
    out_ref, y_ref = oracle_full(w, inp)
    e_out, e_y = check_parity(w, out, y, out_ref, y_ref)
    print(f"widest R=16 {w.name}: rel-L2(out)={e_out:.3e} max|dy|={e_y:.3e}")


def test_widest_channels_r64_zero_gate():
    """C = 864, the widest plan with R = 64 (L = 2^19), checked by a property
    that holds at any size: with G = 0 the mix is zero and y = LayerNorm(x).
    Seeded inputs are drawn on the device (4 x 0.9 GB)."""
    from sub_quadratic_attention_b200.binding import SpectreMix

    B, L, H, D, F = 1, 2 ** 19, 1, 864, 5000
    C = H * D
    g = torch.Generator(device="cuda").manual_seed(864)
    q, k, v, x = (torch.randn(B, L, C, generator=g, device="cuda").bfloat16() for _ in range(4))
    G = torch.zeros(H, L // 2 + 1, device="cuda")
    gamma = 1.0 + 0.1 * torch.randn(C, generator=g, device="cuda")
    beta = 0.1 * torch.randn(C, generator=g, device="cuda")
    with SpectreMix(B, L, H, D, F, "bf16") as mix:
        assert mix.plan[0] == 64
        y = mix(q, k, v, x, G, gamma, beta)
        torch.cuda.synchronize()
    ref = torch.nn.functional.layer_norm(x.float(), (C,), gamma, beta, eps=1e-5)
    err = float((y.float() - ref).abs().max())
    assert err <= 2e-2, err
    print(f"widest R=64 zero gate: max|dy|={err:.3e}")
