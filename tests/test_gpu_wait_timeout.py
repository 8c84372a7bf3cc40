"""The bounded tensor-core wait, made to run out on the GPU without a fault.

With the test option SPECTRE_OPT_TEST_WAIT_TIMEOUT, block 0 of the tensor-core
slice pass issues no MMA and waits only a few 1 ms polls on its MMA barrier.
Nothing is in flight, so the wait simply gives up: the block records the
timeout in the device error word, sets the scales of its unfinished slices to
NaN (so y is NaN), releases its tensor memory and returns.  The context stays
usable: the status is reported once, then cleared, and the next normal run of
the same plan is parity-green against the oracle.
"""
import pytest
import torch

from helpers import check_parity, oracle_full
from sub_quadratic_attention_b200 import binding as b
from sub_quadratic_attention_b200.workloads import custom, make_inputs

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_poisons_y_and_recovers():
    w = custom(1, 65536, 1, 16, 8192, dtype="bf16", name="wait_timeout")
    inp = make_inputs(w)
    d = {k: v.cuda() for k, v in inp.items()}
    with b.SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps) as mix:
        assert mix.slice_pass == "tensor_cores"
        b.spectre_mix_set_option(mix.handle, b.SPECTRE_OPT_TEST_WAIT_TIMEOUT, 1)
        y = torch.zeros_like(d["x"])
        mix(d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y=y)
        assert b.spectre_mix_device_status(mix.handle) == b.SPECTRE_ERR_TIMEOUT
        assert torch.isnan(y.float()).all()
        assert b.spectre_mix_device_status(mix.handle) == b.SPECTRE_OK   # cleared

        b.spectre_mix_set_option(mix.handle, b.SPECTRE_OPT_TEST_WAIT_TIMEOUT, 0)
        out = torch.empty((w.B, w.L, w.C), dtype=torch.float32, device="cuda")
        mix(d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y=y, out=out)
        assert b.spectre_mix_device_status(mix.handle) == b.SPECTRE_OK
    out_ref, y_ref = oracle_full(w, inp)
    check_parity(w, out.cpu(), y.cpu(), out_ref, y_ref)


def test_wait_timeout_option_is_validated():
    with b.SpectreMix(1, 256, 1, 16, 129, "f32") as mix:
        with pytest.raises(b.SpectreMixError):
            b.spectre_mix_set_option(mix.handle, b.SPECTRE_OPT_TEST_WAIT_TIMEOUT, 2)
        # no effect on a plan with the CUDA-core slice pass
        b.spectre_mix_set_option(mix.handle, b.SPECTRE_OPT_TEST_WAIT_TIMEOUT, 1)
        assert mix.slice_pass == "cuda_cores"
