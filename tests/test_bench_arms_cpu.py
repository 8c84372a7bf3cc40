"""bench.py's GPU arms run on the CPU against a fake library and fake CUDA
events, to check the JSON line they assemble: the contract's keys, the
roofline and ALU objects, e2e byte counts and the launch count.  The numbers
are the fakes' (every event record advances a clock by 0.1 ms); the real
timings come only from a B200."""
import argparse
import json

import pytest
import torch

import bench
from sub_quadratic_attention_b200 import binding
from sub_quadratic_attention_b200.workloads import DCT_WORKLOADS, WORKLOADS

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "e2e", "gpu_launches", "roofline",
        "cpu_baseline", "clocks"}


class FakeEvent:
    clock = 0.0

    def __init__(self, enable_timing=False):
        self.ts = None

    def record(self, stream=None):
        FakeEvent.clock += 0.1
        self.ts = FakeEvent.clock

    def elapsed_time(self, other):
        return other.ts - self.ts


class FakeSpectreMix:
    def __init__(self, B, L, H, D, F, dtype, eps, tensor_cores=None, norm=None,
                 complex_gate=False, block_len=None):
        self.handle = 1
        self.plan = (16, 4096, 9, 16, 5)      # R, M, slices, channels per wave, launches
        self.slice_pass = "cuda_cores"

    def close(self):
        pass


class FakeDctMix:
    def __init__(self, d, dtype, eps):
        self.handle = 2

    def close(self):
        pass


def _profiled(h, q, k, v, x, G, gamma, beta, y, events, stream):
    for e in events:
        e.record(stream)


@pytest.fixture
def fake_gpu(monkeypatch):
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(binding, "SpectreMix", FakeSpectreMix)
    monkeypatch.setattr(binding, "DctMix", FakeDctMix)
    noop = lambda *a, **k: None
    for name in ("spectre_mix_run", "spectre_mix_run_host", "dct_mix_run", "dct_mix_run_host"):
        monkeypatch.setattr(binding, name, noop)
    monkeypatch.setattr(binding, "spectre_mix_run_profiled", _profiled)


def _args(**kw):
    a = dict(steps=2, warmup=3, cpu_seconds=0.2, no_cpu_baseline=False, norm="post_ln",
             complex_gate=False, cuda_core_slices=False, block_len=0)
    a.update(kw)
    return argparse.Namespace(**a)


def _line(capsys):
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_spectral_arm_line(fake_gpu, capsys):
    w = WORKLOADS["tiny_fp32"]
    bench.native_arm(_args(), w, 0, 1, 0, device=torch.device("cpu"))
    d = _line(capsys)
    assert KEYS <= set(d)
    assert d["gpu_launches"] == 5 * 2 and d["n_gpus"] == 1 and d["scaling"] == "weak"
    assert abs(d["ms_per_step"] - 0.1) < 1e-9                      # one fake event tick per step
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["kernel"] in ("rows_fwd", "slices", "rows_inv_ln")
    assert r["alu"]["bound"] == "alu" and r["alu"]["method_flops"] == bench.method_flops(w)
    assert r["path"]["algorithmic_bytes"] == w.algorithmic_bytes()
    n = w.B * w.L * w.C
    assert d["e2e"]["h2d_bytes_per_step"] == 4 * n * 4 + w.H * (w.L // 2 + 1) * 4 + 2 * w.C * 4
    assert d["e2e"]["d2h_bytes_per_step"] == n * 4
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] > 0


def test_spectral_arm_block_and_complex_gate(fake_gpu, capsys):
    w = WORKLOADS["tiny_fp32"]
    bench.native_arm(_args(block_len=64, complex_gate=True, no_cpu_baseline=True), w, 0, 1, 0,
                     device=torch.device("cpu"))
    d = _line(capsys)
    assert d["config"]["block_len"] == 64 and d["roofline"]["plan"]["gate"] == "complex"
    # the gate the plan reads: [H, 64/2 + 1] (re, im) pairs
    assert d["e2e"]["h2d_bytes_per_step"] == 4 * 256 * 16 * 4 + 1 * 33 * 2 * 4 + 2 * 16 * 4


def test_dct_arm_line(fake_gpu, capsys):
    w = DCT_WORKLOADS["dct_tiny_fp32"]
    bench.dct_arm(_args(), w, 0, 1, 0, device=torch.device("cpu"))
    d = _line(capsys)
    assert KEYS <= set(d)
    assert d["gpu_launches"] == 2 and d["config"]["d"] == 64
    r = d["roofline"]
    assert r["kernel"] == "dct_mix" and r["units_per_launch"] == w.T
    assert abs(r["achieved"] - w.algorithmic_bytes() / 0.1e-3 / 1e9) < 0.01
    assert r["alu"]["method_flops"] == bench.dct_method_flops(w)
    assert d["e2e"]["h2d_bytes_per_step"] == w.T * 64 * 4 + 3 * 64 * 4
    assert d["e2e"]["d2h_bytes_per_step"] == w.T * 64 * 4 + 5 * w.T
