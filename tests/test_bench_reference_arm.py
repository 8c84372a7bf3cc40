"""bench.py's reference arm (the fp64 oracle on the host cores) end to end on
the CPU: one JSON line carrying the contract's keys, for the spectral mix and
for the DCT mix."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline",
        "e2e"}


@pytest.mark.parametrize("workload", ["tiny_fp32", "dct_tiny_fp32"])
def test_reference_arm_prints_one_contract_line(workload):
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", workload,
                          "--steps", "2", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == workload
    assert d["steps"] == 2 and d["warmup"] == 3


def test_warmup_below_three_is_refused():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--warmup", "2"],
                         cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert out.returncode != 0
