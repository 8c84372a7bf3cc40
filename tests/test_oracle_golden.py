"""Regression: the oracle and the seeded input recipe still reproduce the
stored fixtures written by ``tests/golden/make_golden.py`` (oracle only)."""
import json
import os

import numpy as np
import pytest

import oracle
from sub_quadratic_attention_b200.workloads import WORKLOADS, make_inputs

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("name", ["tiny_fp32", "fp32_mid"])
def test_oracle_reproduces_fixture(name):
    with open(os.path.join(HERE, f"{name}_oracle.json")) as f:
        doc = json.load(f)
    w = WORKLOADS[name]
    t = make_inputs(w)
    out, y = oracle.spectre_mix(t["q"], t["k"], t["v"], t["x"], t["G"], t["gamma"], t["beta"],
                                H=w.H, F=w.F, eps=w.eps, tokens=doc["tokens"])
    ch = doc["channels"]
    assert np.allclose(out[:, :, ch], np.array(doc["out"]), rtol=1e-12, atol=1e-15)
    assert np.allclose(y[:, :, ch], np.array(doc["y"]), rtol=1e-12, atol=1e-12)
