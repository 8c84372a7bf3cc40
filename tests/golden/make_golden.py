"""Write the oracle regression fixtures in this folder.

Calls only the CPU oracle (``oracle/``) on the seeded workloads.  The values are
oracle outputs, not figures printed on the pages: the pages print no worked
numeric example of the mixer.  They pin the oracle and the input recipe against
silent drift; the oracle's correctness itself is pinned by
``tests/test_oracle_pins.py``.

Usage: python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from sub_quadratic_attention_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

TOKENS = {"tiny_fp32": [0, 1, 77, 128, 255], "fp32_mid": [0, 1, 2048, 4095]}


def main():
    for name, toks in TOKENS.items():
        w = WORKLOADS[name]
        t = make_inputs(w)
        out, y = oracle.spectre_mix(t["q"], t["k"], t["v"], t["x"], t["G"], t["gamma"],
                                    t["beta"], H=w.H, F=w.F, eps=w.eps, tokens=toks)
        chans = list(range(0, w.C, max(1, w.C // 8)))
        doc = {
            "workload": name,
            "source": "oracle/spectre_oracle.c via tests/golden/make_golden.py",
            "tokens": toks,
            "channels": chans,
            "out": out[:, :, chans].tolist(),
            "y": y[:, :, chans].tolist(),
        }
        with open(os.path.join(HERE, f"{name}_oracle.json"), "w") as f:
            json.dump(doc, f, indent=1)
        print("wrote", name)


if __name__ == "__main__":
    main()
