"""Run the mix on a named workload a few times, for external profilers.

    python -m sub_quadratic_attention_b200.profile_run --workload bf16_long --warmup 2 --steps 3

No timing: each step is one ``spectre_mix_run`` (three kernel launches) on
inputs resident in device memory, followed by a device synchronise.  Profilers
select launches with their own skip/count options (3 launches per step).
"""
from __future__ import annotations

import argparse

import torch

from sub_quadratic_attention_b200 import binding
from sub_quadratic_attention_b200.workloads import WORKLOADS, make_inputs


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="bf16_long", choices=sorted(WORKLOADS))
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--cuda-core-slices", action="store_true",
                    help="force the CUDA-core slice pass (default: tensor cores where the plan "
                         "allows)")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    d = {k: v.cuda() for k, v in make_inputs(w).items()}
    y = torch.empty_like(d["x"])
    with binding.SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps,
                            tensor_cores=False if args.cuda_core_slices else None) as mix:
        for _ in range(args.warmup + args.steps):
            mix(d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y=y)
            torch.cuda.synchronize()
        print(f"{w.name}: {args.warmup + args.steps} steps, plan R,M,slices = {mix.plan}, "
              f"slice pass {mix.slice_pass}")


if __name__ == "__main__":
    main()
