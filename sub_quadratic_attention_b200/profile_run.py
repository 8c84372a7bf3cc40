"""Run the mix on a named workload a few times, for external profilers.

    python -m sub_quadratic_attention_b200.profile_run --workload bf16_long --warmup 2 --steps 3
    python -m sub_quadratic_attention_b200.profile_run --workload bf16_very_long --heads 1 --steps 1

No timing: each step is one ``spectre_mix_run`` on inputs resident in device
memory, followed by a device synchronise.  ``--heads`` (and ``--batch``)
shrink a workload to fewer heads (batch rows) with the same kernels and launch
shapes per channel, for captures that must stay small.  ``--workload dct_*``
runs the DCT mix instead.  Profilers select launches with their own
skip/count options.
"""
from __future__ import annotations

import argparse

import torch

from sub_quadratic_attention_b200 import binding
from sub_quadratic_attention_b200.workloads import (DCT_WORKLOADS, WORKLOADS, custom, make_dct_inputs,
                                                    make_inputs)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="bf16_long", choices=sorted(WORKLOADS) + sorted(DCT_WORKLOADS))
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--heads", type=int, default=0, help="run with this many heads instead")
    ap.add_argument("--batch", type=int, default=0, help="run with this many batch rows instead")
    ap.add_argument("--cuda-core-slices", action="store_true",
                    help="force the CUDA-core slice pass (default: tensor cores where the plan "
                         "allows)")
    ap.add_argument("--row-tensor-cores", action="store_true",
                    help="the row pass on the tensor cores (plan option)")
    args = ap.parse_args()
    if args.workload in DCT_WORKLOADS:
        w = DCT_WORKLOADS[args.workload]
        d = {k: v.cuda() for k, v in make_dct_inputs(w).items()}
        with binding.DctMix(w.d, w.dtype, w.eps) as m:
            for _ in range(args.warmup + args.steps):
                m(d["x"], d["w"], d["gamma"], d["beta"], w.tau)
                torch.cuda.synchronize()
        print(f"{w.name}: {args.warmup + args.steps} steps")
        return
    w = WORKLOADS[args.workload]
    if args.heads or args.batch:
        w = custom(args.batch or w.B, w.L, args.heads or w.H, w.D, w.F, dtype=w.dtype,
                   qkv_scale=w.qkv_scale, x_scale=w.x_scale, gate=w.gate, gamma=w.gamma,
                   beta=w.beta, name=f"{w.name}_small", index=w.index)
    d = {k: v.cuda() for k, v in make_inputs(w).items()}
    y = torch.empty_like(d["x"])
    with binding.SpectreMix(w.B, w.L, w.H, w.D, w.F, w.dtype, w.eps,
                            tensor_cores=False if args.cuda_core_slices else None,
                            row_tensor_cores=args.row_tensor_cores) as mix:
        for _ in range(args.warmup + args.steps):
            mix(d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y=y)
            torch.cuda.synchronize()
        print(f"{w.name}: {args.warmup + args.steps} steps, plan R,M,slices,chunk,launches = {mix.plan}, "
              f"slice pass {mix.slice_pass}")


if __name__ == "__main__":
    main()
