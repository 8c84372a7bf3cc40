#!/usr/bin/env python
"""Benchmark of the SPECTRE spectral mix on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One step = one pass of the whole path (row pass, slice pass, inverse row pass
with residual + LayerNorm) over one batch of the bf16 long workload
(B=1, L=65536, H=8, D=64, F=8192), inputs resident in HBM.  L2 is flushed
(256 MiB memset) before every timed step; the flush is outside the timed
interval.  Each step is timed with CUDA events on the launching stream; a
second set of steps through the library's profiled entry point (same
launches, one after another) gives the per-kernel breakdown.  With N > 1 (torchrun, one process per GPU) every rank mixes its own
batch -- no data crosses GPUs -- and the reported time is the max over ranks.

The ``e2e`` figure times the host-buffer entry point: per step, H2D copies of
q, k, v, x, G, gamma, beta from pinned memory, the mix, and the D2H copy of y.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload (rank 0 only).

``--workload dct_d256`` or ``dct_d1024`` times the per-token DCT mix with
spectral-entropy routing instead (x [B, L, d] bf16, one kernel per step), with
the same L2 flush, timing, e2e, roofline, clocks and CPU-oracle legs.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "spectral-mix tokens/s at B1 L65536 H8 D64 bf16; achieved HBM GB/s vs peak"
WORKLOAD = "bf16_long"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "source": "fallback"}
FP32_LANES_PER_SM = 128
NUM_SMS = 148


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def _code_only(text: str) -> str:
    """C/C++ source without comments and with whitespace collapsed: what the
    compiler sees, so editing a comment does not change the hash."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":                       # string or character literal
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_hash(path: str = "spectre") -> str:
    """Hash of one path's code in the library (comments and whitespace
    ignored); the ncu traffic in profiles/traffic.txt is used only under the
    hash it was captured on.  path "spectre": csrc/ and include/ without the
    DCT mix's files (named dct_*); path "dct": the DCT mix's files and the
    headers they include (spectre_mix.h, fft_regs.cuh)."""
    files = sorted(glob.glob(os.path.join(ROOT, "sub_quadratic_attention_b200", "csrc", "*")) +
                   glob.glob(os.path.join(ROOT, "include", "*.h")))
    if path == "dct":
        files = [f for f in files if os.path.basename(f).startswith("dct_") or
                 os.path.basename(f) in ("spectre_mix.h", "fft_regs.cuh")]
    else:
        files = [f for f in files if not os.path.basename(f).startswith("dct_")]
    h = hashlib.sha1()
    for f in files:
        with open(f, encoding="utf-8", errors="replace") as fh:
            h.update(os.path.basename(f).encode())
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:12]


def ncu_traffic(workload: str, path: str = "spectre", kernels: int = 3):
    """DRAM bytes per step from profiles/traffic.txt, if taken on this source."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None, {}
    cur = source_hash(path)
    per = {}
    with open(p) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if len(parts) != 4:
                continue
            wl, hsh, kern, nbytes = parts
            if wl == workload and hsh == cur:
                per[kern] = float(nbytes)
    if len(per) == kernels:
        return sum(per.values()), per
    return None, {}


def path_dtype(w, slice_pass: str) -> str:
    """What the path computes in: fp32 arithmetic on the CUDA cores, and for
    the tensor-core slice pass fp16 DFT operands with fp32 accumulation."""
    io = "bf16 I/O" if w.dtype == "bf16" else "f32 I/O"
    if slice_pass == "tensor_cores":
        return f"f32 ({io}; tensor-core DFT passes: f16 operands, f32 accumulate)"
    return f"f32 ({io})"


def method_flops(w) -> float:
    """The method's own arithmetic per step, counted on a radix-2 model: four
    real transforms of length L per channel (q, k, v forward, out inverse) at
    2.5 L log2 L flops each, about 14 flops per kept bin for the gated
    product, and about 10 per element for the residual and LayerNorm."""
    lg = math.log2(w.L)
    return w.B * w.C * (4 * 2.5 * w.L * lg + 14 * w.F) + 10 * w.B * w.L * w.C


def alu_roofline(flops: float, ms: float, sm_mhz) -> dict:
    """The plain-ALU ceiling beside the HBM fraction: NUM_SMS x
    FP32_LANES_PER_SM fp32 lanes, 2 flops a fused multiply-add, at the
    median SM clock seen under load (the nominal 1965 MHz if none)."""
    mhz = float(sm_mhz) if sm_mhz else 1965.0
    peak = NUM_SMS * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
    achieved = flops / (ms * 1e-3) / 1e12
    return {"bound": "alu", "method_flops": flops, "achieved": round(achieved, 3),
            "peak": round(peak, 2), "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "peak_source": f"{NUM_SMS} SMs x {FP32_LANES_PER_SM} fp32 lanes x 2 flops (FMA) at "
                           f"{mhz:.0f} MHz"}


def dominant_roofline(alg_bytes, units, kernel_ms, launches, kernel_traffic, names, peak_gbs):
    """Roofline of the dominant kernel (the largest time per step).

    alg_bytes: the path's algorithmic bytes per step over `units` (token,
    channel) elements, so alg_bytes / units is the per-unit figure.  A
    launch of kernel i processes units / launches[i] elements, and achieved
    is those elements' algorithmic bytes over the kernel's average launch
    time kernel_ms[i] / launches[i].  traffic: that kernel's measured DRAM
    bytes per launch (kernel_traffic: bytes per step by kernel name), or
    None."""
    dom = max(range(len(kernel_ms)), key=lambda i: kernel_ms[i])
    n = launches[dom]
    per_unit = alg_bytes / units
    units_per_launch = units / n
    launch_ms = kernel_ms[dom] / n
    achieved = per_unit * units_per_launch / (launch_ms * 1e-3) / 1e9
    step_traffic = kernel_traffic.get(names[dom])
    return {
        "bound": "hbm", "achieved": round(achieved, 2), "peak": peak_gbs, "unit": "GB/s",
        "frac": round(achieved / peak_gbs, 4),
        "traffic": None if step_traffic is None else step_traffic / n,
        "kernel": names[dom], "bytes_per_unit": round(per_unit, 4),
        "units_per_launch": units_per_launch, "launch_ms": round(launch_ms, 5),
    }


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML polling thread)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4, "gpu_idle": 0x1,
        "applications_clocks_setting": 0x2, "sync_boost": 0x10, "display_clock_setting": 0x100,
    }

    def __init__(self, torch_device: int):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            self._nv = pynvml
            p = torch.cuda.get_device_properties(torch_device)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            try:
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(torch_device)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report that, do not guess
            self.err = repr(e)
            self.max_mhz = None

    def _loop(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._loop, daemon=True)
            self._t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:  # very short region: nearest samples around it
            inside = sorted(self.samples, key=lambda s: abs(s[0] - (t0 + t1) / 2))[:3]
        mhz = [s[1] for s in inside]
        mask = 0
        for s in inside:
            mask |= s[2]
        reasons = [k for k, bit in self.REASONS.items() if mask & bit and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside)}


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
def time_oracle_sample(w, inputs, target_s: float):
    """Time the oracle on the first nch channels (all tokens, all batch rows),
    growing nch until one call takes about target_s.  Returns
    (tokens-equivalent per second, seconds, nch, threads)."""
    import oracle

    nthreads = os.cpu_count() or 1
    nch = 8
    while True:
        t0 = time.perf_counter()
        oracle.spectre_out(inputs["q"], inputs["k"], inputs["v"], inputs["G"], H=w.H, F=w.F,
                           c0=0, c1=nch, nthreads=nthreads)
        dt = time.perf_counter() - t0
        if dt >= target_s or nch >= w.C:
            break
        grow = max(2, int(target_s / max(dt, 1e-3)))
        nch = min(w.C, nch * grow)
    tokens = w.B * w.L * nch / w.C
    return tokens / dt, dt, nch, nthreads


def reference_arm(args, w, rank, world):
    if rank != 0:
        return
    from sub_quadratic_attention_b200.workloads import make_inputs

    inputs = make_inputs(w)
    per_step = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    # size the sample once, then time every step on that sample
    rate, dt, nch, nthreads = time_oracle_sample(w, inputs, per_step)
    import oracle

    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.spectre_out(inputs["q"], inputs["k"], inputs["v"], inputs["G"], H=w.H, F=w.F,
                           c0=0, c1=nch, nthreads=nthreads)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    mean = sum(times) / len(times)
    tokens = w.B * w.L * nch / w.C
    value = tokens / mean
    sample = (f"oracle (fp64, own FFT, OpenMP) on channels 0..{nch - 1} of {w.C}, all "
              f"{w.B * w.L} tokens, pre-LayerNorm output; tokens/s scaled by {nch}/{w.C}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(w, world, pw=None):
    cfg = {"workload": w.name, "B": w.B, "L": w.L, "H": w.H, "D": w.D, "C": w.C, "F": w.F,
           "io_dtype": w.dtype, "global_batch": w.B * world, "seq_len": w.L,
           "parallelism": f"dp{world} (independent batch per rank, no data-path collective)",
           "l2": "flushed before every timed step (256 MiB memset, outside the timed interval); "
                 "inputs 268 MB also exceed L2"}
    if pw is not None and pw is not w:
        cfg.update({"workload": pw.name, "block_len": pw.L, "F": pw.F,
                    "mode": f"blockwise: the mix within each block of {pw.L} tokens "
                            f"({w.B * w.L // pw.L} blocks), gate [H, {pw.L // 2 + 1}]"})
    return cfg


def block_view(w, inputs, n):
    """Blockwise mode's plan shape and inputs: the workload's q, k, v, x viewed
    as B L / n sequences of n tokens (same memory), the first n/2 + 1 bins of
    its gate, and F scaled by n / L (the same fraction of bins kept)."""
    from sub_quadratic_attention_b200.workloads import custom

    if n < 2 or w.L % n:
        raise SystemExit(f"--block-len must divide L = {w.L}")
    F = max(1, min(n // 2 + 1, w.F * n // w.L))
    pw = custom(w.B * (w.L // n), n, w.H, w.D, F, dtype=w.dtype, qkv_scale=w.qkv_scale,
                x_scale=w.x_scale, gate=w.gate, gamma=w.gamma, beta=w.beta,
                name=f"{w.name}_block{n}", index=w.index)
    shape = (pw.B, pw.L, pw.C)
    out = {k: inputs[k].view(shape) for k in ("q", "k", "v", "x")}
    out.update(G=inputs["G"][:, :n // 2 + 1].contiguous(), gamma=inputs["gamma"],
               beta=inputs["beta"])
    return pw, out


# ---------------------------------------------------------------------------
# native arm
# ---------------------------------------------------------------------------
def _device(local_rank, device):
    """The rank's CUDA device, made current; ``device`` overrides it (the CPU
    tests of the JSON assembly run the arms with a fake library)."""
    import torch

    if device is not None:
        return device
    torch.cuda.set_device(local_rank)
    return torch.device("cuda", local_rank)


def native_arm(args, w, rank, world, local_rank, device=None):
    import torch
    import torch.distributed as dist

    from sub_quadratic_attention_b200 import binding
    from sub_quadratic_attention_b200.ranks import job_throughput, max_over_ranks, rank_seed_offset
    from sub_quadratic_attention_b200.workloads import make_inputs

    dev = _device(local_rank, device)
    inputs = make_inputs(w, seed_offset=rank_seed_offset(rank))
    pw = w          # the shape the plan runs: w itself, or its blocks in blockwise mode
    if args.block_len:
        pw, inputs = block_view(w, inputs, args.block_len)
    d = {k: v.to(dev) for k, v in inputs.items()}
    y = torch.empty_like(d["x"])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    mix = binding.SpectreMix(w.B, w.L, w.H, w.D, pw.F, w.dtype, w.eps,
                             tensor_cores=False if args.cuda_core_slices else None,
                             norm=args.norm, complex_gate=args.complex_gate,
                             block_len=args.block_len or None)
    if args.complex_gate:   # the workload's gate with a one-token relative phase e^{-2 pi i f / L}
        fr = torch.arange(pw.L // 2 + 1, device=dev, dtype=torch.float64)
        d["G"] = torch.polar(d["G"].double(), -2 * math.pi * fr / pw.L).to(torch.complex64)
        d["G"] = torch.view_as_real(d["G"]).contiguous()
    h = mix.handle

    def barrier():
        if world > 1:
            dist.barrier()

    # warm-up
    for _ in range(args.warmup):
        flush.zero_()
        binding.spectre_mix_run(h, d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y,
                                stream)
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.05)
    R, M, nf, wave_ch, nlaunch = mix.plan
    nchunks = (nlaunch - 1) // 2
    step_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_host0 = time.perf_counter()
    for i in range(args.steps):
        flush.zero_()
        step_ev[i][0].record(stream)
        binding.spectre_mix_run(h, d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"], d["beta"], y,
                                stream)
        step_ev[i][1].record(stream)
    torch.cuda.synchronize()
    t_host1 = time.perf_counter()
    barrier()
    sampler.stop()
    clocks = sampler.summary(t_host0, t_host1)
    step_ms = [e[0].elapsed_time(e[1]) for e in step_ev]

    # per-kernel breakdown: the profiled entry point runs the same launches one
    # after another on one stream, with an event before each launch
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(nlaunch + 1)]
              for _ in range(args.steps)]
    for ev in events:  # torch creates the CUDA event on its first record
        for e in ev:
            e.record(stream)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        binding.spectre_mix_run_profiled(h, d["q"], d["k"], d["v"], d["x"], d["G"], d["gamma"],
                                         d["beta"], y, events[i], stream)
    torch.cuda.synchronize()
    seq_ms = [e[0].elapsed_time(e[-1]) for e in events]
    # launch i of a step: row pass of chunk i//2 (even i), slice pass (odd i),
    # inverse row pass (last); per-kernel time = sum over its launches
    kern_ms = [[0.0] * args.steps for _ in range(3)]
    for s_i, e in enumerate(events):
        for i in range(nlaunch):
            kind = 2 if i == nlaunch - 1 else (i % 2)
            kern_ms[kind][s_i] += e[i].elapsed_time(e[i + 1])
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / args.steps
    tokens_per_step = w.B * w.L * world
    value = job_throughput(w.B * w.L, world, args.steps, total_ms)

    # ---- end-to-end through the host-buffer entry point
    pinned = {k: v.pin_memory() for k, v in inputs.items()}
    pinned["G"] = d["G"].cpu().pin_memory()   # the gate as the plan reads it (real, or (re, im))
    y_host = torch.empty_like(pinned["x"]).pin_memory()
    for _ in range(2):
        binding.spectre_mix_run_host(h, pinned["q"], pinned["k"], pinned["v"], pinned["x"],
                                     pinned["G"], pinned["gamma"], pinned["beta"], y_host, stream)
    torch.cuda.synchronize()
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        e2e_ev[i][0].record(stream)
        binding.spectre_mix_run_host(h, pinned["q"], pinned["k"], pinned["v"], pinned["x"],
                                     pinned["G"], pinned["gamma"], pinned["beta"], y_host, stream)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_total = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in e2e_ev), dev)
    e2e_value = job_throughput(w.B * w.L, world, args.steps, e2e_total)
    nelem = w.B * w.L * w.C
    h2d = 4 * nelem * w.elem_bytes + pinned["G"].numel() * 4 + 2 * w.C * 4
    d2h = nelem * w.elem_bytes

    # ---- roofline of the path against measured HBM bandwidth
    peaks = load_peaks()
    alg_bytes = pw.algorithmic_bytes() + (w.H * pw.F * 4 if args.complex_gate else 0)   # (re, im) gate
    achieved = alg_bytes / (ms_per_step * 1e-3) / 1e9
    traffic, per_kernel_traffic = ncu_traffic(pw.name)
    names = ["rows_fwd", "slices", "rows_inv_ln"]
    kmean = [sum(k) / len(k) for k in kern_ms]
    ksum = sum(kmean)
    kernels = [{"name": n, "ms": round(m, 5), "share": round(m / ksum, 4),
                "launches_per_step": (nchunks if i < 2 else 1),
                "dram_bytes": per_kernel_traffic.get(n)} for i, (n, m) in enumerate(zip(names, kmean))]
    dom = max(range(3), key=lambda i: kmean[i])
    roofline = dominant_roofline(alg_bytes, w.B * w.L * w.C, kmean, [nchunks, nchunks, 1],
                                 per_kernel_traffic, names, peaks["hbm_gbs"])
    roofline.update({
        "peak_source": f"{peaks['source']} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
        if peaks["source"] == "measured" else "fallback 6.65 TB/s",
        "scope": "dominant kernel: algorithmic bytes per (token, channel) element (q,k,v,x "
                 "read + G[:, :F] + gamma, beta read + y written, over B L C) x the elements "
                 "one launch processes, over its average launch time (CUDA events on the "
                 "launch stream, profiled steps); traffic: its ncu DRAM bytes per launch",
        "path": {"achieved": round(achieved, 2), "frac": round(achieved / peaks["hbm_gbs"], 4),
                 "frac_of_8TBps_nominal": round(achieved / 8000.0, 4), "traffic": traffic,
                 "algorithmic_bytes": alg_bytes,
                 "scope": "whole step: algorithmic bytes over the timed step time"},
        "alu": alu_roofline(method_flops(pw), ms_per_step, clocks.get("sm_mhz")),
        "kernels": kernels, "dominant_kernel": names[dom],
        "kernels_note": "per-kernel times from the profiled entry point, which runs the launches "
                        "one after another on one stream (sequential step "
                        f"{sum(seq_ms) / len(seq_ms):.4f} ms); the timed step overlaps each chunk's "
                        "row pass with the previous chunk's slice pass on two streams",
        "plan": {"R": R, "M": M, "slices_per_channel": nf, "channels_per_wave": wave_ch,
                 "chunks": nchunks, "launches_per_step": nlaunch,
                 "slice_pass": mix.slice_pass, "norm": args.norm,
                 "gate": "complex" if args.complex_gate else "real",
                 "block_len": args.block_len or None},
    })

    # ---- CPU baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, dt, nch, nthreads = time_oracle_sample(pw, inputs, args.cpu_seconds)
        cpu = {"value": rate, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
               "sample": f"oracle (fp64) on channels 0..{nch - 1} of {w.C}, all {w.B * w.L} "
                         f"tokens, pre-LayerNorm output, {dt:.1f} s; tokens/s scaled by "
                         f"{nch}/{w.C}"}

    if world > 1:
        gathered = [None] * world
        dist.all_gather_object(gathered, clocks)
        reasons = sorted({r for c in gathered for r in c.get("reasons", [])})
        clocks = dict(clocks)
        clocks["reasons"] = reasons
        clocks["per_rank_sm_mhz"] = [c.get("sm_mhz") for c in gathered]

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": path_dtype(w, mix.slice_pass),
            "data": f"synthetic (seeded; shapes and distributions of the {w.name} workload)",
            "config": config_dict(w, world, pw),
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": nlaunch * args.steps,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "clocks": clocks,
            "hbm_gbs_achieved": round(achieved, 2),
        }
        print(json.dumps(line), flush=True)
    mix.close()


# ---------------------------------------------------------------------------
# DCT mix (per-token DCT, spectral entropy, route, LayerNorm(x + iDCT(DCT(x) w)))
# ---------------------------------------------------------------------------
def dct_metric(w) -> str:
    return (f"dct-mix tokens/s at B{w.B} L{w.L} d{w.d} {w.dtype}; achieved HBM GB/s vs peak")


def dct_method_flops(w) -> float:
    """Per token: its half of one d-point complex FFT each way (5 d log2 d
    flops per transform, shared by two rows), about 30 flops per coefficient
    for the split, entropy, filter and re-twiddle, and about 10 per element
    for the residual and LayerNorm."""
    return w.T * (5.0 * w.d * math.log2(w.d) + 40.0 * w.d)


def dct_config(w, world):
    return {"workload": w.name, "B": w.B, "L": w.L, "d": w.d, "tau": w.tau, "io_dtype": w.dtype,
            "global_batch": w.B * world, "seq_len": w.L,
            "parallelism": f"dp{world} (independent tokens per rank, no data-path collective)",
            "l2": "flushed before every timed step (256 MiB memset, outside the timed interval); "
                  f"x alone is {w.T * w.d * w.elem_bytes / 1e6:.0f} MB"}


def time_dct_oracle_sample(w, inputs, target_s: float):
    """Time the oracle on the first n token rows, growing n until one call
    takes about target_s.  Returns (tokens per second, seconds, n, threads)."""
    import oracle

    nthreads = os.cpu_count() or 1
    x = inputs["x"].reshape(-1, w.d)
    n = 64
    while True:
        t0 = time.perf_counter()
        oracle.dct_mix(x[:n], inputs["w"], inputs["gamma"], inputs["beta"], eps=w.eps, tau=w.tau,
                       nthreads=nthreads)
        dt = time.perf_counter() - t0
        if dt >= target_s or n >= w.T:
            break
        n = min(w.T, n * max(2, int(target_s / max(dt, 1e-3))))
    return n / dt, dt, n, nthreads


def dct_reference_arm(args, w, rank, world):
    if rank != 0:
        return
    from sub_quadratic_attention_b200.workloads import make_dct_inputs

    inputs = make_dct_inputs(w)
    per_step = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    _, _, n, nthreads = time_dct_oracle_sample(w, inputs, per_step)
    import oracle

    x = inputs["x"].reshape(-1, w.d)[:n]
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.dct_mix(x, inputs["w"], inputs["gamma"], inputs["beta"], eps=w.eps, tau=w.tau,
                       nthreads=nthreads)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    mean = sum(times) / len(times)
    value = n / mean
    sample = f"oracle (fp64, O(d^2) DCT sums, OpenMP) on the first {n} of {w.T} token rows"
    print(json.dumps({
        "impl": "reference", "metric": dct_metric(w), "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": dct_config(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def dct_arm(args, w, rank, world, local_rank, device=None):
    import torch
    import torch.distributed as dist

    from sub_quadratic_attention_b200 import binding
    from sub_quadratic_attention_b200.ranks import job_throughput, max_over_ranks, rank_seed_offset
    from sub_quadratic_attention_b200.workloads import make_dct_inputs

    dev = _device(local_rank, device)
    inputs = make_dct_inputs(w, seed_offset=rank_seed_offset(rank))
    d = {k: v.to(dev) for k, v in inputs.items()}
    lead = (w.B, w.L)
    y = torch.empty_like(d["x"])
    H = torch.empty(lead, dtype=torch.float32, device=dev)
    route = torch.empty(lead, dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    mix = binding.DctMix(w.d, w.dtype, w.eps)
    h = mix.handle

    def step():
        binding.dct_mix_run(h, w.T, d["x"], d["w"], d["gamma"], d["beta"], w.tau, y, H, route,
                            stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.05)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    barrier()
    sampler.stop()
    clocks = sampler.summary(t0, t1)
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(w.T, world, args.steps, total_ms)

    # e2e through the host-buffer entry point
    pinned = {k: v.pin_memory() for k, v in inputs.items()}
    y_h = torch.empty_like(pinned["x"]).pin_memory()
    H_h = torch.empty(lead, dtype=torch.float32).pin_memory()
    r_h = torch.empty(lead, dtype=torch.uint8).pin_memory()

    def host_step():
        binding.dct_mix_run_host(h, w.T, pinned["x"], pinned["w"], pinned["gamma"],
                                 pinned["beta"], w.tau, y_h, H_h, r_h, stream)

    for _ in range(2):
        host_step()
    torch.cuda.synchronize()
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        e2e_ev[i][0].record(stream)
        host_step()
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_total = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in e2e_ev), dev)
    e2e_value = job_throughput(w.T, world, args.steps, e2e_total)
    es = w.elem_bytes
    h2d = w.T * w.d * es + 3 * w.d * 4
    d2h = w.T * w.d * es + 5 * w.T

    peaks = load_peaks()
    alg = w.algorithmic_bytes()
    achieved = alg / (ms_per_step * 1e-3) / 1e9
    traffic, _ = ncu_traffic(w.name, path="dct", kernels=1)
    roofline = {
        "bound": "hbm", "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
        "kernel": "dct_mix", "bytes_per_unit": round(alg / w.T, 4), "units_per_launch": w.T,
        "launch_ms": round(ms_per_step, 5),
        "peak_source": f"{peaks['source']} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
        if peaks["source"] == "measured" else "fallback 6.65 TB/s",
        "scope": "the step's one kernel: algorithmic bytes per token (x read and y written, "
                 "d values each, H and route written; w, gamma, beta once per launch) x the "
                 "tokens of a launch, over its CUDA-event time",
        "alu": alu_roofline(dct_method_flops(w), ms_per_step, clocks.get("sm_mhz")),
    }
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, dt, n, nthreads = time_dct_oracle_sample(w, inputs, args.cpu_seconds)
        cpu = {"value": rate, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
               "sample": f"oracle (fp64) on the first {n} of {w.T} token rows, {dt:.1f} s"}
    if world > 1:
        gathered = [None] * world
        dist.all_gather_object(gathered, clocks)
        clocks = dict(clocks)
        clocks["reasons"] = sorted({r for c in gathered for r in c.get("reasons", [])})
    if rank == 0:
        print(json.dumps({
            "metric": dct_metric(w), "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": f"synthetic (seeded; half smooth, half white token rows, d = {w.d})",
            "config": dct_config(w, world),
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps,
            "roofline": roofline, "cpu_baseline": cpu, "clocks": clocks,
            "routed_fraction": round(float(route.float().mean().item()), 4),
            "hbm_gbs_achieved": round(achieved, 2),
        }), flush=True)
    mix.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--norm", choices=["post_ln", "pre_ln", "post_rms", "pre_rms"], default="post_ln",
                    help="normalisation: LayerNorm(out + x) (default), LayerNorm(out) + x, or the "
                         "RMSNorm forms")
    ap.add_argument("--complex-gate", action="store_true",
                    help="time a complex gate (the workload's G with a relative-position phase)")
    ap.add_argument("--block-len", type=int, default=0,
                    help="blockwise mode: mix within blocks of this many tokens (must divide L)")
    ap.add_argument("--cuda-core-slices", action="store_true",
                    help="force the CUDA-core slice pass (plan option; default: tensor cores "
                         "where the plan allows)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        # launched without torchrun for N > 1, or mismatched: trust the launcher's world size
        if world == 1 and args.gpus > 1:
            print(json.dumps({"error": "run N > 1 under torchrun (one process per GPU)"}),
                  flush=True)
            sys.exit(2)

    from sub_quadratic_attention_b200.workloads import DCT_WORKLOADS, WORKLOADS

    dct = args.workload in DCT_WORKLOADS
    if not dct and args.workload not in WORKLOADS:
        ap.error(f"unknown workload {args.workload}")
    w = DCT_WORKLOADS[args.workload] if dct else WORKLOADS[args.workload]
    if args.impl == "reference":
        (dct_reference_arm if dct else reference_arm)(args, w, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        (dct_arm if dct else native_arm)(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
