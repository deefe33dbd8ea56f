#!/usr/bin/env python
"""Benchmark of the NVFP4 hot path on B200: quantize (MSE weights, absmax
activations), W4A4 GEMM, dequantize -- one JSON line on rank 0.

Workload (default ``dense31b_m8192``, the 31B-class dense layer): per step
  1. quantize W  (21504 x 5376, 0.015*t4) with MSE block scales,
  2. quantize W2 (5376 x 21504, 0.015*t4) with MSE block scales,
  3. quantize X  (8192 x 5376, N(0,1)) and X2 (8192 x 21504, N(0,1)) with absmax scales,
  4. C1 = X W^T  (M=8192, N=21504, K=5376) and C2 = X2 W2^T (M=8192, N=5376, K=21504),
  5. dequantize X's NVFP4 copy back to BF16 (the reconstruction).
All inputs are seeded synthetic tensors (there is no dataset); the step touches
~1.3 GB, far more than the 126 MB L2, so no extra flush is needed between steps.

value = GEMM FLOPs of all ranks' steps / max-over-ranks device time of the K timed
steps (TFLOP/s of the whole step, quantization included).  ``roofline`` is the
GEMM kernel against the FP4 tensor peak derived from the measured BF16 peak;
``components`` gives every kernel group's own rate.  ``e2e`` repeats the step
through the same C-ABI calls from pinned host buffers, with the host->device
copies of the step's inputs and the device->host copies of C1 and C2 timed.
``cpu_baseline`` times the CPU oracle (single thread) on a bounded sample of the
same step and extrapolates to the full step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    "dense31b_m8192": dict(M=8192, K1=5376, N1=21504, K2=21504, N2=5376),
    "dense31b_m256": dict(M=256, K1=5376, N1=21504, K2=21504, N2=5376),
    "prefill8b": dict(M=4096, K1=4096, N1=14336, K2=14336, N2=4096),
}

FP4_PER_BF16 = 4.0  # nominal dense ratio: 9 PFLOP/s FP4 vs 2.25 PFLOP/s BF16


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=sorted(WORKLOADS), default="dense31b_m8192")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--seed", type=int, default=0)
    return p.parse_args()


KERNEL_SOURCES = {"gemm": ["gemm_sm100.cu", "ptx.cuh", "internal.h"],
                  "quantize": ["quantize.cu", "ptx.cuh", "internal.h"]}


def source_hash(kernel: str = "gemm") -> str:
    """Hash of the source files a kernel is built from (ncu summaries record it, so
    counters taken on an older kernel are never reported for a newer one)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "w4a4_gemm_quantize_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sust=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sust=1400.0, source="fallback")


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, only if it was taken on
    the current kernel sources (the summary records the source hash)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_hash") != source_hash(kernel):
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        rows = []
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), power=float(f[3]), hw=f[5], hwt=f[6], swt=f[7],
                                 pcap=f[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        load = [r for r in rows if r["power"] > 300] or rows
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# ------------------------------------------------------------------------------------------------
# distributed plumbing (one process per GPU; weak scaling: every rank runs its own step)
# ------------------------------------------------------------------------------------------------

def dist_setup(n_gpus: int):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    if world != n_gpus:
        print(f"warning: --gpus {n_gpus} but WORLD_SIZE {world}", file=sys.stderr)
    return rank, world, local


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, flops_per_step: float, ms: float) -> float:
    """Whole-job TFLOP/s under weak scaling: every rank runs `steps` steps of its own
    problem, timed as the slowest rank's `ms`."""
    return world * steps * flops_per_step / (ms * 1e-3) / 1e12


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------

def make_inputs(cfg, seed: int, rank: int):
    import workloads
    s = seed + 1000 * rank
    return {
        "W": workloads.t4_weight(cfg["N1"], cfg["K1"], seed=s, stream=workloads.STREAM_W),
        "W2": workloads.t4_weight(cfg["N2"], cfg["K2"], seed=s, stream=workloads.STREAM_W2),
        "X": workloads.activation(cfg["M"], cfg["K1"], seed=s, stream=workloads.STREAM_X, n_outlier_channels=0),
        "X2": workloads.activation(cfg["M"], cfg["K2"], seed=s, stream=workloads.STREAM_X2, n_outlier_channels=0),
    }


class Step:
    """All device buffers of one step and the C-ABI calls that make it."""

    def __init__(self, cfg, inputs_cpu, device):
        import torch
        import w4a4_gemm_quantize_b200 as nv
        self.nv = nv
        self.cfg = cfg
        self.x = {k: v.to(device) for k, v in inputs_cpu.items()}
        M = cfg["M"]
        self.q = {
            "W": nv.nvfp4_quantize(self.x["W"], "mse"),
            "W2": nv.nvfp4_quantize(self.x["W2"], "mse"),
            "X": nv.nvfp4_quantize(self.x["X"], "absmax"),
            "X2": nv.nvfp4_quantize(self.x["X2"], "absmax"),
        }
        self.c1 = torch.empty((M, cfg["N1"]), dtype=torch.bfloat16, device=device)
        self.c2 = torch.empty((M, cfg["N2"]), dtype=torch.bfloat16, device=device)
        self.xhat = torch.empty((M, cfg["K1"]), dtype=torch.bfloat16, device=device)
        self.ws = {k: torch.empty(256, dtype=torch.uint8, device=device) for k in ("W", "W2", "X", "X2", "g1", "g2")}
        self.launches = 0

    def groups(self):
        nv = self.nv
        return [
            ("quantize_mse_W", lambda: nv.nvfp4_quantize(self.x["W"], "mse", out=self.q["W"], workspace=self.ws["W"])),
            ("quantize_mse_W2", lambda: nv.nvfp4_quantize(self.x["W2"], "mse", out=self.q["W2"],
                                                          workspace=self.ws["W2"])),
            ("quantize_absmax_X", lambda: nv.nvfp4_quantize(self.x["X"], "absmax", out=self.q["X"],
                                                            workspace=self.ws["X"])),
            ("quantize_absmax_X2", lambda: nv.nvfp4_quantize(self.x["X2"], "absmax", out=self.q["X2"],
                                                             workspace=self.ws["X2"])),
            ("gemm_1", lambda: nv.nvfp4_gemm(self.q["X"], self.q["W"], out=self.c1, workspace=self.ws["g1"])),
            ("gemm_2", lambda: nv.nvfp4_gemm(self.q["X2"], self.q["W2"], out=self.c2, workspace=self.ws["g2"])),
            ("dequantize_X", lambda: nv.nvfp4_dequantize(self.q["X"], out=self.xhat)),
        ]

    def run(self, events=None):
        n = 0
        for i, (name, fn) in enumerate(self.groups()):
            if events is not None:
                events[name][0].record()
            fn()
            n += self.nv.last_launch_count()
            if events is not None:
                events[name][1].record()
        self.launches += n
        return n


def work_units(cfg):
    M = cfg["M"]
    flops = 2 * M * cfg["N1"] * cfg["K1"] + 2 * M * cfg["N2"] * cfg["K2"]
    elems = {"quantize_mse_W": cfg["N1"] * cfg["K1"], "quantize_mse_W2": cfg["N2"] * cfg["K2"],
             "quantize_absmax_X": M * cfg["K1"], "quantize_absmax_X2": M * cfg["K2"], "dequantize_X": M * cfg["K1"]}
    return flops, elems


def gemm_kernel_name(M: int, N: int) -> str:
    """The kernel the library picks for an M x N output (its launch dispatch)."""
    if M <= 32:
        return "gemm_decode_kernel (tcgen05 mxf4nvf4, stream-K)"
    if M > 128 and N > 128:
        return "gemm_pair_kernel (tcgen05 cta_group::2 mxf4nvf4)"
    return "gemm_kernel (tcgen05 mxf4nvf4)"


def run_ours(args, rank, world, local):
    import torch
    import w4a4_gemm_quantize_b200 as nv
    nv.load_library()
    device = torch.device("cuda", local)
    cfg = WORKLOADS[args.workload]
    inputs = make_inputs(cfg, args.seed, rank)
    step = Step(cfg, inputs, device)
    stream = torch.cuda.current_stream(device)
    names = [n for n, _ in step.groups()]

    for _ in range(max(args.warmup, 3)):
        step.run()
    torch.cuda.synchronize(device)
    barrier(world)

    events = {n: [] for n in names}
    ev_all = []
    step.launches = 0
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize(device)
        t_start.record(stream)
        for _ in range(args.steps):
            ev = {n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for n in names}
            step.run(ev)
            ev_all.append(ev)
        t_end.record(stream)
        torch.cuda.synchronize(device)
        barrier(world)
    ms_local = t_start.elapsed_time(t_end)
    ms = max_over_ranks(ms_local, world, device)
    per_group = {n: statistics.mean(e[n][0].elapsed_time(e[n][1]) for e in ev_all) for n in names}

    flops, elems = work_units(cfg)
    peaks = load_peaks()
    value = job_throughput(world, args.steps, flops, ms)
    step_ms = ms / args.steps

    # roofline of the dominant kernel: the first GEMM launch (M x N1 x K1)
    gemm_tflops = 2 * cfg["M"] * cfg["N1"] * cfg["K1"] / (per_group["gemm_1"] * 1e-3) / 1e12
    long_region = ms * 1e-3 > 1.0
    bf16_peak = peaks["bf16_sust"] if long_region else peaks["bf16"]
    fp4_peak = bf16_peak * FP4_PER_BF16
    traffic = profiled_traffic("gemm", args.workload)
    roofline = {"bound": "tensor", "achieved": round(gemm_tflops, 1), "peak": round(fp4_peak, 1),
                "unit": "TFLOP/s", "frac": round(gemm_tflops / fp4_peak, 4), "traffic": traffic,
                "kernel": f"{gemm_kernel_name(cfg['M'], cfg['N1'])}, launch gemm_1 (M x N1 x K1)",
                "peak_source": f"{peaks['source']} bf16 {'sustained' if long_region else 'burst'} x {FP4_PER_BF16:g}"}
    comps = {}
    for n in names:
        if n.startswith("gemm"):
            M, N, K = (cfg["M"], cfg["N1"], cfg["K1"]) if n == "gemm_1" else (cfg["M"], cfg["N2"], cfg["K2"])
            t = 2 * M * N * K / (per_group[n] * 1e-3) / 1e12
            comps[n] = {"us": round(per_group[n] * 1e3, 1), "TFLOP/s": round(t, 1), "frac_fp4_peak": round(t / fp4_peak, 4)}
        else:
            # quantize (two-pass, the per-tensor scale computed in the step): 2 B read by
            # the amax pass + 2 B read and 0.5625 B written by the encode pass; dequantize:
            # 0.5625 B read + 2 B written
            bpe = 2.5625 if n.startswith("dequantize") else 4.5625
            gbs = elems[n] * bpe / (per_group[n] * 1e-3) / 1e9
            comps[n] = {"us": round(per_group[n] * 1e3, 1), "GB/s": round(gbs, 1),
                        "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "bytes_per_elem": bpe}

    e2e = run_e2e(args, step, inputs, device, world) if args.e2e_steps > 0 else None
    launches = step.launches // args.steps * args.steps
    out = {
        "metric": "NVFP4 quantize GB/s and W4A4 GEMM TFLOPS on 1 B200, % of roofline",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 codes, e4m3 block scales, fp32 accumulation, bf16 out)", "data": "synthetic",
        "config": {"workload": args.workload, **cfg, "global_batch": cfg["M"] * world,
                   "parallelism": f"independent replicas x{world}",
                   "l2": "inputs larger than L2 (the step touches ~1.3 GB)",
                   "step": "MSE-quantize W, W2; absmax-quantize X, X2; C1 = X W^T; C2 = X2 W2^T; dequantize X"},
        "roofline": roofline, "components": comps, "gpu_launches": launches,
        "clocks": clk.summary(), "e2e": e2e,
        "cpu_baseline": None,
    }
    return out


def run_e2e(args, step, inputs, device, world):
    """Same step from pinned host buffers: H2D inputs, C-ABI calls, D2H outputs, all timed."""
    import torch
    host_in = {k: v.pin_memory() for k, v in inputs.items()}
    host_c1 = torch.empty(step.c1.shape, dtype=torch.bfloat16).pin_memory()
    host_c2 = torch.empty(step.c2.shape, dtype=torch.bfloat16).pin_memory()
    stream = torch.cuda.current_stream(device)

    def one():
        for k, v in host_in.items():
            step.x[k].copy_(v, non_blocking=True)
        step.run()
        host_c1.copy_(step.c1, non_blocking=True)
        host_c2.copy_(step.c2, non_blocking=True)

    one()
    torch.cuda.synchronize(device)
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(args.e2e_steps):
        one()
    e.record(stream)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(s.elapsed_time(e), world, device)
    flops, _ = work_units(step.cfg)
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = host_c1.numel() * 2 + host_c2.numel() * 2
    return {"value": round(world * args.e2e_steps * flops / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
            "ms_per_step": round(ms / args.e2e_steps, 3)}


# ------------------------------------------------------------------------------------------------
# the CPU oracle on a bounded sample of the same step (cpu_baseline and --impl reference)
# ------------------------------------------------------------------------------------------------

SAMPLE = dict(w_rows=48, x_rows=8, out_m=2, out_n=8)


def oracle_sample_step(cfg, inputs):
    """Run the oracle on a row sample of every tensor of the step and extrapolate
    each part to the full step by its share of rows / outputs.  Returns
    (extrapolated full-step seconds, sample seconds)."""
    import numpy as np
    import oracle
    import workloads
    t_total = 0.0
    est = 0.0
    q = {}
    for name, mode, rows in (("W", oracle.SCALE_MSE, SAMPLE["w_rows"]), ("W2", oracle.SCALE_MSE, SAMPLE["w_rows"]),
                             ("X", oracle.SCALE_ABSMAX, SAMPLE["x_rows"]), ("X2", oracle.SCALE_ABSMAX, SAMPLE["x_rows"])):
        bits = workloads.bf16_bits(inputs[name])
        t0 = time.perf_counter()
        sg = oracle.global_scale(bits)                      # full-tensor amax (not sampled)
        t1 = time.perf_counter()
        codes, sc, _, _ = oracle.quantize(np.ascontiguousarray(bits[:rows]), mode, sg)
        t2 = time.perf_counter()
        q[name] = (codes, sc, sg)
        t_total += t2 - t0
        est += (t1 - t0) + (t2 - t1) * bits.shape[0] / rows
    for a, b, M, N in (("X", "W", cfg["M"], cfg["N1"]), ("X2", "W2", cfg["M"], cfg["N2"])):
        mi = np.repeat(np.arange(SAMPLE["out_m"]), SAMPLE["out_n"])
        ni = np.tile(np.arange(SAMPLE["out_n"]), SAMPLE["out_m"])
        t0 = time.perf_counter()
        oracle.gemm_f64_at(*q[a], *q[b], mi, ni)
        t1 = time.perf_counter()
        t_total += t1 - t0
        est += (t1 - t0) * (M * N) / mi.size
    codes, sc, sg = q["X"]
    t0 = time.perf_counter()
    oracle.dequantize(codes, sc, sg)
    t1 = time.perf_counter()
    t_total += t1 - t0
    est += (t1 - t0) * cfg["M"] / codes.shape[0]
    return est, t_total


def sample_desc(cfg):
    return (f"oracle (1 thread) on a row sample of the step: full-tensor amax of W, W2, X, X2; quantize "
            f"{SAMPLE['w_rows']} rows of W and W2 (MSE) and {SAMPLE['x_rows']} rows of X, X2 (absmax); "
            f"{SAMPLE['out_m']}x{SAMPLE['out_n']} outputs of each float64 GEMM; dequantize the X sample; "
            f"each part extrapolated to the full step by its share of rows/outputs")


def cpu_baseline(cfg, inputs):
    import oracle
    oracle.build()
    est, sample_s = oracle_sample_step(cfg, inputs)
    flops, _ = work_units(cfg)
    return {"value": flops / est / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": sample_desc(cfg), "sample_seconds": round(sample_s, 2),
            "extrapolated_step_seconds": round(est, 1)}


def run_reference(args, rank, world):
    cfg = WORKLOADS[args.workload]
    if rank != 0:
        return None
    import oracle
    oracle.build()
    inputs = make_inputs(cfg, args.seed, 0)
    flops, _ = work_units(cfg)
    for _ in range(args.warmup):
        oracle_sample_step(cfg, inputs)
    ests, samples = [], []
    for _ in range(args.steps):
        est, s = oracle_sample_step(cfg, inputs)
        ests.append(est)
        samples.append(s)
    est = statistics.mean(ests)
    value = flops / est / 1e12
    base = {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": sample_desc(cfg),
            "sample_seconds_per_step": round(statistics.mean(samples), 2)}
    return {
        "impl": "reference",
        "metric": "NVFP4 quantize GB/s and W4A4 GEMM TFLOPS on 1 B200, % of roofline",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(est * 1e3, 1), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 GEMM reference, binary32 quantizer (CPU oracle)", "data": "synthetic",
        "config": {"workload": args.workload, **cfg},
        "cpu_baseline": base,
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            out = run_reference(args, rank, world)
        else:
            out = run_ours(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                cfg = WORKLOADS[args.workload]
                out["cpu_baseline"] = cpu_baseline(cfg, make_inputs(cfg, args.seed, 0))
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
