#!/usr/bin/env python
"""Benchmark of the NVFP4 hot path on B200 -- one JSON line on rank 0.

Workloads (``--workload``; seeded synthetic tensors shaped like the pages' layers,
there is no dataset):

* ``dense31b_m8192`` (default), ``dense31b_m256``, ``dense31b_m1`` -- the 31B-class
  dense layer: quantize W (21504 x 5376) and W2 (5376 x 21504), 0.015 Student-t(4),
  with MSE block scales; quantize X (M x 5376) and X2 (M x 21504), N(0,1), with
  absmax scales; C1 = X W^T, C2 = X2 W2^T; dequantize X.
* ``prefill8b`` -- 8B-class prefill: X_up 4096 x 4096 and X_down 4096 x 14336 (4
  outlier channels x50) quantized on the fly (absmax), then C_up = X_up W_up^T
  (14336 x 4096) and C_down = X_down W_down^T (4096 x 14336); weights N(0, 0.02),
  quantized once before timing (MSE).
* ``decode_m1``, ``decode_m8``, ``decode_m32`` -- 8B-class decode: X M x 4096 quantized
  on the fly, then the GEMM against the pre-quantized 14336 x 4096 weight.
* ``mse4096`` -- MSE-vs-absmax scale search: quantize a 4096 x 4096 0.02 Student-t(3)
  weight with MSE block scales (8 candidates); the absmax quantization and both
  mean block errors are reported alongside.
* ``pr1`` -- the PR1 reference: quantize W 256 x 256 and X 16 x 256 (absmax), GEMM
  16 x 256 x 256 (launch-bound).

A step is one pass over every kernel group of the workload.  Each group's C-ABI
calls are captured once into a CUDA graph and replayed, and each replay is timed
with CUDA events on the launching stream; ``value`` is the workload's total work
(GEMM FLOPs, or algorithmic bytes for the quantize-only and decode workloads) of
all ranks' steps over the slowest rank's device time.  Steps whose working set is
smaller than twice the 126 MB L2 cycle through enough copies of their inputs and
outputs that no step finds its data in L2 (``pr1``: a 256 MB L2 flush before each
step, outside the step's events).  ``roofline`` is the group with the largest share
of the step time against its bound (FP4 tensor peak = measured BF16 peak x 4, or
the measured HBM copy bandwidth).  ``e2e`` repeats the step from pinned host
buffers through the same C-ABI calls, host->device copies of the step's inputs and
device->host copies of its results inside the timed region.  ``cpu_baseline`` times
the CPU oracle on a bounded sample of the same step, on one thread and on every
host core, and extrapolates each part to the full step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 quantize GB/s and W4A4 GEMM TFLOPS on 1 B200, % of roofline"
FP4_PER_BF16 = 4.0   # nominal dense ratio: 9 PFLOP/s FP4 vs 2.25 PFLOP/s BF16
L2_BYTES = 126 * 2 ** 20
QUANT_BPE_TWO_PASS = 4.5625   # amax read 2 B + encode read 2 B + codes 0.5 B + scales 0.0625 B
QUANT_BPE_GIVEN_SCALE = 2.5625
DEQUANT_BPE = 2.5625

WORKLOADS = {
    "dense31b_m8192": dict(kind="dense31b", M=8192, K1=5376, N1=21504, K2=21504, N2=5376),
    "dense31b_m256": dict(kind="dense31b", M=256, K1=5376, N1=21504, K2=21504, N2=5376),
    "dense31b_m1": dict(kind="dense31b", M=1, K1=5376, N1=21504, K2=21504, N2=5376),
    "prefill8b": dict(kind="prefill", M=4096, K_up=4096, N_up=14336, K_down=14336, N_down=4096),
    "decode_m1": dict(kind="decode", M=1, N=14336, K=4096),
    "decode_m8": dict(kind="decode", M=8, N=14336, K=4096),
    "decode_m32": dict(kind="decode", M=32, N=14336, K=4096),
    "mse4096": dict(kind="mse", rows=4096, cols=4096),
    "decode_m32_lora16": dict(kind="decode_lora", M=32, N=14336, K=4096, R=16),
    "decode_m32_lora64": dict(kind="decode_lora", M=32, N=14336, K=4096, R=64),
    "prefill8b_lora16": dict(kind="prefill_lora", M=4096, K_up=4096, N_up=14336, K_down=14336, N_down=4096, R=16),
    "prefill8b_lora64": dict(kind="prefill_lora", M=4096, K_up=4096, N_up=14336, K_down=14336, N_down=4096, R=64),
    "pr1": dict(kind="pr1", M=16, N=256, K=256),
}


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=sorted(WORKLOADS), default="dense31b_m8192")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="rough budget of the oracle timing (both legs together)")
    p.add_argument("--seed", type=int, default=0)
    return p.parse_args(argv)


KERNEL_SOURCES = {"gemm": ["gemm_sm100.cu", "ptx.cuh", "internal.h"],
                  "quantize": ["quantize.cu", "quant_block.cuh", "ptx.cuh", "internal.h"],
                  "lora": ["lora.cu", "gemm_sm100.cu", "quant_block.cuh", "ptx.cuh", "internal.h"]}
KERNEL_FAMILY = {"gemm_pair_kernel": "gemm", "gemm_decode_kernel": "gemm", "gemm_kernel": "gemm",
                 "gemm_pair_kernel_lora": "lora", "gemm_decode_kernel_lora": "lora", "quantize_kernel": "quantize",
                 "dequantize_kernel": "quantize"}


def group_kernel(group: str, cfg: dict, family: str):
    """(file tag, description) of the kernel that dominates a group's time."""
    if family == "gemm":
        n_of = {"gemm_1": "N1", "gemm_2": "N2", "gemm_up": "N_up", "gemm_down": "N_down", "gemm": "N", "linear": "N",
                "linear_lora": "N", "linear_lora_up": "N_up", "linear_lora_down": "N_down"}
        M, N = cfg["M"], cfg[n_of[group]]
        tag = "gemm_decode_kernel" if M <= 32 else ("gemm_pair_kernel" if M > 128 and N > 128 else "gemm_kernel")
        desc = {"gemm_decode_kernel": "gemm_decode_kernel (tcgen05 mxf4nvf4, 128-row weight tiles)",
                "gemm_pair_kernel": "gemm_pair_kernel (tcgen05 cta_group::2 mxf4nvf4)",
                "gemm_kernel": "gemm_kernel (tcgen05 mxf4nvf4)"}[tag]
        if group == "linear":
            desc = "quantize_kernel + " + desc + " (one nvfp4_linear call)"
        if group.startswith("linear_lora"):
            tag += "_lora"
            desc = ("lora_down_kernel + quantize_kernel + " + desc +
                    " with the low-rank MMAs in the FP4 accumulator (one nvfp4_linear_lora call)")
        return tag, desc
    if group.startswith("quantize"):
        return "quantize_kernel", "amax_kernel + quantize_kernel"
    return "dequantize_kernel", "dequantize_kernel"


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


def profiled_traffic(tag: str, workload: str, group: str):
    """DRAM bytes per launch of a group's dominant kernel from the committed ncu summary
    profiles/<kernel>_<workload>_<group>.md, only if it was taken on the current kernel
    sources (the summary records their hash)."""
    path = os.path.join(ROOT, "profiles", f"{tag}_{workload}_{group}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_hash") != source_hash(KERNEL_FAMILY[tag]):
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
        self.lines = []

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


def job_throughput(world: int, steps: int, work_per_step: float, ms: float, scale: float = 1e12) -> float:
    """Whole-job rate under weak scaling: every rank runs `steps` steps of its own
    problem, timed as the slowest rank's `ms` (scale 1e12: TFLOP/s, 1e9: GB/s)."""
    return world * steps * work_per_step / (ms * 1e-3) / scale


# ------------------------------------------------------------------------------------------------
# the workloads: inputs, kernel groups and their algorithmic work
# ------------------------------------------------------------------------------------------------

def gemm_work(M, N, K):
    """FLOPs and algorithmic HBM bytes of one W4A4 GEMM launch (codes + scales of both
    operands once, C written once in BF16)."""
    return {"flops": 2.0 * M * N * K, "bytes": (M + N) * K * 0.5625 + 2.0 * M * N}


def lora_work(M, N, K, R):
    """The low-rank linear layer's FLOPs (W4A4 GEMM plus both low-rank products) and
    algorithmic bytes (weight codes and scales, X in BF16, the factors, t, C)."""
    w = gemm_work(M, N, K)
    return {"flops": w["flops"] + 2.0 * M * K * R + 2.0 * M * N * R,
            "bytes": N * K * 0.5625 + M * K * 2.0 + (R * K + N * R) * 2.0 + 2.0 * M * N}


def host_inputs(cfg, seed: int, rank: int):
    """The workload's seeded BF16 host tensors."""
    import workloads as W
    s = seed + 1000 * rank
    k = cfg["kind"]
    if k == "dense31b":
        return {"W": W.t4_weight(cfg["N1"], cfg["K1"], seed=s, stream=W.STREAM_W),
                "W2": W.t4_weight(cfg["N2"], cfg["K2"], seed=s, stream=W.STREAM_W2),
                "X": W.activation(cfg["M"], cfg["K1"], seed=s, stream=W.STREAM_X, n_outlier_channels=0),
                "X2": W.activation(cfg["M"], cfg["K2"], seed=s, stream=W.STREAM_X2, n_outlier_channels=0)}
    if k in ("prefill_lora", "decode_lora"):
        base = host_inputs({**cfg, "kind": k.split("_")[0]}, seed, rank)
        R = cfg["R"]
        for suf, (n, kk) in ((("_up", (cfg["N_up"], cfg["K_up"])), ("_down", (cfg["N_down"], cfg["K_down"])))
                             if k == "prefill_lora" else (("", (cfg["N"], cfg["K"])),)):
            base["A" + suf] = W.to_bf16(W.normal((R, kk), s, 11, 0.02))
            base["B" + suf] = W.to_bf16(W.normal((n, R), s, 12, 0.1))
        return base
    if k == "prefill":
        return {"W_up": W.gaussian_weight(cfg["N_up"], cfg["K_up"], 0.02, seed=s, stream=W.STREAM_W),
                "W_down": W.gaussian_weight(cfg["N_down"], cfg["K_down"], 0.02, seed=s, stream=W.STREAM_W2),
                "X_up": W.activation(cfg["M"], cfg["K_up"], seed=s, stream=W.STREAM_X),
                "X_down": W.activation(cfg["M"], cfg["K_down"], seed=s, stream=W.STREAM_X2)}
    if k == "decode":
        return {"W": W.gaussian_weight(cfg["N"], cfg["K"], 0.02, seed=s, stream=W.STREAM_W),
                "X": W.activation(cfg["M"], cfg["K"], seed=s + cfg["M"], stream=W.STREAM_X)}
    if k == "mse":
        return {"W": W.mse_weight(cfg["rows"], cfg["cols"], seed=s)}
    if k == "pr1":
        d = W.pr1(seed=s)
        return {"W": d["w"], "X": d["x"]}
    raise ValueError(k)


# Each step's inputs copied from the host in the end-to-end measurement (weights that
# the step only reads are resident model parameters), and the results read back.
E2E_INPUTS = {"dense31b": ["W", "W2", "X", "X2"], "prefill": ["X_up", "X_down"], "decode": ["X"],
              "mse": ["W"], "pr1": ["W", "X"], "prefill_lora": ["X_up", "X_down"], "decode_lora": ["X"]}


def describe(cfg):
    k = cfg["kind"]
    return {
        "dense31b": "MSE-quantize W, W2; absmax-quantize X, X2; C1 = X W^T; C2 = X2 W2^T; dequantize X",
        "prefill": "absmax-quantize X_up, C_up = X_up W_up^T; absmax-quantize X_down, C_down = X_down W_down^T "
                   "(weights MSE-quantized once before timing)",
        "decode": "C = Q(X) W^T in one kernel: X's absmax block scales computed on the fly under a calibrated "
                  "per-tensor scale (weight MSE-quantized once before timing)",
        "mse": "MSE-quantize W (8 candidate scales, global scale computed in the step)",
        "decode_lora": f"C = Q(X) W^T + (X A^T) B^T, rank {cfg.get('R')}: the low-rank down-projection, then one "
                       "kernel quantizing X and adding B t to the FP4 accumulator (calibrated activation scale)",
        "prefill_lora": f"up and down projections with a rank-{cfg.get('R')} low-rank branch: down-projection, "
                        "absmax quantization of X, CTA-pair GEMM with the low-rank MMAs (calibrated activation scale)",
        "pr1": "absmax-quantize W and X, C = X W^T",
    }[k]


class Replica:
    """One copy of a step's device buffers and its kernel groups (C-ABI calls)."""

    def __init__(self, cfg, host, device, nv):
        import torch
        self.nv = nv
        self.cfg = cfg
        self.x = {k: v.to(device) for k, v in host.items()}
        k = cfg["kind"]
        self.out = {}
        self.ws = {}
        q = self.q = {}
        if k == "dense31b":
            M = cfg["M"]
            q["W"] = nv.nvfp4_quantize(self.x["W"], "mse")
            q["W2"] = nv.nvfp4_quantize(self.x["W2"], "mse")
            q["X"] = nv.nvfp4_quantize(self.x["X"], "absmax")
            q["X2"] = nv.nvfp4_quantize(self.x["X2"], "absmax")
            self.out["C1"] = torch.empty((M, cfg["N1"]), dtype=torch.bfloat16, device=device)
            self.out["C2"] = torch.empty((M, cfg["N2"]), dtype=torch.bfloat16, device=device)
            self.out["Xhat"] = torch.empty((M, cfg["K1"]), dtype=torch.bfloat16, device=device)
            self._ws(device, [("g1", M, cfg["N1"], cfg["K1"]), ("g2", M, cfg["N2"], cfg["K2"])],
                     ["W", "W2", "X", "X2"])
        elif k == "prefill":
            M = cfg["M"]
            q["W_up"] = nv.nvfp4_quantize(self.x["W_up"], "mse")
            q["W_down"] = nv.nvfp4_quantize(self.x["W_down"], "mse")
            q["X_up"] = nv.nvfp4_quantize(self.x["X_up"], "absmax")
            q["X_down"] = nv.nvfp4_quantize(self.x["X_down"], "absmax")
            self.out["C_up"] = torch.empty((M, cfg["N_up"]), dtype=torch.bfloat16, device=device)
            self.out["C_down"] = torch.empty((M, cfg["N_down"]), dtype=torch.bfloat16, device=device)
            self._ws(device, [("g_up", M, cfg["N_up"], cfg["K_up"]), ("g_down", M, cfg["N_down"], cfg["K_down"])],
                     ["X_up", "X_down"])
        elif k == "decode":
            q["W"] = nv.nvfp4_quantize(self.x["W"], "mse")
            # the activation's per-tensor scale, calibrated once (amax / 2688 of a sample
            # activation); the block scales are computed on every call
            self.x_scale = nv.nvfp4_quantize(self.x["X"], "absmax").global_scale.clone()
            self.out["C"] = torch.empty((cfg["M"], cfg["N"]), dtype=torch.bfloat16, device=device)
            self.ws["lin"] = torch.empty(nv.load_library().nvfp4_linear_workspace_bytes(cfg["M"], cfg["N"], cfg["K"]),
                                         dtype=torch.uint8, device=device)
        elif k == "mse":
            q["W"] = nv.nvfp4_quantize(self.x["W"], "mse", block_err=True)
            self._ws(device, [], ["W"])
        elif k in ("decode_lora", "prefill_lora"):
            lib = nv.load_library()
            R = cfg["R"]
            self.x_scale = {}
            sufs = [("_up", cfg.get("N_up"), cfg.get("K_up")), ("_down", cfg.get("N_down"), cfg.get("K_down"))] \
                if k == "prefill_lora" else [("", cfg["N"], cfg["K"])]
            for suf, n, kk in sufs:
                q["W" + suf] = nv.nvfp4_quantize(self.x["W" + suf], "mse")
                self.x_scale[suf] = nv.nvfp4_quantize(self.x["X" + suf], "absmax").global_scale.clone()
                self.out["C" + suf] = torch.empty((cfg["M"], n), dtype=torch.bfloat16, device=device)
                self.ws["lin" + suf] = torch.empty(lib.nvfp4_linear_lora_workspace_bytes(cfg["M"], n, kk, R),
                                                   dtype=torch.uint8, device=device)
        elif k == "pr1":
            q["W"] = nv.nvfp4_quantize(self.x["W"], "absmax")
            q["X"] = nv.nvfp4_quantize(self.x["X"], "absmax")
            self.out["C"] = torch.empty((cfg["M"], cfg["N"]), dtype=torch.bfloat16, device=device)
            self._ws(device, [("g", cfg["M"], cfg["N"], cfg["K"])], ["W", "X"])

    def _ws(self, device, gemms, quants):
        import torch
        lib = self.nv.load_library()
        for name, M, N, K in gemms:
            self.ws[name] = torch.empty(lib.nvfp4_gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device=device)
        for name in quants:
            self.ws[name] = torch.empty(256, dtype=torch.uint8, device=device)

    def nbytes(self):
        t = 0
        for d in (self.x, self.out, self.ws):
            t += sum(v.numel() * v.element_size() for v in d.values())
        for v in self.q.values():
            t += v.nbytes()
        return t

    def _quant(self, name, mode):
        nv = self.nv
        return lambda: nv.nvfp4_quantize(self.x[name], mode, out=self.q[name], workspace=self.ws[name])

    def _lora(self, suf):
        nv = self.nv
        return lambda: nv.linear_lora(self.x["X" + suf], self.q["W" + suf], self.x["A" + suf], self.x["B" + suf],
                                      x_global_scale=self.x_scale[suf], out=self.out["C" + suf],
                                      workspace=self.ws["lin" + suf])

    def _gemm(self, a, b, c, ws):
        nv = self.nv
        return lambda: nv.nvfp4_gemm(self.q[a], self.q[b], out=self.out[c], workspace=self.ws[ws])

    def groups(self):
        """[(name, callable, work, kernel family)] in step order."""
        nv, cfg, k = self.nv, self.cfg, self.cfg["kind"]

        def qwork(name):
            return {"bytes": self.x[name].numel() * QUANT_BPE_TWO_PASS}

        if k == "dense31b":
            M = cfg["M"]
            return [
                ("quantize_mse_W", self._quant("W", "mse"), qwork("W"), "quantize"),
                ("quantize_mse_W2", self._quant("W2", "mse"), qwork("W2"), "quantize"),
                ("quantize_absmax_X", self._quant("X", "absmax"), qwork("X"), "quantize"),
                ("quantize_absmax_X2", self._quant("X2", "absmax"), qwork("X2"), "quantize"),
                ("gemm_1", self._gemm("X", "W", "C1", "g1"), gemm_work(M, cfg["N1"], cfg["K1"]), "gemm"),
                ("gemm_2", self._gemm("X2", "W2", "C2", "g2"), gemm_work(M, cfg["N2"], cfg["K2"]), "gemm"),
                ("dequantize_X", lambda: nv.nvfp4_dequantize(self.q["X"], out=self.out["Xhat"]),
                 {"bytes": self.x["X"].numel() * DEQUANT_BPE}, "quantize"),
            ]
        if k == "prefill":
            M = cfg["M"]
            return [
                ("quantize_absmax_X_up", self._quant("X_up", "absmax"), qwork("X_up"), "quantize"),
                ("gemm_up", self._gemm("X_up", "W_up", "C_up", "g_up"), gemm_work(M, cfg["N_up"], cfg["K_up"]),
                 "gemm"),
                ("quantize_absmax_X_down", self._quant("X_down", "absmax"), qwork("X_down"), "quantize"),
                ("gemm_down", self._gemm("X_down", "W_down", "C_down", "g_down"),
                 gemm_work(M, cfg["N_down"], cfg["K_down"]), "gemm"),
            ]
        if k == "decode":
            M, N, K = cfg["M"], cfg["N"], cfg["K"]
            work = gemm_work(M, N, K)
            work = {"flops": work["flops"], "bytes": work["bytes"] - M * K * 0.5625 + M * K * 2.0}
            return [("linear", lambda: nv.linear(self.x["X"], self.q["W"], x_global_scale=self.x_scale,
                                                 out=self.out["C"], workspace=self.ws["lin"]), work, "gemm")]
        if k in ("decode_lora", "prefill_lora"):
            out = []
            sufs = [("_up", cfg["N_up"], cfg["K_up"]), ("_down", cfg["N_down"], cfg["K_down"])] \
                if k == "prefill_lora" else [("", cfg["N"], cfg["K"])]
            for suf, n, kk in sufs:
                out.append(("linear_lora" + suf, self._lora(suf), lora_work(cfg["M"], n, kk, cfg["R"]), "gemm"))
            return out
        if k == "mse":
            return [("quantize_mse_W", lambda: nv.nvfp4_quantize(self.x["W"], "mse", out=self.q["W"],
                                                                 workspace=self.ws["W"]), qwork("W"), "quantize")]
        if k == "pr1":
            return [
                ("quantize_absmax_W", self._quant("W", "absmax"), qwork("W"), "quantize"),
                ("quantize_absmax_X", self._quant("X", "absmax"), qwork("X"), "quantize"),
                ("gemm", self._gemm("X", "W", "C", "g"), gemm_work(cfg["M"], cfg["N"], cfg["K"]), "gemm"),
            ]
        raise ValueError(k)

    def results(self):
        """Device tensors the end-to-end measurement reads back after each step."""
        k = self.cfg["kind"]
        if k == "mse":
            return [self.q["W"].codes, self.q["W"].scales]
        return [v for name, v in self.out.items() if name != "Xhat"]


def step_units(cfg, groups):
    """(total work of one step, unit, scale): GEMM FLOPs in TFLOP/s where the step has a
    compute-bound GEMM, otherwise algorithmic bytes in GB/s."""
    k = cfg["kind"]
    if k in ("decode", "mse", "decode_lora"):
        return sum(w["bytes"] for _, _, w, _ in groups), "GB/s", 1e9
    return sum(w.get("flops", 0.0) for _, _, w, fam in groups if fam == "gemm"), "TFLOP/s", 1e12


def group_rate(work, us, peaks, long_region):
    """A group's achieved rate and its roofline: the slower of its tensor time and its
    HBM time decides the bound."""
    bf16 = peaks["bf16_sust"] if long_region else peaks["bf16"]
    fp4 = bf16 * FP4_PER_BF16
    t_tensor = work.get("flops", 0.0) / (fp4 * 1e12)
    t_hbm = work.get("bytes", 0.0) / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm and work.get("flops"):
        ach = work["flops"] / (us * 1e-6) / 1e12
        return {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp4, 1), "unit": "TFLOP/s",
                "frac": round(ach / fp4, 4),
                "peak_source": f"{peaks['source']} bf16 {'sustained' if long_region else 'burst'} x {FP4_PER_BF16:g}"}
    ach = work["bytes"] / (us * 1e-6) / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4), "peak_source": f"{peaks['source']} HBM copy bandwidth"}


def config_of(workload, world):
    cfg = WORKLOADS[workload]
    batch = cfg.get("M", cfg.get("rows"))
    return {"workload": workload, **{k: v for k, v in cfg.items() if k != "kind"},
            "global_batch": batch * world, "parallelism": f"independent replicas x{world}",
            "step": describe(cfg)}


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------

def run_ours(args, rank, world, local, host):
    import torch
    import w4a4_gemm_quantize_b200 as nv
    nv.load_library()
    device = torch.device("cuda", local)
    cfg = WORKLOADS[args.workload]
    first = Replica(cfg, host, device, nv)
    foot = first.nbytes()
    flush = None
    if cfg["kind"] == "pr1":
        reps = [first]
        flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=device)
        l2_note = "L2 flushed (256 MB write) before every step, outside the step's events"
    elif foot < 2 * L2_BYTES:
        n = math.ceil(2 * L2_BYTES / foot) + 1
        reps = [first] + [Replica(cfg, host, device, nv) for _ in range(n - 1)]
        l2_note = f"{n} copies of the step's buffers used in turn ({foot / 1e6:.1f} MB each), so no step finds its data in L2"
    else:
        reps = [first]
        l2_note = f"inputs larger than L2 (the step touches {foot / 1e6:.0f} MB)"
    stream = torch.cuda.current_stream(device)
    names = [g[0] for g in first.groups()]
    works = {g[0]: g[2] for g in first.groups()}
    families = {g[0]: g[3] for g in first.groups()}

    # Every kernel group runs as a CUDA graph of its C-ABI calls (captured after a first
    # direct call), so the step's device time is the kernels', not the host's launch
    # overhead; programmatic dependent launch carries into the graph's edges.
    for rep in reps:
        for _, fn, _, _ in rep.groups():
            fn()
    torch.cuda.synchronize(device)
    graphs, counts = [], []
    for rep in reps:
        gs, cs = {}, {}
        for name, fn, _, _ in rep.groups():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
                cs[name] = nv.last_launch_count()
            gs[name] = g
        graphs.append(gs)
        counts.append(cs)
    torch.cuda.synchronize(device)

    def run_step(i, events=None):
        gs, n = graphs[i % len(reps)], 0
        for name in names:
            if events is not None:
                events[name][0].record(stream)
            gs[name].replay()
            n += counts[i % len(reps)][name]
            if events is not None:
                events[name][1].record(stream)
        return n

    for i in range(max(args.warmup, 3)):
        if flush is not None:
            flush.zero_()
        run_step(i)
    torch.cuda.synchronize(device)
    barrier(world)

    ev_all = []
    launches = 0
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize(device)
        t_start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            ev = {n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for n in names}
            launches += run_step(i, ev)
            ev_all.append(ev)
        t_end.record(stream)
        torch.cuda.synchronize(device)
        barrier(world)
    if flush is None:
        ms_local = t_start.elapsed_time(t_end)
    else:  # the steps' own spans, without the flushes between them
        ms_local = sum(e[names[0]][0].elapsed_time(e[names[-1]][1]) for e in ev_all)
    ms = max_over_ranks(ms_local, world, device)
    per_group = {n: statistics.mean(e[n][0].elapsed_time(e[n][1]) for e in ev_all) * 1e3 for n in names}  # us

    peaks = load_peaks()
    groups = first.groups()
    work, unit, scale = step_units(cfg, groups)
    value = job_throughput(world, args.steps, work, ms, scale)
    step_ms = ms / args.steps
    long_region = ms * 1e-3 > 1.0
    comps = {}
    for n in names:
        r = group_rate(works[n], per_group[n], peaks, long_region)
        comps[n] = {"us": round(per_group[n], 2), r["unit"]: r["achieved"], "frac": r["frac"], "bound": r["bound"]}
    dom = max(names, key=lambda n: per_group[n])
    roof = group_rate(works[dom], per_group[dom], peaks, long_region)
    tag, kname = group_kernel(dom, cfg, families[dom])
    roof.update({"traffic": profiled_traffic(tag, args.workload, dom),
                 "kernel": f"{kname}, group {dom}", "group_share_of_step": round(per_group[dom] / (step_ms * 1e3), 4)})
    roof = {k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic", "kernel", "peak_source",
                                 "group_share_of_step")}
    extra = {}
    if cfg["kind"] == "mse":
        extra = mse_vs_absmax(first, nv)

    e2e = run_e2e(args, first, host, device, world, cfg, groups) if args.e2e_steps > 0 else None
    out = {
        "metric": METRIC,
        "value": round(value, 3), "unit": unit, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 codes, e4m3 block scales, fp32 accumulation, bf16 out)", "data": "synthetic",
        "config": {**config_of(args.workload, world), "l2": l2_note},
        "roofline": roof, "components": comps, "gpu_launches": launches,
        "clocks": clk.summary(), "e2e": e2e, "cpu_baseline": None, **extra,
    }
    return out


def mse_vs_absmax(rep, nv):
    """Mean per-block squared error of the MSE and absmax scale choices on the weight."""
    qa = nv.nvfp4_quantize(rep.x["W"], "absmax", block_err=True)
    qm = nv.nvfp4_quantize(rep.x["W"], "mse", block_err=True)
    ea, em = qa.block_err.double().mean().item(), qm.block_err.double().mean().item()
    return {"block_sse": {"absmax_mean": ea, "mse_mean": em, "ratio_absmax_over_mse": ea / em if em else None}}


def run_e2e(args, rep, host, device, world, cfg, groups):
    """The same step from pinned host buffers: H2D inputs, C-ABI calls, D2H results, all timed."""
    import torch
    names = E2E_INPUTS[cfg["kind"]]
    host_in = {k: host[k].pin_memory() for k in names}
    outs = rep.results()
    host_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    stream = torch.cuda.current_stream(device)

    def one():
        for k, v in host_in.items():
            rep.x[k].copy_(v, non_blocking=True)
        for _, fn, _, _ in rep.groups():
            fn()
        for h, o in zip(host_out, outs):
            h.copy_(o, non_blocking=True)

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
    work, unit, scale = step_units(cfg, groups)
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(h.numel() * h.element_size() for h in host_out)
    return {"value": round(job_throughput(world, args.e2e_steps, work, ms, scale), 4), "unit": unit,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
            "ms_per_step": round(ms / args.e2e_steps, 4)}


# ------------------------------------------------------------------------------------------------
# the CPU oracle on a bounded sample of the same step (cpu_baseline and --impl reference)
# ------------------------------------------------------------------------------------------------

def _split_rows(n, parts):
    import numpy as np
    b = np.linspace(0, n, min(n, parts) + 1).astype(np.int64)
    return [(int(x), int(y)) for x, y in zip(b[:-1], b[1:]) if y > x]


class OracleStep:
    """The workload's step on the CPU oracle (``threads`` host threads; the oracle's C
    code runs without the Python lock).  Each part is timed on a sample sized to the
    budget -- the whole tensor where that fits -- and extrapolated by its share of
    rows or outputs."""

    def __init__(self, cfg, host, threads, budget_s):
        import numpy as np
        import oracle
        import workloads
        self.np, self.oracle = np, oracle
        self.cfg, self.threads, self.budget = cfg, threads, budget_s
        self.bits = {k: workloads.bf16_bits(v) for k, v in host.items()}
        oracle.build()
        oracle.e4m3_encode(1.0)  # fill the oracle's table before threads share it
        self.parts = []   # (name, sampled units, full units, seconds)

    def _pool_map(self, fn, items):
        if self.threads == 1 or len(items) == 1:
            return [fn(x) for x in items]
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(self.threads) as ex:
            return list(ex.map(fn, items))

    def quantize(self, name, mode, share):
        """Global scale over the whole tensor (cheap), then the encode on a row sample."""
        np, oracle = self.np, self.oracle
        bits = self.bits[name]
        rows = bits.shape[0]
        t0 = time.perf_counter()
        sg = oracle.global_scale(bits)
        t_amax = time.perf_counter() - t0
        # calibrate on one row per thread, then size the sample to the part's budget share
        probe = min(rows, self.threads)
        t0 = time.perf_counter()
        self._pool_map(lambda ab: oracle.quantize(np.ascontiguousarray(bits[ab[0]:ab[1]]), mode, sg),
                       _split_rows(probe, self.threads))
        per_row = (time.perf_counter() - t0) / probe
        n = int(min(rows, max(probe, self.budget * share / max(per_row, 1e-9))))
        t0 = time.perf_counter()
        res = self._pool_map(lambda ab: oracle.quantize(np.ascontiguousarray(bits[ab[0]:ab[1]]), mode, sg),
                             _split_rows(n, self.threads * 2))
        t = time.perf_counter() - t0
        codes = np.concatenate([r[0] for r in res])
        scales = np.concatenate([r[1] for r in res])
        self.parts.append((f"quantize {name}", n, rows, t_amax + t * rows / n))
        return codes, scales, sg

    def gemm(self, name, a, b, M, N, share):
        """Sampled outputs among the quantized sample rows of both operands."""
        np, oracle = self.np, self.oracle
        ra, rb = a[0].shape[0], b[0].shape[0]
        r = np.random.default_rng(0)
        probe = 64
        mi, ni = r.integers(0, ra, probe), r.integers(0, rb, probe)
        t0 = time.perf_counter()
        oracle.gemm_f64_at(*a, *b, mi, ni)
        per_out = (time.perf_counter() - t0) / probe / self.threads
        n = int(min(M * N, max(probe, self.budget * share / max(per_out, 1e-12))))
        mi, ni = r.integers(0, ra, n), r.integers(0, rb, n)
        chunks = np.array_split(np.arange(n), self.threads * 2)
        t0 = time.perf_counter()
        self._pool_map(lambda ii: oracle.gemm_f64_at(*a, *b, mi[ii], ni[ii]), [c for c in chunks if c.size])
        t = time.perf_counter() - t0
        self.parts.append((name, n, M * N, t * (M * N) / n))

    def lora(self, name, suf, M, share):
        """The low-rank term on a row sample (t for the rows, then t B^T for all columns)."""
        np, oracle = self.np, self.oracle
        x, A, B = self.bits["X" + suf], self.bits["A" + suf], self.bits["B" + suf]
        t0 = time.perf_counter()
        oracle.lora_f64(np.ascontiguousarray(x[:1]), A, B)
        per_row = time.perf_counter() - t0
        n = int(min(M, max(self.threads, self.budget * share * self.threads / max(per_row, 1e-9))))
        t0 = time.perf_counter()
        self._pool_map(lambda ab: oracle.lora_f64(np.ascontiguousarray(x[ab[0]:ab[1]]), A, B),
                       _split_rows(n, self.threads))
        t = time.perf_counter() - t0
        self.parts.append((name, n, M, t * M / n))

    def dequantize(self, name, q, rows_full):
        np, oracle = self.np, self.oracle
        codes, scales, sg = q
        t0 = time.perf_counter()
        self._pool_map(lambda ab: oracle.dequantize(codes[ab[0]:ab[1]], scales[ab[0]:ab[1]], sg),
                       _split_rows(codes.shape[0], self.threads))
        t = time.perf_counter() - t0
        self.parts.append((name, codes.shape[0], rows_full, t * rows_full / codes.shape[0]))

    def run(self):
        o, cfg, k = self.oracle, self.cfg, self.cfg["kind"]
        self.parts = []
        if k == "dense31b":
            w = self.quantize("W", o.SCALE_MSE, 0.3)
            w2 = self.quantize("W2", o.SCALE_MSE, 0.3)
            x = self.quantize("X", o.SCALE_ABSMAX, 0.05)
            x2 = self.quantize("X2", o.SCALE_ABSMAX, 0.05)
            self.gemm("gemm_1", x, w, cfg["M"], cfg["N1"], 0.14)
            self.gemm("gemm_2", x2, w2, cfg["M"], cfg["N2"], 0.14)
            self.dequantize("dequantize X", x, cfg["M"])
        elif k == "prefill":
            xu = self.quantize("X_up", o.SCALE_ABSMAX, 0.15)
            xd = self.quantize("X_down", o.SCALE_ABSMAX, 0.15)
            wu = self.quantize("W_up", o.SCALE_ABSMAX, 0.05)    # operands for the GEMM sample (not timed in the step)
            wd = self.quantize("W_down", o.SCALE_ABSMAX, 0.05)
            self.parts = [p for p in self.parts if not p[0].startswith("quantize W")]
            self.gemm("gemm_up", xu, wu, cfg["M"], cfg["N_up"], 0.3)
            self.gemm("gemm_down", xd, wd, cfg["M"], cfg["N_down"], 0.3)
        elif k == "decode":
            x = self.quantize("X", o.SCALE_ABSMAX, 0.1)
            wq = self.quantize("W", o.SCALE_ABSMAX, 0.2)
            self.parts = [p for p in self.parts if p[0] != "quantize W"]
            self.gemm("gemm", x, wq, cfg["M"], cfg["N"], 0.7)
        elif k in ("decode_lora", "prefill_lora"):
            sufs = [("_up", "N_up"), ("_down", "N_down")] if k == "prefill_lora" else [("", "N")]
            for suf, nkey in sufs:
                xq = self.quantize("X" + suf, o.SCALE_ABSMAX, 0.1 / len(sufs))
                wq = self.quantize("W" + suf, o.SCALE_ABSMAX, 0.1 / len(sufs))
                self.parts = [p for p in self.parts if p[0] != "quantize W" + suf]
                self.gemm("gemm" + suf, xq, wq, cfg["M"], cfg[nkey], 0.5 / len(sufs))
                self.lora("lora" + suf, suf, cfg["M"], 0.3 / len(sufs))
        elif k == "mse":
            self.quantize("W", o.SCALE_MSE, 1.0)
        elif k == "pr1":
            wq = self.quantize("W", o.SCALE_ABSMAX, 0.3)
            xq = self.quantize("X", o.SCALE_ABSMAX, 0.1)
            self.gemm("gemm", xq, wq, cfg["M"], cfg["N"], 0.6)
        return sum(p[3] for p in self.parts)

    def describe(self):
        s = "; ".join(f"{n}: {u} of {f} {'rows' if n.startswith(('quantize', 'dequantize', 'lora')) else 'outputs'}"
                      for n, u, f, _ in self.parts)
        return f"oracle on {self.threads} host thread(s): {s}; each part extrapolated to the full step"

    def extrapolated(self):
        return any(u < f for _, u, f, _ in self.parts)


def oracle_rate(cfg, step_seconds):
    """The oracle's rate in the workload's unit (work per extrapolated step time)."""
    work, unit, scale = step_units(cfg, _static_groups(cfg))
    return work / step_seconds / scale, unit


def _static_groups(cfg):
    """The workload's groups with their algorithmic work, without device buffers."""
    k = cfg["kind"]

    def q(rows, cols):
        return {"bytes": rows * cols * QUANT_BPE_TWO_PASS}

    if k == "dense31b":
        M = cfg["M"]
        return [("quantize_mse_W", None, q(cfg["N1"], cfg["K1"]), "quantize"),
                ("quantize_mse_W2", None, q(cfg["N2"], cfg["K2"]), "quantize"),
                ("quantize_absmax_X", None, q(M, cfg["K1"]), "quantize"),
                ("quantize_absmax_X2", None, q(M, cfg["K2"]), "quantize"),
                ("gemm_1", None, gemm_work(M, cfg["N1"], cfg["K1"]), "gemm"),
                ("gemm_2", None, gemm_work(M, cfg["N2"], cfg["K2"]), "gemm"),
                ("dequantize_X", None, {"bytes": M * cfg["K1"] * DEQUANT_BPE}, "quantize")]
    if k == "prefill":
        M = cfg["M"]
        return [("quantize_absmax_X_up", None, q(M, cfg["K_up"]), "quantize"),
                ("gemm_up", None, gemm_work(M, cfg["N_up"], cfg["K_up"]), "gemm"),
                ("quantize_absmax_X_down", None, q(M, cfg["K_down"]), "quantize"),
                ("gemm_down", None, gemm_work(M, cfg["N_down"], cfg["K_down"]), "gemm")]
    if k == "decode":
        M, N, K = cfg["M"], cfg["N"], cfg["K"]
        w = gemm_work(M, N, K)
        return [("linear", None, {"flops": w["flops"], "bytes": w["bytes"] - M * K * 0.5625 + M * K * 2.0}, "gemm")]
    if k == "decode_lora":
        return [("linear_lora", None, lora_work(cfg["M"], cfg["N"], cfg["K"], cfg["R"]), "gemm")]
    if k == "prefill_lora":
        return [("linear_lora_up", None, lora_work(cfg["M"], cfg["N_up"], cfg["K_up"], cfg["R"]), "gemm"),
                ("linear_lora_down", None, lora_work(cfg["M"], cfg["N_down"], cfg["K_down"], cfg["R"]), "gemm")]
    if k == "mse":
        return [("quantize_mse_W", None, q(cfg["rows"], cfg["cols"]), "quantize")]
    if k == "pr1":
        return [("quantize_absmax_W", None, q(cfg["N"], cfg["K"]), "quantize"),
                ("quantize_absmax_X", None, q(cfg["M"], cfg["K"]), "quantize"),
                ("gemm", None, gemm_work(cfg["M"], cfg["N"], cfg["K"]), "gemm")]
    raise ValueError(k)


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(cfg, host, budget_s):
    """The oracle timed on one thread and on every host core (same sample rules)."""
    cores = host_cores()
    legs = {}
    for threads, share in ((1, 0.4), (cores, 0.6)):
        st = OracleStep(cfg, host, threads, budget_s * share)
        est = st.run()
        value, unit = oracle_rate(cfg, est)
        legs[threads] = {"value": value, "unit": unit, "threads": threads, "sample": st.describe(),
                         "extrapolated": st.extrapolated(), "step_seconds": round(est, 3)}
    allc = legs[cores]
    return {"value": allc["value"], "unit": allc["unit"], "cores": cores, "kind": "oracle",
            "sample": allc["sample"], "extrapolated": allc["extrapolated"],
            "step_seconds": allc["step_seconds"], "host_cores": cores, "nproc": os.cpu_count(),
            "single_thread": legs[1]}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on every host core, rank 0 only."""
    cfg = WORKLOADS[args.workload]
    if rank != 0:
        return None
    host = host_inputs(cfg, args.seed, 0)
    cores = host_cores()
    budget = getattr(args, "cpu_seconds", 12.0) / 4  # per step: K + W steps stay within a few minutes
    st = OracleStep(cfg, host, cores, budget)
    for _ in range(args.warmup):
        st.run()
    ests = []
    for _ in range(args.steps):
        ests.append(st.run())
    est = statistics.mean(ests) if ests else st.run()
    value, unit = oracle_rate(cfg, est)
    base = {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": st.describe(),
            "extrapolated": st.extrapolated(), "nproc": os.cpu_count()}
    return {
        "impl": "reference", "metric": METRIC,
        "value": value, "unit": unit, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(est * 1e3, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 GEMM reference, binary32 quantizer (CPU oracle)", "data": "synthetic",
        "config": config_of(args.workload, world),
        "extrapolated": st.extrapolated(),
        "cpu_baseline": base,
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            out = run_reference(args, rank, world)
        else:
            cfg = WORKLOADS[args.workload]
            host = host_inputs(cfg, args.seed, rank)
            out = run_ours(args, rank, world, local, host)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(cfg, host, args.cpu_seconds)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
