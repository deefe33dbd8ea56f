"""Run one kernel of the library on one shape a few times (for profilers such as ncu).

    python -m w4a4_gemm_quantize_b200.profile_case gemm --M 8192 --N 21504 --K 5376 --reps 3
    python -m w4a4_gemm_quantize_b200.profile_case quantize --rows 21504 --cols 5376 --mode mse

Inputs are seeded synthetic tensors (N(0,1) activations, 0.015 * Student-t(4)
weights); only the tensors of that one call live on the device.  The first call
is a warm-up, then `reps` more launches follow.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import workloads  # noqa: E402
import w4a4_gemm_quantize_b200 as nv  # noqa: E402


def main():
    p = argparse.ArgumentParser()
    p.add_argument("kernel", choices=["gemm", "quantize", "dequantize"])
    p.add_argument("--M", type=int, default=8192)
    p.add_argument("--N", type=int, default=21504)
    p.add_argument("--K", type=int, default=5376)
    p.add_argument("--rows", type=int, default=21504)
    p.add_argument("--cols", type=int, default=5376)
    p.add_argument("--mode", choices=["absmax", "mse"], default="mse")
    p.add_argument("--given-scale", action="store_true", help="pass a global scale (no amax pass)")
    p.add_argument("--reps", type=int, default=3)
    a = p.parse_args()
    torch.cuda.set_device(0)
    if a.kernel == "gemm":
        A = nv.nvfp4_quantize(workloads.activation(a.M, a.K, n_outlier_channels=0).cuda(), "absmax")
        B = nv.nvfp4_quantize(workloads.t4_weight(a.N, a.K).cuda(), "mse")
        C = nv.nvfp4_gemm(A, B)
        for _ in range(a.reps):
            nv.nvfp4_gemm(A, B, out=C)
    else:
        x = workloads.t4_weight(a.rows, a.cols).cuda()
        q = nv.nvfp4_quantize(x, a.mode)
        gs = q.global_scale.clone() if a.given_scale else None
        if a.kernel == "quantize":
            for _ in range(a.reps):
                nv.nvfp4_quantize(x, a.mode, global_scale=gs, out=q)
        else:
            out = nv.nvfp4_dequantize(q)
            for _ in range(a.reps):
                nv.nvfp4_dequantize(q, out=out)
    torch.cuda.synchronize()
    print("done")


if __name__ == "__main__":
    main()
