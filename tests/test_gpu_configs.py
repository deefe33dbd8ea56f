"""GPU parity on the full-size workloads that the benchmark runs.

* 31B-class dense layer: W 21504 x 5376 and W2 5376 x 21504 (0.015 Student-t(4),
  MSE block scales), X ~ N(0,1); the W4A4 GEMM at M = 8192, 256 and 1 against
  both weights, with operands quantized by the oracle; sampled outputs, every row
  of the last 256-row tile and the full first and last 256 x 256 tiles (M = 1
  compared in full).  The GPU MSE quantizer on W2 against the oracle (sampled rows).
* The W4A4 linear layer (activation quantized on the fly, then the GEMM, one
  stream): prefill up / down projections and decode M in {1, 8, 32}, against the
  oracle's quantization of both operands and its float64 GEMM.
* Repeated launches of the CTA-pair GEMM on the prefill and 31B shapes give
  bit-identical results (a race between the kernel's roles would show as a
  difference between launches).

Sources: the page "NVFP4 en difusión: la misma cuantización, un motor
completamente distinto", section 2 "NVFP4 sin vLLM: torch._scaled_mm a mano"
(out = (A s_a)(B s_b)^T, activation quantized at runtime); the 31B-class layer
is the page "Tu pipeline NVFP4: meter 62 GB de modelo en 24 GB de laptop"
(Gemma-4 31B) as a shape.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_quantize_b200 as nv
from helpers import check_gemm, check_gemm_large, gemm_ref_block, operand, oracle_quantize, upload

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=None)
def dense31b_operands():
    w = workloads.t4_weight(21504, 5376, seed=0, stream=workloads.STREAM_W)
    w2 = workloads.t4_weight(5376, 21504, seed=0, stream=workloads.STREAM_W2)
    return {"w": operand(oracle_quantize(w, oracle.SCALE_MSE)), "w2": operand(oracle_quantize(w2, oracle.SCALE_MSE))}


@functools.lru_cache(maxsize=None)
def dense31b_activation(m, k):
    stream = workloads.STREAM_X if k == 5376 else workloads.STREAM_X2
    x = workloads.activation(m, k, seed=0, stream=stream, n_outlier_channels=0)
    return operand(oracle_quantize(x, oracle.SCALE_ABSMAX))


@pytest.mark.parametrize("M", [8192, 256, 1])
@pytest.mark.parametrize("which", ["w", "w2"])
def test_dense31b_gemm(cuda_device, M, which):
    """C = X W^T (K=5376, N=21504) and X2 W2^T (K=21504, N=5376) at M = 8192, 256, 1."""
    b = dense31b_operands()[which]
    K = b[0].shape[1] * 2
    a = dense31b_activation(M, K)
    out = nv.nvfp4_gemm(upload(a), upload(b))
    torch.cuda.synchronize()
    if M == 1:
        ref, absum = gemm_ref_block(a, b, 0, 1, 0, b[0].shape[0])
        check_gemm(out.float().cpu().numpy(), ref, absum, where=f"31B M=1 {which}")
    else:
        check_gemm_large(out, a, b, where=f"31B M={M} {which}", seed=M)


def test_dense31b_w2_mse_quantize_sampled(cuda_device):
    """The GPU MSE quantizer on the second 31B weight (5376 x 21504): codes, scales,
    block errors and the global scale bit-exact with the oracle on sampled rows."""
    x = workloads.t4_weight(5376, 21504, seed=0, stream=workloads.STREAM_W2)
    q = nv.nvfp4_quantize(x.cuda(), "mse", block_err=True)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, 1, 5375], np.random.default_rng(3).choice(5376, 29, replace=False)]))
    sg = oracle.global_scale(x)
    assert q.global_scale.item() == sg
    codes, sc, _, err = oracle.quantize(np.ascontiguousarray(workloads.bf16_bits(x)[rows]), oracle.SCALE_MSE, sg)
    assert np.array_equal(q.codes.cpu().numpy()[rows], codes)
    lin = oracle.unswizzle_scales(q.scales.cpu().numpy(), 5376, 21504 // 16)
    assert np.array_equal(lin[rows], sc)
    assert np.array_equal(q.block_err.cpu().numpy()[rows].view(np.uint32), err.view(np.uint32))


# --- the W4A4 linear layer: activation quantized on the fly, then the GEMM ------------------------

@functools.lru_cache(maxsize=None)
def weight_pair(n, k, stream):
    """A 0.02-Gaussian weight: its BF16 values and the oracle's MSE quantization."""
    w = workloads.gaussian_weight(n, k, 0.02, seed=0, stream=stream)
    return w, operand(oracle_quantize(w, oracle.SCALE_MSE))


def run_linear(x, w_cpu, w_op, where):
    wq = nv.nvfp4_quantize(w_cpu.cuda(), "mse")
    out = nv.linear(x.cuda(), wq)
    torch.cuda.synchronize()
    a = operand(oracle_quantize(x, oracle.SCALE_ABSMAX))
    M, N = out.shape
    if M <= 32:
        ref, absum = gemm_ref_block(a, w_op, 0, M, 0, N)
        check_gemm(out.float().cpu().numpy(), ref, absum, where=where)
    else:
        check_gemm_large(out, a, w_op, where=where)


def test_linear_prefill_up(cuda_device):
    """Prefill up projection: X 4096 x 4096 (4 outlier channels x50), W 14336 x 4096."""
    w, w_op = weight_pair(14336, 4096, workloads.STREAM_W)
    x = workloads.activation(4096, 4096, seed=0, stream=workloads.STREAM_X)
    run_linear(x, w, w_op, "prefill up")


def test_linear_prefill_down(cuda_device):
    """Prefill down projection: X 4096 x 14336, W 4096 x 14336 (56 K-tiles)."""
    w, w_op = weight_pair(4096, 14336, workloads.STREAM_W2)
    x = workloads.activation(4096, 14336, seed=0, stream=workloads.STREAM_X2)
    run_linear(x, w, w_op, "prefill down")


@pytest.mark.parametrize("M", [1, 8, 32])
def test_linear_decode(cuda_device, M):
    """Decode: X M x 4096 with 4 outlier channels x50 against the 14336 x 4096 weight."""
    w, w_op = weight_pair(14336, 4096, workloads.STREAM_W)
    x = workloads.activation(M, 4096, seed=M, stream=workloads.STREAM_X)
    run_linear(x, w, w_op, f"decode M={M}")


# --- repeated launches are bit-identical ----------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(4096, 14336, 4096), (4096, 4096, 14336), (8192, 21504, 5376),
                                   (8192, 5376, 21504)])
def test_pair_kernel_repeated_launches_identical(cuda_device, M, N, K):
    """Ten back-to-back launches of the CTA-pair GEMM on one stream give the same bits."""
    A = nv.nvfp4_quantize(workloads.activation(M, K, seed=1, n_outlier_channels=0).cuda(), "absmax")
    B = nv.nvfp4_quantize(workloads.t4_weight(N, K, seed=1).cuda(), "absmax")
    ws = torch.empty(nv.load_library().nvfp4_gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    first = nv.nvfp4_gemm(A, B, workspace=ws)
    outs = [torch.empty_like(first) for _ in range(9)]
    for out in outs:  # enqueued back to back: each launch overlaps the previous one's tail
        nv.nvfp4_gemm(A, B, out=out, workspace=ws)
    assert nv.read_device_error(ws) == 0
    for i, out in enumerate(outs):
        assert torch.equal(out, first), f"launch {i + 2} differs from the first"
