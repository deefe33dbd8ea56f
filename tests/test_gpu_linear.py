"""GPU parity of the W4A4 linear layer: the activation quantized on the call, then
the GEMM -- nvfp4_linear through the quantizer and the GEMM (chained with
programmatic dependent launch), and for M <= 32 nvfp4_linear_fused, one kernel in
which every CTA quantizes the activation K-tiles it consumes.

Two references: the standalone path (nvfp4_quantize with absmax scales, then
nvfp4_gemm), which must give the same bits, and the oracle (its quantization of
both operands and its float64 GEMM), within the GEMM acceptance test of
``helpers.check_gemm``.  Page: "NVFP4 en difusión: la misma cuantización, un motor
completamente distinto", section 2 (the activation is quantized on every forward,
block by block, out = (A s_a)(B s_b)^T in BF16) and section 3 (quantization fused
into the matmul kernel).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_quantize_b200 as nv
from helpers import check_gemm, gemm_ref_block, operand, oracle_quantize

pytestmark = pytest.mark.gpu


def standalone(x, wq, gs=None):
    xq = nv.nvfp4_quantize(x, "absmax", "swizzled", global_scale=gs)
    return nv.nvfp4_gemm(xq, wq)


def run_case(x_cpu, w_cpu, w_mode="mse", gs=None, where="", fused=False):
    x = x_cpu.cuda()
    wq = nv.nvfp4_quantize(w_cpu.cuda(), w_mode)
    gs_t = None if gs is None else torch.tensor([gs], dtype=torch.float32, device="cuda")
    ws = torch.full((nv.load_library().nvfp4_linear_workspace_bytes(x.shape[0], w_cpu.shape[0], x.shape[1]),),
                    0x5A, dtype=torch.uint8, device="cuda")  # any content on entry
    out = nv.linear(x, wq, x_global_scale=gs_t, workspace=ws, fused=fused)
    assert nv.read_device_error(ws) == 0
    ref_out = standalone(x, wq, gs_t)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out), f"{where}: linear differs from quantize + gemm"
    a = operand(oracle_quantize(x_cpu, oracle.SCALE_ABSMAX, sg=gs))
    b = operand(oracle_quantize(w_cpu, {"mse": oracle.SCALE_MSE, "absmax": oracle.SCALE_ABSMAX}[w_mode]))
    ref, absum = gemm_ref_block(a, b, 0, x.shape[0], 0, w_cpu.shape[0])
    check_gemm(out.float().cpu().numpy(), ref, absum, where=where)
    return out


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("M,N,K", [(1, 14336, 4096), (8, 14336, 4096), (32, 14336, 4096), (7, 520, 96),
                                   (3, 136, 544), (32, 384, 8192), (24, 1000, 2080), (1, 128, 32)])
def test_small_m_matches_standalone_and_oracle(cuda_device, M, N, K, fused):
    """M <= 32 (global scale from the amax pass): ragged N, partial K-tiles, K cut into
    many stream-K segments; the fused kernel gives the same bits."""
    x = workloads.activation(M, K, seed=M + K, n_outlier_channels=min(4, K // 16))
    w = workloads.gaussian_weight(N, K, 0.02, seed=N)
    run_case(x, w, where=f"{'fused' if fused else 'linear'} {M}x{N}x{K}", fused=fused)


@pytest.mark.parametrize("fused,launches", [(False, 2), (True, 1)])
@pytest.mark.parametrize("M,N,K", [(8, 14336, 4096), (1, 520, 96), (32, 136, 544)])
def test_small_m_with_given_global_scale(cuda_device, M, N, K, fused, launches):
    """A caller-supplied activation scale (as a calibrated one would be): no amax pass,
    and the same bits as nvfp4_quantize given that scale followed by nvfp4_gemm."""
    x = workloads.activation(M, K, seed=3 * M + K)
    w = workloads.gaussian_weight(N, K, 0.02, seed=N + 1)
    run_case(x, w, gs=0.0213, where=f"given scale {M}x{N}x{K} fused={fused}", fused=fused)
    gs = torch.tensor([0.0213], dtype=torch.float32, device="cuda")
    wq = nv.nvfp4_quantize(w.cuda(), "mse")
    nv.linear(x.cuda(), wq, x_global_scale=gs, fused=fused)
    assert nv.last_launch_count() == launches


@pytest.mark.parametrize("M,N,K", [(33, 520, 96), (129, 136, 544), (300, 1000, 2080)])
def test_large_m_matches_standalone_and_oracle(cuda_device, M, N, K):
    x = workloads.activation(M, K, seed=M, n_outlier_channels=2)
    w = workloads.gaussian_weight(N, K, 0.02, seed=N + 2)
    run_case(x, w, where=f"linear {M}x{N}x{K}")
    run_case(x, w, gs=0.05, where=f"linear given scale {M}x{N}x{K}")


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("M,which", [(1, "w"), (1, "w2"), (32, "w")])
def test_31b_decode_shapes(cuda_device, M, which, fused):
    """The 31B-class layer at decode sizes: K=5376 / N=21504 and K=21504 / N=5376."""
    n, k, stream = (21504, 5376, workloads.STREAM_W) if which == "w" else (5376, 21504, workloads.STREAM_W2)
    w = workloads.t4_weight(n, k, seed=0, stream=stream)
    x = workloads.activation(M, k, seed=M, n_outlier_channels=0)
    run_case(x, w, where=f"31B M={M} {which} fused={fused}", fused=fused)


@pytest.mark.parametrize("fused", [False, True])
def test_edge_values(cuda_device, fused):
    """Zero rows, -0, a huge value next to tiny ones, BF16 subnormals in the activation."""
    M, N, K = 6, 256, 256
    a = np.random.default_rng(9).standard_normal((M, K)).astype(np.float32)
    a[0] = 0.0
    a[1] = -0.0
    a[2, :16] = np.float32(1e-40)
    a[3, 7] = 3.0e4
    a[4, 100:116] = -a[4, 100:116] * 1e-30
    x = workloads.to_bf16(a)
    w = workloads.gaussian_weight(N, K, 0.02, seed=5)
    run_case(x, w, w_mode="absmax", where=f"edge values fused={fused}", fused=fused)
    z = workloads.to_bf16(np.zeros((4, K), np.float32))
    out = nv.linear(z.cuda(), nv.nvfp4_quantize(w.cuda(), "absmax"), fused=fused)
    assert not out.float().abs().sum().item()


@pytest.mark.parametrize("fused", [False, True])
def test_repeated_calls_identical(cuda_device, fused):
    """Back-to-back calls on one workspace (the tile counters reset themselves) give the
    same bits, and a different activation in between does not leak into the next call."""
    N, K = 14336, 4096
    wq = nv.nvfp4_quantize(workloads.gaussian_weight(N, K, 0.02, seed=11).cuda(), "mse")
    x1 = workloads.activation(32, K, seed=1).cuda()
    x2 = workloads.activation(32, K, seed=2, factor=500.0).cuda()
    ws = torch.empty(nv.load_library().nvfp4_linear_workspace_bytes(32, N, K), dtype=torch.uint8, device="cuda")
    first = nv.linear(x1, wq, workspace=ws, fused=fused)
    outs = []
    for i in range(6):
        outs.append(nv.linear(x2 if i % 2 else x1, wq, workspace=ws, fused=fused))
    assert nv.read_device_error(ws) == 0
    ref2 = standalone(x2, wq)
    for i, o in enumerate(outs):
        assert torch.equal(o, ref2 if i % 2 else first), f"call {i + 2}"


@pytest.mark.parametrize("M,N,K", [(7, 520, 96), (32, 136, 544), (129, 520, 96)])
def test_linear_writes_stay_in_bounds(cuda_device, M, N, K):
    """C (with ldc > N) and the workspace inside canary margins."""
    from test_gpu_bounds import FILL, Guarded
    x = workloads.activation(M, K, seed=M)
    wq = nv.nvfp4_quantize(workloads.gaussian_weight(N, K, 0.02, seed=N).cuda(), "mse")
    ldc = N + 8
    g_c = Guarded(M * ldc * 2)
    c_full = g_c.view(torch.bfloat16, (M, ldc))
    g_ws = Guarded(nv.load_library().nvfp4_linear_workspace_bytes(M, N, K))
    out = nv.linear(x.cuda(), wq, out=c_full[:, :N], workspace=g_ws.inner)
    assert nv.read_device_error(g_ws.inner) == 0
    g_c.check("C")
    g_ws.check("workspace")
    assert (c_full[:, N:].contiguous().view(torch.uint8).cpu().numpy() == FILL).all()
    assert torch.equal(out, standalone(x.cuda(), wq))
