"""GPU parity of the W4A4 GEMM against the oracle's float64 reference.

Operands are quantized by the oracle (so these tests do not lean on the GPU
quantizer) and uploaded; C = (A s_a)(B s_b)^T s_gA s_gB comes back in BF16 and is
checked element by element by ``helpers.check_gemm``: the stated accumulation bound
|C - ref| <= 1e-3 * S + 1e-6 (S = sum_k |a_k b_k|) plus half a BF16 ulp of C for the
output rounding, every element outside the bare bound within one ulp of
BF16_RNE(ref), and at least 90 % of the elements equal to BF16_RNE(ref).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_quantize_b200 as nv
from helpers import check_gemm, upload

pytestmark = pytest.mark.gpu


def oracle_operand(x_cpu, mode=oracle.SCALE_ABSMAX):
    codes, sc, sg, _ = oracle.quantize(x_cpu, mode)
    return codes, sc, sg


def check(c_gpu, ref, absum):
    check_gemm(c_gpu, ref, absum)


def run_full(a, b, M, N, K):
    A, B = upload(a), upload(b)
    out = nv.nvfp4_gemm(A, B)
    ws_bytes = nv.load_library().nvfp4_gemm_workspace_bytes(M, N, K)
    ws = torch.full((ws_bytes,), 0xAB, dtype=torch.uint8, device="cuda")  # content on entry is arbitrary
    out2 = nv.nvfp4_gemm(A, B, workspace=ws)
    assert nv.read_device_error(ws) == 0
    assert torch.equal(out, out2)  # deterministic
    ref, absum = oracle.gemm_f64(*a, *b)
    check(out.float().cpu().numpy(), ref, absum)
    return out


def test_pr1_reference_config(cuda_device):
    """W4A4 GEMM M=16, N=256, K=256 on the PR1 tensors (absmax scales)."""
    d = workloads.pr1(seed=0)
    run_full(oracle_operand(d["x"]), oracle_operand(d["w"]), 16, 256, 256)


@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (7, 136, 32), (128, 256, 256), (200, 320, 544),
                                   (129, 384, 1056), (300, 520, 2080), (256, 512, 4096)])
def test_ragged_shapes_full_compare(cuda_device, M, N, K):
    """Several tiles in M and N, partial K-tiles (K % 256 != 0, K % 64 == 32), N not
    a multiple of 128 (a tile whose second scale group is absent)."""
    xa = workloads.activation(M, K, seed=M, n_outlier_channels=min(4, K // 16))
    xb = workloads.gaussian_weight(N, K, 0.02, seed=N)
    run_full(oracle_operand(xa), oracle_operand(xb, oracle.SCALE_MSE), M, N, K)


@pytest.mark.parametrize("M,N,K", [(1280, 4096, 128), (2176, 2560, 96)])
def test_more_tiles_than_sms_full_compare(cuda_device, M, N, K):
    """More output tiles than SMs, so each persistent CTA walks several tiles (and the
    grouped tile order ends on a partial group of row tiles)."""
    xa = workloads.activation(M, K, seed=M + 1, n_outlier_channels=2)
    xb = workloads.gaussian_weight(N, K, 0.02, seed=N + 1)
    run_full(oracle_operand(xa), oracle_operand(xb, oracle.SCALE_MSE), M, N, K)


@pytest.mark.parametrize("M,N,K", [(24, 1000, 2080), (2, 384, 8192), (32, 14336, 512)])
def test_small_m_stream_k_full_compare(cuda_device, M, N, K):
    """The small-M kernel (weights on the 128-row MMA side, the weight stream split evenly
    over the SMs): ragged N, a partial last K-tile, tiles cut into up to 32 segments
    (N=384, K=8192: one K-tile per CTA) and the ordered partial reduction."""
    xa = workloads.activation(M, K, seed=M + 7, n_outlier_channels=2)
    xb = workloads.gaussian_weight(N, K, 0.02, seed=N + 7)
    run_full(oracle_operand(xa), oracle_operand(xb, oracle.SCALE_MSE), M, N, K)


def test_bounded_wait_gives_up_and_reports(cuda_device):
    """A device-side wait on a barrier nothing completes gives up after its limit,
    writes its status word, and the context keeps working afterwards."""
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    nv.selftest_wait_timeout(ws, timeout_us=20000)
    assert nv.read_device_error(ws) == 0x600
    d = workloads.pr1(seed=0)
    run_full(oracle_operand(d["x"]), oracle_operand(d["w"]), 16, 256, 256)


def test_zero_and_sign_cases(cuda_device):
    M, N, K = 64, 256, 256
    z = workloads.to_bf16(np.zeros((M, K), np.float32))
    w = workloads.gaussian_weight(N, K, 1.0, seed=3)
    out = nv.nvfp4_gemm(upload(oracle_operand(z)), upload(oracle_operand(w)))
    assert not out.float().abs().sum().item()
    neg = workloads.to_bf16(-workloads.gaussian_weight(M, K, 1.0, seed=4).float().numpy())
    run_full(oracle_operand(neg), oracle_operand(w), M, N, K)


def test_integer_grid_special_case(cuda_device):
    """All block scales 1 and s_g = 1: C is an exact integer matmul / 4."""
    r = np.random.default_rng(12)
    M, N, K = 130, 264, 320
    ca = r.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    cb = r.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = np.full((M, K // 16), 0x38, np.uint8)
    sb = np.full((N, K // 16), 0x38, np.uint8)
    run_full((ca, sa, np.float32(1)), (cb, sb, np.float32(1)), M, N, K)


def _sampled(M, N, K, a, b, out, n_samples=3000, seed=0):
    r = np.random.default_rng(seed)
    mi = np.concatenate([r.integers(0, M, n_samples), np.repeat(np.arange(min(M, 128)), 4),
                         np.full(64, M - 1)])
    ni = np.concatenate([r.integers(0, N, n_samples), r.integers(0, N, 4 * min(M, 128)),
                         np.arange(N - 64, N)])
    ref, absum = oracle.gemm_f64_at(*a, *b, mi, ni)
    got = out.float().cpu().numpy()[mi, ni]
    check(got, ref, absum)


def test_decode_config(cuda_device):
    """Decode linear: M in {1, 8, 32}, K=4096, N=14336 (weights pre-quantized)."""
    w = oracle_operand(workloads.gaussian_weight(14336, 4096, 0.02, seed=0), oracle.SCALE_MSE)
    W = upload(w)
    for m in (1, 8, 32):
        x = oracle_operand(workloads.activation(m, 4096, seed=m))
        out = nv.nvfp4_gemm(upload(x), W)
        ref, absum = oracle.gemm_f64(*x, *w)
        check(out.float().cpu().numpy(), ref, absum)


def test_prefill_config_sampled(cuda_device):
    """Prefill linear M=4096, K=4096, N=14336 at full size, sampled outputs."""
    M, N, K = 4096, 14336, 4096
    a = oracle_operand(workloads.activation(M, K, seed=0))
    b = oracle_operand(workloads.gaussian_weight(N, K, 0.02, seed=0), oracle.SCALE_ABSMAX)
    out = nv.nvfp4_gemm(upload(a), upload(b))
    _sampled(M, N, K, a, b, out)


def test_prefill_down_projection_sampled(cuda_device):
    """Down projection M=4096, K=14336, N=4096 (56 K-tiles)."""
    M, N, K = 4096, 4096, 14336
    a = oracle_operand(workloads.activation(M, K, seed=1, stream=workloads.STREAM_X2))
    b = oracle_operand(workloads.gaussian_weight(N, K, 0.02, seed=1, stream=workloads.STREAM_W2))
    out = nv.nvfp4_gemm(upload(a), upload(b))
    _sampled(M, N, K, a, b, out, seed=1)


def test_shared_tiles_stream_k_sampled(cuda_device):
    """M=2560, N=2048, K=12288: 80 tiles of 256 x 256 on the CTA pairs with 48 K-tiles
    each, so the last round's work is spread over every pair and most tiles are split
    along K between two pairs (partial sums through the workspace, the second piece adds
    them).  Sampled outputs against the FP64 reference, two launches bitwise equal on a
    workspace whose content on entry is arbitrary, no device-side timeout."""
    M, N, K = 2560, 2048, 12288
    a = oracle_operand(workloads.activation(M, K, seed=5, n_outlier_channels=4))
    b = oracle_operand(workloads.gaussian_weight(N, K, 0.02, seed=5), oracle.SCALE_MSE)
    A, B = upload(a), upload(b)
    ws_bytes = nv.load_library().nvfp4_gemm_workspace_bytes(M, N, K)
    ws = torch.full((ws_bytes,), 0xAB, dtype=torch.uint8, device="cuda")
    out = nv.nvfp4_gemm(A, B, workspace=ws)
    assert nv.read_device_error(ws) == 0
    out2 = nv.nvfp4_gemm(A, B, workspace=ws)
    assert nv.read_device_error(ws) == 0
    assert torch.equal(out, out2)
    _sampled(M, N, K, a, b, out, n_samples=8000, seed=5)


def test_scaled_mm_library_pin_of_the_oracle(cuda_device):
    """Pin the oracle's nibble order and swizzled scale layout against a library
    routine: torch._scaled_mm (cuBLASLt NVFP4) reads the oracle's bytes and must
    agree with the oracle's float64 GEMM."""
    if not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("torch has no float4_e2m1fn_x2")
    M, N, K = 128, 256, 512
    a = oracle_operand(workloads.activation(M, K, seed=9))
    b = oracle_operand(workloads.gaussian_weight(N, K, 0.02, seed=9), oracle.SCALE_MSE)
    A = torch.from_numpy(a[0]).cuda().view(torch.float4_e2m1fn_x2)
    B = torch.from_numpy(b[0]).cuda().view(torch.float4_e2m1fn_x2)
    sa = torch.from_numpy(oracle.swizzle_scales(a[1])).cuda().view(torch.float8_e4m3fn)
    sb = torch.from_numpy(oracle.swizzle_scales(b[1])).cuda().view(torch.float8_e4m3fn)
    try:
        out = torch._scaled_mm(A, B.t(), scale_a=sa, scale_b=sb, out_dtype=torch.float32)
    except (RuntimeError, TypeError) as e:
        pytest.skip(f"torch._scaled_mm rejects NVFP4 here: {e}")
    got = out.double().cpu().numpy() * float(a[2]) * float(b[2])
    ref, absum = oracle.gemm_f64(*a, *b)
    assert np.all(np.abs(got - ref) <= 1e-5 * absum + 1e-9)
