"""GPU parity of the MXFP4 path (quantize, dequantize, GEMM) against the oracle.

MXFP4 as the OCP Microscaling Formats (MX) v1.0 specification defines it (the
pages name the format without its block size or scale type): E2M1 codes in
32-value blocks with an E8M0 power-of-two scale, no per-tensor scale.  Codes and
scales must be bit-exact; the GEMM (block-scaled tcgen05 MMA with 32-value UE8M0
scales) must pass ``helpers.check_gemm`` against the oracle's float64 product.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_quantize_b200 as nv
from helpers import check_gemm, sample_positions

pytestmark = pytest.mark.gpu


def mx_inputs(rows, cols, seed):
    r = np.random.default_rng(seed)
    a = (r.standard_t(3, size=(rows, cols)) * 0.02).astype(np.float32)
    if rows > 4 and cols >= 64:
        a[0, :32] = 0.0
        a[1, 32:64] = -0.0
        a[2, :32] *= 1e-30                       # far below the rest: its own small power of two
        a[3, 7] = 3.0e4
        a[4, :32] = np.float32(1e-40)            # BF16 subnormals
    return workloads.to_bf16(a)


@pytest.mark.parametrize("rows,cols", [(1, 32), (7, 96), (129, 544), (300, 4096), (1000, 1024)])
@pytest.mark.parametrize("layout", ["swizzled", "linear"])
def test_mx_quantize_bit_exact(cuda_device, rows, cols, layout):
    x = mx_inputs(rows, cols, seed=rows + cols)
    q = nv.mxfp4_quantize(x.cuda(), layout)
    torch.cuda.synchronize()
    codes, sc = oracle.quantize_mx(x)
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    got = q.scales.cpu().numpy()
    if layout == "swizzled":
        assert np.array_equal(got, oracle.swizzle_scales(sc))      # padding included
    else:
        assert np.array_equal(got.reshape(sc.shape), sc)
    out = nv.mxfp4_dequantize(q)
    assert np.array_equal(workloads.bf16_bits(out.cpu()), oracle.dequantize_mx(codes, sc))


def upload(codes, sc):
    rows, half = codes.shape
    return nv.MXFP4Tensor(torch.from_numpy(np.ascontiguousarray(codes)).cuda(),
                          torch.from_numpy(oracle.swizzle_scales(sc)).cuda(), rows, half * 2, nv.SF_SWIZZLED)


@pytest.mark.parametrize("M,N,K", [(1, 136, 32), (7, 520, 96), (32, 14336, 4096), (3, 384, 8192),
                                   (129, 136, 544), (300, 520, 2080), (256, 512, 4096), (64, 1000, 160)])
def test_mx_gemm_full_compare(cuda_device, M, N, K):
    a = oracle.quantize_mx(workloads.activation(M, K, seed=M, n_outlier_channels=min(4, K // 32)))
    b = oracle.quantize_mx(workloads.gaussian_weight(N, K, 0.02, seed=N))
    ws = torch.full((nv.load_library().nvfp4_gemm_workspace_bytes(M, N, K),), 0x77, dtype=torch.uint8, device="cuda")
    out = nv.mxfp4_gemm(upload(*a), upload(*b), workspace=ws)
    assert nv.read_device_error(ws) == 0
    again = nv.mxfp4_gemm(upload(*a), upload(*b), workspace=ws)
    assert torch.equal(out, again)
    ref, absum = oracle.gemm_mx_f64(*a, *b)
    check_gemm(out.float().cpu().numpy(), ref, absum, where=f"mxfp4 {M}x{N}x{K}")


def test_mx_gemm_prefill_sampled(cuda_device):
    """Prefill size (4096 x 14336 x 4096) on the GPU quantizer's operands (bit-exact with the
    oracle's, checked on sampled rows) against the oracle's product at sampled outputs."""
    M, N, K = 4096, 14336, 4096
    xa = workloads.activation(M, K, seed=0)
    xb = workloads.gaussian_weight(N, K, 0.02, seed=0)
    A, B = nv.mxfp4_quantize(xa.cuda()), nv.mxfp4_quantize(xb.cuda())
    out = nv.mxfp4_gemm(A, B)
    torch.cuda.synchronize()
    mi, ni = sample_positions(M, N, n_random=2000)
    rows_a, rows_b = np.unique(mi), np.unique(ni)
    a_codes, a_sc = oracle.quantize_mx(np.ascontiguousarray(workloads.bf16_bits(xa)[rows_a]))
    b_codes, b_sc = oracle.quantize_mx(np.ascontiguousarray(workloads.bf16_bits(xb)[rows_b]))
    assert np.array_equal(A.codes.cpu().numpy()[rows_a], a_codes)
    assert np.array_equal(oracle.unswizzle_scales(A.scales.cpu().numpy(), M, K // 32)[rows_a], a_sc)
    ia = np.searchsorted(rows_a, mi)
    ib = np.searchsorted(rows_b, ni)
    ref, absum = oracle.gemm_mx_f64_at(a_codes, a_sc, b_codes, b_sc, ia, ib)
    check_gemm(out.float().cpu().numpy()[mi, ni], ref, absum, where="mxfp4 prefill sampled")
