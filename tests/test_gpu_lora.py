"""GPU parity of the W4A4 linear layer with a low-rank branch (nvfp4_linear_lora).

y = Q(x) W^T + (x A^T) B^T -- the page "NVFP4 en difusión: la misma cuantización, un
motor completamente distinto", section 3 ("¿Cómo fine-tuneás algo que ya está en 4
bits?"): the low-rank term is computed in 16 bits and added to the quantized matmul
inside the kernel, never merged into the 4-bit weights.  Reading: t = BF16(A x)
with FP32 accumulation, then B t added to the W4A4 accumulator before the single
BF16 rounding of the result.

Reference: the oracle's quantization of x (absmax) and W (MSE), its float64 GEMM
(ref, S = sum |a b|) and its low-rank term (u = t B^T in float64 with the oracle's
BF16 t, S_u = sum |t b|).  The tolerance per element is the stated accumulation
bound over both sums, 1e-3 (S + S_u) + 1e-6, plus half a BF16 ulp of the result,
plus sum_j |B[n, j]| ulp(t[m, j]): the order of t's FP32 accumulation is left open by
the reading, so the GPU's t may round to the neighbouring BF16 value (t itself is
checked to be within one ulp, and equal on nearly every element).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_quantize_b200 as nv
from helpers import bf16_rne, bf16_ulp, gemm_ref_block, operand, oracle_quantize, rows_of

pytestmark = pytest.mark.gpu


def factors(N, K, R, seed):
    """LoRA factors: A (R x K) ~ N(0, 0.02), B (N x R) ~ N(0, 0.1) -- a low-rank term
    large enough that dropping it, or scaling it wrongly, breaks the bound."""
    return (workloads.to_bf16(workloads.normal((R, K), seed, 11, 0.02)),
            workloads.to_bf16(workloads.normal((N, R), seed, 12, 0.1)))


def check_lora(c, ref, absum, u, absum_u, t_ref, b_bits, rows, where):
    c = np.asarray(c, np.float64)
    t_ulp = bf16_ulp(workloads.from_bits(t_ref).double().numpy())
    b_abs = np.abs(workloads.from_bits(b_bits).double().numpy())
    t_term = t_ulp @ b_abs.T                      # sum_j ulp(t[m, j]) |B[n, j]|
    expect = ref + u
    err = np.abs(c - expect)
    allow = 1e-3 * (absum + absum_u) + 1e-6 + 0.5 * bf16_ulp(c) + t_term
    bad = err > allow
    assert not bad.any(), (f"{where}: {int(bad.sum())} out of bound; worst excess {(err - allow).max():.3e} at "
                           f"{np.unravel_index(np.argmax(err - allow), err.shape)}")
    # the low-rank term matters at this scale: leaving it out would fail the bound
    assert (np.abs(u) > 1e-3 * absum + 1e-6 + 0.5 * bf16_ulp(expect)).mean() > 0.5, where
    exact = float(np.mean(c == bf16_rne(expect)))
    assert exact >= 0.75, f"{where}: only {exact:.3f} equal BF16(ref + u)"


def run(M, N, K, R, gs=None, row_blocks=None, seed=0, where=""):
    x = workloads.activation(M, K, seed=seed + M, n_outlier_channels=min(4, K // 16))
    w = workloads.gaussian_weight(N, K, 0.02, seed=seed + N)
    A, B = factors(N, K, R, seed)
    wq = nv.nvfp4_quantize(w.cuda(), "mse")
    gs_t = None if gs is None else torch.tensor([gs], dtype=torch.float32, device="cuda")
    ws = torch.full((nv.load_library().nvfp4_linear_lora_workspace_bytes(M, N, K, R),), 0x3C, dtype=torch.uint8,
                    device="cuda")
    t_out = torch.empty((M, R), dtype=torch.bfloat16, device="cuda")
    out = nv.linear_lora(x.cuda(), wq, A.cuda(), B.cuda(), x_global_scale=gs_t, t_out=t_out, workspace=ws)
    assert nv.read_device_error(ws) == 0
    again = nv.linear_lora(x.cuda(), wq, A.cuda(), B.cuda(), x_global_scale=gs_t, workspace=ws)
    assert torch.equal(out, again), f"{where}: a second call on the same workspace differs"
    a = operand(oracle_quantize(x, oracle.SCALE_ABSMAX, sg=gs))
    b = operand(oracle_quantize(w, oracle.SCALE_MSE))
    got = out.float().cpu().numpy()
    t_gpu = workloads.bf16_bits(t_out.cpu())
    xb, Ab, Bb = workloads.bf16_bits(x), workloads.bf16_bits(A), workloads.bf16_bits(B)
    for (r0, r1) in (row_blocks or [(0, M)]):
        ref, absum = gemm_ref_block(a, b, r0, r1, 0, N)
        u, absum_u, t_ref = oracle.lora_f64(np.ascontiguousarray(xb[r0:r1]), Ab, Bb)
        d = np.abs(workloads.from_bits(t_gpu[r0:r1]).double().numpy() - workloads.from_bits(t_ref).double().numpy())
        assert np.all(d <= bf16_ulp(workloads.from_bits(t_ref).double().numpy())), f"{where}: t off by more than an ulp"
        assert np.mean(t_gpu[r0:r1] == t_ref) >= 0.98, f"{where}: t differs from the oracle's too often"
        check_lora(got[r0:r1], ref, absum, u, absum_u, t_ref, Bb, (r0, r1), f"{where} rows {r0}:{r1}")
    return out


@pytest.mark.parametrize("M,N,K,R", [(1, 14336, 4096, 64), (8, 14336, 4096, 16), (32, 14336, 4096, 64),
                                     (7, 520, 96, 16), (32, 384, 8192, 32), (3, 136, 544, 48)])
def test_lora_small_m(cuda_device, M, N, K, R):
    """M <= 32: the activation quantized and the low-rank term added inside the decode kernel."""
    run(M, N, K, R, where=f"lora {M}x{N}x{K} r{R}")


@pytest.mark.parametrize("M,N,K,R", [(8, 520, 544, 64), (64, 520, 544, 16)])
def test_lora_given_global_scale(cuda_device, M, N, K, R):
    run(M, N, K, R, gs=0.05, where=f"lora given scale {M}x{N}x{K} r{R}")


@pytest.mark.parametrize("M,N,K,R", [(64, 520, 544, 16), (129, 136, 544, 64), (300, 1000, 2080, 48),
                                     (260, 264, 96, 16)])
def test_lora_large_m(cuda_device, M, N, K, R):
    """M > 32: the CTA-pair GEMM with the low-rank MMAs (small M and N included)."""
    run(M, N, K, R, where=f"lora {M}x{N}x{K} r{R}")


@pytest.mark.parametrize("R", [16, 64])
def test_lora_prefill(cuda_device, R):
    """Prefill up projection (4096 x 14336 x 4096): the first and last 64 rows in full."""
    run(4096, 14336, 4096, R, row_blocks=[(0, 64), (4032, 4096)], where=f"lora prefill r{R}")


@pytest.mark.parametrize("M,N,K,R", [(300, 520, 544, 16), (4096, 4096, 512, 16), (2048, 14336, 4096, 64)])
def test_lora_zero_factors_equal_the_plain_linear(cuda_device, M, N, K, R):
    """With B = 0 the layer is the plain W4A4 linear layer, bit for bit -- also with many
    tiles per CTA pair, where the low-rank MMAs that open each tile's accumulator must
    complete before the tile's first FP4 MMA (MMAs of different shapes on one
    accumulator are not ordered by issue; a K-tile's products would be lost)."""
    x = workloads.activation(M, K, seed=5).cuda()
    wq = nv.nvfp4_quantize(workloads.gaussian_weight(N, K, 0.02, seed=5).cuda(), "mse")
    A = workloads.to_bf16(workloads.normal((R, K), 5, 11, 0.02)).cuda()
    B = torch.zeros((N, R), dtype=torch.bfloat16, device="cuda")
    for m in (M, 8):
        out = nv.linear_lora(x[:m], wq, A, B)
        plain = nv.linear(x[:m], wq)
        assert torch.equal(out, plain), f"{m}x{N}x{K}: {int((out != plain).sum())} elements differ"
