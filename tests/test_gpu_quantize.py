"""GPU parity of the quantizer and dequantizer against the CPU oracle (bit-exact).

Every call goes through the C ABI (ctypes binding over libnvfp4_b200.so).  The
oracle is given the same BF16 bytes; codes, scales (including the zero padding of
the swizzled layout), the global scale and the per-block errors must match bit
for bit.  Workloads: the pages' configurations (PR1 reference, the MSE-vs-absmax
4096x4096 Student-t weight, 8B-class and 31B-class linears) and edge cases.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_quantize_b200 as nv

pytestmark = pytest.mark.gpu

MODES = {"absmax": oracle.SCALE_ABSMAX, "mse": oracle.SCALE_MSE, "four_over_six": oracle.SCALE_FOUR_OVER_SIX}
ALL_MODES = list(MODES)


def _f32_bits(v):
    return np.array([v], np.float32).view(np.uint32)[0]


def run_and_compare(x_cpu, mode, layout="swizzled", sg=None, rows_sample=None):
    """Quantize on the GPU and compare with the oracle (optionally on sampled rows)."""
    x = x_cpu.cuda()
    gs_in = None if sg is None else torch.tensor([sg], dtype=torch.float32, device="cuda")
    q = nv.nvfp4_quantize(x, mode, layout, global_scale=gs_in, block_err=True)
    torch.cuda.synchronize()
    rows, cols = x_cpu.shape
    nblk = cols // 16
    sg_ref = oracle.global_scale(x_cpu) if sg is None else np.float32(sg)
    assert _f32_bits(q.global_scale.item()) == _f32_bits(sg_ref), (q.global_scale.item(), sg_ref)
    bits = workloads.bf16_bits(x_cpu)
    sel = np.arange(rows) if rows_sample is None else np.asarray(rows_sample)
    codes, sc_lin, _, err = oracle.quantize(np.ascontiguousarray(bits[sel]), MODES[mode], sg_ref)
    g_codes = q.codes.cpu().numpy()[sel]
    assert np.array_equal(g_codes, codes), _first_diff(g_codes, codes)
    g_sc = q.scales.cpu().numpy()
    if layout == "swizzled":
        g_lin = oracle.unswizzle_scales(g_sc, rows, nblk)[sel]
        # every padding byte of the swizzled buffer is zero
        pad = oracle.swizzle_scales(np.ones((rows, nblk), np.uint8)) == 0
        assert not g_sc[pad].any(), "swizzle padding not zero"
    else:
        g_lin = g_sc.reshape(rows, nblk)[sel]
    assert np.array_equal(g_lin, sc_lin), _first_diff(g_lin, sc_lin)
    g_err = q.block_err.cpu().numpy()[sel]
    assert np.array_equal(g_err.view(np.uint32), err.view(np.uint32)), _first_diff(g_err, err)
    return q


def _first_diff(a, b):
    idx = np.argwhere(a != b)
    if idx.size == 0:
        return "equal"
    i = tuple(idx[0])
    return f"{len(idx)} mismatches; first at {i}: gpu={a[i]!r} oracle={b[i]!r}"


# --- the pages' workloads -----------------------------------------------------------------------

@pytest.mark.parametrize("mode", ALL_MODES)
@pytest.mark.parametrize("layout", ["swizzled", "linear"])
def test_pr1_reference_config(cuda_device, mode, layout):
    d = workloads.pr1(seed=0)
    run_and_compare(d["w"], mode, layout)
    run_and_compare(d["x"], mode, layout)


@pytest.mark.parametrize("mode", ALL_MODES)
def test_mse_workload_small_full_compare(cuda_device, mode):
    """0.02 * Student-t(3), 8 x 128-row tiles with a ragged tail of rows."""
    run_and_compare(workloads.mse_weight(1000, 1024, seed=1), mode)


@pytest.mark.parametrize("mode", ["absmax", "mse"])
def test_mse_workload_full_size_sampled(cuda_device, mode):
    """The 4096 x 4096 weight of the MSE-vs-absmax workload; oracle on sampled rows."""
    x = workloads.mse_weight(4096, 4096, seed=0)
    rows = np.unique(np.concatenate([np.arange(0, 4), np.arange(4090, 4096),
                                     np.random.default_rng(0).choice(4096, 48, replace=False)]))
    run_and_compare(x, mode, rows_sample=rows)


def test_four_over_six_blocks_exact_on_one_mapping(cuda_device):
    """Blocks on the E2M1 grid with their maximum on 4 (exact only when the maximum maps to 4)
    and on 6 (exact only when it maps to 6), a zero block and a one-value tie, with s_g = 1:
    the GPU takes the 4 mapping exactly where the oracle does."""
    b4 = [4, 3, 2, 1.5, 1, 0.5, 0, -4, -3, -2, -1.5, -1, -0.5, 0, 4, 2]
    b6 = [6, 4, 3, 2, 1.5, 1, 0.5, 0, -6, -4, -3, -2, -1.5, -1, -0.5, 0]
    a = np.array([b4 + b6, b6 + b4, [0.0] * 16 + [0.0] * 15 + [3.0], [x * 0.25 for x in b4] + b4], np.float32)
    q = run_and_compare(workloads.to_bf16(a), "four_over_six", sg=1.0)
    lin = oracle.unswizzle_scales(q.scales.cpu().numpy(), 4, 2)
    assert lin[0, 0] == 0x38 and lin[1, 1] == 0x38  # E4M3 1.0: the block maximum 4 maps to 4


def test_decode_activations_outlier_channels(cuda_device):
    for m in (1, 8, 32):
        run_and_compare(workloads.activation(m, 4096, seed=m), "absmax")


def test_31b_weight_mse_sampled(cuda_device):
    x = workloads.t4_weight(21504, 5376, seed=0)
    rows = np.unique(np.concatenate([[0, 1, 21503], np.random.default_rng(1).choice(21504, 24, replace=False)]))
    run_and_compare(x, "mse", rows_sample=rows)


def test_prefill_activation_sampled(cuda_device):
    x = workloads.activation(4096, 14336, seed=2, stream=workloads.STREAM_X2)
    rows = np.unique(np.concatenate([[0, 4095], np.random.default_rng(2).choice(4096, 24, replace=False)]))
    run_and_compare(x, "absmax", rows_sample=rows)


# --- edge cases ---------------------------------------------------------------------------------

@pytest.mark.parametrize("mode", ALL_MODES)
def test_edge_values(cuda_device, mode):
    r = np.random.default_rng(5)
    a = (r.standard_t(3, size=(130, 48)) * 0.02).astype(np.float32)
    a[0, :16] = 0.0
    a[1, 16:32] = -0.0
    a[2, :16] = -1e-30                      # far below the tensor maximum: zero scale
    a[3, 5] = 40.0                          # the tensor maximum (its block gets scale 448)
    a[4, :16] = np.float32(1e-40)           # BF16 subnormals
    a[5, 32:48] = r.standard_normal(16) * 1e-4
    a[6, :] = -a[6, :]
    run_and_compare(workloads.to_bf16(a), mode)


@pytest.mark.parametrize("mode", ALL_MODES)
def test_huge_and_tiny_magnitudes(cuda_device, mode):
    """A BF16 value near the format maximum next to ordinary and subnormal values:
    most block scales underflow to E4M3 zero; tiny tensors push s_g to subnormal."""
    a = np.random.default_rng(6).standard_normal((16, 64)).astype(np.float32)
    a[3, 5] = 3.0e38
    run_and_compare(workloads.to_bf16(a), mode)
    b = (np.random.default_rng(7).standard_normal((16, 64)) * 1e-38).astype(np.float32)
    run_and_compare(workloads.to_bf16(b), mode)
    c = np.zeros((2, 32), np.float32)
    c[0, 3] = np.float32(9.2e-41)  # the smallest BF16 subnormal: s_g subnormal, 1/eff overflows
    c[1, 7] = -np.float32(9.2e-41)
    run_and_compare(workloads.to_bf16(c), mode)


def test_rounding_midpoints_with_given_global_scale(cuda_device):
    """Values exactly on E2M1 midpoints (ties go to the even mantissa) and on
    saturation, with s_g = 2^-3 so that the block scale is exactly 1."""
    mids = np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, 5.5, 6.5, 0.2, 0.3, 2.75, 4.5, 1.0, 0.5],
                    np.float32) * np.float32(0.125)
    a = np.stack([mids, -mids, mids[::-1].copy(), np.roll(mids, 3)])
    for mode in ALL_MODES:
        run_and_compare(workloads.to_bf16(a), mode, sg=0.125)


@pytest.mark.parametrize("shape", [(1, 16), (3, 32), (127, 16), (128, 64), (129, 80), (257, 272)])
def test_ragged_shapes(cuda_device, shape):
    a = np.random.default_rng(sum(shape)).standard_normal(shape).astype(np.float32)
    for mode in ALL_MODES:
        for layout in ("swizzled", "linear"):
            run_and_compare(workloads.to_bf16(a), mode, layout)


def test_all_zero_tensor(cuda_device):
    for sgn in (1.0, -1.0):
        a = np.zeros((64, 64), np.float32) * sgn
        q = run_and_compare(workloads.to_bf16(a), "mse")
        assert q.global_scale.item() == 1.0


def test_strided_input(cuda_device):
    base = workloads.mse_weight(96, 512, seed=4)
    x = base.cuda()[:, :256]                     # row stride 512, 256 columns
    q = nv.nvfp4_quantize(x, "mse", "linear", block_err=True)
    codes, sc, sg, err = oracle.quantize(base[:, :256].contiguous(), oracle.SCALE_MSE)
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    assert np.array_equal(q.scales.cpu().numpy(), sc)
    assert q.global_scale.item() == sg


def test_given_global_scale_skips_amax_pass(cuda_device):
    x = workloads.mse_weight(256, 256, seed=8)
    run_and_compare(x, "absmax", sg=0.0123)
    gs = torch.tensor([0.0123], dtype=torch.float32, device="cuda")
    nv.nvfp4_quantize(x.cuda(), "absmax", global_scale=gs)
    assert nv.last_launch_count() == 1  # no amax pass, no padding pass (256 rows, 16 blocks)


def test_empty_tensor(cuda_device):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q = nv.nvfp4_quantize(x, "absmax")
    assert q.codes.numel() == 0
    assert q.global_scale.item() == 1.0


# --- dequantize ---------------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["swizzled", "linear"])
def test_dequantize_bit_exact(cuda_device, layout):
    x = workloads.mse_weight(300, 528, seed=6)
    q = nv.nvfp4_quantize(x.cuda(), "mse", layout)
    out = nv.nvfp4_dequantize(q)
    codes, sc, sg, _ = oracle.quantize(x, oracle.SCALE_MSE)
    ref = oracle.dequantize(codes, sc, sg)
    assert np.array_equal(workloads.bf16_bits(out.cpu()), ref)


def test_dequantize_from_oracle_codes(cuda_device):
    """Dequantize oracle-made codes (every code value, every scale byte but NaN)."""
    r = np.random.default_rng(7)
    rows, cols = 200, 256
    codes = r.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    sc = r.integers(0, 0x7F, size=(rows, cols // 16), dtype=np.uint8)
    sg = np.float32(0.37)
    q = nv.NVFP4Tensor(torch.from_numpy(codes).cuda(), torch.from_numpy(oracle.swizzle_scales(sc)).cuda(),
                       torch.tensor([sg], device="cuda"), rows, cols, nv.SF_SWIZZLED)
    out = nv.nvfp4_dequantize(q)
    assert np.array_equal(workloads.bf16_bits(out.cpu()), oracle.dequantize(codes, sc, sg))


# --- host-side validation on a real device ------------------------------------------------------

def test_validation_errors(cuda_device):
    x = torch.zeros((4, 24), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.nvfp4_quantize(x, "absmax")
    assert e.value.status == 2  # cols % 16
    x = torch.zeros((4, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.nvfp4_quantize(x[:, 1:17], "absmax")  # misaligned start
    assert e.value.status == 3
