"""The quantizer entry point that allocates nothing (nvfp4_quantize_noalloc).

It exists for callers that cannot allocate device memory -- plugins inside a
framework or server that owns every allocation and gives them no workspace, and
latency-critical loops where cudaMalloc would synchronize the device.  It must
give exactly what nvfp4_quantize gives (bit-exact codes, scales, global scale and
block errors, the tolerance the quantizer tests use) on consecutive calls that
share its built-in scratch block.  This file is collected last so that a run
stopping at the first failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_quantize_b200 as nv

pytestmark = pytest.mark.gpu


def _noalloc_via_c_abi(x, mode, layout, gs_in=None):
    """Call the C entry point directly through ctypes, outputs allocated by torch."""
    lib = nv.load_library()
    rows, cols = x.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty(lib.nvfp4_scales_bytes(rows, cols, layout), dtype=torch.uint8, device=x.device)
    gs = torch.empty(1, dtype=torch.float32, device=x.device)
    err = torch.empty((rows, cols // 16), dtype=torch.float32, device=x.device)
    P = ctypes.c_void_p
    st = lib.nvfp4_quantize_noalloc(P(x.data_ptr()), rows, cols, x.stride(0), mode, layout,
                                    None if gs_in is None else P(gs_in.data_ptr()),
                                    P(codes.data_ptr()), P(scales.data_ptr()), P(gs.data_ptr()),
                                    P(err.data_ptr()), P(torch.cuda.current_stream().cuda_stream))
    assert st == 0, nv.STATUS.get(st, st)
    return codes, scales, gs, err


def _same(a, b):
    return np.array_equal(a.cpu().numpy().view(np.uint8), b.cpu().numpy().view(np.uint8))


MODES = [nv.SCALE_ABSMAX, nv.SCALE_MSE, nv.SCALE_FOUR_OVER_SIX]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("layout", [nv.SF_SWIZZLED, nv.SF_LINEAR])
def test_noalloc_matches_quantize_on_two_calls_in_a_row(cuda_device, mode, layout):
    # The first tensor has a much larger maximum than the second, so a scratch
    # word left over from the first call would corrupt the second's global scale.
    first = workloads.activation(200, 1024, seed=31, n_outlier_channels=4, factor=50.0)
    second = workloads.mse_weight(300, 512, seed=32)
    for x_cpu in (first, second):
        x = x_cpu.cuda()
        codes, scales, gs, err = _noalloc_via_c_abi(x, mode, layout)
        ref = nv.nvfp4_quantize(x, mode, layout, block_err=True)
        torch.cuda.synchronize()
        assert _same(codes, ref.codes)
        assert _same(scales, ref.scales.reshape(-1))
        assert _same(gs, ref.global_scale)
        assert _same(err, ref.block_err)
        # and the CPU definition of the method, bit for bit
        o_codes, o_sc, o_sg, o_err = oracle.quantize(x_cpu, mode)
        assert np.array_equal(codes.cpu().numpy(), o_codes)
        lin = oracle.unswizzle_scales(scales.cpu().numpy(), *o_sc.shape) if layout == nv.SF_SWIZZLED \
            else scales.cpu().numpy().reshape(o_sc.shape)
        assert np.array_equal(lin, o_sc)
        assert gs.item() == o_sg
        assert np.array_equal(err.cpu().numpy().view(np.uint32), o_err.view(np.uint32))


@pytest.mark.parametrize("mode", MODES)
def test_noalloc_with_a_given_global_scale(cuda_device, mode):
    """With the caller's global scale the entry point needs no scratch at all; two calls
    in a row with different scales match nvfp4_quantize given the same scale."""
    x = workloads.mse_weight(130, 256, seed=33).cuda()
    for sg in (0.0123, 3.5e-5):
        gs_in = torch.tensor([sg], dtype=torch.float32, device="cuda")
        codes, scales, gs, err = _noalloc_via_c_abi(x, mode, nv.SF_SWIZZLED, gs_in=gs_in)
        ref = nv.nvfp4_quantize(x, mode, "swizzled", global_scale=gs_in, block_err=True)
        torch.cuda.synchronize()
        assert _same(codes, ref.codes) and _same(scales, ref.scales) and _same(err, ref.block_err)
        assert gs.item() == np.float32(sg)
