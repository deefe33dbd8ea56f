"""Bounds of every write: outputs surrounded by canary bytes.

Each output buffer of a call (codes, swizzled and linear scales, block errors, the
global scale, C with a leading dimension larger than N, and the GEMM workspace with
the small-M kernel's partial tiles) is carved out of a larger allocation whose
4 KiB margins on both sides hold a fixed byte pattern.  After the call the margins,
and the columns of C between N and ldc, must be untouched.  The shapes are ragged
(rows 1, 7, 129; N 136, 520; K 32, 96, 544), so partial tiles, clipped tensor-map
boxes and partial quads of scale bytes are all exercised.  This is the test of
out-of-bounds writes that does not need a sanitizer.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_quantize_b200 as nv
from helpers import check_gemm, upload

pytestmark = pytest.mark.gpu

MARGIN = 4096
FILL = 0xA5


class Guarded:
    """`nbytes` bytes of device memory with canary margins on both sides."""

    def __init__(self, nbytes):
        self.nbytes = nbytes
        self.buf = torch.full((MARGIN + nbytes + MARGIN,), FILL, dtype=torch.uint8, device="cuda")
        self.inner = self.buf[MARGIN:MARGIN + nbytes]

    def view(self, dtype, shape):
        return self.inner.view(dtype).view(shape)

    def check(self, what):
        b = self.buf.cpu().numpy()
        lo, hi = b[:MARGIN], b[MARGIN + self.nbytes:]
        assert (lo == FILL).all(), f"{what}: {int((lo != FILL).sum())} bytes written before the buffer"
        assert (hi == FILL).all(), f"{what}: {int((hi != FILL).sum())} bytes written after the buffer"


@pytest.mark.parametrize("rows,cols", [(1, 32), (7, 96), (129, 544), (136, 32), (520, 96)])
@pytest.mark.parametrize("mode", ["absmax", "mse", "four_over_six"])
@pytest.mark.parametrize("layout", ["swizzled", "linear"])
def test_quantize_writes_stay_in_bounds(cuda_device, rows, cols, mode, layout):
    x = workloads.activation(rows, cols, seed=rows + cols, n_outlier_channels=1)
    lay = nv.SF_SWIZZLED if layout == "swizzled" else nv.SF_LINEAR
    nblk = cols // 16
    g_codes = Guarded(nv.codes_bytes(rows, cols))
    g_scales = Guarded(nv.scales_bytes(rows, cols, lay))
    g_gs = Guarded(4)
    g_err = Guarded(rows * nblk * 4)
    g_ws = Guarded(nv.load_library().nvfp4_quantize_workspace_bytes(rows, cols))
    scales = g_scales.inner if lay == nv.SF_SWIZZLED else g_scales.view(torch.uint8, (rows, nblk))
    out = nv.NVFP4Tensor(g_codes.view(torch.uint8, (rows, cols // 2)), scales, g_gs.view(torch.float32, (1,)),
                         rows, cols, lay, g_err.view(torch.float32, (rows, nblk)))
    nv.nvfp4_quantize(x.cuda(), mode, layout, block_err=True, out=out, workspace=g_ws.inner)
    torch.cuda.synchronize()
    for g, what in ((g_codes, "codes"), (g_scales, "scales"), (g_gs, "global scale"), (g_err, "block_err"),
                    (g_ws, "workspace")):
        g.check(what)
    codes, sc, sg, err = oracle.quantize(x, {"absmax": 0, "mse": 1, "four_over_six": 2}[mode])
    assert np.array_equal(out.codes.cpu().numpy(), codes)
    got_sc = out.scales.cpu().numpy()
    if lay == nv.SF_SWIZZLED:
        assert np.array_equal(got_sc, oracle.swizzle_scales(sc))  # padding included
    else:
        assert np.array_equal(got_sc, sc)


@pytest.mark.parametrize("M,N,K", [(1, 136, 32), (7, 520, 96), (129, 136, 544), (7, 136, 544),
                                   (129, 520, 96), (300, 520, 544), (32, 520, 544),
                                   (64, 520, 96), (300, 120, 544)])
def test_gemm_writes_stay_in_bounds(cuda_device, M, N, K):
    """C inside a canary region with ldc > N (the gap columns are checked too), and the
    workspace (status word, tile counters, partial tiles) inside one as well."""
    a = oracle.quantize(workloads.activation(M, K, seed=M, n_outlier_channels=1), oracle.SCALE_ABSMAX)[:3]
    b = oracle.quantize(workloads.gaussian_weight(N, K, 0.02, seed=N), oracle.SCALE_MSE)[:3]
    ldc = N + 24  # a multiple of 8 elements (16 bytes), larger than N
    g_c = Guarded(M * ldc * 2)
    c_full = g_c.view(torch.bfloat16, (M, ldc))
    c = c_full[:, :N]
    ws_bytes = nv.load_library().nvfp4_gemm_workspace_bytes(M, N, K)
    g_ws = Guarded(ws_bytes)
    nv.nvfp4_gemm(upload(a), upload(b), out=c, workspace=g_ws.inner)
    assert nv.read_device_error(g_ws.inner) == 0
    g_c.check("C")
    g_ws.check("workspace")
    gap = c_full[:, N:].contiguous().view(torch.uint8).cpu().numpy()
    assert (gap == FILL).all(), "columns between N and ldc were written"
    ref, absum = oracle.gemm_f64(*a, *b)
    check_gemm(c.float().cpu().numpy(), ref, absum, where=f"guarded {M}x{N}x{K}")


@pytest.mark.parametrize("rows,cols", [(7, 96), (129, 544)])
def test_dequantize_writes_stay_in_bounds(cuda_device, rows, cols):
    x = workloads.mse_weight(rows, cols, seed=rows)
    q = nv.nvfp4_quantize(x.cuda(), "mse")
    ld = cols + 8
    g = Guarded(rows * ld * 2)
    full = g.view(torch.bfloat16, (rows, ld))
    nv.nvfp4_dequantize(q, out=full[:, :cols])
    torch.cuda.synchronize()
    g.check("dequantized output")
    assert (full[:, cols:].contiguous().view(torch.uint8).cpu().numpy() == FILL).all()
    codes, sc, sg, _ = oracle.quantize(x, oracle.SCALE_MSE)
    assert np.array_equal(workloads.bf16_bits(full[:, :cols].contiguous().cpu()), oracle.dequantize(codes, sc, sg))
