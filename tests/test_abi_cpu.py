"""The C-ABI library on a machine without a GPU: it loads, exports every symbol the
header declares, and its host-side logic (size queries, argument validation)
answers before any CUDA call.  No compute call is made here."""
import ctypes
import os
import re

import pytest

import w4a4_gemm_quantize_b200 as nv
from w4a4_gemm_quantize_b200 import build as nvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:nvfp4|mxfp4)_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    nvbuild.build()
    return nv.load_library()


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
        assert n in nv.SIGNATURES, f"binding lacks {n}"
    assert set(nv.SIGNATURES) == set(names)


def test_status_strings(lib):
    for code in range(8):
        s = lib.nvfp4_status_string(code)
        assert s and s != b"unknown status"
    assert lib.nvfp4_status_string(99) == b"unknown status"


def test_size_queries(lib):
    assert lib.nvfp4_codes_bytes(4096, 4096) == 4096 * 2048
    assert lib.nvfp4_scales_bytes(4096, 4096, nv.SF_LINEAR) == 4096 * 256
    assert lib.nvfp4_scales_bytes(4096, 4096, nv.SF_SWIZZLED) == 4096 * 256
    assert lib.nvfp4_scales_bytes(130, 48, nv.SF_SWIZZLED) == 256 * 4   # rows -> 256, 3 blocks -> 4
    assert lib.nvfp4_scales_bytes(1, 16, nv.SF_SWIZZLED) == 128 * 4
    assert lib.nvfp4_quantize_workspace_bytes(1, 16) >= 4
    assert lib.nvfp4_gemm_workspace_bytes(1, 1, 32) >= 4
    assert lib.nvfp4_codes_bytes(-1, 16) == 0


def _q(lib, x=16, rows=4, cols=32, ld=32, mode=0, layout=0, gs=None, codes=16, scales=16, ws=16,
       ws_bytes=256):
    P = ctypes.c_void_p
    return lib.nvfp4_quantize(P(x) if x else None, rows, cols, ld, mode, layout, P(gs) if gs else None,
                              P(codes) if codes else None, P(scales) if scales else None, None, None,
                              P(ws) if ws else None, ws_bytes, None)


def test_quantize_validation_before_any_cuda_call(lib):
    assert _q(lib, cols=24, ld=24) == 2            # cols % 16
    assert _q(lib, rows=-1) == 1                    # negative size
    assert _q(lib, ld=16) == 1                      # ld < cols
    assert _q(lib, mode=5) == 1                     # unknown mode
    assert _q(lib, mode=3) == 1
    assert _q(lib, mode=2) in (4, 5)                # four-over-six is a valid mode
    assert _q(lib, layout=7) == 1                   # unknown layout
    assert _q(lib, x=0) == 1                        # NULL input
    assert _q(lib, ws=0) == 7                       # no workspace, no global scale
    assert _q(lib, ws_bytes=3) == 7                 # workspace too small
    assert _q(lib, x=8) == 3                        # misaligned input
    assert _q(lib, codes=24) == 3                   # misaligned output
    assert _q(lib, ld=36) == 3                      # row stride not 16-byte aligned
    # everything valid: the device check runs and fails without a GPU
    assert _q(lib) in (4, 5)


def test_gemm_validation_before_any_cuda_call(lib):
    P = ctypes.c_void_p

    def g(M=64, N=16, K=64, ldc=16, ptr=16, ws=16, ws_bytes=256, gs=16):
        p = P(ptr) if ptr else None
        return lib.nvfp4_gemm(p, p, P(gs), M, p, p, P(gs), N, K, p, ldc, P(ws) if ws else None, ws_bytes, None)

    assert g(K=48) == 2          # K % 32
    assert g(M=0) == 1
    assert g(ldc=8) == 1         # ldc < N
    assert g(ptr=0) == 1
    assert g(ws=0) == 7
    assert g(ptr=8) == 3
    assert g(ldc=20) == 3
    assert g(gs=2) == 3
    assert g() in (4, 5)
    # small M uses stream-K scratch after the status word: a 256-byte workspace is too small
    need = lib.nvfp4_gemm_workspace_bytes(8, 14336, 4096)
    assert need > 256
    assert g(M=8, N=14336, ldc=14336, K=4096) == 7
    assert g(M=8, N=14336, ldc=14336, K=4096, ws_bytes=need) in (4, 5)
    assert g(M=8, N=14336, ldc=14336, K=4096, ws_bytes=need - 1) == 7


def test_decode_workspace_holds_every_partial_tile():
    """M <= 32: the weight stream (128-row tiles x 256-wide K-tiles) is split evenly over
    up to 296 CTAs; a tile spans at most (KT - 1) // per + 2 CTA ranges (per = units per
    CTA, rounded down), each with a 128 x 32 FP32 partial slot, after the 256-byte status
    block and one counter word per tile (rounded up to 256 bytes)."""
    lib = nv.load_library()
    for (M, N, K) in [(8, 14336, 4096), (1, 21504, 5376), (32, 5376, 21504), (2, 384, 8192), (24, 1000, 2080),
                      (1, 128, 32)]:
        T, KT = -(-N // 128), -(-K // 256)
        U = T * KT
        G = min(296, U)
        per = max(1, U // G)
        segs = min(KT, (KT - 1) // per + 2)
        counters = -(-(T * 4) // 256) * 256
        assert lib.nvfp4_gemm_workspace_bytes(M, N, K) == 256 + counters + T * segs * 128 * 32 * 4, (M, N, K)
    # M in 33..128 (or N <= 128): only the status block
    assert lib.nvfp4_gemm_workspace_bytes(33, 14336, 4096) == 256
    assert lib.nvfp4_gemm_workspace_bytes(4096, 128, 4096) == 256
    # M, N > 128 (CTA pairs on 256 x 256 tiles): a ticket and a flag word per slot, CTA and
    # epilogue warp for 74 slots (rounded up to 256 bytes), then per slot two pieces x two
    # CTAs x 8 warps x 32 x 128 FP32 partial sums
    pair = 256 + -(-(2 * 74 * 2 * 8 * 4) // 256) * 256 + 74 * 2 * 2 * 8 * 32 * 128 * 4
    for (M, N, K) in [(8192, 21504, 5376), (129, 129, 32), (256, 5376, 21504)]:
        assert lib.nvfp4_gemm_workspace_bytes(M, N, K) == pair, (M, N, K)


def test_dequantize_validation(lib):
    P = ctypes.c_void_p
    assert lib.nvfp4_dequantize(P(16), P(16), 0, P(16), 4, 24, P(16), 24, None) == 2
    assert lib.nvfp4_dequantize(P(16), P(16), 0, P(16), 0, 32, P(16), 32, None) == 0  # empty: nothing to do
    assert lib.nvfp4_dequantize(None, P(16), 0, P(16), 4, 32, P(16), 32, None) == 1
    assert lib.nvfp4_dequantize(P(16), P(16), 0, P(16), 4, 32, P(24), 32, None) == 3


def test_read_device_error_needs_workspace(lib):
    assert lib.nvfp4_read_device_error(None, None, None) == 1


def test_selftest_validation(lib):
    P = ctypes.c_void_p
    assert lib.nvfp4_selftest_wait_timeout(None, 1000, None) == 1
    assert lib.nvfp4_selftest_wait_timeout(P(16), 0, None) == 1
    assert lib.nvfp4_selftest_wait_timeout(P(16), 3000000, None) == 1
    assert lib.nvfp4_selftest_wait_timeout(P(8), 1000, None) == 3


def test_binding_constants_match_the_header():
    """The Python binding's enum values and status names are the ones include/nvfp4.h
    declares (parsed from the header text)."""
    hdr = open(HEADER).read()
    enum = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(NVFP4_[A-Z0-9_]+)\s*=\s*(\d+)", hdr)}
    assert enum["NVFP4_SCALE_ABSMAX"] == nv.SCALE_ABSMAX
    assert enum["NVFP4_SCALE_MSE"] == nv.SCALE_MSE
    assert enum["NVFP4_SCALE_FOUR_OVER_SIX"] == nv.SCALE_FOUR_OVER_SIX
    assert enum["NVFP4_SF_SWIZZLED"] == nv.SF_SWIZZLED and enum["NVFP4_SF_LINEAR"] == nv.SF_LINEAR
    status = {v: k for k, v in enum.items() if k == "NVFP4_OK" or k.startswith("NVFP4_ERR_")}
    assert status == nv.STATUS


def test_bench_profile_record_matches_only_its_sources(tmp_path, monkeypatch):
    """bench.py reports the ncu DRAM traffic of a profile summary only while the summary's
    source hash equals the hash of the kernel's current sources."""
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    real_csrc = os.path.join(os.path.dirname(os.path.abspath(bench.__file__)), "w4a4_gemm_quantize_b200", "csrc")
    os.makedirs(tmp_path / "w4a4_gemm_quantize_b200")
    os.symlink(real_csrc, tmp_path / "w4a4_gemm_quantize_b200" / "csrc")
    os.makedirs(tmp_path / "profiles")
    h = bench.source_hash("gemm")
    f = tmp_path / "profiles" / "gemm_pair_kernel_w_gemm_1.md"
    f.write_text(f"- source_hash: `{h}`\n- traffic_bytes_per_launch: 1234\n")
    assert bench.profiled_traffic("gemm_pair_kernel", "w", "gemm_1") == 1234.0
    f.write_text("- source_hash: `0000000000000000`\n- traffic_bytes_per_launch: 1234\n")
    assert bench.profiled_traffic("gemm_pair_kernel", "w", "gemm_1") is None
    assert bench.profiled_traffic("gemm_pair_kernel", "missing", "gemm_1") is None
    # a low-rank group's kernel is hashed with the down-projection's sources too
    assert bench.KERNEL_FAMILY["gemm_pair_kernel_lora"] == "lora" and "lora.cu" in bench.KERNEL_SOURCES["lora"]


def test_noalloc_validation_before_any_cuda_call(lib):
    """The no-allocation quantizer checks its arguments on the host first, then the device
    (without a GPU it reports the device), before it looks up its scratch block."""
    P = ctypes.c_void_p

    def q(x=16, rows=4, cols=32, ld=32, mode=0, layout=0, codes=16, scales=16):
        return lib.nvfp4_quantize_noalloc(P(x) if x else None, rows, cols, ld, mode, layout, None,
                                          P(codes) if codes else None, P(scales) if scales else None, None, None,
                                          None)

    assert q(cols=24, ld=24) == 2
    assert q(rows=-1) == 1
    assert q(mode=9) == 1
    assert q(x=0) == 1
    assert q(x=8) == 3
    assert q(ld=36) == 3
    assert q() in (4, 5)


@pytest.mark.parametrize("entry", ["nvfp4_linear", "nvfp4_linear_fused"])
def test_linear_validation_before_any_cuda_call(lib, entry):
    P = ctypes.c_void_p
    fn = getattr(lib, entry)

    def g(M=8, N=256, K=64, ld=64, ldc=256, ptr=16, ws=16, ws_bytes=1 << 30, x_gs=None):
        p = P(ptr) if ptr else None
        return fn(p, M, K, ld, P(x_gs) if x_gs else None, p, p, P(16), N, p, ldc, P(ws) if ws else None, ws_bytes,
                  None)

    assert g(K=48, ld=48) == 2          # K % 32
    assert g(M=0) == 1
    assert g(ld=32) == 1                # ld_x < K
    assert g(ptr=0) == 1
    assert g(ws=0) == 7
    assert g(ws_bytes=511) == 7
    assert g(ptr=8) == 3
    assert g(x_gs=18) == 3
    assert g() in (4, 5)
    if entry == "nvfp4_linear_fused":
        assert g(M=33) == 2             # the fused kernel is the small-M one


def test_linear_workspace_layout(lib):
    # header, the small-M GEMM's counters and partial tiles, the activation's codes and scales
    for M in (8, 32):
        gemm_scratch = lib.nvfp4_gemm_workspace_bytes(M, 14336, 4096) - 256
        act = -(-(M * 2048) // 256) * 256 + lib.nvfp4_scales_bytes(M, 4096, 0)
        assert lib.nvfp4_linear_workspace_bytes(M, 14336, 4096) >= 512 + gemm_scratch + act
    assert lib.nvfp4_linear_workspace_bytes(4096, 14336, 4096) >= 512 + 4096 * 2048 + 4096 * 256
    # M, N > 128: the CTA-pair GEMM's shared-tile counters and partial tiles come before the
    # activation's codes and scales
    for (M, N, K) in [(4096, 14336, 4096), (8192, 5376, 21504)]:
        gemm_scratch = lib.nvfp4_gemm_workspace_bytes(M, N, K) - 256
        act = -(-(M * K // 2) // 256) * 256 + lib.nvfp4_scales_bytes(M, K, 0)
        assert gemm_scratch > 38_000_000
        assert lib.nvfp4_linear_workspace_bytes(M, N, K) >= 512 + gemm_scratch + act


def test_linear_lora_validation_before_any_cuda_call(lib):
    P = ctypes.c_void_p

    def g(M=8, N=256, K=64, R=16, ptr=16, ws=16, ws_bytes=1 << 30, a=16, b=16, t=None):
        p = P(ptr) if ptr else None
        return lib.nvfp4_linear_lora(p, M, K, K, None, p, p, P(16), N, P(a) if a else None, P(b) if b else None, R,
                                     p, N, P(t) if t else None, P(ws) if ws else None, ws_bytes, None)

    assert g(R=8) == 2                  # rank not a multiple of 16
    assert g(R=80) == 2                 # rank above 64
    assert g(R=0) == 1
    assert g(a=0) == 1 and g(b=0) == 1
    assert g(ws_bytes=100) == 7
    assert g(b=24) == 3 and g(t=40) == 3
    assert g() in (4, 5) and g(R=64, M=4096) in (4, 5)
    small = lib.nvfp4_linear_lora_workspace_bytes(8, 14336, 4096, 64)
    assert small > lib.nvfp4_linear_workspace_bytes(8, 14336, 4096)
