"""NVFP4 quantization and the W4A4 block-scaled GEMM on B200 (sm_100a).

A thin ctypes binding over ``libnvfp4_b200.so`` (declared in ``include/nvfp4.h``).
It only marshals arguments: torch provides device memory and the current CUDA
stream; every step of the computation runs in the library's CUDA kernels.  There
is no CPU fallback: if the library is missing or the device is not sm_100, the
calls raise.

Format and method: web page "Tu pipeline NVFP4: meter 62 GB de modelo en 24 GB
de laptop", section 2 "Qué es realmente NVFP4" (E2M1 codes in blocks of 16
along K, one E4M3 scale per block, one FP32 scale per tensor; absmax or MSE
block scales) and "NVFP4 en difusión: la misma cuantización, un motor
completamente distinto", section 2 (packed (out, in/2) codes, (out, in/16)
scales, out = (A s_a)(B s_b)^T in BF16, activations quantized on every call).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4_b200.so")

SCALE_ABSMAX = 0
SCALE_MSE = 1
SCALE_FOUR_OVER_SIX = 2
SF_SWIZZLED = 0
SF_LINEAR = 1

_MODES = {"absmax": SCALE_ABSMAX, "mse": SCALE_MSE, "four_over_six": SCALE_FOUR_OVER_SIX,
          SCALE_ABSMAX: SCALE_ABSMAX, SCALE_MSE: SCALE_MSE, SCALE_FOUR_OVER_SIX: SCALE_FOUR_OVER_SIX}
_LAYOUTS = {"swizzled": SF_SWIZZLED, "linear": SF_LINEAR, SF_SWIZZLED: SF_SWIZZLED, SF_LINEAR: SF_LINEAR}

STATUS = {0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_SHAPE", 3: "NVFP4_ERR_ALIGNMENT",
          4: "NVFP4_ERR_UNSUPPORTED_DEVICE", 5: "NVFP4_ERR_CUDA", 6: "NVFP4_ERR_TIMEOUT",
          7: "NVFP4_ERR_WORKSPACE"}

# Every symbol include/nvfp4.h declares, with its ctypes signature.
_P, _I64, _SZ, _I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
SIGNATURES = {
    "nvfp4_status_string": ([_I], ctypes.c_char_p),
    "nvfp4_check_device": ([], _I),
    "nvfp4_codes_bytes": ([_I64, _I64], _SZ),
    "nvfp4_scales_bytes": ([_I64, _I64, _I], _SZ),
    "nvfp4_quantize_workspace_bytes": ([_I64, _I64], _SZ),
    "nvfp4_quantize": ([_P, _I64, _I64, _I64, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "nvfp4_dequantize": ([_P, _P, _I, _P, _I64, _I64, _P, _I64, _P], _I),
    "nvfp4_gemm_workspace_bytes": ([_I64, _I64, _I64], _SZ),
    "nvfp4_gemm": ([_P, _P, _P, _I64, _P, _P, _P, _I64, _I64, _P, _I64, _P, _SZ, _P], _I),
    "nvfp4_linear_workspace_bytes": ([_I64, _I64, _I64], _SZ),
    "nvfp4_linear": ([_P, _I64, _I64, _I64, _P, _P, _P, _P, _I64, _P, _I64, _P, _SZ, _P], _I),
    "nvfp4_linear_fused": ([_P, _I64, _I64, _I64, _P, _P, _P, _P, _I64, _P, _I64, _P, _SZ, _P], _I),
    "nvfp4_linear_lora_workspace_bytes": ([_I64, _I64, _I64, _I64], _SZ),
    "nvfp4_linear_lora": ([_P, _I64, _I64, _I64, _P, _P, _P, _P, _I64, _P, _P, _I64, _P, _I64, _P, _P, _SZ, _P], _I),
    "mxfp4_scales_bytes": ([_I64, _I64, _I], _SZ),
    "mxfp4_quantize": ([_P, _I64, _I64, _I64, _I, _P, _P, _P], _I),
    "mxfp4_dequantize": ([_P, _P, _I, _I64, _I64, _P, _I64, _P], _I),
    "mxfp4_gemm": ([_P, _P, _I64, _P, _P, _I64, _I64, _P, _I64, _P, _SZ, _P], _I),
    "nvfp4_read_device_error": ([_P, _P, ctypes.POINTER(ctypes.c_uint32)], _I),
    "nvfp4_last_launch_count": ([], _I),
    "nvfp4_quantize_noalloc": ([_P, _I64, _I64, _I64, _I, _I, _P, _P, _P, _P, _P, _P], _I),
    "nvfp4_selftest_wait_timeout": ([_P, ctypes.c_uint32, _P], _I),
}


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status})")


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the CUDA library (raises if it was not built: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} not found: build it with `python -m w4a4_gemm_quantize_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise Nvfp4Error(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@dataclass
class NVFP4Tensor:
    """A quantized rows x cols tensor: packed codes, E4M3 scales, FP32 global scale."""
    codes: torch.Tensor          # uint8 (rows, cols/2)
    scales: torch.Tensor         # uint8, flat swizzled buffer or (rows, cols/16) linear
    global_scale: torch.Tensor   # float32 (1,)
    rows: int
    cols: int
    layout: int = SF_SWIZZLED
    block_err: Optional[torch.Tensor] = None  # float32 (rows, cols/16)

    def nbytes(self) -> int:
        return self.codes.numel() + self.scales.numel() + 4


def codes_bytes(rows: int, cols: int) -> int:
    return load_library().nvfp4_codes_bytes(rows, cols)


def scales_bytes(rows: int, cols: int, layout=SF_SWIZZLED) -> int:
    return load_library().nvfp4_scales_bytes(rows, cols, _LAYOUTS[layout])


def nvfp4_quantize(x: torch.Tensor, mode="absmax", layout="swizzled", global_scale: Optional[torch.Tensor] = None,
                   block_err: bool = False, out: Optional[NVFP4Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> NVFP4Tensor:
    """Quantize a 2-D BF16 CUDA tensor (row stride multiple of 8, cols % 16 == 0)."""
    lib = load_library()
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda or x.stride(1) != 1:
        raise ValueError("x must be a 2-D row-major bfloat16 CUDA tensor")
    rows, cols = x.shape
    m, lay = _MODES[mode], _LAYOUTS[layout]
    dev = x.device
    if out is None:
        codes = torch.empty(lib.nvfp4_codes_bytes(rows, cols), dtype=torch.uint8, device=dev).view(rows, cols // 2)
        nsf = lib.nvfp4_scales_bytes(rows, cols, lay)
        scales = torch.empty(nsf, dtype=torch.uint8, device=dev)
        if lay == SF_LINEAR:
            scales = scales.view(rows, cols // 16)
        gs = torch.empty(1, dtype=torch.float32, device=dev)
        err = torch.empty((rows, cols // 16), dtype=torch.float32, device=dev) if block_err else None
        out = NVFP4Tensor(codes, scales, gs, rows, cols, lay, err)
    if workspace is None and global_scale is None:
        workspace = torch.empty(lib.nvfp4_quantize_workspace_bytes(rows, cols), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.nvfp4_quantize(_ptr(x), rows, cols, x.stride(0), m, lay, _ptr(global_scale), _ptr(out.codes),
                            _ptr(out.scales), _ptr(out.global_scale), _ptr(out.block_err), _ptr(workspace),
                            ws_bytes, _stream(stream))
    _check(st, "nvfp4_quantize")
    return out


def nvfp4_quantize_noalloc(x: torch.Tensor, mode="absmax", layout="swizzled",
                           global_scale: Optional[torch.Tensor] = None, block_err: bool = False,
                           out: Optional[NVFP4Tensor] = None, stream=None) -> NVFP4Tensor:
    """nvfp4_quantize without a workspace, for callers that cannot allocate device
    memory: the library's own 256-byte scratch block per GPU is used instead.
    Calls that overlap on the GPU share that block and race; serialize them."""
    lib = load_library()
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda or x.stride(1) != 1:
        raise ValueError("x must be a 2-D row-major bfloat16 CUDA tensor")
    rows, cols = x.shape
    lay = _LAYOUTS[layout]
    if out is None:
        dev = x.device
        codes = torch.empty(lib.nvfp4_codes_bytes(rows, cols), dtype=torch.uint8, device=dev).view(rows, cols // 2)
        scales = torch.empty(lib.nvfp4_scales_bytes(rows, cols, lay), dtype=torch.uint8, device=dev)
        if lay == SF_LINEAR:
            scales = scales.view(rows, cols // 16)
        gs = torch.empty(1, dtype=torch.float32, device=dev)
        err = torch.empty((rows, cols // 16), dtype=torch.float32, device=dev) if block_err else None
        out = NVFP4Tensor(codes, scales, gs, rows, cols, lay, err)
    st = lib.nvfp4_quantize_noalloc(_ptr(x), rows, cols, x.stride(0), _MODES[mode], lay, _ptr(global_scale),
                                    _ptr(out.codes), _ptr(out.scales), _ptr(out.global_scale),
                                    _ptr(out.block_err), _stream(stream))
    _check(st, "nvfp4_quantize_noalloc")
    return out


def nvfp4_dequantize(q: NVFP4Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """BF16 reconstruction q * s_b * s_g of a quantized tensor."""
    lib = load_library()
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=torch.bfloat16, device=q.codes.device)
    st = lib.nvfp4_dequantize(_ptr(q.codes), _ptr(q.scales), q.layout, _ptr(q.global_scale), q.rows, q.cols,
                              _ptr(out), out.stride(0), _stream(stream))
    _check(st, "nvfp4_dequantize")
    return out


def nvfp4_gemm(a: NVFP4Tensor, b: NVFP4Tensor, out: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """C = (A s_a)(B s_b)^T s_gA s_gB in BF16; A is M x K, B is N x K, scales swizzled."""
    lib = load_library()
    if a.cols != b.cols:
        raise ValueError("A and B must share K")
    if a.layout != SF_SWIZZLED or b.layout != SF_SWIZZLED:
        raise ValueError("nvfp4_gemm needs swizzled scales")
    M, N, K = a.rows, b.rows, a.cols
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.codes.device)
    if workspace is None:
        workspace = torch.empty(lib.nvfp4_gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device=a.codes.device)
    st = lib.nvfp4_gemm(_ptr(a.codes), _ptr(a.scales), _ptr(a.global_scale), M, _ptr(b.codes), _ptr(b.scales),
                        _ptr(b.global_scale), N, K, _ptr(out), out.stride(0), _ptr(workspace),
                        workspace.numel(), _stream(stream))
    _check(st, "nvfp4_gemm")
    return out


def read_device_error(workspace: torch.Tensor, stream=None) -> int:
    """Synchronize and return the raw device status word of a GEMM workspace (0 = ok)."""
    word = ctypes.c_uint32(0)
    st = load_library().nvfp4_read_device_error(_ptr(workspace), _stream(stream), ctypes.byref(word))
    if st not in (0, 6):
        _check(st, "nvfp4_read_device_error")
    return word.value


def selftest_wait_timeout(workspace: torch.Tensor, timeout_us: int = 20000, stream=None) -> None:
    """Launch the bounded-wait diagnostic (see include/nvfp4.h); read the result with read_device_error."""
    _check(load_library().nvfp4_selftest_wait_timeout(_ptr(workspace), timeout_us, _stream(stream)),
           "nvfp4_selftest_wait_timeout")


def last_launch_count() -> int:
    return load_library().nvfp4_last_launch_count()


def linear(x: torch.Tensor, w: NVFP4Tensor, x_global_scale: Optional[torch.Tensor] = None,
           out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None,
           fused: bool = False) -> torch.Tensor:
    """W4A4 linear layer C = Q(x) w^T in BF16: the activation x (M x K BF16) is
    quantized on this call with absmax block scales -- under `x_global_scale` (a
    device float, e.g. a calibrated activation scale) or, if None, amax(|x|)/2688
    computed on the device -- and multiplied by the pre-quantized weight w (N x K).
    fused=True (M <= 32) quantizes the activation inside the GEMM kernel
    (nvfp4_linear_fused); the result is the same bit for bit."""
    lib = load_library()
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda or x.stride(1) != 1:
        raise ValueError("x must be a 2-D row-major bfloat16 CUDA tensor")
    if w.layout != SF_SWIZZLED or w.cols != x.shape[1]:
        raise ValueError("w must share K with x and have swizzled scales")
    M, K = x.shape
    N = w.rows
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(lib.nvfp4_linear_workspace_bytes(M, N, K), dtype=torch.uint8, device=x.device)
    fn = lib.nvfp4_linear_fused if fused else lib.nvfp4_linear
    st = fn(_ptr(x), M, K, x.stride(0), _ptr(x_global_scale), _ptr(w.codes), _ptr(w.scales),
            _ptr(w.global_scale), N, _ptr(out), out.stride(0), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "nvfp4_linear_fused" if fused else "nvfp4_linear")
    return out


def linear_lora(x: torch.Tensor, w: NVFP4Tensor, lora_a: torch.Tensor, lora_b: torch.Tensor,
                x_global_scale: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                t_out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """W4A4 linear layer with a low-rank branch, y = Q(x) w^T + (x A^T) B^T in BF16:
    lora_a (R x K) and lora_b (N x R) BF16 CUDA tensors, rank R in {16, 32, 48, 64};
    t = x A^T is rounded to BF16 (returned in t_out if given) and t B^T is added to the
    W4A4 GEMM's FP32 accumulator before the single BF16 rounding."""
    lib = load_library()
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda or x.stride(1) != 1:
        raise ValueError("x must be a 2-D row-major bfloat16 CUDA tensor")
    M, K = x.shape
    N, R = w.rows, lora_a.shape[0]
    if w.layout != SF_SWIZZLED or w.cols != K:
        raise ValueError("w must share K with x and have swizzled scales")
    for t, shape in ((lora_a, (R, K)), (lora_b, (N, R))):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"low-rank factors must be contiguous bfloat16 of shapes {(R, K)} and {(N, R)}")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(lib.nvfp4_linear_lora_workspace_bytes(M, N, K, R), dtype=torch.uint8,
                                device=x.device)
    st = lib.nvfp4_linear_lora(_ptr(x), M, K, x.stride(0), _ptr(x_global_scale), _ptr(w.codes), _ptr(w.scales),
                               _ptr(w.global_scale), N, _ptr(lora_a), _ptr(lora_b), R, _ptr(out), out.stride(0),
                               _ptr(t_out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "nvfp4_linear_lora")
    return out


@dataclass
class MXFP4Tensor:
    """A rows x cols tensor in MXFP4: packed E2M1 codes and one E8M0 scale per 32 values."""
    codes: torch.Tensor   # uint8 (rows, cols/2)
    scales: torch.Tensor  # uint8, flat swizzled buffer or (rows, cols/32) linear
    rows: int
    cols: int
    layout: int = SF_SWIZZLED


def mxfp4_quantize(x: torch.Tensor, layout="swizzled", out: Optional[MXFP4Tensor] = None, stream=None) -> MXFP4Tensor:
    """Quantize a 2-D BF16 CUDA tensor (cols % 32 == 0) to MXFP4."""
    lib = load_library()
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda or x.stride(1) != 1:
        raise ValueError("x must be a 2-D row-major bfloat16 CUDA tensor")
    rows, cols = x.shape
    lay = _LAYOUTS[layout]
    if out is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
        scales = torch.empty(lib.mxfp4_scales_bytes(rows, cols, lay), dtype=torch.uint8, device=x.device)
        if lay == SF_LINEAR:
            scales = scales.view(rows, cols // 32)
        out = MXFP4Tensor(codes, scales, rows, cols, lay)
    _check(lib.mxfp4_quantize(_ptr(x), rows, cols, x.stride(0), lay, _ptr(out.codes), _ptr(out.scales),
                              _stream(stream)), "mxfp4_quantize")
    return out


def mxfp4_dequantize(q: MXFP4Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    lib = load_library()
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=torch.bfloat16, device=q.codes.device)
    _check(lib.mxfp4_dequantize(_ptr(q.codes), _ptr(q.scales), q.layout, q.rows, q.cols, _ptr(out), out.stride(0),
                                _stream(stream)), "mxfp4_dequantize")
    return out


def mxfp4_gemm(a: MXFP4Tensor, b: MXFP4Tensor, out: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """C = A B^T in BF16 for MXFP4 operands (A M x K, B N x K, swizzled scales)."""
    lib = load_library()
    if a.cols != b.cols or a.layout != SF_SWIZZLED or b.layout != SF_SWIZZLED:
        raise ValueError("A and B must share K and have swizzled scales")
    M, N, K = a.rows, b.rows, a.cols
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.codes.device)
    if workspace is None:
        workspace = torch.empty(lib.nvfp4_gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device=a.codes.device)
    _check(lib.mxfp4_gemm(_ptr(a.codes), _ptr(a.scales), M, _ptr(b.codes), _ptr(b.scales), N, K, _ptr(out),
                          out.stride(0), _ptr(workspace), workspace.numel(), _stream(stream)), "mxfp4_gemm")
    return out
