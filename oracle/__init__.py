"""CPU oracle for NVFP4 block quantization and the W4A4 GEMM (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``w4a4_gemm_quantize_b200``) never imports it and shares no code with it.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, binary32 round-to-nearest-
even, no FMA contraction, float64 for the GEMM reference); this module only
compiles it with gcc, loads it with ctypes and marshals numpy arrays.  Every
function cites the passage it follows in the C source:

* [G4] "Tu pipeline NVFP4: meter 62 GB de modelo en 24 GB de laptop", section 2
  "Qué es realmente NVFP4" (E2M1 bitfield, grid, q_ij / W^_ij equations,
  two-level scale, absmax and MSE block scales).
* [DF] "NVFP4 en difusión: la misma cuantización, un motor completamente
  distinto", section 2 "NVFP4 sin vLLM: torch._scaled_mm a mano" (packed codes,
  per-16 E4M3 scales along the input dimension, block-scaled GEMM, BF16 out) and
  section 8 "Para practicar" (scale search over factors of the absmax scale).

Parity unpinned: the global-scale formula s_g = amax/2688 and the binary32
operation order are readings (conventions); the tests pin their consequences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libnvfp4_oracle.so")

SCALE_ABSMAX = 0
SCALE_MSE = 1
SCALE_FOUR_OVER_SIX = 2

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (binary32 RNE, no contraction) and return the .so path."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    F = ctypes.c_float
    lib.ora_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.ora_bf16_to_f32.restype = F
    lib.ora_f32_to_bf16.argtypes = [F]
    lib.ora_f32_to_bf16.restype = ctypes.c_uint16
    lib.ora_e2m1_decode.argtypes = [ctypes.c_uint8]
    lib.ora_e2m1_decode.restype = ctypes.c_double
    lib.ora_e2m1_encode_mag.argtypes = [F]
    lib.ora_e2m1_encode_mag.restype = ctypes.c_uint8
    lib.ora_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.ora_e4m3_decode.restype = ctypes.c_double
    lib.ora_e4m3_encode.argtypes = [F]
    lib.ora_e4m3_encode.restype = ctypes.c_uint8
    lib.ora_amax.argtypes = [P, I64, I64, I64]
    lib.ora_amax.restype = F
    lib.ora_global_scale_from_amax.argtypes = [F]
    lib.ora_global_scale_from_amax.restype = F
    lib.ora_global_scale.argtypes = [P, I64, I64, I64]
    lib.ora_global_scale.restype = F
    lib.ora_quantize.argtypes = [P, I64, I64, I64, ctypes.c_int, F, P, P, P]
    lib.ora_quantize.restype = ctypes.c_int
    lib.ora_swizzled_scales_bytes.argtypes = [I64, I64]
    lib.ora_swizzled_scales_bytes.restype = I64
    lib.ora_swizzled_offset.argtypes = [I64, I64, I64]
    lib.ora_swizzled_offset.restype = I64
    lib.ora_swizzle_scales.argtypes = [P, I64, I64, P]
    lib.ora_swizzle_scales.restype = None
    lib.ora_unswizzle_scales.argtypes = [P, I64, I64, P]
    lib.ora_unswizzle_scales.restype = None
    lib.ora_dequantize.argtypes = [P, P, F, I64, I64, P]
    lib.ora_dequantize.restype = None
    lib.ora_gemm_f64.argtypes = [P, P, F, I64, P, P, F, I64, I64, P, P]
    lib.ora_gemm_f64.restype = ctypes.c_int
    lib.ora_gemm_f64_at.argtypes = [P, P, F, P, P, F, I64, P, P, I64, P, P]
    lib.ora_gemm_f64_at.restype = ctypes.c_int
    lib.ora_e2m1_encode_mag_array.argtypes = [P, I64, P]
    lib.ora_e2m1_encode_mag_array.restype = None
    lib.ora_e4m3_encode_array.argtypes = [P, I64, P]
    lib.ora_e4m3_encode_array.restype = None
    lib.ora_f32_to_bf16_array.argtypes = [P, I64, P]
    lib.ora_f32_to_bf16_array.restype = None
    lib.ora_lora_f64.argtypes = [P, I64, I64, P, I64, P, I64, P, P, P]
    lib.ora_lora_f64.restype = ctypes.c_int
    lib.ora_e8m0_decode.argtypes = [ctypes.c_uint8]
    lib.ora_e8m0_decode.restype = ctypes.c_double
    lib.ora_quantize_mx.argtypes = [P, I64, I64, I64, P, P]
    lib.ora_quantize_mx.restype = ctypes.c_int
    lib.ora_dequantize_mx.argtypes = [P, P, I64, I64, P]
    lib.ora_dequantize_mx.restype = None
    lib.ora_gemm_mx_f64_at.argtypes = [P, P, P, P, I64, P, P, I64, P, P]
    lib.ora_gemm_mx_f64_at.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """BF16 input as a C-contiguous uint16 bit array (accepts torch bf16 or uint16)."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        x = x.contiguous().view(dtype=__import__("torch").int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "BF16 inputs are passed as uint16 bit patterns"
    return x


# --- scalar codecs ------------------------------------------------------------------------------

def e2m1_decode(code: int) -> float:
    """[G4] E2M1 bitfield value v(s, e, m) with bias 1 (bit 3 = s, bits 2:1 = e, bit 0 = m)."""
    return _load().ora_e2m1_decode(code)


def e2m1_encode_mag(y: float) -> int:
    """Magnitude code of y >= 0: nearest grid value, ties to even mantissa, saturating at 6."""
    return _load().ora_e2m1_encode_mag(y)


def e4m3_decode(b: int) -> float:
    """E4M3 ("fn") value of byte b: bias 7, subnormals m/8*2^-6, 0x7F = NaN."""
    return _load().ora_e4m3_decode(b)


def e4m3_encode(u: float) -> int:
    """Nearest non-negative finite E4M3 code of u >= 0, ties to even, saturating at 448."""
    return _load().ora_e4m3_encode(u)


def f32_to_bf16_bits(f: float) -> int:
    return _load().ora_f32_to_bf16(f)


def e2m1_encode_mag_array(y) -> np.ndarray:
    y = np.ascontiguousarray(y, np.float32)
    out = np.empty(y.shape, np.uint8)
    _load().ora_e2m1_encode_mag_array(_ptr(y), y.size, _ptr(out))
    return out


def e4m3_encode_array(u) -> np.ndarray:
    u = np.ascontiguousarray(u, np.float32)
    out = np.empty(u.shape, np.uint8)
    _load().ora_e4m3_encode_array(_ptr(u), u.size, _ptr(out))
    return out


def f32_to_bf16_array(f) -> np.ndarray:
    f = np.ascontiguousarray(f, np.float32)
    out = np.empty(f.shape, np.uint16)
    _load().ora_f32_to_bf16_array(_ptr(f), f.size, _ptr(out))
    return out


# --- tensor functions ---------------------------------------------------------------------------

def amax(x) -> float:
    x = _bits(x)
    r, c = x.shape
    return float(_load().ora_amax(_ptr(x), r, c, c))


def global_scale(x) -> np.float32:
    """s_g = RN32(amax/2688) (reading R1), 1.0 for an all-zero tensor."""
    x = _bits(x)
    r, c = x.shape
    return np.float32(_load().ora_global_scale(_ptr(x), r, c, c))


def global_scale_from_amax(a: float) -> np.float32:
    return np.float32(_load().ora_global_scale_from_amax(a))


def quantize(x, mode: int = SCALE_ABSMAX, sg=None):
    """Quantize a rows x cols BF16 tensor (cols % 16 == 0).

    Returns (codes uint8 [rows, cols/2], scales uint8 [rows, cols/16] linear E4M3,
    global scale float32, block_err float32 [rows, cols/16]).  ``sg`` given means a
    caller-supplied global scale; otherwise it is computed from the tensor's amax.
    """
    x = _bits(x)
    rows, cols = x.shape
    if sg is None:
        sg = global_scale(x)
    sg = np.float32(sg)
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    err = np.zeros((rows, cols // 16), np.float32)
    rc = _load().ora_quantize(_ptr(x), rows, cols, cols, int(mode), float(sg), _ptr(codes),
                              _ptr(scales), _ptr(err))
    if rc != 0:
        raise ValueError(f"bad shape {x.shape}")
    return codes, scales, sg, err


def swizzled_scales_bytes(rows: int, nblk: int) -> int:
    return int(_load().ora_swizzled_scales_bytes(rows, nblk))


def swizzle_scales(scales: np.ndarray) -> np.ndarray:
    """Linear (rows, nblk) E4M3 scales -> flat swizzled 128x4-tile buffer (zero padded)."""
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, nblk = scales.shape
    out = np.empty(swizzled_scales_bytes(rows, nblk), np.uint8)
    _load().ora_swizzle_scales(_ptr(scales), rows, nblk, _ptr(out))
    return out


def unswizzle_scales(swz: np.ndarray, rows: int, nblk: int) -> np.ndarray:
    swz = np.ascontiguousarray(swz, dtype=np.uint8)
    assert swz.size >= swizzled_scales_bytes(rows, nblk)
    out = np.empty((rows, nblk), np.uint8)
    _load().ora_unswizzle_scales(_ptr(swz), rows, nblk, _ptr(out))
    return out


def dequantize(codes: np.ndarray, scales: np.ndarray, sg) -> np.ndarray:
    """BF16 bits of RN32(q * RN32(dec(s_b) * s_g)), rounded to BF16 (RNE)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, half = codes.shape
    cols = half * 2
    out = np.empty((rows, cols), np.uint16)
    _load().ora_dequantize(_ptr(codes), _ptr(scales), float(np.float32(sg)), rows, cols, _ptr(out))
    return out


def gemm_f64(a_codes, a_scales, a_sg, b_codes, b_scales, b_sg):
    """FP64 reference of C = (A s_a)(B s_b)^T; returns (C [M, N], S = sum|a b| [M, N])."""
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    b_codes = np.ascontiguousarray(b_codes, np.uint8)
    a_scales = np.ascontiguousarray(a_scales, np.uint8)
    b_scales = np.ascontiguousarray(b_scales, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    assert b_codes.shape[1] * 2 == K
    out = np.empty((M, N), np.float64)
    absum = np.empty((M, N), np.float64)
    rc = _load().ora_gemm_f64(_ptr(a_codes), _ptr(a_scales), float(np.float32(a_sg)), M, _ptr(b_codes),
                              _ptr(b_scales), float(np.float32(b_sg)), N, K, _ptr(out), _ptr(absum))
    if rc != 0:
        raise MemoryError("oracle GEMM work buffer")
    return out, absum


def gemm_f64_at(a_codes, a_scales, a_sg, b_codes, b_scales, b_sg, m_idx, n_idx):
    """The FP64 reference at sampled positions (m_idx[i], n_idx[i]); returns (C, S)."""
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    b_codes = np.ascontiguousarray(b_codes, np.uint8)
    a_scales = np.ascontiguousarray(a_scales, np.uint8)
    b_scales = np.ascontiguousarray(b_scales, np.uint8)
    K = a_codes.shape[1] * 2
    m_idx = np.ascontiguousarray(m_idx, np.int64)
    n_idx = np.ascontiguousarray(n_idx, np.int64)
    assert m_idx.shape == n_idx.shape
    out = np.empty(m_idx.shape, np.float64)
    absum = np.empty(m_idx.shape, np.float64)
    rc = _load().ora_gemm_f64_at(_ptr(a_codes), _ptr(a_scales), float(np.float32(a_sg)), _ptr(b_codes),
                                 _ptr(b_scales), float(np.float32(b_sg)), K, _ptr(m_idx), _ptr(n_idx),
                                 m_idx.size, _ptr(out), _ptr(absum))
    if rc != 0:
        raise MemoryError("oracle GEMM work buffer")
    return out, absum


def lora_f64(x, a, b):
    """Low-rank term of y = W_4bit x + B (A x) (reading R9): x (M, K), a (R, K), b (N, R) BF16.

    Returns (u [M, N] float64, S_u = sum |t b| [M, N], t [M, R] BF16 bits) with
    t = BF16_RNE(RN32(x a^T)) and u = t b^T in binary64."""
    x, a, b = _bits(x), _bits(a), _bits(b)
    M, K = x.shape
    R = a.shape[0]
    N = b.shape[0]
    assert a.shape[1] == K and b.shape[1] == R
    out = np.empty((M, N), np.float64)
    absum = np.empty((M, N), np.float64)
    t = np.empty((M, R), np.uint16)
    rc = _load().ora_lora_f64(_ptr(x), M, K, _ptr(a), R, _ptr(b), N, _ptr(out), _ptr(absum), _ptr(t))
    if rc != 0:
        raise MemoryError("oracle LoRA work buffer")
    return out, absum, t


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """(rows, cols/2) packed bytes -> (rows, cols) 4-bit codes (element 2j = low nibble)."""
    codes = np.asarray(codes, np.uint8)
    out = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    out[:, 0::2] = codes & 0xF
    out[:, 1::2] = codes >> 4
    return out


# --- MXFP4 (outside reading: the OCP Microscaling Formats specification v1.0) ----------------------

def e8m0_decode(b: int) -> float:
    """E8M0 scale byte b -> 2^(b - 127) (0xFF = NaN)."""
    return _load().ora_e8m0_decode(b)


def quantize_mx(x):
    """MXFP4: blocks of 32 along the row, E8M0 scale 2^(floor(log2 amax) - 2), E2M1 elements.

    Returns (codes uint8 [rows, cols/2], scales uint8 [rows, cols/32] linear E8M0)."""
    x = _bits(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 32), np.uint8)
    if _load().ora_quantize_mx(_ptr(x), rows, cols, cols, _ptr(codes), _ptr(scales)) != 0:
        raise ValueError(f"bad shape {x.shape}")
    return codes, scales


def dequantize_mx(codes, scales) -> np.ndarray:
    """BF16 bits of q * 2^(s - 127)."""
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, half = codes.shape
    out = np.empty((rows, half * 2), np.uint16)
    _load().ora_dequantize_mx(_ptr(codes), _ptr(scales), rows, half * 2, _ptr(out))
    return out


def gemm_mx_f64_at(a_codes, a_scales, b_codes, b_scales, m_idx, n_idx):
    """Binary64 C = A B^T of MXFP4 operands at positions (m_idx[i], n_idx[i]); returns (C, S)."""
    a_codes, b_codes = np.ascontiguousarray(a_codes, np.uint8), np.ascontiguousarray(b_codes, np.uint8)
    a_scales, b_scales = np.ascontiguousarray(a_scales, np.uint8), np.ascontiguousarray(b_scales, np.uint8)
    m_idx = np.ascontiguousarray(m_idx, np.int64)
    n_idx = np.ascontiguousarray(n_idx, np.int64)
    out = np.empty(m_idx.shape, np.float64)
    absum = np.empty(m_idx.shape, np.float64)
    if _load().ora_gemm_mx_f64_at(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), a_codes.shape[1] * 2,
                                  _ptr(m_idx), _ptr(n_idx), m_idx.size, _ptr(out), _ptr(absum)) != 0:
        raise MemoryError("oracle GEMM work buffer")
    return out, absum


def gemm_mx_f64(a_codes, a_scales, b_codes, b_scales):
    """Binary64 C = A B^T of MXFP4 operands, all positions; returns (C [M, N], S)."""
    M, N = a_codes.shape[0], b_codes.shape[0]
    mi = np.repeat(np.arange(M), N)
    ni = np.tile(np.arange(N), M)
    c, s = gemm_mx_f64_at(a_codes, a_scales, b_codes, b_scales, mi, ni)
    return c.reshape(M, N), s.reshape(M, N)
