"""Seeded synthetic inputs shaped like the pages' workloads.

This module is shared by the tests, the benchmark and the smoke check.  It holds
no NVFP4 arithmetic: it only draws random numbers (numpy PCG64, keyed by
``(seed, stream)``) and rounds them to BF16 with torch's round-to-nearest-even
cast.  Both the oracle and the CUDA path receive the same BF16 bytes.

Workloads (the shapes are 8B-class and 31B-class transformer linears; the pages
quantize such layers, e.g. Gemma-4 31B, but publish no benchmark suite, so these
synthetic tensors stand in for real weights and activations):

* ``pr1``     W 256x256 and X 16x256 ~ N(0,1), each entry x20 with probability 1 %.
* ``mse``     W 4096x4096 = 0.02 * Student-t(nu=3).
* ``decode``  X Mx4096 ~ N(0,1) with 4 seed-chosen channels x50, M in {1, 8, 32};
              W 14336x4096 ~ N(0, 0.02).
* ``prefill`` X 4096x4096 (up) and 4096x14336 (down) ~ N(0,1) with 4 channels x50;
              W_up 14336x4096, W_down 4096x14336 ~ N(0, 0.02).
* ``dense31b`` W 21504x5376 and W2 5376x21504 = 0.015 * Student-t(nu=4);
              X Mx5376 / Mx21504 ~ N(0,1), M in {1, 256, 8192}.
"""
from __future__ import annotations

import numpy as np
import torch

# Stream ids keep every tensor of a workload independent under one seed.
STREAM_W = 1
STREAM_X = 2
STREAM_W2 = 3
STREAM_X2 = 4
STREAM_OUTLIER = 5


def rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(stream)]))


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32 numpy array -> contiguous CPU torch.bfloat16 tensor (RNE cast)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).contiguous()


def normal(shape, seed: int, stream: int, std: float = 1.0, chunk: int = 1 << 22) -> np.ndarray:
    g = rng(seed, stream)
    n = int(np.prod(shape))
    out = np.empty(n, np.float32)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        out[i:i + m] = g.standard_normal(m, dtype=np.float32) * np.float32(std)
    return out.reshape(shape)


def student_t(shape, nu: int, scale: float, seed: int, stream: int, chunk: int = 1 << 22) -> np.ndarray:
    """scale * Student-t(nu) for an integer nu, drawn as z / sqrt(chi2_nu / nu) with
    z ~ N(0,1) and chi2_nu the sum of nu // 2 terms -2 ln(U) (U uniform on (0, 1]) plus
    one squared normal when nu is odd -- an exact construction of the distribution,
    generated in chunks of `chunk` values."""
    g = rng(seed, stream)
    n = int(np.prod(shape))
    out = np.empty(n, np.float32)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        z = g.standard_normal(m, dtype=np.float32)
        chi = np.zeros(m, np.float32)
        for _ in range(nu // 2):
            chi -= np.float32(2) * np.log1p(-g.random(m, dtype=np.float32))
        if nu % 2:
            chi += g.standard_normal(m, dtype=np.float32) ** 2
        chi = np.maximum(chi, np.float32(1e-30))
        out[i:i + m] = z / np.sqrt(chi / np.float32(nu)) * np.float32(scale)
    return out.reshape(shape)


def with_outlier_entries(a: np.ndarray, prob: float, factor: float, seed: int, stream: int) -> np.ndarray:
    """Multiply each entry by ``factor`` with probability ``prob``."""
    mask = rng(seed, stream).random(size=a.shape) < prob
    out = a.copy()
    out[mask] *= np.float32(factor)
    return out


def with_outlier_channels(a: np.ndarray, n_channels: int, factor: float, seed: int, stream: int) -> np.ndarray:
    """Multiply ``n_channels`` seed-chosen columns (input channels) by ``factor``."""
    cols = rng(seed, stream).choice(a.shape[1], size=n_channels, replace=False)
    out = a.copy()
    out[:, cols] *= np.float32(factor)
    return out


# --- the five workloads ------------------------------------------------------------------------

def pr1(seed: int = 0):
    """W 256x256, X 16x256, N(0,1) with 1 % of entries x20 (absmax scales)."""
    w = with_outlier_entries(normal((256, 256), seed, STREAM_W), 0.01, 20.0, seed, STREAM_OUTLIER)
    x = with_outlier_entries(normal((16, 256), seed, STREAM_X), 0.01, 20.0, seed, STREAM_OUTLIER + 10)
    return {"w": to_bf16(w), "x": to_bf16(x)}


def mse_weight(rows: int = 4096, cols: int = 4096, seed: int = 0):
    """0.02 * Student-t(nu=3) weight (the MSE-vs-absmax workload)."""
    return to_bf16(student_t((rows, cols), 3, 0.02, seed, STREAM_W))


def activation(m: int, k: int, seed: int = 0, stream: int = STREAM_X, n_outlier_channels: int = 4,
               factor: float = 50.0):
    """N(0,1) activation with a few outlier input channels."""
    x = normal((m, k), seed, stream)
    if n_outlier_channels:
        x = with_outlier_channels(x, n_outlier_channels, factor, seed, stream + 100)
    return to_bf16(x)


def gaussian_weight(n: int, k: int, std: float = 0.02, seed: int = 0, stream: int = STREAM_W):
    return to_bf16(normal((n, k), seed, stream, std))


def t4_weight(n: int, k: int, seed: int = 0, stream: int = STREAM_W):
    """0.015 * Student-t(nu=4) weight (31B-class layer)."""
    return to_bf16(student_t((n, k), 4, 0.015, seed, stream))


def decode(m: int, seed: int = 0):
    return {"x": activation(m, 4096, seed), "w": gaussian_weight(14336, 4096, 0.02, seed)}


def prefill(seed: int = 0):
    return {
        "x_up": activation(4096, 4096, seed, STREAM_X),
        "w_up": gaussian_weight(14336, 4096, 0.02, seed, STREAM_W),
        "x_down": activation(4096, 14336, seed, STREAM_X2),
        "w_down": gaussian_weight(4096, 14336, 0.02, seed, STREAM_W2),
    }


def dense31b(m: int, seed: int = 0):
    return {
        "w": t4_weight(21504, 5376, seed, STREAM_W),
        "w2": t4_weight(5376, 21504, seed, STREAM_W2),
        "x": activation(m, 5376, seed, STREAM_X, n_outlier_channels=0),
        "x2": activation(m, 21504, seed, STREAM_X2, n_outlier_channels=0),
    }


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """CPU bf16 tensor -> uint16 numpy view of its bit patterns."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
