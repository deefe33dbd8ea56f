"""Pins of the oracle's MXFP4 functions (CPU).

The pages name MXFP4 ("Cuantización en Producción: AWQ, GPTQ, GGUF K-quants, FP8,
MXFP4/NVFP4", section "MXFP4 / NVFP4: Blackwell agresivo") but give neither its
block size nor its scale type; the oracle follows the public OCP Microscaling
Formats (MX) specification v1.0: 32-value blocks, an E8M0 scale 2^(floor(log2 amax)
- 2) clamped to the E8M0 range, E2M1 elements rounded to nearest (ties to even,
saturating at 6).  These tests check it against a library codec (ml_dtypes'
float8_e8m0fnu and float4_e2m1fn), a restatement with numpy's exact frexp / ldexp,
brute force, the rule's invariant and exact rational sums.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

import oracle
import workloads

E2M1 = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def test_e8m0_decode_matches_ml_dtypes():
    lib = np.arange(255, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    ours = np.array([oracle.e8m0_decode(b) for b in range(255)])
    assert np.array_equal(lib, ours)
    assert np.isnan(oracle.e8m0_decode(255))


def mx_blocks():
    r = np.random.default_rng(7)
    parts = [r.standard_t(3, size=(64, 256)) * 0.02,
             r.standard_normal((32, 256)) * np.repeat(2.0 ** r.uniform(-130, 120, (32, 8)), 32, axis=1),
             np.repeat(r.uniform(-8, 8, (4, 8)), 32, axis=1)]
    z = np.zeros((4, 256))
    z[1] = -0.0
    z[2, 5] = 1e-39                    # a BF16 subnormal alone in its block: the scale clamps
    z[3, 40] = 3.0e38                  # near the BF16 maximum
    parts.append(z)
    g = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    pw = 2.0 ** r.integers(-20, 20, (8, 8))                 # one power of two per block
    on_grid = r.choice(g, (8, 256)) * r.choice([-1, 1], (8, 256)) * np.repeat(pw, 32, axis=1)
    on_grid[:, ::32] = 6 * pw                                 # each block's maximum: 6 times its power
    parts.append(on_grid)
    return workloads.to_bf16(np.concatenate(parts).astype(np.float32))


def restated(x):
    """numpy restatement: shared = floor(log2 amax) - 2 (exact via frexp), clamped to
    [-127, 127], codes = sign | E2M1(|x| / 2^shared) by ml_dtypes' cast."""
    v = x.float().numpy().astype(np.float64).reshape(-1, 32)
    amax = np.abs(v).max(axis=1)
    _, e = np.frexp(np.where(amax > 0, amax, 1.0))
    shared = np.where(amax > 0, e - 1 - 2, -127)
    shared = np.clip(shared, -127, 127)
    y = np.ldexp(np.abs(v), -shared[:, None]).astype(np.float32)
    mag = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 7
    mag = np.where(v == 0, 0, mag)
    codes = (np.signbit(v).astype(np.uint8) << 3) | mag.astype(np.uint8)
    return codes, (shared + 127).astype(np.uint8)


def test_mx_quantize_equals_restatement():
    x = mx_blocks()
    codes, scales = oracle.quantize_mx(x)
    rc, rs = restated(x)
    assert np.array_equal(scales.reshape(-1), rs)
    assert np.array_equal(oracle.unpack_codes(codes).reshape(-1, 32), rc)


def test_mx_block_maximum_lands_in_4_to_8_and_codes_are_nearest():
    """The rule puts the block maximum in [4, 8) times the scale, so its code is 4 or 6
    (values in (6, 8) saturate); brute force: every code is the nearest grid value."""
    x = mx_blocks()
    codes, scales = oracle.quantize_mx(x)
    v = x.float().numpy().astype(np.float64).reshape(-1, 32)
    q = oracle.unpack_codes(codes).reshape(-1, 32)
    X = np.ldexp(1.0, scales.reshape(-1).astype(np.int64) - 127)
    amax = np.abs(v).max(axis=1)
    normal = (amax > 0) & (scales.reshape(-1) > 0) & (scales.reshape(-1) < 254)
    ratio = amax[normal] / X[normal]
    assert np.all((ratio >= 4) & (ratio < 8))
    top = np.take_along_axis(q, np.abs(v).argmax(axis=1)[:, None], axis=1)[:, 0] & 7
    assert set(np.unique(top[normal])) <= {6, 7}            # the codes of 4 and 6
    for i in np.random.default_rng(1).choice(v.shape[0], 40, replace=False):
        for k in range(32):
            y = Fraction(float(abs(v[i, k]))) / Fraction(2) ** (int(scales.reshape(-1)[i]) - 127)
            if y >= 6:
                want = 7
            else:
                d = [abs(y - Fraction(float(E2M1[c]))) for c in range(8)]
                best = min(d)
                cands = [c for c in range(8) if d[c] == best]
                want = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
            if v[i, k] == 0:
                want = 0
            assert (q[i, k] & 7) == want, (i, k, v[i, k], q[i, k], want)


def test_mx_dequantize_round_trips_grid_values():
    """Values that are E2M1 grid points times a block's power of two are reproduced exactly."""
    x = mx_blocks()[-8:]
    codes, scales = oracle.quantize_mx(x)
    assert np.array_equal(oracle.dequantize_mx(codes, scales), workloads.bf16_bits(x))


def test_mx_gemm_reference_exact_on_tiny_k():
    r = np.random.default_rng(3)
    M, N, K = 3, 4, 64
    a = workloads.to_bf16(r.standard_normal((M, K)).astype(np.float32))
    b = workloads.to_bf16(r.standard_normal((N, K)).astype(np.float32))
    ac, asc = oracle.quantize_mx(a)
    bc, bsc = oracle.quantize_mx(b)
    got, absum = oracle.gemm_mx_f64(ac, asc, bc, bsc)
    qa, qb = oracle.unpack_codes(ac), oracle.unpack_codes(bc)
    for m in range(M):
        for n in range(N):
            s = Fraction(0)
            t = Fraction(0)
            for k in range(K):
                va = Fraction(float(E2M1[qa[m, k]])) * Fraction(2) ** (int(asc[m, k // 32]) - 127)
                vb = Fraction(float(E2M1[qb[n, k]])) * Fraction(2) ** (int(bsc[n, k // 32]) - 127)
                s += va * vb
                t += abs(va * vb)
            assert got[m, n] == float(s) and absum[m, n] == float(t)
