"""Helpers shared by the GPU parity tests (test infrastructure; imports the oracle).

* ``oracle_quantize``: the oracle's quantizer on a whole tensor, the rows split
  over host threads (the oracle's C functions run without the Python lock), with
  the global scale computed once from the whole tensor -- the same arithmetic as
  one ``oracle.quantize`` call, only faster on large tensors.
* ``check_gemm``: the GEMM acceptance test, per element, against the oracle's
  float64 product of the dequantized operands (ref) and S = sum_k |a_k b_k|:
    - the accumulation bound stated for the method, |C - ref| <= 1e-3 S + 1e-6,
      plus the rounding of the result to BF16, which the output format forces:
      half a BF16 ulp of C;
    - every element that misses the bare bound (this can happen only through that
      output rounding, when one product dominates the sum) is BF16_RNE(ref) to
      within one BF16 ulp;
    - at least 90 % of the elements equal BF16_RNE(ref) exactly (a wrong scale on a
      few blocks would stay inside the bound but not inside this).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
import workloads

THREADS = max(1, os.cpu_count() or 1)


def oracle_quantize(x, mode=oracle.SCALE_ABSMAX, sg=None):
    """(codes, linear scales, s_g, block_err) of the oracle for a BF16 CPU tensor."""
    bits = workloads.bf16_bits(x) if isinstance(x, torch.Tensor) else np.ascontiguousarray(x)
    rows, cols = bits.shape
    if sg is None:
        sg = oracle.global_scale(bits)
    sg = np.float32(sg)
    if rows * cols < (1 << 20) or THREADS == 1 or rows < 2:
        return oracle.quantize(bits, mode, sg)
    oracle.e4m3_encode(1.0)  # the oracle fills its E4M3 table on first use: do it before threading
    bounds = np.linspace(0, rows, min(rows, THREADS * 4) + 1).astype(np.int64)
    parts = [(int(a), int(b)) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]
    with ThreadPoolExecutor(THREADS) as ex:
        res = list(ex.map(lambda ab: oracle.quantize(np.ascontiguousarray(bits[ab[0]:ab[1]]), mode, sg), parts))
    codes = np.concatenate([r[0] for r in res])
    scales = np.concatenate([r[1] for r in res])
    err = np.concatenate([r[3] for r in res])
    return codes, scales, sg, err


def operand(q):
    """(codes, scales, s_g) of an oracle_quantize result, the GEMM oracle's operand form."""
    return q[0], q[1], q[2]


def rows_of(op, r0, r1):
    """Rows [r0, r1) of an operand (codes, linear scales, s_g)."""
    return np.ascontiguousarray(op[0][r0:r1]), np.ascontiguousarray(op[1][r0:r1]), op[2]


def gemm_ref_at(a, b, mi, ni):
    """oracle.gemm_f64_at over host threads: (ref, S) at positions (mi[i], ni[i])."""
    mi = np.ascontiguousarray(mi, np.int64)
    ni = np.ascontiguousarray(ni, np.int64)
    if mi.size < 256 or THREADS == 1:
        return oracle.gemm_f64_at(*a, *b, mi, ni)
    oracle.e4m3_encode(1.0)
    idx = np.array_split(np.arange(mi.size), THREADS * 2)
    with ThreadPoolExecutor(THREADS) as ex:
        res = list(ex.map(lambda ii: oracle.gemm_f64_at(*a, *b, mi[ii], ni[ii]), idx))
    return np.concatenate([r[0] for r in res]), np.concatenate([r[1] for r in res])


def gemm_ref_block(a, b, m0, m1, n0, n1):
    """The oracle's float64 GEMM on the output block [m0, m1) x [n0, n1)."""
    A = rows_of(a, m0, m1)
    if THREADS == 1 or (n1 - n0) < 64:
        return oracle.gemm_f64(*A, *rows_of(b, n0, n1))
    oracle.e4m3_encode(1.0)
    cuts = np.linspace(n0, n1, min(n1 - n0, THREADS) + 1).astype(np.int64)
    parts = [(int(x), int(y)) for x, y in zip(cuts[:-1], cuts[1:]) if y > x]
    with ThreadPoolExecutor(THREADS) as ex:
        res = list(ex.map(lambda xy: oracle.gemm_f64(*A, *rows_of(b, xy[0], xy[1])), parts))
    return np.concatenate([r[0] for r in res], axis=1), np.concatenate([r[1] for r in res], axis=1)


def bf16_ulp(v):
    """Spacing of BF16 numbers at |v| (the ulp of the binade holding v; the
    subnormal spacing 2^-133 at and below 2^-126)."""
    a = np.abs(np.asarray(v, np.float64))
    _, e = np.frexp(a)                    # a = m 2^e with 0.5 <= m < 1
    e = np.maximum(e - 1, -126)
    return np.where(a == 0, 2.0 ** -133, np.ldexp(1.0, e - 7))


def bf16_rne(v):
    return torch.from_numpy(np.asarray(v, np.float64).astype(np.float32)).to(torch.bfloat16).double().numpy()


def check_gemm(c, ref, absum, min_exact=0.9, where=""):
    """The acceptance test described in the module docstring, element by element."""
    c = np.asarray(c, np.float64)
    err = np.abs(c - ref)
    bare = 1e-3 * absum + 1e-6
    allow = bare + 0.5 * bf16_ulp(c)
    bad = err > allow
    if bad.any():
        i = np.unravel_index(np.argmax(err - allow), err.shape)
        raise AssertionError(f"{where}: {int(bad.sum())} elements out of bound; worst at {i}: C={c[i]!r} "
                             f"ref={ref[i]!r} S={absum[i]!r}")
    over = err > bare
    if over.any():
        rne = bf16_rne(ref[over])
        far = np.abs(c[over] - rne) > bf16_ulp(rne)
        assert not far.any(), f"{where}: {int(far.sum())} elements miss the bare bound by more than output rounding"
    exact = float(np.mean(c == bf16_rne(ref)))
    assert exact >= min_exact, f"{where}: only {exact:.3f} of the elements equal BF16(ref)"
    return exact


def upload(op, device="cuda"):
    """An oracle operand (codes, linear scales, s_g) as a device NVFP4Tensor with swizzled scales."""
    import w4a4_gemm_quantize_b200 as nv
    codes, sc, sg = op
    rows, half = codes.shape
    return nv.NVFP4Tensor(torch.from_numpy(np.ascontiguousarray(codes)).to(device),
                          torch.from_numpy(oracle.swizzle_scales(sc)).to(device),
                          torch.tensor([sg], dtype=torch.float32, device=device), rows, half * 2, nv.SF_SWIZZLED)


def sample_positions(M, N, n_random=3000, tile=256, last_row_cols=32, seed=0):
    """Output positions to check on a large GEMM: random ones, every row of the last
    M-tile (a few random columns each), the last columns of the last row."""
    r = np.random.default_rng(seed)
    mi = [r.integers(0, M, n_random)]
    ni = [r.integers(0, N, n_random)]
    last0 = (M - 1) // tile * tile
    rows = np.repeat(np.arange(last0, M), last_row_cols)
    mi.append(rows)
    ni.append(r.integers(0, N, rows.size))
    mi.append(np.full(min(N, 64), M - 1))
    ni.append(np.arange(N - min(N, 64), N))
    return np.concatenate(mi), np.concatenate(ni)


def check_gemm_large(out, a, b, where, tile=256, seed=0):
    """Sampled positions plus the full first and last tile x tile output blocks."""
    M, N = out.shape
    got = out.float().cpu().numpy()
    mi, ni = sample_positions(M, N, tile=tile, seed=seed)
    ref, absum = gemm_ref_at(a, b, mi, ni)
    check_gemm(got[mi, ni], ref, absum, where=f"{where} sampled")
    m_last = (M - 1) // tile * tile
    n_last = (N - 1) // tile * tile
    for (m0, n0) in {(0, 0), (m_last, n_last)}:
        m1, n1 = min(M, m0 + tile), min(N, n0 + tile)
        ref, absum = gemm_ref_block(a, b, m0, m1, n0, n1)
        check_gemm(got[m0:m1, n0:n1], ref, absum, where=f"{where} tile ({m0},{n0})")
