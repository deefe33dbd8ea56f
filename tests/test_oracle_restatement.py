"""An independent restatement of the block-scale rules, compared bit for bit with the oracle.

The oracle's absmax, MSE and four-over-six block quantization is written a second
time here with other tools -- vectorised numpy binary32 arithmetic, torch's
float8_e4m3fn cast for the E4M3 scale, ml_dtypes' float4_e2m1fn cast for the E2M1
codes, and an exactly rounded binary32 fused multiply-add -- and without calling
the oracle.  On several thousand blocks (Student-t weights, blocks spread over the
whole E4M3 range relative to the global scale, blocks on the grid, all-zero and
-0 blocks, single-outlier blocks) the codes, the scale bytes and the binary32
block errors must equal the oracle's exactly.

Rules restated (page "Tu pipeline NVFP4: meter 62 GB de modelo en 24 GB de
laptop", section 2, boxes "Fundamento matemático: bitfield E2M1 y cuantización
jerárquica" and "Derivación del objetivo de optimización MSE vs Absmax"; the
search over factors of the absmax scale of "NVFP4 en difusión: la misma
cuantización, un motor completamente distinto", section 8 "Para practicar"):
  absmax scale  s = E4M3(RN32(amax_b / RN32(6 s_g)))            (saturating RNE)
  MSE           f = RN32((3+i)/10), i = 7 .. 0; s_f = E4M3(RN32(f v_b)); keep the
                first candidate and later ones only on a strictly smaller error
  four-over-six the absmax scale, then E4M3(RN32(amax_b / RN32(4 s_g))) on a strictly
                smaller error
  encode        eff = RN32(dec(s) s_g), r = RN32(1/eff), code = sign | E2M1(RN32(|x| r))
  error         d_k = fma(-q_k, eff, x_k), e = fma(d_k, d_k, e), k = 0..15
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads

F32 = np.float32


# --- exact binary32 arithmetic helpers ------------------------------------------------------------

def _two_sum(a, b):
    """Knuth's error-free sum of float64 arrays: s = fl(a + b), s + t = a + b exactly."""
    s = a + b
    bb = s - a
    t = (a - (s - bb)) + (b - bb)
    return s, t


def fma32(a, b, c):
    """RN32(a*b + c) for binary32 arrays, rounded once: the product is exact in binary64,
    the sum is carried exactly as s + t, and s is rounded to binary32 with t deciding the
    direction when s falls exactly halfway between two binary32 numbers."""
    a, b, c = (np.asarray(v, F32) for v in (a, b, c))
    p = a.astype(np.float64) * b.astype(np.float64)
    s, t = _two_sum(p, np.broadcast_to(c, p.shape).astype(np.float64))
    r = s.astype(F32)
    toward = np.where(s > r.astype(np.float64), np.inf, -np.inf).astype(F32)
    other = np.nextafter(r, toward)
    mid = (r.astype(np.float64) + other.astype(np.float64)) / 2
    halfway = (s == mid) & (s != r.astype(np.float64)) & (t != 0)
    goes_other = halfway & (np.sign(t) == np.sign(other.astype(np.float64) - r.astype(np.float64)))
    return np.where(goes_other, other, r).astype(F32)


def e4m3_byte(u):
    """Nearest E4M3 byte of u >= 0, ties to even, saturating at 448 (torch's cast)."""
    u = np.minimum(np.asarray(u, F32), F32(448))
    return torch.from_numpy(np.ascontiguousarray(u)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_value(s):
    return torch.from_numpy(np.ascontiguousarray(s, np.uint8)).view(torch.float8_e4m3fn).float().numpy()


E2M1 = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(F32)


def encode(xb, eff):
    """Signed 4-bit codes of blocks xb (n, 16) under per-block eff (n,), and the block errors."""
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        r = F32(1) / eff
        y = np.abs(xb) * r[:, None]
    mag = np.nan_to_num(y, nan=0.0).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 7
    mag = np.where((eff[:, None] == 0) | (xb == 0), 0, mag).astype(np.uint8)
    codes = (np.signbit(xb).astype(np.uint8) << 3) | mag
    q = E2M1[codes]
    e = np.zeros(xb.shape[0], F32)
    for k in range(16):
        d = fma32(-q[:, k], eff, xb[:, k])
        e = fma32(d, d, e)
    return codes, e


def restated_quantize(xb, sg, mode, factors=None):
    """(scale bytes (n,), codes (n, 16), errors (n,)) of blocks xb (n, 16)."""
    xb = np.asarray(xb, F32)
    sg = F32(sg)
    amax = np.abs(xb).max(axis=1)
    vb = amax / (F32(6) * sg)
    if factors is None:
        factors = [F32(3 + i) / F32(10) for i in range(7, -1, -1)] if mode == oracle.SCALE_MSE else [F32(1)]
    best = None
    for f in factors:
        s = e4m3_byte(F32(f) * vb)
        codes, e = encode(xb, e4m3_value(s) * sg)
        if best is None:
            best = [s, codes, e]
        else:
            take = e < best[2]
            best = [np.where(take, s, best[0]), np.where(take[:, None], codes, best[1]), np.where(take, e, best[2])]
    if mode == oracle.SCALE_FOUR_OVER_SIX:
        s = e4m3_byte(amax / (F32(4) * sg))
        codes, e = encode(xb, e4m3_value(s) * sg)
        take = e < best[2]
        best = [np.where(take, s, best[0]), np.where(take[:, None], codes, best[1]), np.where(take, e, best[2])]
    return best


# --- the blocks ---------------------------------------------------------------------------------

def make_blocks():
    """Rows of 256 values (16 blocks each), BF16-rounded; returns the (R, 256) bf16 tensor."""
    r = np.random.default_rng(2024)
    rows = []
    rows.append(r.standard_t(3, size=(160, 256)) * 0.02)                 # MSE workload weights
    rows.append(r.standard_t(4, size=(96, 256)) * 0.015)                 # 31B-class weights
    # blocks spread over ~40 binades below the tensor maximum: block scales run from 448
    # down through the E4M3 subnormals to zero, where candidates collapse to one code
    spread = r.standard_normal((64, 256)) * np.repeat(2.0 ** -r.uniform(0, 40, (64, 16)), 16, axis=1)
    rows.append(spread)
    # blocks on the E2M1 grid (exact under the absmax scale: no candidate can improve)
    g = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    on_grid = r.choice(g, size=(16, 256)) * r.choice([-1, 1], size=(16, 256))
    on_grid[:, ::16] = 6.0
    rows.append(on_grid * 0.125)
    # single-outlier blocks and all-equal blocks
    out = r.standard_normal((16, 256)) * 0.01
    out[:, 5::16] = r.choice([-1, 1], (16, 16)) * r.uniform(0.5, 8, (16, 16))
    rows.append(out)
    rows.append(np.repeat(r.uniform(-2, 2, (8, 16)), 16, axis=1))
    z = np.zeros((4, 256))
    z[1] = -0.0
    z[2, ::3] = -0.0
    rows.append(z)
    a = np.concatenate(rows).astype(np.float32)
    a[0, 7] = 3.0  # the tensor maximum
    return workloads.to_bf16(a)


def _oracle_blocks(x, mode, sg):
    codes, scales, _, err = oracle.quantize(x, mode, sg)
    n = scales.size
    return scales.reshape(n), oracle.unpack_codes(codes).reshape(n, 16), err.reshape(n)


@pytest.fixture(scope="module")
def blocks():
    x = make_blocks()
    xb = x.float().numpy().reshape(-1, 16)
    sg = np.abs(xb).max() / F32(2688)   # reading R1, restated
    assert sg.dtype == F32
    assert sg == oracle.global_scale(x)
    return x, xb, sg


@pytest.mark.parametrize("mode", [oracle.SCALE_ABSMAX, oracle.SCALE_MSE, oracle.SCALE_FOUR_OVER_SIX])
def test_restatement_equals_oracle_bit_for_bit(blocks, mode):
    x, xb, sg = blocks
    assert xb.shape[0] >= 4096
    s_r, c_r, e_r = restated_quantize(xb, sg, mode)
    s_o, c_o, e_o = _oracle_blocks(x, mode, sg)
    bad = np.nonzero(s_r != s_o)[0]
    assert bad.size == 0, f"scale bytes differ on {bad.size} blocks, first {bad[:5]}: {s_r[bad[:5]]} vs {s_o[bad[:5]]}"
    assert np.array_equal(c_r, c_o), f"codes differ on {int((c_r != c_o).any(axis=1).sum())} blocks"
    assert np.array_equal(e_r.view(np.uint32), e_o.view(np.uint32)), \
        f"errors differ on {int((e_r != e_o).sum())} blocks"


def test_mse_choices_are_varied(blocks):
    """The blocks make the MSE walk choose a scale below the absmax one on many blocks,
    with several different factors, so the comparison above exercises the walk.  (On
    these blocks, as on the workloads' weights, the factors 0.3-0.5 never win: clipping
    the block maximum to 6 at such a scale costs more than it saves on the other values.)"""
    x, xb, sg = blocks
    s_abs, _, _ = restated_quantize(xb, sg, oracle.SCALE_ABSMAX)
    s_mse, _, _ = restated_quantize(xb, sg, oracle.SCALE_MSE)
    vb = np.abs(xb).max(axis=1) / (F32(6) * sg)
    chosen = set()
    for i in range(8):
        f = F32(3 + i) / F32(10)
        if ((s_mse == e4m3_byte(f * vb)) & (s_mse != s_abs)).any():
            chosen.add(i)
    assert (s_mse != s_abs).mean() > 0.1
    assert {5, 6} <= chosen and len(chosen) >= 3, chosen


_MSE = [F32(3 + i) / F32(10) for i in range(7, -1, -1)]


@pytest.mark.parametrize("name,factors", [
    ("0.9 dropped", [f for f in _MSE if f != F32(0.9)]),
    ("0.8 read as 0.85", [F32(0.85) if f == F32(0.8) else f for f in _MSE]),
    ("0.9 read as 0.95", [F32(0.95) if f == F32(0.9) else f for f in _MSE]),
])
def test_a_changed_walk_is_detected(blocks, name, factors):
    """The comparison has teeth: a slip in a candidate that wins changes the result on
    some of these blocks."""
    x, xb, sg = blocks
    s_o, c_o, e_o = _oracle_blocks(x, oracle.SCALE_MSE, sg)
    s_m, c_m, e_m = restated_quantize(xb, sg, oracle.SCALE_MSE, factors=factors)
    differs = (s_m != s_o) | (c_m != c_o).any(axis=1) | (e_m.view(np.uint32) != e_o.view(np.uint32))
    assert differs.sum() >= 10, name


def test_an_unfused_error_sum_is_detected(blocks, monkeypatch):
    """The block error is a chain of fused multiply-adds; the same sum with separately
    rounded products and additions gives different binary32 errors on many blocks."""
    x, xb, sg = blocks
    _, _, e_o = _oracle_blocks(x, oracle.SCALE_MSE, sg)
    import test_oracle_restatement as me
    monkeypatch.setattr(me, "fma32", lambda a, b, c: (np.asarray(a, F32) * np.asarray(b, F32)
                                                      + np.asarray(c, F32)).astype(F32))
    _, _, e_m = me.restated_quantize(xb, sg, oracle.SCALE_MSE)
    assert (e_m.view(np.uint32) != e_o.view(np.uint32)).sum() > 100


def test_fma32_against_exact_rationals():
    """The exactly rounded fused multiply-add used above, against rational arithmetic."""
    from fractions import Fraction
    r = np.random.default_rng(5)
    a = (r.standard_normal(400) * 2.0 ** r.integers(-30, 30, 400)).astype(F32)
    b = (r.standard_normal(400) * 2.0 ** r.integers(-30, 30, 400)).astype(F32)
    c = (r.standard_normal(400) * 2.0 ** r.integers(-60, 60, 400)).astype(F32)
    # halfway cases: c = -a*b + a binary32 midpoint's offset
    got = fma32(a, b, c)
    for i in range(a.size):
        exact = Fraction(float(a[i])) * Fraction(float(b[i])) + Fraction(float(c[i]))
        lo = F32(float(exact))
        cands = {lo, np.nextafter(lo, F32(np.inf)), np.nextafter(lo, F32(-np.inf))}
        dist = {v: abs(Fraction(float(v)) - exact) for v in cands}
        best = min(dist.values())
        near = [v for v in cands if dist[v] == best]
        if len(near) > 1:
            near = [v for v in near if (int(np.array(v, F32).view(np.uint32)) & 1) == 0]
        assert got[i] == near[0], (a[i], b[i], c[i], got[i], near[0])
    # a product exactly halfway between two binary32 numbers, nudged by a tiny c
    a2 = np.array([1 + 2.0 ** -12] * 3, F32)
    b2 = np.array([1 + 2.0 ** -12] * 3, F32)    # a*b = 1 + 2^-11 + 2^-24: halfway above 1 + 2^-11
    c2 = np.array([0.0, 2.0 ** -60, -(2.0 ** -60)], F32)
    g2 = fma32(a2, b2, c2)
    base = F32(1 + 2.0 ** -11)
    assert g2[0] == base                       # tie: to even (1 + 2^-11 has an even last bit)
    assert g2[1] == np.nextafter(base, F32(2))
    assert g2[2] == base
