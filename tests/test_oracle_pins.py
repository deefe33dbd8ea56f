"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test checks the oracle against what the pages print, a library routine,
brute force on tiny inputs, or an invariant of the method, chosen so that a
plausible slip (a dropped term, a wrong tie rule, a swapped nibble, a transposed
operand) fails at least one of them.

Pages: [G4] "Tu pipeline NVFP4: meter 62 GB de modelo en 24 GB de laptop";
[DF] "NVFP4 en difusión: la misma cuantización, un motor completamente distinto".
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def f32(v):
    return float(np.float32(v))


# --- E2M1 --------------------------------------------------------------------------------------

def test_e2m1_decode_matches_printed_grid():
    """[G4] box "Fundamento matemático": bitfield evaluation and the grid G_E2M1."""
    rows = read_golden("e2m1_grid.txt")
    assert len(rows) == 16
    for s, e, m, value in rows:
        code = (int(s) << 3) | (int(e) << 1) | int(m)
        got = oracle.e2m1_decode(code)
        assert got == float(value), (code, got, value)
        assert np.signbit(got) == (int(s) == 1)
    printed = sorted({abs(float(r[3])) for r in rows})
    assert printed == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_matches_ml_dtypes():
    """Library routine: ml_dtypes' float4_e2m1fn decodes the same 16 codes."""
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = np.array([oracle.e2m1_decode(c) for c in range(16)])
    assert np.array_equal(lib, ours)
    assert np.array_equal(np.signbit(lib), np.signbit(ours))


def test_e2m1_encode_matches_ml_dtypes_on_every_bf16():
    """Every non-negative BF16 value: RNE to E2M1 with saturation, as ml_dtypes rounds it."""
    bits = np.arange(0, 0x7F81, dtype=np.uint32)  # +0 .. +inf
    y = (bits << 16).view(np.float32)
    ours = oracle.e2m1_encode_mag_array(y)
    lib = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0x7
    bad = np.nonzero(ours != lib)[0]
    assert bad.size == 0, [(float(y[i]), int(ours[i]), int(lib[i])) for i in bad[:10]]


def test_e2m1_encode_bruteforce_exact_midpoints():
    """Brute force in exact rationals around every midpoint of the grid."""
    grid = [Fraction(v).limit_denominator(4) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    probes = []
    for a, b in zip(grid, grid[1:]):
        mid = np.float32(float((a + b) / 2))
        probes += [np.nextafter(mid, np.float32(0)), mid, np.nextafter(mid, np.float32(10))]
    probes += [np.float32(6.0), np.float32(6.5), np.float32(1e30), np.float32(np.inf)]
    for y in probes:
        got = oracle.e2m1_encode_mag(float(y))
        if not np.isfinite(y):
            assert got == 7
            continue
        fy = Fraction(float(y))
        dist = [abs(fy - g) for g in grid]
        best = min(dist)
        cands = [c for c in range(8) if dist[c] == best]
        want = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        assert got == want, (float(y), got, want)


# --- E4M3 --------------------------------------------------------------------------------------

def test_e4m3_decode_matches_torch_all_codes():
    """Library routine: torch.float8_e4m3fn decodes all 256 byte patterns the same."""
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().double().numpy()
    ours = np.array([oracle.e4m3_decode(b) for b in range(256)])
    nan = np.isnan(lib)
    assert np.array_equal(nan, np.isnan(ours))
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(lib[~nan], ours[~nan])
    assert oracle.e4m3_decode(0x7E) == 448.0  # largest finite
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9  # smallest subnormal


def test_e4m3_encode_matches_torch_below_saturation():
    """RNE to E4M3 for a dense sweep of binary32 values in [0, 464), plus every E4M3
    value, every midpoint and their neighbours, against torch's float8_e4m3fn cast."""
    top = np.array([464.0], np.float32).view(np.uint32)[0]
    sweep = np.arange(0, top, 997, dtype=np.uint32).view(np.float32)
    vals = np.array([oracle.e4m3_decode(b) for b in range(0x7F)], np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e3)),
                           vals.astype(np.float32)])
    u = np.concatenate([sweep, near]).astype(np.float32)
    ours = oracle.e4m3_encode_array(u)
    lib = torch.from_numpy(u).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != lib)[0]
    assert bad.size == 0, [(float(u[i]), int(ours[i]), int(lib[i])) for i in bad[:10]]


def test_e4m3_encode_saturates_at_448():
    """Reading R4: values past the largest finite E4M3 clamp to 448 (never NaN)."""
    for u in (448.0, 460.0, 464.0, 480.0, 500.0, 1e6, 3.0e38, float("inf")):
        assert oracle.e4m3_encode(u) == 0x7E


# --- BF16 rounding -----------------------------------------------------------------------------

def test_bf16_rounding_matches_torch():
    r = np.random.default_rng(1)
    bits = r.integers(0, 2**32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    ours = oracle.f32_to_bf16_array(f)
    lib = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)


# --- the worked example and the memory arithmetic -----------------------------------------------

def test_grid_at_scale_0p01_matches_page():
    """[DF] section 3: a block with scale 0.01 can only hold 0, ±0.005, ..., ±0.06."""
    rows = read_golden("grid_scale_0p01.txt")
    scale = float(rows[0][0])
    printed = [float(r[0]) for r in rows[1:]]
    # eff = dec(s_b) * s_g with s_b = 1.0 (E4M3 0x38) and s_g = RN32(0.01).
    codes = np.array([[c | (c + 8) << 4 for c in range(8)]], np.uint8)  # +q in low, -q in high nibble
    out = oracle.dequantize(codes, np.array([[0x38]], np.uint8), np.float32(scale))
    vals = workloads.from_bits(out).float().numpy()[0]
    pos, neg = vals[0::2], vals[1::2]
    want = torch.tensor(printed, dtype=torch.float32).to(torch.bfloat16).float().numpy()
    assert np.array_equal(pos, want)
    assert np.array_equal(neg, -want)


def test_memory_arithmetic_matches_page():
    """4.5 effective bits per weight: codes rows*cols/2 bytes + E4M3 scales rows*cols/16."""
    g = {k: float(v) for k, v in read_golden("memory_arithmetic.txt")}
    x = workloads.to_bf16(np.random.default_rng(0).standard_normal((64, 256), dtype=np.float32))
    codes, scales, sg, _ = oracle.quantize(x)
    n = x.numel()
    assert codes.nbytes / n == g["code_bytes_per_weight"]
    assert scales.nbytes / n == g["scale_bytes_per_weight"]
    bits = 8 * (codes.nbytes + scales.nbytes) / n
    assert bits == g["bits_nvfp4"]
    assert round(100 * scales.nbytes / (codes.nbytes + scales.nbytes)) == g["scale_share_percent"]
    p31 = g["params_31b"]
    for fmt in ("fp32", "bf16", "fp8", "fp4"):
        assert p31 * g["bits_" + fmt] / 8 / 1e9 == g[f"gb_{fmt}_31b"]
    assert round(p31 * bits / 8 / 1e9, 1) == g["gb_nvfp4_31b_text"]
    assert abs(p31 * bits / 8 / 1e9 - g["gb_nvfp4_31b_table"]) < 0.1
    assert g["params_8b"] * 2 / 1e9 == g["gb_bf16_8b"]
    assert g["params_8b"] * bits / 8 / 1e9 == g["gb_nvfp4_8b"]


# --- quantization: brute force and invariants ---------------------------------------------------

def _tiny_tensor(rows=24, cols=128, seed=3):
    r = np.random.default_rng(seed)
    a = (r.standard_t(3, size=(rows, cols)) * 0.02).astype(np.float32)
    a[0, :16] = 0.0                       # all-zero block
    a[1, 16:32] = -0.0                    # negative zeros
    a[2, :16] *= 1e-6                     # block far below the tensor maximum
    a[3, 5] = 40.0                        # the global maximum (its block gets scale 448)
    a[4, 0:16] = np.linspace(-1, 1, 16)   # values spread over the whole grid
    return workloads.to_bf16(a)


def _eff(scales, sg):
    dec = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    return (dec[scales].astype(np.float32) * np.float32(sg)).astype(np.float32)


@pytest.mark.parametrize("mode", [oracle.SCALE_ABSMAX, oracle.SCALE_MSE])
def test_each_code_is_the_nearest_grid_point(mode):
    """[G4] q_ij = argmin_q |W_ij/(s_b s_g) - q|: brute force over all 16 signed codes,
    given the block's effective scale eff = s_b s_g (RN32) and y = |x| * RN32(1/eff)."""
    x = _tiny_tensor()
    codes, scales, sg, _ = oracle.quantize(x, mode)
    xs = x.float().numpy()
    q = oracle.unpack_codes(codes)
    eff = np.repeat(_eff(scales, sg), 16, axis=1)
    grid = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for (i, j), xv in np.ndenumerate(xs):
        e = eff[i, j]
        if e == 0 or xv == 0:
            assert q[i, j] & 7 == 0
        else:
            y = np.float32(np.float32(abs(xv)) * (np.float32(1) / e)) * np.sign(xv)
            d = np.abs(float(y) - grid)
            best = np.nonzero(d == d.min())[0]
            best = [c for c in best if np.sign(grid[c]) == np.sign(xv) or grid[c] == 0]
            if len(best) > 1:
                best = [c for c in best if c % 2 == 0]
            assert (q[i, j] & 7) == (best[0] & 7), (i, j, xv, y, q[i, j], best)
        assert (q[i, j] >> 3) == int(np.signbit(xv))


def test_absmax_largest_element_lands_on_6():
    """[G4] "Derivación ... MSE vs Absmax": absmax makes the block's largest element
    coincide with the grid's extreme 6 (for every block with a normal E4M3 scale)."""
    x = workloads.mse_weight(64, 512, seed=5)
    codes, scales, sg, _ = oracle.quantize(x, oracle.SCALE_ABSMAX)
    q = oracle.unpack_codes(codes).reshape(64, 32, 16)
    xs = np.abs(x.float().numpy()).reshape(64, 32, 16)
    arg = xs.argmax(axis=2)
    top = np.take_along_axis(q, arg[..., None], axis=2)[..., 0] & 7
    normal = scales >= 0x08
    assert normal.sum() > 1000
    assert np.all(top[normal] == 7)


def test_block_with_global_max_gets_largest_scale():
    """Reading R1 (s_g = amax/(6*448)): the block holding the tensor maximum gets
    the largest E4M3 scale 448, so block scales cover the range relative to it."""
    for seed in range(4):
        x = workloads.mse_weight(32, 256, seed=seed)
        codes, scales, sg, _ = oracle.quantize(x, oracle.SCALE_ABSMAX)
        xs = np.abs(x.float().numpy())
        r, c = np.unravel_index(xs.argmax(), xs.shape)
        assert scales[r, c // 16] == 0x7E
        assert scales.max() == 0x7E


def test_global_scale_zero_tensor_and_codes():
    z = workloads.to_bf16(np.zeros((4, 32), np.float32))
    codes, scales, sg, err = oracle.quantize(z)
    assert sg == np.float32(1.0)
    assert not codes.any() and not scales.any() and not err.any()
    nz = workloads.to_bf16(-np.zeros((4, 32), np.float32))
    codes, _, _, _ = oracle.quantize(nz)
    assert np.all(codes == 0x88)  # the sign of -0 is kept (reading R3)


def _sse64(x, codes, scales, sg):
    """Block SSE in float64 from the exact reconstruction q * RN32(dec(s) s_g)."""
    grid = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    q = grid[oracle.unpack_codes(codes)]
    eff = np.repeat(_eff(scales, sg).astype(np.float64), 16, axis=1)
    d = x.float().numpy().astype(np.float64) - q * eff
    return (d * d).reshape(d.shape[0], -1, 16).sum(axis=2)


def test_mse_never_worse_than_absmax_and_ties_keep_absmax():
    """MSE picks among candidates that include the absmax scale, so per block its error
    is never above absmax; where nothing improves it returns the absmax bits."""
    x = workloads.mse_weight(128, 512, seed=7)
    ca, sa, sg, ea = oracle.quantize(x, oracle.SCALE_ABSMAX)
    cm, sm, sg2, em = oracle.quantize(x, oracle.SCALE_MSE)
    assert sg == sg2
    assert np.all(em <= ea)
    s_a, s_m = _sse64(x, ca, sa, sg), _sse64(x, cm, sm, sg)
    assert np.all(s_m <= s_a * (1 + 1e-5) + 1e-30)
    same = em == ea
    assert same.sum() > 0 and (~same).sum() > 0
    assert np.array_equal(sm[same], sa[same])
    blk_eq = np.repeat(same, 8, axis=1)
    assert np.array_equal(cm[blk_eq], ca[blk_eq])
    # the oracle's binary32 block error agrees with the float64 one
    assert np.allclose(em, s_m, rtol=1e-4, atol=1e-12)


def test_exhaustive_scale_search_bounds_mse():
    """Brute force over every finite E4M3 block scale: the best of all 127 is never
    worse than the 8-candidate MSE choice, which is never worse than absmax."""
    x = workloads.mse_weight(8, 64, seed=11)  # 32 blocks
    ca, sa, sg, _ = oracle.quantize(x, oracle.SCALE_ABSMAX)
    cm, sm, _, _ = oracle.quantize(x, oracle.SCALE_MSE)
    s_a, s_m = _sse64(x, ca, sa, sg), _sse64(x, cm, sm, sg)
    xs = x.float().numpy()
    grid = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    dec = torch.arange(128, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for r in range(xs.shape[0]):
        for b in range(xs.shape[1] // 16):
            blk = xs[r, 16 * b:16 * b + 16]
            best = np.inf
            for s in range(1, 0x7F):
                eff = np.float32(dec[s] * np.float32(sg))
                y = (np.abs(blk) * (np.float32(1) / eff)).astype(np.float32)
                qm = y.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
                d = np.abs(blk.astype(np.float64)) - qm * np.float64(eff)
                best = min(best, float((d * d).sum()))
            assert best <= s_m[r, b] * (1 + 1e-6) + 1e-30
            assert s_m[r, b] <= s_a[r, b] * (1 + 1e-5) + 1e-30


# --- four-over-six (reading R8) ------------------------------------------------------------------


def _blocks(rows):
    """BF16 tensor from rows of 16 floats (each row one block)."""
    return workloads.to_bf16(np.asarray(rows, np.float32))


def test_four_over_six_picks_the_exact_4_mapping():
    """A block whose maximum sits on 4 of the grid with every value on the E2M1 grid is exact
    when its maximum maps to 4 (s_b = 1 with s_g = 1) and not when it maps to 6
    (4/6 -> E4M3 0.6875, so 4 lands on 5.8 -> 6): four-over-six must take the 4 mapping,
    absmax must not."""
    vals = [4, 3, 2, 1.5, 1, 0.5, 0, -4, -3, -2, -1.5, -1, -0.5, 0, 4, 2]
    x = _blocks([vals])
    ca, sa, _, ea = oracle.quantize(x, oracle.SCALE_ABSMAX, sg=1.0)
    cf, sf, _, ef = oracle.quantize(x, oracle.SCALE_FOUR_OVER_SIX, sg=1.0)
    assert sa[0, 0] == 0x33 and ea[0, 0] > 0          # E4M3 0.6875 = 1.375 * 2^-1 (0 0110 011)
    assert sf[0, 0] == 0x38 and ef[0, 0] == 0.0       # E4M3 1.0
    grid = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(grid[oracle.unpack_codes(cf)][0], np.asarray(vals, np.float64))


def test_four_over_six_keeps_the_exact_6_mapping():
    """A block exact with its maximum on 6 (s_b = 1): the 4 mapping (s_b = 1.5) puts 4 on
    2.67 -> 3, so four-over-six keeps the absmax bits."""
    x = _blocks([[6, 4, 3, 2, 1.5, 1, 0.5, 0, -6, -4, -3, -2, -1.5, -1, -0.5, 0]])
    ca, sa, _, ea = oracle.quantize(x, oracle.SCALE_ABSMAX, sg=1.0)
    cf, sf, _, ef = oracle.quantize(x, oracle.SCALE_FOUR_OVER_SIX, sg=1.0)
    assert sa[0, 0] == 0x38 and ea[0, 0] == 0.0
    assert np.array_equal(cf, ca) and np.array_equal(sf, sa) and ef[0, 0] == 0.0


def test_four_over_six_ties_keep_the_6_mapping():
    """All-zero and one-value blocks: both mappings give zero error, the 6 mapping stays."""
    x = _blocks([[0.0] * 16, [0.0] * 15 + [3.0]])
    ca, sa, sg, _ = oracle.quantize(x, oracle.SCALE_ABSMAX)
    cf, sf, _, ef = oracle.quantize(x, oracle.SCALE_FOUR_OVER_SIX)
    assert np.array_equal(sf, sa) and np.array_equal(cf, ca)


def test_four_over_six_is_the_better_of_two_and_never_worse_than_absmax():
    """Per block: the chosen scale is the absmax scale or E4M3(amax_b / (4 s_g)) (computed
    here with torch's E4M3 conversion), its float64 error is the smaller of the two
    mappings' (brute-force nearest-grid encode), and never above absmax."""
    x = workloads.mse_weight(64, 256, seed=3)
    ca, sa, sg, ea = oracle.quantize(x, oracle.SCALE_ABSMAX)
    cf, sf, sg2, ef = oracle.quantize(x, oracle.SCALE_FOUR_OVER_SIX)
    assert sg == sg2
    assert np.all(ef <= ea)
    xs = x.float().numpy().reshape(64, -1, 16)
    amax = np.abs(xs).max(axis=2).astype(np.float32)
    v4 = (amax / np.float32(np.float32(4) * np.float32(sg))).astype(np.float32)
    s4 = torch.from_numpy(v4).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.all((sf == sa) | (sf == s4))
    s_a, s_f = _sse64(x, ca, sa, sg), _sse64(x, cf, sf, sg)
    assert np.all(s_f <= s_a * (1 + 1e-5) + 1e-30)
    took4 = (sf == s4) & (sf != sa)
    assert took4.sum() > 0 and (~took4).sum() > 0


# --- LoRA branch (reading R9) ----------------------------------------------------------------------


def _bf16_rand(shape, scale, seed):
    return workloads.to_bf16(np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * scale)


def test_lora_exact_integer_case():
    """Small integers (exact in BF16, products and sums exact, t below 256 so exact in BF16):
    the low-rank term equals the integer matmul B (A x) exactly."""
    r = np.random.default_rng(9)
    x = r.integers(-3, 4, size=(5, 24))
    a = r.integers(-2, 3, size=(4, 24))
    b = r.integers(-3, 4, size=(7, 4))
    t_int = x @ a.T
    assert np.abs(t_int).max() < 256
    u, s_u, t = oracle.lora_f64(workloads.to_bf16(x.astype(np.float32)), workloads.to_bf16(a.astype(np.float32)),
                                workloads.to_bf16(b.astype(np.float32)))
    assert np.array_equal(u, (t_int @ b.T).astype(np.float64))
    assert np.array_equal(s_u, (np.abs(t_int)[:, None, :] * np.abs(b)[None, :, :]).sum(axis=2).astype(np.float64))


def test_lora_intermediate_is_the_bf16_rounded_product():
    """The 16-bit intermediate t is torch's BF16 rounding of the binary32 rounding of A x
    (computed here in float64 by numpy), and u = t B^T."""
    x, a, b = _bf16_rand((6, 96), 1.0, 1), _bf16_rand((16, 96), 0.05, 2), _bf16_rand((40, 16), 0.05, 3)
    u, _, t = oracle.lora_f64(x, a, b)
    xf, af, bf = (v.float().numpy().astype(np.float64) for v in (x, a, b))
    t_ref = torch.from_numpy((xf @ af.T).astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(t, t_ref.view(torch.int16).numpy().view(np.uint16))
    tf = t_ref.float().numpy().astype(np.float64)
    assert np.allclose(u, tf @ bf.T, rtol=1e-12, atol=1e-15)
    assert not np.array_equal(tf, xf @ af.T)  # the rounding is visible at this size


def test_lora_zero_rank_or_zero_b_adds_nothing():
    x, a = _bf16_rand((3, 32), 1.0, 4), _bf16_rand((8, 32), 0.1, 5)
    u, s_u, _ = oracle.lora_f64(x, a, workloads.to_bf16(np.zeros((10, 8), np.float32)))
    assert not u.any() and not s_u.any()
    u0, s0, t0 = oracle.lora_f64(x, a[:0], workloads.to_bf16(np.zeros((10, 0), np.float32)))
    assert u0.shape == (3, 10) and not u0.any() and t0.shape == (3, 0)


def test_merging_a_lora_into_nvfp4_erases_most_of_it():
    """[DF] section 3: in a block whose scale is 0.01 the weights can only be 0, +-0.005,
    +-0.01, +-0.015, +-0.02, +-0.03, +-0.04, +-0.06; a LoRA correction of about 0.001 is a
    tenth of a step, so merging it and quantizing again rounds the correction away.  With
    the block scale exactly 0.01, weights on those levels plus +-0.001 re-quantize to the
    same values everywhere (only the sign of some zeros changes), while the fused low-rank
    branch keeps the term."""
    levels = np.array([0, 0.005, 0.01, 0.015, 0.02, 0.03, 0.04, 0.06], np.float32)
    r = np.random.default_rng(12)
    w = (r.choice(levels, size=(64, 64)) * r.choice([-1, 1], size=(64, 64))).astype(np.float32)
    w[:, ::16] = 0.06                                  # every block's maximum maps to 6: s_b s_g = 0.01
    sg = np.float32(0.01) / np.float32(1.0)            # block scale 1.0 (E4M3 exact), eff = RN32(0.01)
    delta = (r.choice([-1, 1], size=w.shape) * 0.001).astype(np.float32)
    c0, s0, _, _ = oracle.quantize(workloads.to_bf16(w), oracle.SCALE_ABSMAX, sg=sg)
    c1, s1, _, _ = oracle.quantize(workloads.to_bf16(w + delta), oracle.SCALE_ABSMAX, sg=sg)
    assert np.all(s0 == 0x38) and np.array_equal(s0, s1)
    grid = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    q0, q1 = grid[oracle.unpack_codes(c0)], grid[oracle.unpack_codes(c1)]
    assert np.array_equal(q0, q1)                      # every correction rounded away
    # the fused low-rank branch keeps it: a rank-1 branch (A = one row of the correction,
    # B = ones) gives a non-zero B (A x)
    x = workloads.to_bf16(np.ones((1, 64), np.float32))
    a = workloads.to_bf16(delta[:1])                   # r = 1, K = 64
    b = workloads.to_bf16(np.ones((64, 1), np.float32))
    u, _, _ = oracle.lora_f64(x, a, b)
    assert np.all(u != 0)


def test_toy_outlier_experiment_structure():
    """[DF] section 8: 4096 blocks of 16 from N(0, 0.02), one outlier per block scaled
    by 1, 3, 6, 12, 30.  The page prints no numbers; the search never loses to absmax
    and gains most when the block has no dominant outlier."""
    ratios = []
    for i, factor in enumerate((1, 3, 6, 12, 30)):
        a = np.random.default_rng(100 + i).standard_normal((256, 256)).astype(np.float32) * 0.02
        a.reshape(-1, 16)[:, 0] *= factor
        x = workloads.to_bf16(a)
        _, _, _, ea = oracle.quantize(x, oracle.SCALE_ABSMAX)
        _, _, _, em = oracle.quantize(x, oracle.SCALE_MSE)
        ratios.append(ea.astype(np.float64).sum() / em.astype(np.float64).sum())
    assert all(r >= 1.0 for r in ratios)
    assert ratios[0] > 1.05 and ratios[0] > ratios[-1]


# --- scale layouts -----------------------------------------------------------------------------

def test_swizzle_roundtrip_and_padding():
    r = np.random.default_rng(2)
    for rows, nblk in [(1, 1), (16, 16), (130, 5), (256, 8), (300, 33)]:
        lin = r.integers(1, 256, size=(rows, nblk), dtype=np.uint8)
        swz = oracle.swizzle_scales(lin)
        assert swz.size == ((rows + 127) // 128 * 128) * ((nblk + 3) // 4 * 4)
        assert np.array_equal(oracle.unswizzle_scales(swz, rows, nblk), lin)
        assert (swz != 0).sum() == rows * nblk  # every pad byte is zero
        offs = {oracle._load().ora_swizzled_offset(i, j, nblk) for i in range(rows) for j in range(nblk)}
        assert len(offs) == rows * nblk         # a bijection onto the non-pad bytes


def test_swizzle_tile_structure():
    """Within one 512-byte tile, 4 consecutive K-blocks of a row are 4 consecutive
    bytes, and rows 32 apart share a 16-byte line (the layout the tensor-core
    scale-factor copy reads as 32 lines of 16 bytes)."""
    off = oracle._load().ora_swizzled_offset
    nblk = 8
    for rr in range(128):
        base = off(rr, 0, nblk)
        assert [off(rr, c, nblk) - base for c in range(4)] == [0, 1, 2, 3]
        assert off(rr, 4, nblk) == base + 512
        assert off(rr, 0, nblk) // 16 == off(rr % 32, 0, nblk) // 16
    assert off(128, 0, nblk) == 2 * 512


# --- dequantize and GEMM -----------------------------------------------------------------------

def test_dequantize_matches_library_reconstruction():
    """W^ = q * s_b * s_g, rebuilt with ml_dtypes/torch decoders and torch's BF16 cast."""
    x = _tiny_tensor()
    codes, scales, sg, _ = oracle.quantize(x, oracle.SCALE_MSE)
    grid = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    q = grid[oracle.unpack_codes(codes)]
    eff = np.repeat(_eff(scales, sg), 16, axis=1)
    want = torch.from_numpy((q * eff).astype(np.float32)).to(torch.bfloat16)
    got = workloads.from_bits(oracle.dequantize(codes, scales, sg))
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def _operand_values(codes, scales, sg):
    grid = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    dec = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    return grid[oracle.unpack_codes(codes)] * np.repeat(dec[scales], 16, axis=1) * float(sg)


def test_gemm_reference_exact_on_tiny_k():
    """[DF] section 2, out = (A s_a)(B s_b)^T: compare with exact rational sums."""
    xa = _tiny_tensor(6, 64, seed=4)
    xb = _tiny_tensor(5, 64, seed=5)
    ca, sa, ga, _ = oracle.quantize(xa)
    cb, sb, gb, _ = oracle.quantize(xb, oracle.SCALE_MSE)
    ref, absum = oracle.gemm_f64(ca, sa, ga, cb, sb, gb)
    A, B = _operand_values(ca, sa, ga), _operand_values(cb, sb, gb)
    for m in range(A.shape[0]):
        for n in range(B.shape[0]):
            exact = sum(Fraction(a) * Fraction(b) for a, b in zip(A[m], B[n]))
            mag = sum(abs(Fraction(a) * Fraction(b)) for a, b in zip(A[m], B[n]))
            # recursive float64 summation of K terms: |err| <= K * 2^-53 * sum|p|
            bound = Fraction(A.shape[1], 2**53) * mag
            assert abs(Fraction(ref[m, n]) - exact) <= bound
            assert abs(Fraction(absum[m, n]) - mag) <= bound
    # the operand order matters: C is A times B transposed, not B times A
    assert ref.shape == (6, 5)


def test_gemm_reference_integer_special_case():
    """All block scales 1.0 and s_g = 1: 2 * grid values are integers, so C equals an
    exact integer matmul / 4 (a textbook routine)."""
    r = np.random.default_rng(9)
    M, N, K = 9, 7, 96
    ca = r.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    cb = r.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = np.full((M, K // 16), 0x38, np.uint8)
    sb = np.full((N, K // 16), 0x38, np.uint8)
    ref, _ = oracle.gemm_f64(ca, sa, 1.0, cb, sb, 1.0)
    grid2 = (2 * np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)).astype(np.int64)
    ia, ib = grid2[oracle.unpack_codes(ca)], grid2[oracle.unpack_codes(cb)]
    assert np.array_equal(ref * 4, (ia @ ib.T).astype(np.float64))
    # and the sampled form agrees with the full one
    mi, ni = np.array([0, 8, 3]), np.array([6, 0, 2])
    at, _ = oracle.gemm_f64_at(ca, sa, 1.0, cb, sb, 1.0, mi, ni)
    assert np.array_equal(at, ref[mi, ni])
