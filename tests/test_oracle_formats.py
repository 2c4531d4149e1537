"""Pins for the oracle's number formats, random bits and layouts (CPU only).

Each check compares the oracle with something other than itself: values the
pages print, an independent library (ml_dtypes, torch's float8 cast, scipy),
published test vectors, or exact rational arithmetic.
"""
import decimal
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# the E2M1 magnitudes as the Qiita note ("NVFP4データの変換") and the glossary
# ("FP4の仕組み") list them
PAGE_E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _f32_neighbours(points, k=40):
    """points and the k float32 neighbours on each side of each point."""
    out = []
    for p in points:
        b = np.array([p], np.float32).view(np.int32)[0]
        for d in range(-k, k + 1):
            if b + d >= 0:
                out.append(np.array([b + d], np.int32).view(np.float32)[0])
    return np.array(out, np.float32)


def test_e2m1_value_set_matches_pages(orc):
    vals = {orc.e2m1_value(c) for c in range(16)}
    page = set(PAGE_E2M1_VALUES) | {-v for v in PAGE_E2M1_VALUES}
    assert vals == page
    assert len(page) == 15          # 15 distinct values (+0 == -0)
    # codes 0..7 are the magnitudes in increasing order, bit 3 is the sign
    assert [orc.e2m1_value(c) for c in range(8)] == PAGE_E2M1_VALUES
    assert [orc.e2m1_value(c | 8) for c in range(8)] == [-v for v in PAGE_E2M1_VALUES]


def test_e2m1_rne_matches_ml_dtypes(orc):
    rng = np.random.default_rng(1)
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0]
    vals = np.concatenate([
        _f32_neighbours(ties, 64),
        _f32_neighbours([0.0], 64),                      # +0 and subnormals
        (rng.standard_normal(400_000) * 10.0 ** rng.uniform(-4, 3, 400_000)).astype(np.float32),
        np.array([7.0, 100.0, 1e30, np.finfo(np.float32).max], np.float32),
    ])
    vals = np.concatenate([vals, -vals, np.array([-0.0], np.float32)])
    got = orc.e2m1_rne_array(vals)
    want = vals.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"mismatch at {vals[bad[:5]]}: {got[bad[:5]]} vs {want[bad[:5]]}"


def test_e2m1_sign_of_zero_reading(orc):
    # READING: sign copied, so small negatives give the negative-zero code 0x8
    assert orc.e2m1_rne(-0.1) == 0x8
    assert orc.e2m1_rne(-0.25) == 0x8       # tie goes to even code 0
    assert orc.e2m1_rne(0.1) == 0x0
    assert orc.e2m1_rne(-0.0) == 0x8


def test_e4m3_matches_torch_float8_cast(orc):
    # torch rounds to nearest even but gives NaN above 464, so it pins [0, 464]
    grid = [orc.e4m3_value(c) for c in range(0x7F)]
    mids = [(a + b) / 2 for a, b in zip(grid[:-1], grid[1:])]
    rng = np.random.default_rng(2)
    vals = np.concatenate([
        _f32_neighbours(mids + grid, 8),
        np.exp2(rng.uniform(-14, 8.85, 300_000)).astype(np.float32),
        np.array([0.0, 464.0, 2.0 ** -10, 2.0 ** -9, 2.0 ** -6], np.float32),
    ])
    vals = vals[(vals >= 0) & (vals <= 464.0)]
    got = orc.e4m3_rne_sat_array(vals)
    want = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"mismatch at {vals[bad[:5]]}: {got[bad[:5]]} vs {want[bad[:5]]}"
    # ml_dtypes agrees on the same range
    want2 = vals.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(got, want2)


def test_e4m3_saturates_at_448(orc):
    # Qiita note "NVFP4の表現できる最大値": the E4M3 maximum is 448
    assert orc.e4m3_value(0x7E) == 448.0
    for s in [448.0, 460.0, 464.0, 464.1, 480.0, 1e6, 3e38]:
        assert orc.e4m3_rne_sat(s) == 0x7E
    assert 6.0 * orc.e4m3_value(0x7E) == 2688.0


def test_e8m0_rne_against_ml_dtypes_and_ties(orc):
    rng = np.random.default_rng(3)
    m = np.exp2(rng.uniform(-120, 120, 200_000)).astype(np.float32)
    # exact midpoints 1.5 * 2^E of the scale target amax/6 (ties)
    E = rng.integers(-100, 100, 2000)
    tie_targets = (1.5 * np.exp2(E.astype(np.float64))).astype(np.float32)
    m = np.concatenate([m, tie_targets * np.float32(6.0)])
    e = orc.e8m0_exponent_array(m, orc.E8M0_RNE)
    target = m / np.float32(6.0)                      # RN(amax / 6) in float32
    mant = target.view(np.uint32) & 0x7FFFFF
    is_tie = mant == 0x400000
    # non-ties: ml_dtypes rounds to the nearest power of two
    ml = np.log2(target[~is_tie].astype(ml_dtypes.float8_e8m0fnu).astype(np.float64))
    assert np.array_equal(e[~is_tie], ml.astype(np.int32))
    # ties: the even biased exponent
    Et = np.frexp(target[is_tie].astype(np.float64))[1] - 1
    want = np.where((Et + 127) % 2 == 0, Et, Et + 1)
    assert is_tie.sum() > 100
    assert np.array_equal(e[is_tie], want)


def test_e8m0_ceil_and_ocp_floor(orc):
    rng = np.random.default_rng(4)
    m = np.exp2(rng.uniform(-100, 100, 100_000)).astype(np.float32)
    m = np.concatenate([m, (6.0 * np.exp2(np.arange(-20, 20))).astype(np.float32)])
    target = (m / np.float32(6.0)).astype(np.float64)
    e = orc.e8m0_exponent_array(m, orc.E8M0_CEIL).astype(np.float64)
    assert np.all(np.exp2(e) >= target) and np.all(np.exp2(e - 1) < target)
    f = orc.e8m0_exponent_array(m, orc.E8M0_OCP_FLOOR)
    assert np.array_equal(f, np.frexp(m.astype(np.float64))[1] - 1 - 2)
    assert orc.e8m0_exponent(0.0, orc.E8M0_RNE) == -127


def test_philox_known_answers(orc):
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(t, 16) for t in r]
        got = orc.philox4x32_10(v[0:4], v[4:6])
        assert [int(t) for t in got] == v[6:10]


def test_sr_bit_mapping_reading(orc):
    # READING: element i takes half (i mod 2) of word (i mod 8) div 2 of the
    # Philox call with counter (i div 8, 0, 0, 0) and key (seed lo, seed hi)
    seed = 0x0123456789ABCDEF
    for g in [0, 1, 12345, 2 ** 33 + 7]:
        w = orc.philox4x32_10([g & 0xFFFFFFFF, g >> 32, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])
        halves = [(int(w[j // 2]) >> (16 * (j % 2))) & 0xFFFF for j in range(8)]
        assert [orc.sr_bits16(seed, 8 * g + j) for j in range(8)] == halves


def test_sr_bits_are_uniform(orc):
    u = orc.sr_bits16_array(7, 0, 1 << 20)
    counts = np.bincount(u >> 8, minlength=256)
    chi2 = ((counts - counts.mean()) ** 2 / counts.mean()).sum()
    assert chi2 < 400          # 255 dof: mean 255, sd ~22.6


def test_sr_exact_probability(orc):
    """Over all 2^16 values of u the round-up count is ceil(t * 2^16), t the
    exact (rational) fraction of the way from the lower to the upper grid
    value; for t on the 2^-16 lattice this makes the rounding unbiased."""
    grid = [Fraction(v) for v in PAGE_E2M1_VALUES]
    u = np.arange(1 << 16, dtype=np.uint32)
    rng = np.random.default_rng(5)
    vals = list(rng.uniform(0, 6, 60).astype(np.float32)) + [0.0, 0.5, 0.75, 5.9999, 1.0 + 2 ** -16]
    for v in vals:
        a = Fraction(float(np.float32(v)))
        lo = max(i for i, g in enumerate(grid) if g <= a)
        t = (a - grid[lo]) / (grid[lo + 1] - grid[lo])
        codes = orc.e2m1_sr_array(np.full(u.shape, v, np.float32), u)
        assert set(np.unique(codes)) <= {lo, lo + 1}
        ups = int((codes == lo + 1).sum())
        want = -((-t * 65536) // 1)            # ceil
        assert ups == want, (v, ups, want)
        if (t * 65536).denominator == 1:       # on the lattice: exactly unbiased
            mean = (Fraction(ups) * grid[lo + 1] + Fraction(65536 - ups) * grid[lo]) / 65536
            assert mean == a
    # saturation and sign
    assert orc.e2m1_sr(7.5, 0) == 7 and orc.e2m1_sr(-6.0, 65535) == 15
    assert orc.e2m1_sr(-0.3, 0) == 0x9 and orc.e2m1_sr(-0.3, 65535) == 0x8


def test_rht_normalisation_constant(orc):
    decimal.getcontext().prec = 60
    exact = decimal.Decimal(1) / decimal.Decimal(128).sqrt()
    cands = [np.float32(float(exact)), np.nextafter(np.float32(float(exact)), np.float32(0)),
             np.nextafter(np.float32(float(exact)), np.float32(1))]
    nearest = min(cands, key=lambda c: abs(decimal.Decimal(float(c)) - exact))
    assert np.float32(orc.rht_norm(128)) == nearest
    assert orc.rht_norm(16) == 0.25


def test_rht_signs_are_philox_bits(orc):
    seed = 99
    w = orc.philox4x32_10([0, 0, 1, 0], [seed, 0])
    s = orc.rht_signs(seed, 128)
    for k in range(128):
        assert s[k] == (-1.0 if (int(w[k // 32]) >> (k % 32)) & 1 else 1.0)
    assert not np.array_equal(s, orc.rht_signs(seed + 1, 128))


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(6)
    v = np.concatenate([(rng.standard_normal(200_000) * 10.0 ** rng.uniform(-30, 30, 200_000)),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8)])]).astype(np.float32)
    got = orc.f32_to_bf16_array(v)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_swizzled_scale_layout(orc):
    """The 128x4 tile layout: offset (r%32)*16 + ((r/32)%4)*4 + c%4 inside a
    512-byte tile, tiles in row-tile-major order; a bijection on the padded size."""
    rows, cols = 256, 8
    n = orc.scale_bytes(rows, cols, orc.SCALE_SWIZZLED)
    assert n == rows * cols
    offs = {orc.scale_offset(r, c, rows, cols, orc.SCALE_SWIZZLED)
            for r in range(rows) for c in range(cols)}
    assert offs == set(range(n))
    S = orc.SCALE_SWIZZLED
    assert orc.scale_offset(0, 0, rows, cols, S) == 0
    assert orc.scale_offset(0, 1, rows, cols, S) == 1
    assert orc.scale_offset(1, 0, rows, cols, S) == 16
    assert orc.scale_offset(32, 0, rows, cols, S) == 4
    assert orc.scale_offset(127, 3, rows, cols, S) == 511
    assert orc.scale_offset(0, 4, rows, cols, S) == 512
    assert orc.scale_offset(128, 0, rows, cols, S) == 1024
    # padding: 130 rows x 5 scale columns pad to 256 x 8
    assert orc.scale_bytes(130, 5, S) == 256 * 8
    assert orc.scale_bytes(130, 5, orc.SCALE_LINEAR) == 650
