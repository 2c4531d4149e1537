"""Pins of the oracle's FP6 formats and MXFP6 quantizer.

"FP6から考えるLLM量子化" (blog.ast.moe), "FP6で隣り合う値の間隔を見てみる":
the OCP FP6 formats E3M2 and E2M3 (no Inf/NaN, subnormals).  The page prints
E3M2's 8, 10, 12, 14 then 16, 20, 24, 28, the spacing 0.0625 near zero, the
64-fold spread of spacings, E2M3's maximum 7.5, 11 landing on 10 or 12, and
0.1 on 0.125; it also reports that E2M3 tends to be more accurate than E3M2
under MX scaling.  ml_dtypes' float6 types decode and round independently.
"""
import numpy as np
import ml_dtypes
import pytest

FMTS = {0: ml_dtypes.float6_e2m3fn, 1: ml_dtypes.float6_e3m2fn}


def values(orc, fmt):
    return np.array([orc.fp6_value(c, fmt) for c in range(64)], np.float32)


def test_values_printed_on_the_page(orc):
    e3m2 = values(orc, orc.FP6_E3M2)
    pos = sorted(set(e3m2[e3m2 > 0].tolist()))
    assert pos[-8:] == [8, 10, 12, 14, 16, 20, 24, 28]
    assert pos[0] == 0.0625 and pos[1] - pos[0] == 0.0625
    spacings = np.diff(np.array([0.0] + pos))
    assert spacings.max() / spacings.min() == 64
    e2m3 = values(orc, orc.FP6_E2M3)
    assert e2m3.max() == 7.5 and e2m3.min() == -7.5


def test_rounding_examples_from_the_page(orc):
    assert orc.fp6_value(orc.fp6_rne(11.0, orc.FP6_E3M2), orc.FP6_E3M2) in (10.0, 12.0)
    assert orc.fp6_value(orc.fp6_rne(11.0, orc.FP6_E3M2), orc.FP6_E3M2) == 12.0   # tie, even code
    assert orc.fp6_value(orc.fp6_rne(0.1, orc.FP6_E3M2), orc.FP6_E3M2) == 0.125


@pytest.mark.parametrize("fmt", [0, 1])
def test_codes_and_rounding_match_ml_dtypes(orc, fmt):
    ref = np.arange(64, dtype=np.uint8).view(FMTS[fmt]).astype(np.float32)
    np.testing.assert_array_equal(values(orc, fmt), ref)
    rng = np.random.default_rng(fmt)
    top = float(ref.max())
    x = np.concatenate([
        rng.uniform(-1.2 * top, 1.2 * top, 20000),
        (ref[:32, None] + np.array([-1e-7, 0, 1e-7])).ravel(),      # grid points
        ((ref[:31] + ref[1:32]) / 2)[:, None].ravel() * np.array([1]),   # midpoints
        [0.0, -0.0, 1e-30, -1e-30, top * 4, -top * 4]]).astype(np.float32)
    got = np.array([orc.fp6_rne(v, fmt) for v in x], np.uint8)
    want = x.astype(FMTS[fmt]).view(np.uint8)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("fmt,emax,qmax", [(0, 2, 7.5), (1, 4, 28.0)])
def test_mx_exponents(orc, fmt, emax, qmax):
    """OCP floor: floor(log2 m) - emax; RNE: RN(m / qmax) to the nearest power
    of two (checked against ml_dtypes' E8M0 rounding away from ties)."""
    rng = np.random.default_rng(5)
    for m in np.float32(2.0) ** rng.uniform(-30, 30, 200).astype(np.float32):
        x = np.zeros((1, 32), np.float32)
        x[0, 3] = m
        e_floor = int(orc.quantize_mxfp6(x, fmt, orc.E8M0_OCP_FLOOR)["sf"][0]) - 127
        assert e_floor == int(np.floor(np.log2(np.float64(m)))) - emax
        t = np.float32(m) / np.float32(qmax)
        f = float(t) / 2.0 ** np.floor(np.log2(float(t)))
        if abs(f - 1.5) < 1e-6:
            continue
        e_rne = int(orc.quantize_mxfp6(x, fmt, orc.E8M0_RNE)["sf"][0]) - 127
        assert 2.0 ** e_rne == float(np.array([t]).astype(ml_dtypes.float8_e8m0fnu)[0])


def test_packing_worked_group(orc):
    """Four E2M3 codes c0..c3 go to bits 0-5, 6-11, 12-17, 18-23 of three
    little-endian bytes.  With a block maximum of 7.5 the scale is 2^0."""
    x = np.zeros((1, 32), np.float32)
    x[0, :4] = [7.5, -0.125, 1.0, -3.0]
    out = orc.quantize_mxfp6(x, orc.FP6_E2M3)
    assert out["sf"][0] == 127
    codes = [orc.fp6_rne(v, orc.FP6_E2M3) for v in x[0, :4]]
    assert codes == [0x1F, 0x21, 0x08, 0x34]
    w = codes[0] | codes[1] << 6 | codes[2] << 12 | codes[3] << 18
    assert out["q"][0, :3].tolist() == [w & 0xFF, (w >> 8) & 0xFF, w >> 16]


@pytest.mark.parametrize("fmt", [0, 1])
def test_round_trip_on_the_grid(orc, fmt):
    """Grid values times power-of-two block scales come back exactly."""
    rng = np.random.default_rng(6 + fmt)
    grid = values(orc, fmt)
    x = rng.choice(grid, size=(8, 128)).astype(np.float32)
    x[:, ::32] = grid.max()                              # each block reaches the maximum
    scale = np.float32(2.0) ** rng.integers(-10, 10, size=(8, 4)).astype(np.float32)
    x = x * np.repeat(scale, 32, axis=1)
    out = orc.quantize_mxfp6(x, fmt, orc.E8M0_OCP_FLOOR)
    fmt_code = orc.FMT_MXFP6_E2M3 if fmt == 0 else orc.FMT_MXFP6_E3M2
    y = orc.dequantize(fmt_code, out["q"], out["sf"], 8, 128, 1, 32)
    np.testing.assert_array_equal(y, x)


def test_e2m3_beats_e3m2_on_gaussian_blocks(orc):
    rng = np.random.default_rng(7)
    x = rng.standard_normal((256, 1024)).astype(np.float32)
    mse = {}
    for fmt, code in ((0, orc.FMT_MXFP6_E2M3), (1, orc.FMT_MXFP6_E3M2)):
        out = orc.quantize_mxfp6(x, fmt)
        y = orc.dequantize(code, out["q"], out["sf"], 256, 1024, 1, 32)
        mse[fmt] = float(np.mean((y.astype(np.float64) - x) ** 2))
    assert mse[0] < mse[1]
