"""Pins of the oracle's IF3 (the IF idea at 3 bits).

"Adaptive Block-Scaled Data Types" explainer, section 2: per 16-value block the
format is chosen between a float and a scaled integer grid by the smaller
squared error, the choice is flagged in the scale's sign bit, and the idea
extends to 3 bits (IF3).  The reading pinned here: FP3 E2M0 (magnitudes 0, 1,
2, 4) against INT3 (-3..3) scaled by 4/3, codes packed eight per three bytes.
"""
import numpy as np
import pytest

E2M0 = [0.0, 1.0, 2.0, 4.0]


def pack3(codes):
    out = []
    for g in range(0, len(codes), 8):
        w = 0
        for j in range(8):
            w |= codes[g + j] << (3 * j)
        out += [w & 0xFF, (w >> 8) & 0xFF, w >> 16]
    return out


def brute_fp3(v):
    """Nearest E2M0 magnitude by exhaustive search in float64; a tie goes to
    the even code; |v| above 4 saturates; sign bit copied."""
    a = abs(float(v))
    d = [abs(a - g) for g in E2M0]
    best = min(range(4), key=lambda c: (d[c], c % 2))
    return best | (4 if np.signbit(v) else 0)


def unit_scale_tensor(block):
    """Row 0: the test block (maximum 4, so S = 1); row 1 holds 1792 so that
    s_enc = RN(1792 / amax) = 1 and r = 1: v equals x."""
    x = np.zeros((2, 16), np.float32)
    x[0] = block
    x[1, 0] = 1792.0
    return x


def test_constants(orc):
    cu, cd = orc.if3_constants()
    assert cu == 0.75 and cd == np.float32(4 / 3)


def test_fp3_grid(orc):
    assert [orc.fp3_value(c) for c in range(8)] == [0, 1, 2, 4, 0, -1, -2, -4]
    assert np.signbit(orc.fp3_value(4))


def test_fp3_rounding_against_brute_force(orc):
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.uniform(-6, 6, 4000).astype(np.float32),
                           np.float32([0.5, 1.5, 3.0, -0.5, -1.5, -3.0, 4.0, 5.0, -7.5, 0.0,
                                       -0.0, 1e-30, np.nextafter(np.float32(0.5), 1),
                                       np.nextafter(np.float32(3.0), 0)])])
    for v in vals:
        assert orc.fp3_rne(v) == brute_fp3(v), v
    # the ties: 0.5 -> 0, 1.5 -> 2, 3 -> 2 (even codes 0 and 2)
    assert [orc.fp3_rne(v) for v in (0.5, 1.5, 3.0)] == [0, 2, 2]
    # saturation holds for every magnitude, also where float64 distances tie
    assert [orc.fp3_rne(v) for v in (1e30, -3e38, 4.0)] == [3, 7, 3]


def test_block_on_the_fp3_grid_keeps_fp3(orc):
    block = np.array([4, -1, 2, 0, -4, 1, -2, 4, 0, 2, -1, 1, -4, 2, 0, -2], np.float32)
    out = orc.quantize_if3(unit_scale_tensor(block))
    assert out["s_dec"][0] == 1.0
    assert out["sf"][0] == 0x38                          # E4M3 1.0, flag clear
    codes = [brute_fp3(v) for v in block]
    assert codes[:4] == [3, 5, 2, 0]
    assert out["q"][0].tolist() == pack3(codes)
    y = orc.dequantize(orc.FMT_IF3, out["q"], out["sf"], 2, 16, 1, 16, s_dec=1.0)
    np.testing.assert_array_equal(y[0], block)


def test_block_on_the_int3_grid_takes_int3(orc):
    _, cd = orc.if3_constants()
    k = np.array([3, -3, 1, -1, 0, 2, -2, 3, 1, 0, -3, 2, -1, 1, 3, -2])
    block = (k.astype(np.float32) * np.float32(cd)).astype(np.float32)
    assert float(np.abs(block).max()) == 4.0              # 3 * RN(4/3) rounds to 4
    out = orc.quantize_if3(unit_scale_tensor(block))
    assert out["sf"][0] == 0x80 | 0x38                  # flag set, S = 1.0
    assert out["q"][0].tolist() == pack3([int(v) & 0x7 for v in k])
    y = orc.dequantize(orc.FMT_IF3, out["q"], out["sf"], 2, 16, 1, 16, s_dec=1.0)
    np.testing.assert_array_equal(y[0], block)           # exact round trip


def test_block_scale_maps_the_maximum_to_four(orc):
    """S = E4M3(RN(m * s_enc) / 4): a block of maximum 8 beside a tensor
    maximum of 1792 gets S = 2 (0x40)."""
    x = np.zeros((2, 16), np.float32)
    x[0, 3] = 8.0
    x[1, 0] = 1792.0
    out = orc.quantize_if3(x)
    assert out["sf"][0] & 0x7F == 0x40
    y = orc.dequantize(orc.FMT_IF3, out["q"], out["sf"], 2, 16, 1, 16,
                       s_dec=float(out["s_dec"][0]))
    assert y[0, 3] == 8.0 and y[1, 0] == 1792.0


@pytest.mark.parametrize("layout", [0, 1])
def test_each_block_is_the_better_of_fp3_and_int3(orc, layout):
    """Mode 1 (IF3) equals, block by block, mode 0 (FP3 everywhere) or mode 2
    (INT3 everywhere), and the one it keeps has the smaller squared error."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((128, 256)).astype(np.float32)
    x[::3] = rng.uniform(-1, 1, (43, 256)).astype(np.float32)      # flat rows favour INT3
    x[5, 7] = 40.0
    runs = [orc.quantize_if3(x, scale_layout=layout, mode=m) for m in (0, 1, 2)]
    deq = [orc.dequantize(orc.FMT_IF3, r["q"], r["sf"], 128, 256, 1, 16,
                          s_dec=float(r["s_dec"][0]), scale_layout=layout).astype(np.float64)
           for r in runs]
    err = [((d - x) ** 2).reshape(128, 16, 16).sum(axis=2) for d in deq]
    same_fp = (deq[1] == deq[0]).reshape(128, 16, 16).all(axis=2)
    same_int = (deq[1] == deq[2]).reshape(128, 16, 16).all(axis=2)
    assert np.all(same_fp | same_int)
    took_int = same_int & ~same_fp
    assert np.all(err[1] <= np.minimum(err[0], err[2]) * (1 + 1e-6) + 1e-30)
    assert 0 < took_int.mean() < 1


def test_if3_beats_both_fixed_formats(orc):
    rng = np.random.default_rng(12)
    x = rng.standard_normal((256, 512)).astype(np.float32)
    mse = []
    for m in (0, 1, 2):
        r = orc.quantize_if3(x, mode=m)
        y = orc.dequantize(orc.FMT_IF3, r["q"], r["sf"], 256, 512, 1, 16,
                           s_dec=float(r["s_dec"][0]))
        mse.append(float(np.mean((y.astype(np.float64) - x) ** 2)))
    assert mse[1] < mse[0] and mse[1] < mse[2]


def test_int3_codes_against_a_float64_restatement(orc):
    """Mode 2 codes on a random tensor equal clamp(rint(v * 0.75), -3, 3) of
    v = x * r computed here from the stored scale, in two's complement."""
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((16, 64)) * 3).astype(np.float32)
    out = orc.quantize_if3(x, mode=2)
    amax = np.float32(np.abs(x).max())
    s_enc = np.float32(np.float32(1792.0) / amax)
    sf = out["sf"].reshape(16, 4)
    q = out["q"].reshape(16, 24)
    for r in range(16):
        for b in range(4):
            S = np.float32(orc.e4m3_value(int(sf[r, b]) & 0x7F))
            rf = np.float32(s_enc / S)
            v = (x[r, 16 * b:16 * b + 16] * rf).astype(np.float32)
            k = np.clip(np.rint((v * np.float32(0.75)).astype(np.float32)), -3, 3).astype(int)
            assert q[r, 6 * b:6 * b + 6].tolist() == pack3([int(c) & 7 for c in k])
