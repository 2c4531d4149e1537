"""Pins of the oracle's IF6 (the IF idea at 6 bits).

"Adaptive Block-Scaled Data Types" explainer, section 2: per 16-value block the
format is chosen between a float and a scaled integer grid by the smaller
squared error, the choice is flagged in the scale's sign bit, and the idea
extends to 6 bits (IF6).  The reading pinned here: FP6 E2M3 (largest 7.5)
against INT6 (-31..31) scaled by 7.5/31, codes packed four per three bytes.
"""
import numpy as np
import pytest


def pack6(codes):
    out = []
    for g in range(0, len(codes), 4):
        w = codes[g] | codes[g + 1] << 6 | codes[g + 2] << 12 | codes[g + 3] << 18
        out += [w & 0xFF, (w >> 8) & 0xFF, w >> 16]
    return out


def unit_scale_tensor(block):
    """Row 0: the test block (maximum 7.5 or just under, so S = 1); row 1 holds
    3360 so that s_enc = RN(3360 / amax) = 1 and r = 1: v equals x."""
    x = np.zeros((2, 16), np.float32)
    x[0] = block
    x[1, 0] = 3360.0
    return x


def test_constants(orc):
    cu, cd = orc.if6_constants()
    assert cu == np.float32(31 / 7.5) and cd == np.float32(7.5 / 31)


def test_block_on_the_fp6_grid_keeps_fp6(orc):
    block = np.array([7.5, -0.125, 1.0, -3.0, 0.875, 5.5, -6.5, 0.0,
                      2.25, -1.125, 4.0, 0.5, -0.375, 3.75, -7.0, 1.875], np.float32)
    out = orc.quantize_if6(unit_scale_tensor(block))
    assert out["s_dec"][0] == 1.0
    assert out["sf"][0] == 0x38                         # E4M3 1.0, flag clear
    codes = [orc.fp6_rne(v, orc.FP6_E2M3) for v in block]
    assert codes[:4] == [0x1F, 0x21, 0x08, 0x34]
    assert out["q"][0].tolist() == pack6(codes)


def test_block_on_the_int6_grid_takes_int6(orc):
    _, cd = orc.if6_constants()
    k = np.array([31, -30, 17, -1, 0, 5, -13, 22, 29, -31, 2, -7, 11, 25, -19, 3])
    block = (k.astype(np.float32) * np.float32(cd)).astype(np.float32)
    assert float(np.abs(block).max()) == 7.5              # 31 * RN(7.5/31) rounds to 7.5
    out = orc.quantize_if6(unit_scale_tensor(block))
    assert out["sf"][0] == 0x80 | 0x38                  # flag set, S = 1.0
    assert out["q"][0].tolist() == pack6([int(v) & 0x3F for v in k])
    y = orc.dequantize(orc.FMT_IF6, out["q"], out["sf"], 2, 16, 1, 16, s_dec=1.0)
    np.testing.assert_array_equal(y[0], block)          # exact round trip


@pytest.mark.parametrize("layout", [0, 1])
def test_each_block_is_the_better_of_fp6_and_int6(orc, layout):
    """Mode 1 (IF6) equals, block by block, mode 0 (FP6 everywhere) or mode 2
    (INT6 everywhere), and the one it keeps has the smaller squared error."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal((128, 256)).astype(np.float32)
    x[::3] = rng.uniform(-1, 1, (43, 256)).astype(np.float32)      # flat rows favour INT6
    x[5, 7] = 40.0
    runs = [orc.quantize_if6(x, scale_layout=layout, mode=m) for m in (0, 1, 2)]
    deq = [orc.dequantize(orc.FMT_IF6, r["q"], r["sf"], 128, 256, 1, 16,
                          s_dec=float(r["s_dec"][0]), scale_layout=layout).astype(np.float64)
           for r in runs]
    err = [((d - x) ** 2).reshape(128, 16, 16).sum(axis=2) for d in deq]
    same_fp = (deq[1] == deq[0]).reshape(128, 16, 16).all(axis=2)
    same_int = (deq[1] == deq[2]).reshape(128, 16, 16).all(axis=2)
    assert np.all(same_fp | same_int)
    took_int = same_int & ~same_fp
    # the kept candidate is never worse than the other beyond rounding noise
    assert np.all(err[1] <= np.minimum(err[0], err[2]) * (1 + 1e-6) + 1e-30)
    assert 0 < took_int.mean() < 1


def test_if6_beats_both_fixed_formats(orc):
    rng = np.random.default_rng(10)
    x = rng.standard_normal((256, 512)).astype(np.float32)
    mse = []
    for m in (0, 1, 2):
        r = orc.quantize_if6(x, mode=m)
        y = orc.dequantize(orc.FMT_IF6, r["q"], r["sf"], 256, 512, 1, 16, s_dec=float(r["s_dec"][0]))
        mse.append(float(np.mean((y.astype(np.float64) - x) ** 2)))
    assert mse[1] < mse[0] and mse[1] < mse[2]
