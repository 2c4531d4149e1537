"""Pins of the oracle's comparison formats: 4/6 and NVINT4.

"Adaptive Block-Scaled Data Types" (gist.science explainer) contrasts IF4
with two alternatives.
- Four over six maps each block maximum to 4 instead of 6 and loses the codes
  +-6 (section 1).
- NVINT4 is INT4 with NVFP4's block scaling (section 4).
The oracle reads NVINT4 as IF4's INT4 candidate in every block.  The pins
below are worked by hand: exact codes and scales of grid-representable
blocks, the tensor-scale constant, the missing codes, and lossless round
trips.
"""
import numpy as np

E2M1_CODE = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}


def code_of(v):
    c = E2M1_CODE[abs(v)]
    return c | (8 if v < 0 else 0)


def test_four_over_six_tensor_scale_uses_4_times_448(orc):
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 1792.0
    assert orc.quantize_four_over_six(x)["s_dec"][0] == np.float32(1.0)
    x[0, 0] = 3584.0
    assert orc.quantize_four_over_six(x)["s_dec"][0] == np.float32(2.0)
    # NVFP4 keeps 2688 = 6 * 448
    assert orc.quantize_nvfp4(x)["s_dec"][0] == np.float32(3584.0 / 2688.0)


def test_four_over_six_worked_blocks(orc):
    """amax = 1792 gives s_enc = 1.  Block 0 has maximum 4, so S = E4M3(4 / 4)
    = 1 (byte 0x38) and the values keep their own codes.  Block 1 holds the
    tensor maximum 1792: S = E4M3(1792 / 4) = 448 (0x7E), r = 1 / 448, and
    1792 -> 4, 896 -> 2, -448 -> -1."""
    b0 = [4.0, -3.0, 2.0, 1.5, 1.0, -0.5, 0.0, 0.5, -4.0, 3.0, -2.0, 1.0, 0.0, -1.5, 2.0, 0.5]
    b1 = [1792.0, 896.0, -448.0] + [0.0] * 13
    x = np.array([b0 + b1], np.float32)
    out = orc.quantize_four_over_six(x)
    assert out["sf_row"].tolist() == [0x38, 0x7E]
    want0 = [code_of(v) for v in b0]
    want1 = [code_of(v / 448.0) for v in b1]
    codes = [int(out["q_row"][0, j // 2] >> (4 * (j % 2))) & 0xF for j in range(32)]
    assert codes == want0 + want1
    # with the NVFP4 divisor 6 (and the same s_enc = 1) block 0's scale is
    # E4M3(4 / 6) instead
    assert orc.quantize_nvfp4(x, amax=2688.0)["sf_row"][0] == orc.e4m3_rne_sat(4.0 / 6.0) != 0x38


def test_four_over_six_never_uses_6(orc):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    x[:, ::37] *= 30.0
    for layouts in (orc.ROWWISE, orc.COLWISE):
        out = orc.quantize_four_over_six(x, layouts=layouts)
        q = out["q_row" if layouts == orc.ROWWISE else "q_col"]
        nib = np.concatenate([q & 0xF, q >> 4]).ravel()
        assert not np.any((nib & 7) == 7)
        assert np.any((nib & 7) == 6)            # the block maxima land on 4


def test_four_over_six_round_trip_and_transpose(orc):
    """Grid values times power-of-two block scales come back exactly, and the
    column-wise output is the row-wise output of the transpose."""
    rng = np.random.default_rng(2)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4], np.float32)
    x = rng.choice(grid, size=(32, 64)) * rng.choice([-1, 1], size=(32, 64))
    x = x.astype(np.float32)
    x[:, ::16] = 4.0                              # every row block has maximum 4
    x[::16, :] = 4.0                              # every column block too
    scale = np.float32(2.0) ** rng.integers(-3, 4, size=(32, 4)).astype(np.float32)
    x = x * np.repeat(scale, 16, axis=1)
    # a tensor amax of 1792 gives s_enc = s_dec = 1, so every step is exact
    out = orc.quantize_four_over_six(x, layouts=orc.ROWWISE | orc.COLWISE, amax=1792.0)
    y = orc.dequantize(orc.FMT_NVFP4, out["q_row"], out["sf_row"], 32, 64, 1, 16,
                       s_dec=out["s_dec"][0])
    np.testing.assert_array_equal(y, x)
    t = orc.quantize_four_over_six(np.ascontiguousarray(x.T), layouts=orc.ROWWISE, amax=1792.0)
    np.testing.assert_array_equal(out["q_col"], t["q_row"])
    np.testing.assert_array_equal(out["sf_col"], t["sf_row"])


def test_nvint4_worked_block(orc):
    """amax = 2688 gives s_enc = 1; a block with maximum 6 has S = 1 and
    r = 1, so v = x.  Values RN(k * RN(6/7)) come back as k, every block is
    flagged INT4, and the IF4 dequantization returns them exactly."""
    c67 = np.float32(6.0) / np.float32(7.0)
    ks = np.array([7, -7, 3, 0, -1, 5, 2, -4, 6, 1, -2, -6, 4, -3, 0, -5], np.int32)
    b = (ks.astype(np.float32) * c67).astype(np.float32)
    x = np.zeros((1, 32), np.float32)
    x[0, :16] = b
    x[0, 16] = 2688.0
    out = orc.quantize_if4(x, int4_only=True)
    assert np.all(out["sf"] & 0x80)
    assert out["sf"][0] & 0x7F == 0x38            # S = 1
    codes = [int(out["q"][0, j // 2] >> (4 * (j % 2))) & 0xF for j in range(16)]
    assert codes == [int(k) & 0xF for k in ks]
    y = orc.dequantize(orc.FMT_IF4, out["q"], out["sf"], 1, 32, 1, 16, s_dec=out["s_dec"][0])
    np.testing.assert_array_equal(y[0, :16], b)


def test_if4_is_the_better_of_nvfp4_and_nvint4_per_block(orc):
    """IF4 keeps, per block, whichever candidate has the smaller squared
    error: its codes agree with NVFP4's where the flag is clear and with
    NVINT4's where it is set, and both kinds occur on mixed data."""
    rng = np.random.default_rng(3)
    x = np.where(rng.random((128, 256)) < 0.5, rng.standard_normal((128, 256)),
                 rng.uniform(-1, 1, (128, 256))).astype(np.float32)
    a = float(np.abs(x).max())
    if4 = orc.quantize_if4(x, amax=a)
    fp = orc.quantize_if4(x, amax=a, allow_int4=False)
    it = orc.quantize_if4(x, amax=a, int4_only=True)
    flag = (if4["sf"] & 0x80) != 0
    assert 0 < flag.mean() < 1
    q_blocks = if4["q"].reshape(128, 16, 8)
    want = np.where(flag.reshape(128, 16, 1), it["q"].reshape(128, 16, 8),
                    fp["q"].reshape(128, 16, 8))
    np.testing.assert_array_equal(q_blocks, want)
    np.testing.assert_array_equal(if4["sf"] & 0x7F, fp["sf"])
    np.testing.assert_array_equal(it["sf"], fp["sf"] | 0x80)


def test_mse_order_on_gaussian_blocks(orc):
    """Table 1 of the explainer reports IF4 below NVFP4 on N(0, 1) blocks.
    Dequantized MSE on 2^16 Gaussian blocks: IF4 < NVFP4 and IF4 < NVINT4."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((1024, 1024)).astype(np.float32)
    a = float(np.abs(x).max())

    def mse(out, fmt):
        y = orc.dequantize(fmt, out["q"], out["sf"], 1024, 1024, 1, 16, s_dec=out["s_dec"][0])
        return float(np.mean((y.astype(np.float64) - x) ** 2))

    m_if4 = mse(orc.quantize_if4(x, amax=a), orc.FMT_IF4)
    m_fp = mse(orc.quantize_if4(x, amax=a, allow_int4=False), orc.FMT_IF4)
    m_int = mse(orc.quantize_if4(x, amax=a, int4_only=True), orc.FMT_IF4)
    assert m_if4 < m_fp and m_if4 < m_int
    out46 = orc.quantize_four_over_six(x, amax=a)
    y46 = orc.dequantize(orc.FMT_NVFP4, out46["q_row"], out46["sf_row"], 1024, 1024, 1, 16,
                         s_dec=out46["s_dec"][0])
    m46 = float(np.mean((y46.astype(np.float64) - x) ** 2))
    assert np.isfinite(m46) and m46 > 0
