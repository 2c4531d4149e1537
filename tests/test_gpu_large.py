"""GPU parity at a tensor of more than 2^31 elements (the 64-bit index paths).

A 32768 x 65600 BF16 tensor (2.15e9 elements, 4.3 GB) takes the kernels'
64-bit index paths.  The whole tensor is too large for the oracle, so the
checks are the ones that hold at any size: the tensor amax against a planted
maximum at the very last element, and sampled rows (first, second, middle,
last) against the oracle run on those rows alone.  The row-wise formats are
row-independent once the tensor amax is given, so that comparison is exact.
The formats whose blocks span rows (row+col NVFP4 and MXFP4, 2D, the RHT
along tokens) are compared on bands of whole blocks (first, middle, last).
Round to nearest, except in the stochastic-rounding tests: their bits depend
on the global element index, so the oracle runs on the band with the band's
first row (row0 / token0) and draws the same bits.
"""
import pytest
import torch

import fp4_block_scaled_04_b200 as fq

from test_gpu_parity import DEV, assert_same, bits, host

pytestmark = pytest.mark.gpu

R, C = 32768, 65600
PEAK = 768.0                      # exact in BF16
ROWS = [0, 1, R // 2 + 3, R - 1]


@pytest.fixture(scope="module")
def big():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    free, _ = torch.cuda.mem_get_info()
    if free < 24 * 2**30:
        pytest.skip("needs about 24 GB of free device memory")
    fq.lib()
    g = torch.Generator(device=DEV).manual_seed(1234)
    x = torch.randn((R, C), generator=g, dtype=torch.bfloat16, device=DEV)
    x.clamp_(-60.0, 60.0)
    x[R - 1, C - 1] = -PEAK                # the maximum |x| sits in the last element
    x[R // 2, 7] = 512.0
    amax = torch.tensor([PEAK], dtype=torch.float32, device=DEV)
    yield x, amax
    del x
    torch.cuda.empty_cache()


def sample(t):
    return host(t[ROWS])


def test_large_amax(big):
    x, _ = big
    assert R * C > 2**31
    assert float(fq.fp4q_amax(x).item()) == PEAK


def test_large_nvfp4_rowwise_and_dequant(orc, big):
    x, amax = big
    out = fq.fp4q_quantize_nvfp4(x, layouts=fq.ROWWISE, amax=amax)
    want = orc.quantize_nvfp4(bits(x[ROWS]), layouts=orc.ROWWISE, amax=PEAK)
    assert_same("s_dec", host(out["s_dec"]), want["s_dec"])
    assert_same("q_row", sample(out["q_row"]), want["q_row"])
    assert_same("sf_row", sample(out["sf_row"].view(R, C // 16)), want["sf_row"])
    y = fq.fp4q_dequantize(fq.FMT_NVFP4, out["q_row"], out["sf_row"], R, C,
                           tensor_scale=out["s_dec"], out_dtype=torch.bfloat16)
    yw = orc.dequantize(orc.FMT_NVFP4, want["q_row"], want["sf_row"], len(ROWS), C, 1, 16,
                        s_dec=float(want["s_dec"][0]), out_dtype=orc.BF16)
    assert_same("y", sample(y), yw)


def test_large_mxfp6(orc, big):
    x, _ = big
    out = fq.fp4q_quantize_mxfp6(x, fq.FP6_E2M3)
    want = orc.quantize_mxfp6(bits(x[ROWS]), orc.FP6_E2M3)
    assert_same("q", sample(out["q"]), want["q"])
    assert_same("sf", sample(out["sf"].view(R, C // 32)), want["sf"])


@pytest.mark.parametrize("fmt", ["if4", "if6", "if3"])
def test_large_if(orc, big, fmt):
    x, amax = big
    if fmt == "if4":
        out = fq.fp4q_quantize_if4(x, amax=amax)
        want = orc.quantize_if4(bits(x[ROWS]), amax=PEAK)
    elif fmt == "if6":
        out = fq.fp4q_quantize_if6(x, amax=amax)
        want = orc.quantize_if6(bits(x[ROWS]), amax=PEAK)
    else:
        out = fq.fp4q_quantize_if3(x, amax=amax)
        want = orc.quantize_if3(bits(x[ROWS]), amax=PEAK)
    assert_same("s_dec", host(out["s_dec"]), want["s_dec"])
    assert_same("q", sample(out["q"]), want["q"])
    assert_same("sf", sample(out["sf"].view(R, C // 16)), want["sf"])


# Row bands for the formats whose blocks or tiles span rows: a band of whole
# column blocks (16 rows; 32 for MXFP4; the transform's 16- or 128-token
# groups) gives, on the oracle run on the band alone, the same column-wise
# codes and scales as the whole tensor once the tensor amax is given.
def bands(n):
    return [0, (R // 2 // n) * n + n, R - n]


def test_large_nvfp4_rowcol(orc, big):
    x, amax = big
    out = fq.fp4q_quantize_nvfp4(x, layouts=fq.ROWWISE | fq.COLWISE, amax=amax)
    for r0 in bands(16):
        want = orc.quantize_nvfp4(bits(x[r0:r0 + 16]), layouts=3, amax=PEAK)
        assert_same("q_row", host(out["q_row"][r0:r0 + 16]), want["q_row"])
        assert_same("sf_row", host(out["sf_row"].view(R, C // 16)[r0:r0 + 16]), want["sf_row"])
        assert_same("q_col", host(out["q_col"][:, r0 // 2:r0 // 2 + 8]), want["q_col"])
        assert_same("sf_col", host(out["sf_col"].view(C, R // 16)[:, r0 // 16:r0 // 16 + 1]),
                    want["sf_col"])


def test_large_mxfp4_rowcol(orc, big):
    x, _ = big
    out = fq.fp4q_quantize_mxfp4(x, layouts=fq.ROWWISE | fq.COLWISE)
    for r0 in bands(32):
        want = orc.quantize_mxfp4(bits(x[r0:r0 + 32]), layouts=3)
        assert_same("q_row", host(out["q_row"][r0:r0 + 32]), want["q_row"])
        assert_same("sf_row", host(out["sf_row"].view(R, C // 32)[r0:r0 + 32]), want["sf_row"])
        assert_same("q_col", host(out["q_col"][:, r0 // 2:r0 // 2 + 16]), want["q_col"])
        assert_same("sf_col", host(out["sf_col"].view(C, R // 32)[:, r0 // 32:r0 // 32 + 1]),
                    want["sf_col"])


def test_large_2d(orc, big):
    x, amax = big
    out = fq.fp4q_quantize_2d(x, amax=amax)
    for r0 in bands(16):
        want = orc.quantize_2d(bits(x[r0:r0 + 16]), amax=PEAK)
        assert_same("q_w", host(out["q_w"][r0:r0 + 16]), want["q_w"])
        assert_same("q_wt", host(out["q_wt"][:, r0 // 2:r0 // 2 + 8]), want["q_wt"])
        assert_same("sf_tiles", host(out["sf_tiles"].view(R // 16, C // 16)[r0 // 16]),
                    want["sf_tiles"])


@pytest.mark.parametrize("n", [16, 128])
def test_large_rht(orc, big, n):
    """The transform works within 16- or 128-token groups and its signs repeat
    per group, so a band of whole groups is transformed and quantized as in
    the whole tensor; the transform's amax is given (any positive value is a
    valid caller amax) so that the band needs no global reduction."""
    x, _ = big
    a = 16384.0
    out = fq.fp4q_quantize_rht_sr(x, n, round=fq.RNE,
                                  amax_rht=torch.tensor([a], dtype=torch.float32, device=DEV))
    for r0 in bands(n):
        want = orc.quantize_rht(bits(x[r0:r0 + n]), n, round=orc.RNE, amax_rht=a)
        assert_same("s_dec", host(out["s_dec"]), want["s_dec"])
        assert_same("q_t", host(out["q_t"][:, r0 // 2:r0 // 2 + n // 2]), want["q_t"])
        assert_same("sf_t", host(out["sf_t"].view(C, R // 16)[:, r0 // 16:r0 // 16 + n // 16]),
                    want["sf_t"])


@pytest.mark.parametrize("layouts", [1, 3])
def test_large_nvfp4_sr(orc, big, layouts):
    """Stochastic rounding at more than 2^31 elements: the oracle runs on a
    band with the band's first row, so that its SR bits come from the whole
    tensor's flat index, as the kernel's do."""
    x, amax = big
    out = fq.fp4q_quantize_nvfp4(x, layouts=layouts, round=fq.SR, seed=21, amax=amax)
    for r0 in bands(16):
        want = orc.quantize_nvfp4(bits(x[r0:r0 + 16]), layouts=layouts, round=orc.SR, seed=21,
                                  amax=PEAK, row0=r0)
        assert_same("q_row", host(out["q_row"][r0:r0 + 16]), want["q_row"])
        assert_same("sf_row", host(out["sf_row"].view(R, C // 16)[r0:r0 + 16]), want["sf_row"])
        if layouts & fq.COLWISE:
            assert_same("q_col", host(out["q_col"][:, r0 // 2:r0 // 2 + 8]), want["q_col"])


@pytest.mark.parametrize("n", [16, 128])
def test_large_rht_sr(orc, big, n):
    x, _ = big
    a = 16384.0
    out = fq.fp4q_quantize_rht_sr(x, n, round=fq.SR, seed=23,
                                  amax_rht=torch.tensor([a], dtype=torch.float32, device=DEV))
    for r0 in bands(n):
        want = orc.quantize_rht(bits(x[r0:r0 + n]), n, round=orc.SR, seed=23, amax_rht=a,
                                token0=r0)
        assert_same("q_t", host(out["q_t"][:, r0 // 2:r0 // 2 + n // 2]), want["q_t"])
        assert_same("sf_t", host(out["sf_t"].view(C, R // 16)[:, r0 // 16:r0 // 16 + n // 16]),
                    want["sf_t"])
