"""GPU parity at a tensor of more than 2^31 elements (the 64-bit index paths).

A 32768 x 65600 BF16 tensor (2.15e9 elements, 4.3 GB) takes the kernels'
64-bit index paths.  The whole tensor is too large for the oracle, so the
checks are the ones that hold at any size: the tensor amax against a planted
maximum at the very last element, and sampled rows (first, second, middle,
last) against the oracle run on those rows alone.  The row-wise formats are
row-independent once the tensor amax is given, so that comparison is exact.
Round to nearest throughout (the stochastic-rounding bits depend on the
global element index).
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
