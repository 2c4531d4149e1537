"""GPU parity of the comparison formats, through the C ABI, against the oracle.

NVINT4 and four-over-six are the alternatives the "Adaptive Block-Scaled Data
Types" explainer measures IF4 against (sections 1 and 4).  Codes, scale bytes
(with the INT4 flags), tensor scales and dequantized values must match the
oracle bit for bit.
"""
import numpy as np
import pytest
import torch

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import workloads

from test_gpu_parity import DEV, DTYPES, assert_same, bits, host, randmat

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape,layout", [((16, 16), 0), ((48, 80), 0), ((80, 336), 0),
                                          ((128, 256), 1), ((256, 64), 1)])
def test_nvint4(orc, dtype, shape, layout):
    x = randmat(*shape, dtype, seed=61)
    got = fq.fp4q_quantize_nvint4(x.to(DEV), scale_layout=layout)
    want = orc.quantize_if4(bits(x), scale_layout=layout, int4_only=True)
    for k in ("s_dec", "q", "sf"):
        assert_same(k, host(got[k]), want[k])
    y = fq.fp4q_dequantize(fq.FMT_IF4, got["q"], got["sf"], *shape, tensor_scale=got["s_dec"],
                           scale_layout=layout)
    yw = orc.dequantize(orc.FMT_IF4, want["q"], want["sf"], *shape, 1, 16,
                        s_dec=want["s_dec"][0], scale_layout=layout)
    assert_same("y", host(y), yw)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("layouts", [1, 2, 3])
@pytest.mark.parametrize("shape,layout", [((16, 16), 0), ((48, 80), 0), ((80, 144), 0),
                                          ((208, 336), 0), ((128, 256), 1), ((256, 512), 1)])
def test_four_over_six(orc, dtype, layouts, shape, layout):
    x = randmat(*shape, dtype, seed=62)
    got = fq.fp4q_quantize_four_over_six(x.to(DEV), layouts=layouts, scale_layout=layout)
    want = orc.quantize_four_over_six(bits(x), layouts=layouts, scale_layout=layout)
    for k in want:
        assert_same(k, host(got[k]), want[k])


def test_four_over_six_given_amax_and_dequant(orc):
    x = randmat(256, 256, torch.bfloat16, seed=63)
    a = float(np.float32(torch.abs(x.float()).max().item()) * np.float32(1.5))
    amax = torch.tensor([a], dtype=torch.float32, device=DEV)
    got = fq.fp4q_quantize_four_over_six(x.to(DEV), layouts=3, amax=amax,
                                         scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_four_over_six(bits(x), layouts=3, amax=a, scale_layout=orc.SCALE_SWIZZLED)
    for k in want:
        assert_same(k, host(got[k]), want[k])
    y = fq.fp4q_dequantize(fq.FMT_NVFP4, got["q_col"], got["sf_col"], 256, 256,
                           tensor_scale=got["s_dec"], scale_layout=fq.SCALE_SWIZZLED,
                           out_dtype=torch.bfloat16)
    yw = orc.dequantize(orc.FMT_NVFP4, want["q_col"], want["sf_col"], 256, 256, 1, 16,
                        s_dec=want["s_dec"][0], scale_layout=orc.SCALE_SWIZZLED,
                        out_dtype=orc.BF16)
    assert_same("y", host(y), yw)


def test_variants_empty():
    x = torch.empty((0, 32), dtype=torch.bfloat16, device=DEV)
    amax = torch.tensor([1792.0], device=DEV)
    out = fq.fp4q_quantize_four_over_six(x, layouts=1, amax=amax)
    assert out["s_dec"].item() == 1.0
    amax = torch.tensor([2688.0], device=DEV)
    out = fq.fp4q_quantize_nvint4(x, amax=amax)
    assert out["s_dec"].item() == 1.0


def test_variants_activation_fullsize(orc):
    """The activation workload (8192x4096 BF16), swizzled scales, both calls."""
    x = workloads.activation()
    xb = bits(x)
    xd = x.to(DEV)
    got = fq.fp4q_quantize_four_over_six(xd, layouts=3, scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_four_over_six(xb, layouts=3, scale_layout=orc.SCALE_SWIZZLED)
    for k in want:
        assert_same(k, host(got[k]), want[k])
    got = fq.fp4q_quantize_nvint4(xd, scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_if4(xb, scale_layout=orc.SCALE_SWIZZLED, int4_only=True)
    for k in want:
        assert_same(k, host(got[k]), want[k])
