"""GPU parity of IF6 (FP6 E2M3 or INT6 per 16-value block), through the C ABI.

"Adaptive Block-Scaled Data Types" explainer, section 2 (the IF idea extends
to 6 bits).  Codes, flagged scale bytes, the tensor scale and the dequantized
values must match the oracle bit for bit.
"""
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


def check(orc, x, layout, amax=None, out_dtype=torch.float32):
    rows, cols = x.shape
    got = fq.fp4q_quantize_if6(x.to(DEV), scale_layout=layout,
                               amax=None if amax is None else torch.tensor([amax], device=DEV))
    want = orc.quantize_if6(bits(x), amax=amax, scale_layout=layout)
    for k in ("s_dec", "q", "sf"):
        assert_same(k, host(got[k]), want[k])
    y = fq.fp4q_dequantize(fq.FMT_IF6, got["q"], got["sf"], rows, cols, 1, 16,
                           tensor_scale=got["s_dec"], scale_layout=layout, out_dtype=out_dtype)
    yw = orc.dequantize(orc.FMT_IF6, want["q"], want["sf"], rows, cols, 1, 16,
                        s_dec=float(want["s_dec"][0]), scale_layout=layout,
                        out_dtype=orc.FP32 if out_dtype == torch.float32 else orc.BF16)
    assert_same("y", host(y), yw)
    return want


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (48, 80), (130, 336), (257, 1024)])
def test_if6_linear(orc, dtype, shape):
    check(orc, randmat(*shape, dtype, seed=101), 0)


@pytest.mark.parametrize("shape", [(128, 64), (256, 512)])
def test_if6_swizzled_bf16_out(orc, shape):
    check(orc, randmat(*shape, torch.bfloat16, seed=102), 1, out_dtype=torch.bfloat16)


def test_if6_mixed_blocks_and_given_amax(orc):
    """Uniform blocks (INT6 wins) beside heavy-tailed ones (FP6 wins), and a
    caller amax above the data's."""
    x = workloads.if4_blocks(rows=128, cols=512)
    a = float(torch.abs(x.float()).max().item()) * 1.25
    want = check(orc, x, 1, amax=a)
    flags = want["sf"] >= 0x80
    assert 0.05 < flags.mean() < 0.95


def test_if6_strided_input(orc):
    base = randmat(64, 96, torch.float32, seed=103).to(DEV)
    x = base[:, :64]
    got = fq.fp4q_quantize_if6(x)
    want = orc.quantize_if6(bits(x))
    for k in ("s_dec", "q", "sf"):
        assert_same(k, host(got[k]), want[k])


def test_if6_degenerate(orc):
    x = torch.zeros((32, 64), dtype=torch.bfloat16)
    x[3, 5] = 1e-38
    x[7, :16] = -2.0
    check(orc, x, 0)
    e = torch.empty((0, 32), dtype=torch.bfloat16, device=DEV)
    out = fq.fp4q_quantize_if6(e, amax=torch.tensor([3360.0], device=DEV))
    assert out["s_dec"].item() == 1.0


def test_if6_rejects_cols_not_16():
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_quantize_if6(torch.zeros((16, 24), dtype=torch.bfloat16, device=DEV))


def test_if6_fullsize(orc):
    """The IF4 workload (16384x8192 BF16), swizzled scales."""
    x = workloads.if4_blocks()
    got = fq.fp4q_quantize_if6(x.to(DEV), scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_if6(bits(x), scale_layout=orc.SCALE_SWIZZLED)
    for k in ("s_dec", "q", "sf"):
        assert_same(k, host(got[k]), want[k])
