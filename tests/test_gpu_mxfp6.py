"""GPU parity of MXFP6 (E2M3 and E3M2 with E8M0 block scales), through the C ABI.

"FP6から考えるLLM量子化" (blog.ast.moe), "FP6で隣り合う値の間隔を見てみる":
the two OCP FP6 element formats under 32-value power-of-two scaling.  Codes
(packed four per three bytes), scale bytes and dequantized values must match
the oracle bit for bit, for every E8M0 rule, both scale layouts and both input
types.
"""
import numpy as np
import pytest
import torch

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import workloads

from test_gpu_parity import DEV, DTYPES, assert_same, bits, host, randmat

pytestmark = pytest.mark.gpu

FMT_CODE = {fq.FP6_E2M3: fq.FMT_MXFP6_E2M3, fq.FP6_E3M2: fq.FMT_MXFP6_E3M2}
QMAX = {fq.FP6_E2M3: 7.5, fq.FP6_E3M2: 28.0}


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def check(orc, x, fmt, mode, layout, out_dtype=torch.float32):
    rows, cols = x.shape
    got = fq.fp4q_quantize_mxfp6(x.to(DEV), fmt, mode, scale_layout=layout)
    want = orc.quantize_mxfp6(bits(x), fmt, mode, scale_layout=layout)
    assert_same("q", host(got["q"]), want["q"])
    assert_same("sf", host(got["sf"]), want["sf"])
    y = fq.fp4q_dequantize(FMT_CODE[fmt], got["q"], got["sf"], rows, cols, 1, 32,
                           scale_layout=layout, out_dtype=out_dtype)
    yw = orc.dequantize(FMT_CODE[fmt], want["q"], want["sf"], rows, cols, 1, 32,
                        scale_layout=layout,
                        out_dtype=orc.FP32 if out_dtype == torch.float32 else orc.BF16)
    assert_same("y", host(y), yw)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("fmt", [fq.FP6_E2M3, fq.FP6_E3M2])
@pytest.mark.parametrize("mode", [fq.E8M0_RNE, fq.E8M0_CEIL, fq.E8M0_OCP_FLOOR])
@pytest.mark.parametrize("shape", [(1, 32), (3, 64), (130, 96), (257, 416)])
def test_mxfp6_linear(orc, dtype, fmt, mode, shape):
    check(orc, randmat(*shape, dtype, seed=91), fmt, mode, fq.SCALE_LINEAR)


@pytest.mark.parametrize("fmt", [fq.FP6_E2M3, fq.FP6_E3M2])
@pytest.mark.parametrize("shape", [(128, 128), (256, 512)])
def test_mxfp6_swizzled_bf16_out(orc, fmt, shape):
    check(orc, randmat(*shape, torch.bfloat16, seed=92), fmt, fq.E8M0_RNE, fq.SCALE_SWIZZLED,
          out_dtype=torch.bfloat16)


@pytest.mark.parametrize("fmt", [fq.FP6_E2M3, fq.FP6_E3M2])
@pytest.mark.parametrize("mode", [fq.E8M0_RNE, fq.E8M0_CEIL, fq.E8M0_OCP_FLOOR])
def test_mxfp6_exponent_edges(orc, fmt, mode):
    """Block maxima on the E8M0 decision points: RN(m / qmax) exactly at 1.5 *
    2^E (the RNE tie), just either side of it, exact powers of two, the FP32
    extremes (the exponent clamps at -127 and at the top) and all-zero
    blocks."""
    q = np.float32(QMAX[fmt])
    maxima = []
    for E in (-20, -3, 0, 1, 2, 7, 40):
        t = np.float32(1.5) * np.float32(2.0) ** E
        m = t * q
        maxima += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(np.inf)),
                   np.float32(2.0) ** E]
    maxima += [np.float32(3.0e38), np.float32(1e-45), np.float32(1.2e-38), np.float32(0.0)]
    rows = len(maxima)
    g = np.random.default_rng(93)
    x = (g.uniform(-1, 1, (rows, 64)) * np.array(maxima, np.float64)[:, None]).astype(np.float32)
    x[:, 5] = np.array(maxima, np.float32)
    x[:, 37] = -np.array(maxima, np.float32)
    check(orc, torch.from_numpy(x), fmt, mode, fq.SCALE_LINEAR)


def test_mxfp6_grid_values_and_signed_zero(orc):
    """Every FP6 code's value (and values midway between neighbours) under a
    unit scale, negative zero and tiny negatives that round to zero."""
    for fmt in (fq.FP6_E2M3, fq.FP6_E3M2):
        vals = np.array([orc.fp6_value(c, fmt) for c in range(64)], np.float32)
        pos = np.sort(vals[:32])
        mids = (pos[:-1] + pos[1:]) / 2
        row = np.concatenate([vals, mids, -mids, [-0.0, -1e-30, 1e-30, -1e-3]]).astype(np.float32)
        row = np.resize(row, 192)
        row[::32] = pos[-1]                     # each block's maximum is the format's maximum
        check(orc, torch.from_numpy(row.reshape(1, -1).copy()), fmt, fq.E8M0_OCP_FLOOR,
              fq.SCALE_LINEAR)


def test_mxfp6_strided_input(orc):
    base = randmat(64, 160, torch.bfloat16, seed=94).to(DEV)
    x = base[:, :128]                           # ld = 160
    got = fq.fp4q_quantize_mxfp6(x, fq.FP6_E3M2)
    want = orc.quantize_mxfp6(bits(x), fq.FP6_E3M2)
    assert_same("q", host(got["q"]), want["q"])
    assert_same("sf", host(got["sf"]), want["sf"])


def test_mxfp6_empty():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    out = fq.fp4q_quantize_mxfp6(x)
    assert out["q"].numel() == 0


def test_mxfp6_rejects_cols_not_32():
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_quantize_mxfp6(torch.zeros((16, 48), dtype=torch.bfloat16, device=DEV))


@pytest.mark.parametrize("fmt", [fq.FP6_E2M3, fq.FP6_E3M2])
def test_mxfp6_activation_fullsize(orc, fmt):
    """The activation workload (8192x4096 BF16), swizzled scales."""
    x = workloads.activation()
    check(orc, x, fmt, fq.E8M0_RNE, fq.SCALE_SWIZZLED, out_dtype=torch.bfloat16)
