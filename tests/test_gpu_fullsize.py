"""GPU parity at the benchmark sizes, with the calls bench.py times.

Each workload is generated from its seed, quantized on the GPU exactly as
the benchmark does (tensor amax computed on the device first and passed in),
and every output byte is compared with the oracle run over the whole tensor
on the host.
"""
import numpy as np
import pytest
import torch

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import workloads

from test_gpu_parity import assert_same, bits, host

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def test_small_matrix_quant_dequant(orc):
    """256x256 BF16, NVFP4 1x16 + FP32 dequant."""
    x = workloads.small_matrix()
    xd = x.to(DEV)
    amax = fq.fp4q_amax(xd)
    got = fq.fp4q_quantize_nvfp4(xd, layouts=fq.ROWWISE, amax=amax)
    y = fq.fp4q_dequantize(fq.FMT_NVFP4, got["q_row"], got["sf_row"], 256, 256,
                           tensor_scale=got["s_dec"])
    want = orc.quantize_nvfp4(bits(x), layouts=orc.ROWWISE)
    for k in ("s_dec", "q_row", "sf_row"):
        assert_same(k, host(got[k]), want[k])
    yw = orc.dequantize(orc.FMT_NVFP4, want["q_row"], want["sf_row"], 256, 256,
                        s_dec=float(want["s_dec"][0]))
    assert_same("dequant", host(y), yw)


def test_activation_nvfp4_and_mxfp4_rowcol(orc):
    """8192x4096 BF16 activation: NVFP4 row+col from one read, and MXFP4."""
    x = workloads.activation()
    xb = bits(x)
    xd = x.to(DEV)
    amax = fq.fp4q_amax(xd)
    assert_same("amax", host(amax), np.array([orc.amax(xb)], np.float32))
    got = fq.fp4q_quantize_nvfp4(xd, layouts=3, amax=amax, scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_nvfp4(xb, layouts=3, scale_layout=orc.SCALE_SWIZZLED)
    for k in ("s_dec", "q_row", "sf_row", "q_col", "sf_col"):
        assert_same(k, host(got[k]), want[k])
    got = fq.fp4q_quantize_mxfp4(xd, layouts=3, scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_mxfp4(xb, layouts=3, scale_layout=orc.SCALE_SWIZZLED)
    for k in ("q_row", "sf_row", "q_col", "sf_col"):
        assert_same("mx " + k, host(got[k]), want[k])


def test_weight_2d(orc):
    """14336x4096 FP32 weight, 16x16 tiles, W and W^T; q(W) = q(W^T)^T."""
    w = workloads.weight()
    wd = w.to(DEV)
    amax = fq.fp4q_amax(wd)
    got = fq.fp4q_quantize_2d(wd, amax=amax)
    want = orc.quantize_2d(bits(w))
    for k in ("s_dec", "q_w", "q_wt", "sf_tiles"):
        assert_same(k, host(got[k]), want[k])


@pytest.mark.parametrize("n", [16, 128])
def test_gradient_rht(orc, n):
    """8192x5120 BF16 Student-t gradient, RHT(n) + NVFP4 of dY^T, SR and RNE."""
    dy = workloads.gradient()
    db = bits(dy)
    dd = dy.to(DEV)
    a = fq.fp4q_rht_amax(dd, n, seed=0)
    for rnd in (fq.SR, fq.RNE):
        got = fq.fp4q_quantize_rht_sr(dd, n, round=rnd, seed=0, amax_rht=a,
                                      scale_layout=fq.SCALE_SWIZZLED)
        want = orc.quantize_rht(db, n, round=rnd, seed=0, scale_layout=orc.SCALE_SWIZZLED)
        for k in ("s_dec", "q_t", "sf_t"):
            assert_same(f"n={n} round={rnd} {k}", host(got[k]), want[k])


def test_if4_quant_dequant(orc):
    """16384x8192 BF16 mixed uniform / Laplace blocks: IF4 and BF16 dequant."""
    x = workloads.if4_blocks()
    xb = bits(x)
    xd = x.to(DEV)
    amax = fq.fp4q_amax(xd)
    got = fq.fp4q_quantize_if4(xd, amax=amax, scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_if4(xb, scale_layout=orc.SCALE_SWIZZLED)
    for k in ("s_dec", "q", "sf"):
        assert_same(k, host(got[k]), want[k])
    flags = (want["sf"] & 0x80) != 0
    assert 0.05 < flags.mean() < 0.95
    y = fq.fp4q_dequantize(fq.FMT_IF4, got["q"], got["sf"], 16384, 8192,
                           tensor_scale=got["s_dec"], scale_layout=fq.SCALE_SWIZZLED,
                           out_dtype=torch.bfloat16)
    yw = orc.dequantize(orc.FMT_IF4, want["q"], want["sf"], 16384, 8192,
                        s_dec=float(want["s_dec"][0]), scale_layout=orc.SCALE_SWIZZLED,
                        out_dtype=orc.BF16)
    assert_same("dequant", host(y), yw)
