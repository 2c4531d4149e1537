"""Consumer check: a block-scaled FP4 GEMM reads the quantized outputs as they are.

Qiita note on NVFP4 training: the quantized operands feed FP4 GEMMs (Fprop
X W^T, Dgrad, Wgrad).  The swizzled scale layout is the 128x4 tile layout that
block-scaled tensor-core GEMMs read, so the library's outputs go straight into
the vendor's block-scaled GEMM (reached through torch.nn.functional.scaled_mm).
The product must equal the exact product of the dequantized operands up to
FP32 accumulation error.  Where the installed library offers no such GEMM,
the test is skipped and says so.

This checks the byte layout against an implementation that is not ours: the
E2M1 nibble order, the E4M3 scale bytes and the 128x4 scale tiles (which
MXFP4 shares).  The installed library's MXFP4 (1x32, E8M0) GEMM path is not
used: its products came out uncorrelated with the operands even though the
same codes and tile layout pass through its NVFP4 path exactly.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import fp4_block_scaled_04_b200 as fq

from test_gpu_parity import DEV, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g) * torch.exp2(torch.randint(-4, 5, (M, 1), generator=g).float())
    w = torch.randn(N, K, generator=g) * 0.05
    w[:, torch.randint(0, K, (8,), generator=g)] *= 20.0
    return x.to(torch.bfloat16).to(DEV), w.to(torch.bfloat16).to(DEV)


def scaled_mm_or_skip(*args, **kw):
    try:
        return F.scaled_mm(*args, **kw)
    except (RuntimeError, NotImplementedError, TypeError, ValueError) as e:
        pytest.skip(f"no block-scaled FP4 GEMM in the installed library: {str(e)[:200]}")


def check_against_exact(c, ya, yb):
    """c [M, N] from the GEMM; ya [M, K], yb [N, K] the dequantized operands
    (FP32, exact).  Every product of two dequantized values is exact in FP32,
    so only the accumulation rounds: |c - ya yb^T| <= (K + 2) 2^-22 (|ya|
    |yb|^T) + tiny (four times the plain FP32 bound, leaving room for the
    tensor cores' accumulation order).  A misplaced scale or nibble is off by
    the size of the values themselves."""
    a = ya.astype(np.float64)
    b = yb.astype(np.float64)
    exact = a @ b.T
    bound = (a.shape[1] + 2) * 2.0 ** -22 * (np.abs(a) @ np.abs(b).T) + 1e-30
    err = np.abs(c.astype(np.float64) - exact)
    worst = float(np.max(err / bound))
    assert worst <= 1.0, f"GEMM differs from the exact product by {worst:.3g} x the bound"
    # and it is not trivially zero
    assert np.linalg.norm(exact) > 0


@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (256, 128, 1024)])
def test_nvfp4_operands_in_block_scaled_gemm(M, N, K):
    x, w = operands(M, N, K, seed=81)
    sw = fq.SCALE_SWIZZLED
    ox = fq.fp4q_quantize_nvfp4(x, layouts=fq.ROWWISE, scale_layout=sw)
    ow = fq.fp4q_quantize_nvfp4(w, layouts=fq.ROWWISE, scale_layout=sw)
    A = ox["q_row"].view(torch.float4_e2m1fn_x2)                # [M, K/2]
    B = ow["q_row"].view(torch.float4_e2m1fn_x2).t()            # [K/2, N], column-major
    sa = ox["sf_row"].view(torch.float8_e4m3fn)
    sb = ow["sf_row"].view(torch.float8_e4m3fn)
    c = scaled_mm_or_skip(A, B, sa, F.ScalingType.BlockWise1x16, sb, F.ScalingType.BlockWise1x16,
                          swizzle_a=F.SwizzleType.SWIZZLE_32_4_4,
                          swizzle_b=F.SwizzleType.SWIZZLE_32_4_4, output_dtype=torch.float32)
    # the GEMM applies the block scales; the tensor scales are applied outside,
    # so the operands are dequantized with s_dec = 1
    one = torch.ones(1, device=DEV)
    ya = fq.fp4q_dequantize(fq.FMT_NVFP4, ox["q_row"], ox["sf_row"], M, K, tensor_scale=one,
                            scale_layout=sw)
    yb = fq.fp4q_dequantize(fq.FMT_NVFP4, ow["q_row"], ow["sf_row"], N, K, tensor_scale=one,
                            scale_layout=sw)
    check_against_exact(host(c), host(ya), host(yb))


def test_wgrad_operands_from_the_column_wise_copies():
    """Wgrad = dY^T X: both operands are the column-wise (transposed) outputs,
    whose rows run along tokens -- the contraction dimension."""
    T, Co, Ci = 512, 128, 256
    g = torch.Generator().manual_seed(83)
    dy = (torch.randn(T, Co, generator=g) * 1e-2).to(torch.bfloat16).to(DEV)
    x = torch.randn(T, Ci, generator=g).to(torch.bfloat16).to(DEV)
    sw = fq.SCALE_SWIZZLED
    od = fq.fp4q_quantize_nvfp4(dy, layouts=fq.COLWISE, scale_layout=sw)   # dY^T [Co, T/2]
    ox = fq.fp4q_quantize_nvfp4(x, layouts=fq.COLWISE, scale_layout=sw)    # X^T [Ci, T/2]
    A = od["q_col"].view(torch.float4_e2m1fn_x2)
    B = ox["q_col"].view(torch.float4_e2m1fn_x2).t()
    c = scaled_mm_or_skip(A, B, od["sf_col"].view(torch.float8_e4m3fn), F.ScalingType.BlockWise1x16,
                          ox["sf_col"].view(torch.float8_e4m3fn), F.ScalingType.BlockWise1x16,
                          swizzle_a=F.SwizzleType.SWIZZLE_32_4_4,
                          swizzle_b=F.SwizzleType.SWIZZLE_32_4_4, output_dtype=torch.float32)
    one = torch.ones(1, device=DEV)
    ya = fq.fp4q_dequantize(fq.FMT_NVFP4, od["q_col"], od["sf_col"], Co, T, tensor_scale=one,
                            scale_layout=sw)
    yb = fq.fp4q_dequantize(fq.FMT_NVFP4, ox["q_col"], ox["sf_col"], Ci, T, tensor_scale=one,
                            scale_layout=sw)
    check_against_exact(host(c), host(ya), host(yb))
