"""GPU parity of the tensor-core MXFP4 GEMM (fp4q_gemm_mxfp4) against the
oracle's gemm_block_scaled with MXFP4 operands, through the C ABI.

Ultralytics glossary "FP4", section "FP4の仕組み": MXFP4 gives 32 E2M1 values
one power-of-two E8M0 scale and has no tensor scale; the AIBR summary of
Quartet trains with MXFP4 linear layers on Blackwell.  This GEMM reads
fp4q_quantize_mxfp4's codes and swizzled scales as they are, which checks
that layout against the tensor core's block-scaled MMA (kind::mxf4 block32).
The tensor core accumulates in FP32 in its own order, so the comparison is
against the exact product of the dequantized operands with the FP32
accumulation bound used for the NVFP4 GEMM: every product of two dequantized
values is exact, only the K additions round, |C - exact| <= (K + 2) 2^-22
(|A| |B|^T), plus one rounding for the output type.  A misplaced code
nibble, scale byte or tile is off by the size of the values.
"""
import numpy as np
import pytest
import torch

import fp4_block_scaled_04_b200 as fq

from test_gpu_parity import DEV, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def random_operand(rows, K, seed):
    """Random codes and E8M0 scale bytes (2^-6 .. 2^5), the scale matrix
    [rows, K/32] in the swizzled layout (a permutation of random bytes is
    random bytes)."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    sf = rng.integers(121, 133, rows * K // 32, dtype=np.uint8)
    return q, sf


def check(orc, qa, sfa, qb, sfb, M, N, K, c, out_bits=24):
    exact = orc.gemm_block_scaled(qa, sfa, qb, sfb, M, N, K, fmt=orc.FMT_MXFP4,
                                  scale_layout=orc.SCALE_SWIZZLED)
    a = orc.dequantize(orc.FMT_MXFP4, qa, sfa, M, K, 1, 32,
                       scale_layout=orc.SCALE_SWIZZLED).astype(np.float64)
    b = orc.dequantize(orc.FMT_MXFP4, qb, sfb, N, K, 1, 32,
                       scale_layout=orc.SCALE_SWIZZLED).astype(np.float64)
    mag = np.abs(a) @ np.abs(b).T
    bound = (K + 2) * 2.0 ** -22 * mag + np.abs(exact) * 2.0 ** -out_bits + 1e-30
    err = np.abs(c.astype(np.float64) - exact)
    worst = float(np.max(err / bound))
    assert worst <= 1.0, f"GEMM differs from the exact product by {worst:.3g} x the bound"
    assert np.linalg.norm(exact) > 0


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 128, 512), (128, 384, 1024),
                                   (384, 256, 768), (256, 512, 2048)])
def test_mxfp4_gemm_random_codes_and_scales(orc, M, N, K):
    qa, sfa = random_operand(M, K, 1)
    qb, sfb = random_operand(N, K, 2)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    c = fq.fp4q_gemm_mxfp4(torch.from_numpy(qa).to(DEV), torch.from_numpy(sfa).to(DEV),
                           torch.from_numpy(qb).to(DEV), torch.from_numpy(sfb).to(DEV), K,
                           status=status)
    assert int(status.item()) == 0
    check(orc, qa, sfa, qb, sfb, M, N, K, host(c))


def test_mxfp4_gemm_one_hot_selects_columns(orc):
    """B rows one-hot at 1.0 (code 0x2, scale 2^0): C is a column selection of
    the dequantized A, exact in every FP32 order; a scale byte read from the
    wrong half of its 32-bit cell or the wrong tile shows up as a power of two."""
    M, N, K = 256, 256, 512
    qa, sfa = random_operand(M, K, 3)
    rng = np.random.default_rng(4)
    kn = rng.permutation(K)[:N]
    cb = np.zeros((N, K), np.uint8)
    cb[np.arange(N), kn] = 0x2
    qb = (cb[:, 0::2] | (cb[:, 1::2] << 4)).astype(np.uint8)
    sfb = np.full(N * K // 32, 127, np.uint8)
    c = fq.fp4q_gemm_mxfp4(torch.from_numpy(qa).to(DEV), torch.from_numpy(sfa).to(DEV),
                           torch.from_numpy(qb).to(DEV), torch.from_numpy(sfb).to(DEV), K)
    want = orc.gemm_block_scaled(qa, sfa, qb, sfb, M, N, K, fmt=orc.FMT_MXFP4,
                                 scale_layout=orc.SCALE_SWIZZLED)
    np.testing.assert_array_equal(host(c).astype(np.float64), want)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_mxfp4_fprop_from_quantized_activations_and_weights(orc, out_dtype):
    """Fprop: X [M, K] and W [N, K] through fp4q_quantize_mxfp4 (row-wise,
    swizzled E8M0 scales), then C = X_q W_q^T."""
    M, N, K = 256, 512, 1024
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(M, K, generator=g) * 3).to(torch.bfloat16).to(DEV)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    sw = fq.SCALE_SWIZZLED
    ox = fq.fp4q_quantize_mxfp4(x, layouts=fq.ROWWISE | fq.COLWISE, scale_layout=sw)
    ow = fq.fp4q_quantize_mxfp4(w, layouts=fq.ROWWISE, scale_layout=sw)
    c = fq.fp4q_gemm_mxfp4(ox["q_row"], ox["sf_row"], ow["q_row"], ow["sf_row"], K,
                           out_dtype=out_dtype)
    check(orc, host(ox["q_row"]), host(ox["sf_row"]), host(ow["q_row"]), host(ow["sf_row"]),
          M, N, K, host(c.float()), out_bits=24 if out_dtype == torch.float32 else 8)
    ref = (x.float() @ w.float().t()).cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(host(c.float()) - ref) / np.linalg.norm(ref)
    assert rel < 0.3, rel


def test_mxfp4_wgrad_from_column_wise_copies(orc):
    """Wgrad = dY^T X from the column-wise copies (rows along tokens, the
    contraction dimension)."""
    T, Co, Ci = 512, 128, 256
    g = torch.Generator().manual_seed(12)
    dy = (torch.randn(T, Co, generator=g) * 1e-3).to(torch.bfloat16).to(DEV)
    x = torch.randn(T, Ci, generator=g).to(torch.bfloat16).to(DEV)
    sw = fq.SCALE_SWIZZLED
    od = fq.fp4q_quantize_mxfp4(dy, layouts=fq.COLWISE, scale_layout=sw)
    ox = fq.fp4q_quantize_mxfp4(x, layouts=fq.COLWISE, scale_layout=sw)
    c = fq.fp4q_gemm_mxfp4(od["q_col"], od["sf_col"], ox["q_col"], ox["sf_col"], T)
    check(orc, host(od["q_col"]), host(od["sf_col"]), host(ox["q_col"]), host(ox["sf_col"]),
          Co, Ci, T, host(c))


def test_mxfp4_gemm_rejects_ragged_shapes():
    q = torch.zeros((128, 64), dtype=torch.uint8, device=DEV)
    s = torch.zeros(128 * 4, dtype=torch.uint8, device=DEV)
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_gemm_mxfp4(q, s, q, s, 128)             # K % 256
