"""GPU parity of the tensor-core NVFP4 GEMM (fp4q_gemm_nvfp4) against the
oracle's gemm_block_scaled, through the C ABI.

Qiita note on NVFP4 training: the quantized operands feed the FP4 GEMMs
(Fprop X W^T from the row-wise copies, Wgrad dY^T X from the column-wise
ones).  The GEMM accumulates in FP32 in the tensor core's own order, so the
comparison is against the exact product of the dequantized operands with
the FP32 accumulation bound: every product of two dequantized values is
exact, only the K additions round, |C - exact| <= (K + 2) 2^-22 (|A| |B|^T)
(four times the textbook bound, leaving room for the hardware's order),
plus one rounding for the tensor-scale product and one for the output type.
A misplaced code nibble, scale byte or tile is off by the size of the values.
"""
import numpy as np
import pytest
import torch

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import workloads

from test_gpu_parity import DEV, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def random_operand(rows, K, seed):
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    sf = rng.integers(0x20, 0x50, rows * K // 16, dtype=np.uint8)   # E4M3 2^-4 .. 2^3
    return q, sf


def check(orc, qa, sfa, qb, sfb, M, N, K, c, alpha=1.0, out_bits=24):
    exact = orc.gemm_block_scaled(qa, sfa, qb, sfb, M, N, K)
    a = orc.dequantize(orc.FMT_NVFP4, qa, sfa, M, K, 1, 16, s_dec=1.0,
                       scale_layout=orc.SCALE_SWIZZLED).astype(np.float64)
    b = orc.dequantize(orc.FMT_NVFP4, qb, sfb, N, K, 1, 16, s_dec=1.0,
                       scale_layout=orc.SCALE_SWIZZLED).astype(np.float64)
    mag = np.abs(a) @ np.abs(b).T
    bound = alpha * (K + 2) * 2.0 ** -22 * mag + abs(alpha * exact) * (2.0 ** -23 + 2.0 ** -out_bits)
    bound += 1e-30
    err = np.abs(c.astype(np.float64) - alpha * exact)
    worst = float(np.max(err / bound))
    assert worst <= 1.0, f"GEMM differs from the exact product by {worst:.3g} x the bound"
    assert np.linalg.norm(exact) > 0


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 128, 512), (128, 384, 1024),
                                   (384, 256, 768), (256, 256, 4096),
                                   # M and N multiples of 256: the two-SM (cluster) kernel
                                   (256, 512, 512), (512, 256, 1024), (768, 768, 256),
                                   (1024, 1024, 2048)])
def test_gemm_random_codes_and_scales(orc, M, N, K):
    qa, sfa = random_operand(M, K, 1)
    qb, sfb = random_operand(N, K, 2)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    c = fq.fp4q_gemm_nvfp4(torch.from_numpy(qa).to(DEV), torch.from_numpy(sfa).to(DEV),
                           torch.from_numpy(qb).to(DEV), torch.from_numpy(sfb).to(DEV), K,
                           status=status)
    assert int(status.item()) == 0
    check(orc, qa, sfa, qb, sfb, M, N, K, host(c))


@pytest.mark.parametrize("M,N", [(256, 128), (512, 256)])
def test_gemm_one_hot_selects_columns(orc, M, N):
    """B rows one-hot at 1.0: C is a column selection of dequantized A, which
    every FP32 order computes exactly (both kernels: N = 128 and the two-SM
    form)."""
    K = 512
    qa, sfa = random_operand(M, K, 3)
    rng = np.random.default_rng(4)
    kn = rng.permutation(K)[:N]
    cb = np.zeros((N, K), np.uint8)
    cb[np.arange(N), kn] = 0x2
    qb = (cb[:, 0::2] | (cb[:, 1::2] << 4)).astype(np.uint8)
    sfb = np.full(N * K // 16, 0x38, np.uint8)
    c = fq.fp4q_gemm_nvfp4(torch.from_numpy(qa).to(DEV), torch.from_numpy(sfa).to(DEV),
                           torch.from_numpy(qb).to(DEV), torch.from_numpy(sfb).to(DEV), K)
    want = orc.gemm_block_scaled(qa, sfa, qb, sfb, M, N, K)
    np.testing.assert_array_equal(host(c).astype(np.float64), want)


def quantized(x):
    o = fq.fp4q_quantize_nvfp4(x, layouts=fq.ROWWISE | fq.COLWISE, scale_layout=fq.SCALE_SWIZZLED)
    return o


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_fprop_from_quantized_activations_and_weights(orc, out_dtype):
    """Fprop: X [M, K] and W [N, K] through fp4q_quantize_nvfp4 (row-wise,
    swizzled scales), then C = s_x s_w (X_q W_q^T)."""
    M, N, K = (256, 384, 1024) if out_dtype == torch.bfloat16 else (512, 512, 1024)
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(M, K, generator=g) * 3).to(torch.bfloat16).to(DEV)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    ox, ow = quantized(x), quantized(w)
    c = fq.fp4q_gemm_nvfp4(ox["q_row"], ox["sf_row"], ow["q_row"], ow["sf_row"], K,
                           tensor_scale_a=ox["s_dec"], tensor_scale_b=ow["s_dec"],
                           out_dtype=out_dtype)
    alpha = float(np.float32(ox["s_dec"].item()) * np.float32(ow["s_dec"].item()))
    check(orc, host(ox["q_row"]), host(ox["sf_row"]), host(ow["q_row"]), host(ow["sf_row"]),
          M, N, K, host(c.float()), alpha=alpha, out_bits=24 if out_dtype == torch.float32 else 8)


def test_wgrad_from_column_wise_copies(orc):
    """Wgrad = dY^T X: both operands are the column-wise outputs (rows run
    along tokens, the contraction dimension)."""
    T, Co, Ci = 512, 128, 256
    g = torch.Generator().manual_seed(12)
    dy = (torch.randn(T, Co, generator=g) * 1e-3).to(torch.bfloat16).to(DEV)
    x = torch.randn(T, Ci, generator=g).to(torch.bfloat16).to(DEV)
    od, ox = quantized(dy), quantized(x)
    c = fq.fp4q_gemm_nvfp4(od["q_col"], od["sf_col"], ox["q_col"], ox["sf_col"], T,
                           tensor_scale_a=od["s_dec"], tensor_scale_b=ox["s_dec"])
    alpha = float(np.float32(od["s_dec"].item()) * np.float32(ox["s_dec"].item()))
    check(orc, host(od["q_col"]), host(od["sf_col"]), host(ox["q_col"]), host(ox["sf_col"]),
          Co, Ci, T, host(c), alpha=alpha)


def test_gemm_strided_output_and_empty_k():
    M, N, K = 128, 128, 256
    qa, sfa = random_operand(M, K, 5)
    qb, sfb = random_operand(N, K, 6)
    big = torch.full((M, N + 64), 7.0, device=DEV)
    view = big[:, :N]
    fq.fp4q_gemm_nvfp4(torch.from_numpy(qa).to(DEV), torch.from_numpy(sfa).to(DEV),
                       torch.from_numpy(qb).to(DEV), torch.from_numpy(sfb).to(DEV), K, out=view)
    assert torch.all(big[:, N:] == 7.0)                 # nothing written past ldc's row
    z = torch.full((M, N), 5.0, device=DEV)
    e = torch.empty((M, 0), dtype=torch.uint8, device=DEV)
    fq.fp4q_gemm_nvfp4(e, e, torch.empty((N, 0), dtype=torch.uint8, device=DEV), e, 0, out=z)
    assert torch.all(z == 0)


def test_gemm_rejects_ragged_shapes():
    q = torch.zeros((128, 64), dtype=torch.uint8, device=DEV)
    s = torch.zeros(128 * 8, dtype=torch.uint8, device=DEV)
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_gemm_nvfp4(q, s, q, s, 128)             # K % 256
    q2 = torch.zeros((96, 128), dtype=torch.uint8, device=DEV)
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_gemm_nvfp4(q2, s, q, s, 256)            # M % 128


def test_dgrad_from_the_backward_call(orc):
    """Dgrad = dY W: A is the row-wise dY from fp4q_quantize_backward (the
    contraction runs over the output features), B is the column-wise copy of
    W [N_out, K_in], i.e. W^T [K_in, N_out] row-wise."""
    T, Nout, Kin = 256, 512, 384
    g = torch.Generator().manual_seed(13)
    dy = (torch.randn(T, Nout, generator=g) * 1e-3).to(torch.bfloat16).to(DEV)
    w = (torch.randn(Nout, Kin, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    sw = fq.SCALE_SWIZZLED
    ob = fq.fp4q_quantize_backward(dy, 16, round=fq.SR, seed_row=5, seed_col=6, scale_layout=sw)
    ow = fq.fp4q_quantize_nvfp4(w, layouts=fq.COLWISE, scale_layout=sw)
    c = fq.fp4q_gemm_nvfp4(ob["q_row"], ob["sf_row"], ow["q_col"], ow["sf_col"], Nout,
                           tensor_scale_a=ob["s_dec_row"], tensor_scale_b=ow["s_dec"])
    alpha = float(np.float32(ob["s_dec_row"].item()) * np.float32(ow["s_dec"].item()))
    check(orc, host(ob["q_row"]), host(ob["sf_row"]), host(ow["q_col"]), host(ow["sf_col"]),
          T, Kin, Nout, host(c), alpha=alpha)
    # and it estimates the unquantized product
    ref = (dy.float() @ w.float()).cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(host(c) - ref) / np.linalg.norm(ref)
    assert rel < 0.3, rel                # about 0.17 from NVFP4 and SR noise


@pytest.mark.parametrize("n", [16, 128])
def test_wgrad_from_rht_operands_with_the_same_signs(orc, n):
    """Qiita note, "ランダムアダマール変換": Wgrad multiplies the transformed
    dY^T and X^T; with the same random signs the transform cancels
    ((H S dY)^T (H S X) c^2 = dY^T X), so the GEMM of the two RHT outputs
    estimates dY^T X."""
    T, Co, Ci = 512, 128, 256
    g = torch.Generator().manual_seed(14)
    dy = (torch.randn(T, Co, generator=g) * 1e-3).to(torch.bfloat16).to(DEV)
    x = torch.randn(T, Ci, generator=g).to(torch.bfloat16).to(DEV)
    sw = fq.SCALE_SWIZZLED
    od = fq.fp4q_quantize_rht_sr(dy, n, round=fq.SR, seed=21, scale_layout=sw)
    ox = fq.fp4q_quantize_rht_sr(x, n, round=fq.SR, seed=21, scale_layout=sw)
    c = fq.fp4q_gemm_nvfp4(od["q_t"], od["sf_t"], ox["q_t"], ox["sf_t"], T,
                           tensor_scale_a=od["s_dec"], tensor_scale_b=ox["s_dec"])
    alpha = float(np.float32(od["s_dec"].item()) * np.float32(ox["s_dec"].item()))
    check(orc, host(od["q_t"]), host(od["sf_t"]), host(ox["q_t"]), host(ox["sf_t"]),
          Co, Ci, T, host(c), alpha=alpha)
    ref = (dy.float().t() @ x.float()).cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(host(c) - ref) / np.linalg.norm(ref)
    assert rel < 0.3, rel                # about 0.2 from NVFP4 and SR noise
    # with different signs the transform does not cancel
    ox2 = fq.fp4q_quantize_rht_sr(x, n, round=fq.SR, seed=22, scale_layout=sw)
    c2 = fq.fp4q_gemm_nvfp4(od["q_t"], od["sf_t"], ox2["q_t"], ox2["sf_t"], T,
                            tensor_scale_a=od["s_dec"], tensor_scale_b=ox2["s_dec"])
    rel2 = np.linalg.norm(host(c2) - ref) / np.linalg.norm(ref)
    assert rel2 > 1.0, rel2              # about 1.5: uncorrelated with dY^T X


def test_gemm_wait_that_runs_out_sets_status_and_leaves_the_context_usable(orc):
    """Failure detection without a GPU fault: the test hook withholds the
    operand loads, so the tensor-core thread's bounded wait (about a second)
    runs out; the kernel must report it through status and return, and the
    next GEMM must be correct."""
    M, N, K = 128, 128, 256
    qa, sfa = random_operand(M, K, 7)
    qb, sfb = random_operand(N, K, 8)
    ta, tsa, tb, tsb = (torch.from_numpy(a).to(DEV) for a in (qa, sfa, qb, sfb))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    c = torch.empty((M, N), device=DEV)
    rc = fq.lib().fp4q_gemm_nvfp4_withhold_loads(
        fq._ptr(ta), fq._ptr(tsa), None, fq._ptr(tb), fq._ptr(tsb), None, M, N, K, fq._ptr(c),
        1, N, fq._ptr(status), fq._stream(ta.device))
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    status.zero_()
    c = fq.fp4q_gemm_nvfp4(ta, tsa, tb, tsb, K, status=status)
    assert int(status.item()) == 0
    check(orc, qa, sfa, qb, sfb, M, N, K, host(c))


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 384, 1024), (512, 256, 2048)])
def test_if4_operand_in_the_tensor_core_gemm(orc, M, N, K):
    """IF4 x NVFP4: the IF4 operand split into FP4 blocks and the two E2M1
    parts of its INT4 blocks, one GEMM pass with an FP4 and an INT4
    accumulator.  Compared with the exact product of the dequantized IF4 and
    NVFP4 operands, with room for three FP32 accumulation chains, the RN(6/7)
    factor and the output addition."""
    x = workloads.if4_blocks(rows=M, cols=K).to(DEV)
    g = torch.Generator().manual_seed(15)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16).to(DEV)
    sw = fq.SCALE_SWIZZLED
    ox = fq.fp4q_quantize_if4(x, scale_layout=sw)
    ow = fq.fp4q_quantize_nvfp4(w, scale_layout=sw)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    c = fq.fp4q_gemm_if4_nvfp4(ox["q"], ox["sf"], ow["q_row"], ow["sf_row"], K,
                               tensor_scale_a=ox["s_dec"], tensor_scale_b=ow["s_dec"],
                               status=status)
    assert int(status.item()) == 0
    qa, sa, qb, sb = host(ox["q"]), host(ox["sf"]), host(ow["q_row"]), host(ow["sf_row"])
    assert 0.05 < np.mean(sa >= 0x80) < 0.95          # both kinds of block present
    alpha = float(np.float32(ox["s_dec"].item()) * np.float32(ow["s_dec"].item()))
    exact = orc.gemm_block_scaled(qa, sa, qb, sb, M, N, K, fmt=orc.FMT_IF4)
    a = orc.dequantize(orc.FMT_IF4, qa, sa, M, K, 1, 16, s_dec=1.0,
                       scale_layout=orc.SCALE_SWIZZLED).astype(np.float64)
    b = orc.dequantize(orc.FMT_NVFP4, qb, sb, N, K, 1, 16, s_dec=1.0,
                       scale_layout=orc.SCALE_SWIZZLED).astype(np.float64)
    bound = alpha * (3 * K + 16) * 2.0 ** -22 * (np.abs(a) @ np.abs(b).T) \
        + abs(alpha * exact) * 2.0 ** -21 + 1e-30
    worst = float(np.max(np.abs(host(c).astype(np.float64) - alpha * exact) / bound))
    assert worst <= 1.0, f"IF4 GEMM differs from the exact product by {worst:.3g} x the bound"
