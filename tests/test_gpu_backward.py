"""GPU parity of the fused backward call (both dY operands from one read).

Qiita note on NVFP4 training, "誤差逆伝播と転置" and "ランダムアダマール変換":
Dgrad consumes dY row-wise and Wgrad consumes dY^T after the random Hadamard
transform.  fp4q_quantize_backward must reproduce, bit for bit, the oracle's
row-wise NVFP4 of dY (seed_row) and its RHT + column-wise NVFP4 (seed_col).
"""
import numpy as np
import pytest
import torch

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import workloads

from test_gpu_parity import DEV, DTYPES, assert_same, bits, host, randmat

pytestmark = pytest.mark.gpu

KEYS = ("s_dec_row", "q_row", "sf_row", "s_dec_col", "q_t", "sf_t")


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def check(orc, dy, n, rnd, layout, amax_row=None, amax_rht=None, seeds=(3, 4)):
    got = fq.fp4q_quantize_backward(
        dy.to(DEV), n, round=rnd, seed_row=seeds[0], seed_col=seeds[1], scale_layout=layout,
        amax_row=None if amax_row is None else torch.tensor([amax_row], device=DEV),
        amax_rht=None if amax_rht is None else torch.tensor([amax_rht], device=DEV))
    want = orc.quantize_backward(bits(dy), n, round=rnd, seed_row=seeds[0], seed_col=seeds[1],
                                 amax_row=amax_row, amax_rht=amax_rht, scale_layout=layout)
    for k in KEYS:
        assert_same(k, host(got[k]), want[k])


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("rnd", [0, 1])
@pytest.mark.parametrize("n,shape", [(16, (16, 16)), (16, (48, 80)), (16, (144, 208)),
                                     (128, (128, 48)), (128, (256, 96))])
def test_backward_linear(orc, dtype, rnd, n, shape):
    check(orc, randmat(*shape, dtype, seed=71), n, rnd, 0)


@pytest.mark.parametrize("rnd", [0, 1])
@pytest.mark.parametrize("n", [16, 128])
def test_backward_zero_scale_blocks(orc, rnd, n):
    """Blocks whose scale code is 0 (factor 0: signed zeros) in both outputs."""
    from test_gpu_parity import wide_range
    check(orc, wide_range(256, 48, torch.bfloat16, seed=43), n, rnd, 0)


@pytest.mark.parametrize("rnd", [0, 1])
@pytest.mark.parametrize("n", [16, 128])
def test_backward_swizzled_given_amaxes(orc, rnd, n):
    dy = randmat(256, 128, torch.bfloat16, seed=72)
    a = float(torch.abs(dy.float()).max().item())
    rht = orc.rht(bits(dy), n, seed=4)
    ar = float(np.abs(rht).max())
    check(orc, dy, n, rnd, 1, amax_row=a, amax_rht=ar)


def test_backward_same_seed_draws_independent_of_operand(orc):
    """With seed_row == seed_col the two outputs still match the oracle (the
    row path and the column path use the same counters, each on its own
    values)."""
    check(orc, randmat(64, 64, torch.float32, seed=73), 16, 1, 0, seeds=(9, 9))


def test_backward_empty():
    dy = torch.empty((0, 32), dtype=torch.bfloat16, device=DEV)
    out = fq.fp4q_quantize_backward(dy, 16, amax_row=torch.tensor([2688.0], device=DEV),
                                    amax_rht=torch.tensor([5376.0], device=DEV))
    assert out["s_dec_row"].item() == 1.0 and out["s_dec_col"].item() == 2.0


def test_backward_rejects_cols_not_16():
    dy = torch.zeros((16, 24), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_quantize_backward(dy, 16)


@pytest.mark.parametrize("n,rnd", [(16, 1), (128, 0)])
def test_backward_gradient_fullsize(orc, n, rnd):
    """The gradient workload (8192x5120 BF16), swizzled scales."""
    check(orc, workloads.gradient(), n, rnd, 1, seeds=(0, 0))
