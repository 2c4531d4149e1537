"""fp4q_quantize_nvfp4_noalloc against fp4q_quantize_nvfp4, through the C ABI.

The no-allocation variant is for callers that cannot allocate device memory
(a host application or framework that owns every device buffer): it keeps
the tensor amax in the library's own device array instead of a caller
workspace.  Its outputs must be byte-identical to the workspace version's.
Two calls in a row, the first on a tensor with the larger amax, check that the
shared array is cleared between calls rather than keeping the previous amax.

The file name makes pytest collect it last.
"""
import ctypes

import pytest
import torch

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import workloads

pytestmark = pytest.mark.gpu


def _outputs(rows, cols, dev, scale_layout):
    return {
        "s_dec": torch.full((1,), -1.0, dtype=torch.float32, device=dev),
        "q_row": torch.full((rows, cols // 2), 0xAA, dtype=torch.uint8, device=dev),
        "sf_row": torch.full((fq.fp4q_scale_bytes(rows, cols, 16, scale_layout),), 0xAA,
                             dtype=torch.uint8, device=dev),
        "q_col": torch.full((cols, rows // 2), 0xAA, dtype=torch.uint8, device=dev),
        "sf_col": torch.full((fq.fp4q_scale_bytes(cols, rows, 16, scale_layout),), 0xAA,
                             dtype=torch.uint8, device=dev),
    }


def _noalloc(x, out, rnd, seed, scale_layout):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rows, cols = x.shape
    status = fq.lib().fp4q_quantize_nvfp4_noalloc(
        p(x), 0 if x.dtype == torch.bfloat16 else 1, rows, cols, x.stride(0),
        fq.ROWWISE | fq.COLWISE, rnd, seed, None, p(out["s_dec"]), p(out["q_row"]),
        p(out["sf_row"]), p(out["q_col"]), p(out["sf_col"]), scale_layout,
        ctypes.c_void_p(torch.cuda.current_stream(x.device).cuda_stream))
    assert status == 0, fq.fp4q_status_string(status)


@pytest.mark.parametrize("dtype,rnd,scale_layout", [
    (torch.bfloat16, fq.RNE, fq.SCALE_SWIZZLED),
    (torch.float32, fq.SR, fq.SCALE_LINEAR),
])
def test_noalloc_matches_workspace_version_twice(dtype, rnd, scale_layout):
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    rows, cols = 256, 512
    big = workloads.activation(seed=11, rows=rows, cols=cols).to(dtype).to(dev)
    small = (workloads.activation(seed=12, rows=rows, cols=cols, n_outlier_cols=0)
             .to(dtype).to(dev))
    assert float(big.abs().max()) > 4 * float(small.abs().max())
    for x, seed in ((big, 5), (small, 6)):
        want = fq.fp4q_quantize_nvfp4(x, layouts=fq.ROWWISE | fq.COLWISE, round=rnd, seed=seed,
                                      scale_layout=scale_layout)
        got = _outputs(rows, cols, dev, scale_layout)
        _noalloc(x, got, rnd, seed, scale_layout)
        torch.cuda.synchronize(dev)
        for k in ("s_dec", "q_row", "sf_row", "q_col", "sf_col"):
            assert torch.equal(got[k].view(torch.uint8), want[k].view(torch.uint8)), k


def test_noalloc_refuses_host_input():
    x = torch.zeros(16, 16, dtype=torch.bfloat16)
    out = _outputs(16, 16, torch.device("cuda", 0), fq.SCALE_LINEAR)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    status = fq.lib().fp4q_quantize_nvfp4_noalloc(
        p(x), 0, 16, 16, 16, fq.ROWWISE, fq.RNE, 0, None, p(out["s_dec"]), p(out["q_row"]),
        p(out["sf_row"]), None, None, fq.SCALE_LINEAR, None)
    assert fq.fp4q_status_string(status) == "FP4Q_ERR_INVALID_ARG"
