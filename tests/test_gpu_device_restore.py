"""The C ABI runs each call on the device that holds its input and gives the
caller's current device back on return (include/fp4q.h, conventions).

With one GPU the check is that a call leaves device 0 current. With two or
more, a call on a tensor of device 1, made while device 0 is current, must
leave device 0 current. It must also write the same bytes as the same call
made on device 0.
"""
import pytest
import torch

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import workloads

pytestmark = pytest.mark.gpu


def test_a_call_leaves_the_current_device_as_it_was():
    torch.cuda.set_device(0)
    x = workloads.activation(rows=256, cols=256).to("cuda:0")
    fq.fp4q_quantize_nvfp4(x, layouts=fq.ROWWISE | fq.COLWISE)
    fq.fp4q_quantize_nvfp4_noalloc(
        x, {"s_dec": torch.empty(1, device="cuda:0"),
            "q_row": torch.empty((256, 128), dtype=torch.uint8, device="cuda:0"),
            "sf_row": torch.empty(256 * 16, dtype=torch.uint8, device="cuda:0")})
    torch.cuda.synchronize()
    assert torch.cuda.current_device() == 0


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs two GPUs")
def test_a_call_on_another_device_restores_the_callers_device():
    torch.cuda.set_device(0)
    x = workloads.activation(rows=256, cols=256)
    o1 = fq.fp4q_quantize_nvfp4(x.to("cuda:1"), layouts=fq.ROWWISE | fq.COLWISE)
    assert torch.cuda.current_device() == 0
    o0 = fq.fp4q_quantize_nvfp4(x.to("cuda:0"), layouts=fq.ROWWISE | fq.COLWISE)
    torch.cuda.synchronize("cuda:1")
    torch.cuda.synchronize("cuda:0")
    for k in o0:
        assert torch.equal(o0[k].cpu(), o1[k].cpu()), k
    assert torch.cuda.current_device() == 0
