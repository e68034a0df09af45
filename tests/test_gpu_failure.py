"""The bounded-wait failure path on the GPU, made to run out on purpose: one
thread waits on a barrier nothing arrives on, with a ~2 ms budget.  The host
must read NVFP4_ERR_TIMEOUT from nvfp4_check_device_error, the record must be
cleared by that check, and the context must stay usable.  No fault, no hang."""
import pytest
import torch

import nvfp4_w4a4_gated_b200 as nv

pytestmark = pytest.mark.gpu


def test_bounded_wait_expiry_is_reported_and_cleared(cuda_dev):
    nv.check_device_error()                 # start from a clean record
    nv.selftest_wait_timeout(1 << 22)
    with pytest.raises(nv.NVFP4Error) as ei:
        nv.check_device_error()
    assert ei.value.status == 5 and "bounded wait" in str(ei.value)
    nv.check_device_error()                 # the check cleared the record
    # the context still works: a quantisation runs and checks clean
    x = torch.randn((128, 256), device="cuda").to(torch.bfloat16)
    q = nv.nvfp4_quantize(x)
    torch.cuda.synchronize()
    nv.check_device_error()
    assert float(q.scale.item()) > 0
