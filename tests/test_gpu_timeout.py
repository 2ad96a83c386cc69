"""The timeout path of the tensor-core GEMM, exercised without a fault (GPU).

Every on-chip wait of the library gives up after a bounded time, reports
MOE_STATUS_TIMEOUT and unwinds (loads already issued are waited for, TMEM
is freed). moe_debug_stall_next_gemms makes the next grouped-GEMM launch wait
on a barrier that nothing signals, so that wait runs out on a normal
problem. The call must return with the status bit set, and the next normal
call on the same stream must give the usual result bit for bit.
"""
import pytest
import torch

import combine_router_gemm_softmax_b200 as M

from gpu_cases import DeviceCase, parity_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["small_ragged", "small_pair"])
def test_gemm_wait_timeout_is_reported_and_the_context_stays_usable(name):
    """small_ragged runs single-CTA tiles, small_pair CTA-pair tiles, whose
    timeout also stops the partner CTA through its shared-memory flag."""
    torch.cuda.set_device(0)
    dc = DeviceCase(parity_case(name)[0])
    y_ref = dc.layer()["y"].clone()
    torch.cuda.synchronize()
    assert int(dc.status.item()) == 0
    assert M.lib().moe_debug_stall_next_gemms(1) == M.MOE_OK
    try:
        dc.status.zero_()
        dc.layer()
        torch.cuda.synchronize()
        assert int(dc.status.item()) & M.MOE_STATUS_TIMEOUT
    finally:
        M.lib().moe_debug_stall_next_gemms(0)
    dc.status.zero_()
    y = dc.layer()["y"]
    torch.cuda.synchronize()
    assert int(dc.status.item()) == 0
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
