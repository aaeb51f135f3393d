"""Failure detection without a GPU fault: a device wait on an mbarrier nothing
arrives at gives up after its bound, records the timeout in the device error
word, and the CUDA context stays usable for the next call."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import dual_window_attention_b200 as ttcd
    ttcd.get_device_error()  # clear
    assert ttcd.test_bounded_wait(2_000_000) == ttcd.OK  # 2 ms bound
    st, flags = ttcd.get_device_error()
    assert st == ttcd.ERR_TIMEOUT and flags & 1
    assert ttcd.get_device_error()[0] == ttcd.OK  # reading clears it
    q = torch.randn(1, 256, 2, 64, device="cuda").bfloat16()
    k = torch.randn(1, 256, 1, 64, device="cuda").bfloat16()
    o_T, o_S, _, _ = ttcd.dual_window_attn(q, k, k, 16, 64)
    torch.cuda.synchronize()
    assert torch.isfinite(o_T).all() and ttcd.get_device_error()[0] == ttcd.OK
