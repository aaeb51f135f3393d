"""Failure detection without a GPU fault: a device wait on an mbarrier nothing
arrives at gives up after its bound, records the timeout in a status word, and
the CUDA context stays usable for the next call.

Status words are per call: a block forward or MLP keeps its word in its own
workspace, so a timeout on one stream is not seen, and not cleared, by a caller
on another stream; the entry points without a workspace share one word per
device."""
import pytest
import torch

from tests.helpers import TOL_OUT, oracle_block, rel_max, to_device
from ttcd_workloads import BlockShape, make_block_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import dual_window_attention_b200 as ttcd
    ttcd.get_device_error()  # clear
    assert ttcd.test_bounded_wait(2_000_000) == ttcd.OK  # 2 ms bound, per-device word
    st, flags = ttcd.get_device_error()
    assert st == ttcd.ERR_TIMEOUT and flags & 1
    assert ttcd.get_device_error()[0] == ttcd.OK  # reading clears it
    q = torch.randn(1, 256, 2, 64, device="cuda").bfloat16()
    k = torch.randn(1, 256, 1, 64, device="cuda").bfloat16()
    o_T, o_S, _, _ = ttcd.dual_window_attn(q, k, k, 16, 64)
    torch.cuda.synchronize()
    assert torch.isfinite(o_T).all() and ttcd.get_device_error()[0] == ttcd.OK


def test_status_is_per_workspace_on_two_streams():
    """Stream 1: a wait that nothing ends gives up and records a timeout in
    workspace A.  Stream 2, at the same time: a block forward on workspace B.
    B reports OK (and its output matches the oracle), A reports the timeout
    once, and the per-device word stays clear."""
    import dual_window_attention_b200 as ttcd
    shape = BlockShape("status_two_streams", "bf16", B=1, T=300, d_model=128, n_q_heads=4,
                       n_kv_heads=2, head_dim=64, d_ff=256, w_S=48, w_T=200, chunk=64, conv_k=4)
    p = ttcd.BlockParams.from_shape(shape)
    inp = make_block_inputs(shape, seed=21)
    x, w = to_device(inp)
    ws_a = ttcd.alloc_workspace(ttcd.STATUS_BYTES)
    ws_b = ttcd.alloc_workspace(ttcd.block_forward_workspace_size(p))
    ttcd.get_device_error()  # clear the per-device word
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    assert ttcd.test_bounded_wait(50_000_000, status=ws_a, stream=s1) == ttcd.OK  # 50 ms
    with torch.cuda.stream(s2):
        out, _, _ = ttcd.block_forward(x, w["beta"], w, p, workspace=ws_b, stream=s2)
    assert ttcd.check_device_status(ws_b, s2) == ttcd.OK
    assert ttcd.check_device_status(ws_a, s1) == ttcd.ERR_TIMEOUT
    assert ttcd.check_device_status(ws_a, s1) == ttcd.OK  # reading clears it
    assert ttcd.get_device_error()[0] == ttcd.OK
    torch.cuda.synchronize()
    assert rel_max(out, oracle_block(shape, inp)["out"]) <= TOL_OUT


def test_decode_state_holds_its_own_status():
    """A wait that gives up while targeting a decode state is reported by that
    state's check, not by the per-device word."""
    import dual_window_attention_b200 as ttcd
    shape = BlockShape("status_decode", "bf16", B=1, T=1, d_model=128, n_q_heads=2,
                       n_kv_heads=1, head_dim=64, d_ff=256, w_S=8, w_T=32, chunk=64, conv_k=4)
    inp = make_block_inputs(shape, seed=22)
    _, w = to_device(inp)
    dec = ttcd.Decoder(w, ttcd.BlockParams.from_shape(shape))
    assert dec.check_status() == ttcd.OK
    ttcd.get_device_error()
    assert ttcd.test_bounded_wait(2_000_000, status=dec.state) == ttcd.OK
    assert dec.check_status() == ttcd.ERR_TIMEOUT
    assert dec.check_status() == ttcd.OK and ttcd.get_device_error()[0] == ttcd.OK
