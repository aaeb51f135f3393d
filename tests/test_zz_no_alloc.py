"""ttcd_fastweight_mlp_noalloc: the fast-weight MLP for callers that cannot hand
the library scratch memory (a host framework owning the whole device pool, or a
loop that may not call cudaMalloc).  Its scratch is a fixed array inside the
library, so these checks compare it with ttcd_fastweight_mlp, which takes a
caller workspace, over several calls in a row.  Each call leaves the shared
array holding data of another shape: other sequence lengths, a chunk of 96 whose
padding rows sit where the previous call kept real tokens, an fp32 call and a
sequence shorter than one chunk (the fp32-operand route).  A buffer that a call
read without writing first would carry the previous call's values and fail the
comparison.

This file sorts last so that a run stopping at the first failure has already
run every other test.
"""
import ctypes

import pytest
import torch

from tests.helpers import TOL_OUT, TOL_STATE, rel_fro, rel_max
from ttcd_workloads import BlockShape, make_mlp_inputs

BASE = BlockShape("noalloc_bf16", "bf16", B=2, T=700, d_model=128, n_q_heads=1, n_kv_heads=1,
                  head_dim=64, d_ff=256, w_S=1, w_T=1, chunk=128, conv_k=4)
# Call order: each shape after the first finds the previous one's data in the array.
SEQUENCE = [
    (BASE, 11),
    (BASE.with_(name="noalloc_chunk96", B=1, T=500, chunk=96, conv_k=3), 12),
    (BASE.with_(name="noalloc_f32", dtype="f32", B=1, T=300, chunk=64), 13),
    (BASE.with_(name="noalloc_short", B=1, T=50, chunk=128), 14),
    (BASE, 15),
]


def _lib():
    import dual_window_attention_b200 as ttcd
    return ttcd, ttcd.load_library()


def _call_noalloc(ttcd, lib, dev, p, h_S=True):
    """Direct C-ABI call of ttcd_fastweight_mlp_noalloc."""
    y = torch.empty_like(dev["u_S"])
    state = torch.empty(p.B, p.d_model, p.d_ff, device="cuda", dtype=torch.float32)
    pc, wc = p.c(), ttcd._weights(dev)
    st = lib.ttcd_fastweight_mlp_noalloc(
        dev["u_T"].data_ptr(), dev["u_S"].data_ptr(), dev["h_S"].data_ptr() if h_S else None,
        dev["beta"].data_ptr(), ctypes.byref(wc), ctypes.byref(pc), None, state.data_ptr(),
        y.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == ttcd.OK, ttcd.status_string(st)
    return y, state


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_over_calls_of_other_shapes():
    ttcd, lib = _lib()
    for shape, seed in SEQUENCE:
        p = ttcd.BlockParams.from_shape(shape)
        assert ttcd.fastweight_mlp_workspace_size(p) <= lib.ttcd_fastweight_mlp_noalloc_capacity()
        inp = make_mlp_inputs(shape, seed=seed)
        dev = {k: v.cuda() for k, v in inp.items()}
        y_ref, s_ref, ws = ttcd.fastweight_mlp(dev["u_T"], dev["u_S"], dev["beta"], dev, p,
                                               h_S=dev["h_S"], state_out=True)
        assert ttcd.check_device_status(ws) == ttcd.OK
        y, s = _call_noalloc(ttcd, lib, dev, p)
        torch.cuda.synchronize()
        assert ttcd.get_device_error()[0] == ttcd.OK
        assert rel_max(y, y_ref) <= TOL_OUT, shape.name
        assert rel_fro(s, s_ref) <= TOL_STATE, shape.name


@pytest.mark.gpu
def test_noalloc_python_wrapper():
    """The binding's wrapper: y allocated when not given, state_out=True allocates."""
    ttcd, _ = _lib()
    shape = BASE.with_(name="noalloc_wrapper", T=333)
    p = ttcd.BlockParams.from_shape(shape)
    dev = {k: v.cuda() for k, v in make_mlp_inputs(shape, seed=16).items()}
    y_ref, s_ref, _ = ttcd.fastweight_mlp(dev["u_T"], dev["u_S"], dev["beta"], dev, p,
                                          h_S=dev["h_S"], state_out=True)
    y, s = ttcd.fastweight_mlp_noalloc(dev["u_T"], dev["u_S"], dev["beta"], dev, p,
                                       h_S=dev["h_S"], state_out=True)
    torch.cuda.synchronize()
    assert ttcd.get_device_error()[0] == ttcd.OK
    assert y.shape == dev["u_S"].shape and s.shape == (p.B, p.d_model, p.d_ff)
    assert rel_max(y, y_ref) <= TOL_OUT
    assert rel_fro(s, s_ref) <= TOL_STATE


def test_noalloc_rejects_problems_larger_than_its_scratch():
    ttcd, lib = _lib()
    big = ttcd.BlockParams(B=1, T=65536, d_model=1024, n_q_heads=16, n_kv_heads=8, head_dim=128,
                           d_ff=3072, w_S=512, w_T=8192, chunk=1024)
    assert ttcd.fastweight_mlp_workspace_size(big) > lib.ttcd_fastweight_mlp_noalloc_capacity()
    fake = 1 << 20
    w = ttcd._Weights(*([fake] * 10))
    pc = big.c()
    st = lib.ttcd_fastweight_mlp_noalloc(fake, fake, None, fake, ctypes.byref(w), ctypes.byref(pc),
                                         None, None, fake, None)
    assert st == ttcd.ERR_WORKSPACE
