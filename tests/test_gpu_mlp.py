"""GPU parity of ttcd_fastweight_mlp (the in-place fast-weight MLP alone).

papernotes.org review "Learning What to Remember", 关键设计 2-3; podcast cue 29.
Inputs u_T, u_S are drawn directly (teacher = student + noise), so this checks
the MLP path independently of attention, including a nonzero incoming state.
"""
import numpy as np
import pytest
import torch

from oracle import ttcd_oracle as orc
from tests.helpers import TOL_OUT, TOL_STATE, np64, rel_fro, rel_max
from ttcd_workloads import QWEN3_0P6B_64K, BlockShape, make_mlp_inputs

pytestmark = pytest.mark.gpu

MLP_SHAPES = [
    BlockShape("mlp_bf16", "bf16", B=2, T=1100, d_model=192, n_q_heads=1, n_kv_heads=1,
               head_dim=64, d_ff=384, w_S=1, w_T=1, chunk=256, conv_k=4),
    BlockShape("mlp_f32_chunk40", "f32", B=1, T=333, d_model=64, n_q_heads=1, n_kv_heads=1,
               head_dim=64, d_ff=128, w_S=1, w_T=1, chunk=40, conv_k=2),
    # d and f ragged for the chunk scan's 256 x 192 CTA-pair tiles: the last
    # pair of rows has one CTA with 64 valid rows and one with none, the last
    # column tile 64 valid key columns in its first CTA and none in its second
    BlockShape("mlp_bf16_pair_ragged", "bf16", B=2, T=700, d_model=320, n_q_heads=1,
               n_kv_heads=1, head_dim=64, d_ff=448, w_S=1, w_T=1, chunk=192, conv_k=3),
    # bf16 shorter than one chunk: the fp32-operand route
    BlockShape("mlp_bf16_short", "bf16", B=2, T=70, d_model=128, n_q_heads=1, n_kv_heads=1,
               head_dim=64, d_ff=256, w_S=1, w_T=1, chunk=128, conv_k=4),
]


@pytest.fixture(scope="module")
def ttcd():
    import dual_window_attention_b200 as m
    m.load_library()
    return m


@pytest.mark.parametrize("shape", MLP_SHAPES, ids=lambda s: s.name)
@pytest.mark.parametrize("with_state", [False, True])
def test_fastweight_mlp_parity(ttcd, shape, with_state):
    inp = make_mlp_inputs(shape, seed=0)
    dev = {k: v.cuda() for k, v in inp.items()}
    state_in = None
    if with_state:
        g = torch.Generator().manual_seed(5)
        state_in = 0.02 * torch.randn(shape.B, shape.d_model, shape.d_ff, generator=g)
    p = ttcd.BlockParams.from_shape(shape)
    y, state, ws = ttcd.fastweight_mlp(dev["u_T"], dev["u_S"], dev["beta"], dev, p,
                                       h_S=dev["h_S"],
                                       state_in=None if state_in is None else state_in.cuda(),
                                       state_out=True)
    assert ttcd.check_device_status(ws) == ttcd.OK
    n = {k: np64(v) for k, v in inp.items()}
    ref = orc.fastweight_mlp(n["u_T"], n["u_S"], n["beta"], n["w_gate"], n["w_up"], n["w_down"],
                             n["w_proj"], n["conv_T"], n["conv_S"], shape.chunk, shape.l2_eps,
                             h_S=n["h_S"], state_in=None if state_in is None else np64(state_in),
                             keep_prefixes=False)
    assert rel_max(y, ref["out"]) <= TOL_OUT
    assert rel_fro(state, ref["state_out"]) <= TOL_STATE


def test_fastweight_mlp_qwen3_full_length(ttcd):
    """The Qwen3-0.6B-shaped MLP at T = 65536 (d 1024, f 3072, C 1024): all 64
    chunks of the fp32 prefix scan.  Every output row, and the state after the
    last chunk (the quantity most exposed to accumulation drift), against the
    float64 oracle (about 17 GB of host memory and a minute of CPU time)."""
    shape = QWEN3_0P6B_64K
    inp = make_mlp_inputs(shape, seed=0)
    dev = {k: v.cuda() for k, v in inp.items()}
    p = ttcd.BlockParams.from_shape(shape)
    y, state, ws = ttcd.fastweight_mlp(dev["u_T"], dev["u_S"], dev["beta"], dev, p,
                                       h_S=dev["h_S"], state_out=True)
    assert ttcd.check_device_status(ws) == ttcd.OK
    y, state = y.cpu(), state.cpu()
    del dev, ws
    torch.cuda.empty_cache()
    n = {k: np64(v) for k, v in inp.items()}
    del inp
    ref = orc.fastweight_mlp(n["u_T"], n["u_S"], n["beta"], n["w_gate"], n["w_up"], n["w_down"],
                             n["w_proj"], n["conv_T"], n["conv_S"], shape.chunk, shape.l2_eps,
                             h_S=n["h_S"], keep_prefixes=False)
    e_out, e_state = rel_max(y, ref["out"]), rel_fro(state, ref["state_out"])
    print(f"\nqwen3 MLP T=65536: out max-rel {e_out:.2e}, state rel-Frobenius {e_state:.2e}")
    assert e_out <= TOL_OUT
    assert e_state <= TOL_STATE
