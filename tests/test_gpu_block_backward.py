"""GPU parity of ttcd_block_backward against the float64 oracle's
block_backward (pinned by central differences of the block forward and by
library autograd of a plain sliding-window block in test_oracle_grad.py).

papernotes.org review "Learning What to Remember", 方法详解 flowchart A-F and
关键设计 2-3 (the block), 局限与展望 (training differentiates it); podcast cue 51
(W_proj, the convs and the write gate are trained by the next-token loss).

Tolerance: every gradient within relative Frobenius 2e-2 of the oracle's, the
state gradient within 5e-3 (the bounds of the MLP backward, whose chains are
the longest: the attention and RMSNorm steps add one or two bf16 roundings of
dh, dO and dqkv at 2^-9 each, inside the same margin).
"""
import pytest
import torch

from oracle.ttcd_oracle_grad import block_backward as oracle_block_backward
from tests.helpers import np64, rel_fro
from ttcd_workloads import QWEN3_0P6B_64K, BlockShape, make_block_inputs

pytestmark = pytest.mark.gpu

TOL_GRAD = 2e-2
TOL_GRAD_STATE = 5e-3
NAMES = ["x", "beta", "state_in", "w_qkv", "w_o", "g_attn", "g_mlp", "w_gate", "w_up", "w_down",
         "w_proj", "conv_T", "conv_S"]

SHAPES = [
    # two full chunks and a partial one, GQA 2:1, hd 64
    BlockShape("blk_bwd_hd64", "bf16", B=2, T=300, d_model=128, n_q_heads=4, n_kv_heads=2,
               head_dim=64, d_ff=256, w_S=40, w_T=150, chunk=128, conv_k=4),
    # hd 128, GQA 4:1, chunk 96 (padded), conv width 3, teacher window > T
    BlockShape("blk_bwd_hd128", "bf16", B=1, T=260, d_model=256, n_q_heads=4, n_kv_heads=1,
               head_dim=128, d_ff=512, w_S=64, w_T=400, chunk=96, conv_k=3),
]


@pytest.fixture(scope="module")
def ttcd():
    import dual_window_attention_b200 as m
    m.load_library()
    return m


def _case(shape, seed):
    inp = make_block_inputs(shape, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    d_out = torch.randn(shape.B, shape.T, shape.d_model, generator=g).to(torch.bfloat16)
    d_state = 0.1 * torch.randn(shape.B, shape.d_model, shape.d_ff, generator=g)
    state_in = 0.02 * torch.randn(shape.B, shape.d_model, shape.d_ff, generator=g)
    return inp, d_out, d_state, state_in


def _check(ttcd, shape, inp, d_out, d_state, state_in):
    w = {k: v.cuda() for k, v in inp["layers"][0].items()}
    x = inp["x"].cuda()
    p = ttcd.BlockParams.from_shape(shape)
    got, ws = ttcd.block_backward(x, w["beta"], w, p, d_out.cuda(),
                                  state_in=None if state_in is None else state_in.cuda(),
                                  d_state_out=None if d_state is None else d_state.cuda())
    torch.cuda.synchronize()
    assert ttcd.check_device_status(ws) == ttcd.OK
    wn = {k: np64(v) for k, v in inp["layers"][0].items()}
    ref = oracle_block_backward(
        np64(inp["x"]), wn["beta"], wn, np64(d_out), n_q_heads=shape.n_q_heads,
        n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, w_S=shape.w_S, w_T=shape.w_T,
        chunk=shape.chunk, rms_eps=shape.rms_eps, l2_eps=shape.l2_eps,
        rope_theta=shape.rope_theta, state_in=None if state_in is None else np64(state_in),
        d_state_out=None if d_state is None else np64(d_state))
    errs = {k: rel_fro(got[k].cpu(), ref[k]) for k in NAMES}
    print(f"\n{shape.name}: " + ", ".join(f"{k} {v:.2e}" for k, v in errs.items()))
    for k in NAMES:
        assert errs[k] <= (TOL_GRAD_STATE if k == "state_in" else TOL_GRAD), (k, errs[k])


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
@pytest.mark.parametrize("with_state", [False, True], ids=["zero_state", "state"])
def test_block_backward_parity(ttcd, shape, with_state):
    inp, d_out, d_state, state_in = _case(shape, seed=11)
    if not with_state:
        d_state, state_in = None, None
    _check(ttcd, shape, inp, d_out, d_state, state_in)


def test_block_backward_qwen3_shape(ttcd):
    """The Qwen3-0.6B-shaped block (d 1024, 16/8 heads of 128, f 3072, C 1024,
    w_S 512, w_T 8192) over one full chunk and a partial one of 76 tokens."""
    shape = QWEN3_0P6B_64K.with_(name="block_bwd_qwen3_T1100", T=1100)
    inp, d_out, d_state, state_in = _case(shape, seed=13)
    _check(ttcd, shape, inp, d_out, d_state, state_in)
