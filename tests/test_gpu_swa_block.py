"""GPU parity of the plain sliding-window block and of stacks with a TTT layer subset.

A layer outside the TTT layer set of an IP-TTCD model (GitHub README "TTCD",
"Model configuration": ttt_layers; window_size is every layer's window, the
teacher window w_T) is a pre-norm block with one sliding window and the static
SwiGLU MLP: ttcd_swa_block_forward.  It is compared with the float64 oracle's
swa_block_forward (max|d|/max|ref| <= 1e-2).  A stack mixing both kinds of
layers (block_stack_forward with ttt_layers) is checked layer by layer: each
layer's oracle input is the GPU's output of the layer before, and IP-TTCD layers
are compared with the oracle's block, plain ones with its plain block.
"""
import numpy as np
import pytest
import torch

from tests.helpers import TOL_OUT, np64, rel_max, to_device
from ttcd_workloads import TINY_F32, BlockShape, make_block_inputs

pytestmark = pytest.mark.gpu

SHAPES = [
    BlockShape("swa_bf16", "bf16", B=2, T=300, d_model=128, n_q_heads=4, n_kv_heads=2,
               head_dim=64, d_ff=256, w_S=16, w_T=64, chunk=128, conv_k=4),
    # hd 128, a window past several 128-key tiles, d and f not multiples of 256
    BlockShape("swa_bf16_hd128", "bf16", B=1, T=1100, d_model=320, n_q_heads=4, n_kv_heads=2,
               head_dim=128, d_ff=448, w_S=64, w_T=500, chunk=256, conv_k=4),
    # a window longer than the sequence: plain causal attention
    BlockShape("swa_bf16_full_causal", "bf16", B=1, T=200, d_model=128, n_q_heads=2, n_kv_heads=2,
               head_dim=64, d_ff=192, w_S=8, w_T=4096, chunk=64, conv_k=2),
    TINY_F32,
]


@pytest.fixture(scope="module")
def ttcd():
    import dual_window_attention_b200 as m
    m.load_library()
    return m


def _oracle_swa(shape, x, w):
    from oracle import ttcd_oracle as orc
    return orc.swa_block_forward(np64(x), {k: np64(v) for k, v in w.items()},
                                 n_q_heads=shape.n_q_heads, n_kv_heads=shape.n_kv_heads,
                                 head_dim=shape.head_dim, window=shape.w_T,
                                 rms_eps=shape.rms_eps, rope_theta=shape.rope_theta)["out"]


def _oracle_ttcd(shape, x, w):
    from oracle import ttcd_oracle as orc
    ww = {k: np64(v) for k, v in w.items()}
    return orc.block_forward(np64(x), ww["beta"], ww, n_q_heads=shape.n_q_heads,
                             n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim,
                             w_S=shape.w_S, w_T=shape.w_T, chunk=shape.chunk,
                             rms_eps=shape.rms_eps, l2_eps=shape.l2_eps,
                             rope_theta=shape.rope_theta)["out"]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_swa_block_parity(ttcd, shape):
    inp = make_block_inputs(shape, seed=21)
    x, w = to_device(inp)
    # the plain block reads none of the fast-weight inputs
    for k in ("w_proj", "conv_T", "conv_S", "beta"):
        w.pop(k)
    p = ttcd.BlockParams.from_shape(shape)
    out, ws = ttcd.swa_block_forward(x, w, p)
    torch.cuda.synchronize()
    assert ttcd.check_device_status(ws) == ttcd.OK
    err = rel_max(out, _oracle_swa(shape, inp["x"], inp["layers"][0]))
    print(f"{shape.name}: out max-rel {err:.2e}")
    assert err <= TOL_OUT


def test_swa_block_equals_ttcd_block_with_one_window_and_no_update(ttcd):
    """Within bf16 rounding: the IP-TTCD block with w_S = w_T and beta = 0 is the plain block."""
    shape = SHAPES[0].with_(w_S=64, w_T=64)
    inp = make_block_inputs(shape, seed=22)
    x, w = to_device(inp)
    p = ttcd.BlockParams.from_shape(shape)
    plain, _ = ttcd.swa_block_forward(x, w, p)
    full, _, _ = ttcd.block_forward(x, torch.zeros_like(w["beta"]), w, p)
    torch.cuda.synchronize()
    assert rel_max(plain, full) <= TOL_OUT


def test_stack_with_ttt_layer_subset(ttcd):
    shape = SHAPES[0].with_(name="stack4", n_layers=4)
    inp = make_block_inputs(shape, seed=23)
    x = inp["x"].cuda()
    layers = [{k: v.cuda() for k, v in lw.items()} for lw in inp["layers"]]
    p = ttcd.BlockParams.from_shape(shape)
    ttt = {1, 3}
    outs = []
    last = ttcd.block_stack_forward(x, layers, p, ttt_layers=ttt,
                                    on_layer=lambda l, o: outs.append(o.cpu()))
    torch.cuda.synchronize()
    assert len(outs) == 4 and torch.equal(last.cpu(), outs[-1])
    for l in range(4):
        x_in = inp["x"] if l == 0 else outs[l - 1]
        ref = (_oracle_ttcd if l in ttt else _oracle_swa)(shape, x_in, inp["layers"][l])
        err = rel_max(outs[l], ref)
        print(f"layer {l} ({'IP-TTCD' if l in ttt else 'plain'}): max-rel {err:.2e}")
        assert err <= TOL_OUT, (l, err)
