"""GPU parity of ttcd_fastweight_mlp_backward against the float64 oracle's
fastweight_mlp_backward (itself pinned by central differences of the MLP
forward in test_oracle_grad.py).

papernotes.org review "Learning What to Remember", 关键设计 2-3 (the write
rule) and 局限与展望 (training the block); podcast cue 51 (W_proj, the convs
and the write gate are trained through the writes).

Tolerance: every gradient within relative Frobenius 2e-2 of the oracle's.  The
GPU contracts bf16 operands with fp32 accumulation; the longest chain from d_y
to a weight gradient rounds to bf16 five times (Z_S or u, the per-chunk G_i,
the row gradients dRt and s dRt, dM or [da | db]), each a relative 2^-9
(3.9e-3 worst case, about 2.3e-3 rms for a uniformly distributed rounding), so
the rms error of a product of five such roundings is about sqrt(5) x 2.3e-3 =
5e-3 and the bound leaves a factor 4 for cancellation in the sums.  The read
path's gradients (state_in, and u_S through W_down + S_i) pass two roundings and
are held to 5e-3.
"""
import numpy as np
import pytest
import torch

from oracle.ttcd_oracle_grad import fastweight_mlp_backward as oracle_mlp_backward
from tests.helpers import np64, rel_fro
from ttcd_workloads import QWEN3_0P6B_64K, BlockShape, make_mlp_inputs

pytestmark = pytest.mark.gpu

TOL_GRAD = 2e-2
TOL_GRAD_READ = 5e-3
NAMES = ["u_T", "u_S", "beta", "state_in", "w_gate", "w_up", "w_down", "w_proj", "conv_T",
         "conv_S"]

SHAPES = [
    # four full chunks and a partial one (1100 = 4 x 256 + 76)
    BlockShape("bwd_partial_chunk", "bf16", B=2, T=1100, d_model=192, n_q_heads=1, n_kv_heads=1,
               head_dim=64, d_ff=384, w_S=1, w_T=1, chunk=256, conv_k=4),
    # a chunk that is not a multiple of 64 (padded to 128) and conv width 3
    BlockShape("bwd_chunk96_k3", "bf16", B=1, T=500, d_model=128, n_q_heads=1, n_kv_heads=1,
               head_dim=64, d_ff=256, w_S=1, w_T=1, chunk=96, conv_k=3),
    # the widest conv, three sequences
    BlockShape("bwd_k8_B3", "bf16", B=3, T=300, d_model=128, n_q_heads=1, n_kv_heads=1,
               head_dim=64, d_ff=320, w_S=1, w_T=1, chunk=128, conv_k=8),
    # shorter than one chunk
    BlockShape("bwd_short", "bf16", B=2, T=70, d_model=128, n_q_heads=1, n_kv_heads=1,
               head_dim=64, d_ff=256, w_S=1, w_T=1, chunk=128, conv_k=4),
]


@pytest.fixture(scope="module")
def ttcd():
    import dual_window_attention_b200 as m
    m.load_library()
    return m


def _grad_inputs(shape, seed):
    g = torch.Generator().manual_seed(seed)
    d_y = torch.randn(shape.B, shape.T, shape.d_model, generator=g).to(torch.bfloat16)
    d_state = 0.1 * torch.randn(shape.B, shape.d_model, shape.d_ff, generator=g)
    state_in = 0.02 * torch.randn(shape.B, shape.d_model, shape.d_ff, generator=g)
    return d_y, d_state, state_in


def _run(ttcd, shape, inp, d_y, d_state, state_in, beta=None):
    dev = {k: v.cuda() for k, v in inp.items()}
    beta = dev["beta"] if beta is None else beta.cuda()
    p = ttcd.BlockParams.from_shape(shape)
    g, ws = ttcd.fastweight_mlp_backward(
        dev["u_T"], dev["u_S"], beta, dev, p, d_y.cuda(),
        state_in=None if state_in is None else state_in.cuda(),
        d_state_out=None if d_state is None else d_state.cuda())
    torch.cuda.synchronize()
    assert ttcd.check_device_status(ws) == ttcd.OK
    return {k: v.cpu() for k, v in g.items()}


def _oracle(shape, inp, d_y, d_state, state_in, beta=None):
    n = {k: np64(v) for k, v in inp.items()}
    return oracle_mlp_backward(
        n["u_T"], n["u_S"], n["beta"] if beta is None else np64(beta), n["w_gate"], n["w_up"],
        n["w_down"], n["w_proj"], n["conv_T"], n["conv_S"], shape.chunk, shape.l2_eps, np64(d_y),
        state_in=None if state_in is None else np64(state_in),
        d_state_out=None if d_state is None else np64(d_state))


def _check(got, ref, tag):
    errs = {k: rel_fro(got[k], ref[k]) for k in NAMES}
    print(f"\n{tag}: " + ", ".join(f"{k} {v:.2e}" for k, v in errs.items()))
    for k in NAMES:
        tol = TOL_GRAD_READ if k == "state_in" else TOL_GRAD
        assert errs[k] <= tol, (k, errs[k])


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
@pytest.mark.parametrize("with_state", [False, True], ids=["zero_state", "state"])
def test_mlp_backward_parity(ttcd, shape, with_state):
    inp = make_mlp_inputs(shape, seed=1)
    d_y, d_state, state_in = _grad_inputs(shape, seed=2)
    if not with_state:
        d_state, state_in = None, None
    got = _run(ttcd, shape, inp, d_y, d_state, state_in)
    ref = _oracle(shape, inp, d_y, d_state, state_in)
    _check(got, ref, f"{shape.name} {'state' if with_state else 'zero state'}")


def test_mlp_backward_without_writes_leaves_the_write_path_at_zero(ttcd):
    """beta = 0: nothing is written, so W_proj and the two convs, whose only
    route to the loss is the fast-weight write, get exactly zero (the review's
    关键设计 3: Delta W = beta R K^T); the read path still gets its gradients."""
    shape = SHAPES[0]
    inp = make_mlp_inputs(shape, seed=3)
    d_y, _, _ = _grad_inputs(shape, seed=4)
    beta0 = torch.zeros(shape.B, shape.T)
    got = _run(ttcd, shape, inp, d_y, None, None, beta=beta0)
    for k in ("w_proj", "conv_T", "conv_S"):
        assert torch.count_nonzero(got[k]) == 0, k
    ref = _oracle(shape, inp, d_y, None, None, beta=beta0)
    assert rel_fro(got["state_in"], ref["state_in"]) <= TOL_GRAD_READ
    for k in ("u_S", "w_down", "beta"):
        assert rel_fro(got[k], ref[k]) <= TOL_GRAD, k


def test_mlp_backward_qwen3_shape(ttcd):
    """The Qwen3-0.6B-shaped MLP (d 1024, f 3072, C 1024, k 4) over two full
    chunks and a partial one of 100 tokens: every gradient against the oracle."""
    shape = QWEN3_0P6B_64K.with_(name="mlp_bwd_qwen3_T2148", T=2148)
    inp = make_mlp_inputs(shape, seed=5)
    d_y, d_state, state_in = _grad_inputs(shape, seed=6)
    got = _run(ttcd, shape, inp, d_y, d_state, state_in)
    ref = _oracle(shape, inp, d_y, d_state, state_in)
    _check(got, ref, shape.name)
