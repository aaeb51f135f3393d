"""GPU parity of token-by-token decode (ttcd_block_decode) against the
float64 oracle's block forward.

The block is causal (papernotes.org review "Learning What to Remember",
方法详解: windowed attention over earlier tokens, causal short convs, an
exclusive prefix over chunks), so decoding tokens 0..T-1 one at a time must
give the rows of the block forward over those T tokens, and the fast-weight
state after token T-1 must be the forward's state_out (partial last chunk
included).  Tolerances: outputs max|d|/max|ref| <= 1e-2, state relative
Frobenius <= 5e-3.
"""
import pytest
import torch

from tests.helpers import TOL_OUT, TOL_STATE, oracle_block, rel_fro, rel_max, to_device
from ttcd_workloads import BlockShape, make_block_inputs

pytestmark = pytest.mark.gpu

DEC_A = BlockShape("decode_hd64", "bf16", B=2, T=300, d_model=128, n_q_heads=4, n_kv_heads=2,
                   head_dim=64, d_ff=256, w_S=64, w_T=256, chunk=128, conv_k=4)
DEC_B = BlockShape("decode_hd128_chunk96", "bf16", B=1, T=230, d_model=256, n_q_heads=4,
                   n_kv_heads=1, head_dim=128, d_ff=512, w_S=40, w_T=150, chunk=96, conv_k=3)
# nine sequences: 2B = 18 rows take the tensor-core GEMM path instead of the GEMV
DEC_C = DEC_A.with_(name="decode_batch9_gemm_path", B=9, T=150)
# six sequences: the B-row products (QKV, r) on the GEMV, the 2B-row products
# (o_proj, gate/up) on the tensor-core GEMM
DEC_E = DEC_A.with_(name="decode_batch6_mixed_path", B=6, T=140)
# eight query heads per KV head at hd 32, a teacher window of two 256-key splits
DEC_D = BlockShape("decode_hd32_gqa8", "bf16", B=2, T=340, d_model=128, n_q_heads=8,
                   n_kv_heads=1, head_dim=32, d_ff=256, w_S=48, w_T=300, chunk=128, conv_k=4)


@pytest.fixture(scope="module")
def ttcd():
    import dual_window_attention_b200 as m
    m.load_library()
    return m


def _decode_all(ttcd, shape, inp, state_in=None):
    x, w = to_device(inp)
    p = ttcd.BlockParams.from_shape(shape)
    dec = ttcd.Decoder(w, p, state_in=state_in)
    ys = [dec.step(x[:, t].contiguous(), w["beta"][:, t].contiguous()) for t in range(shape.T)]
    assert dec.check_status() == ttcd.OK
    return torch.stack(ys, dim=1), dec.state_out(), x, w, p


@pytest.mark.parametrize("shape", [DEC_A, DEC_B, DEC_C, DEC_D, DEC_E], ids=lambda s: s.name)
def test_decode_matches_block_forward(ttcd, shape):
    inp = make_block_inputs(shape, seed=4)
    y, state, x, w, p = _decode_all(ttcd, shape, inp)
    ref = oracle_block(shape, inp)
    assert rel_max(y, ref["out"]) <= TOL_OUT
    assert rel_fro(state, ref["state_out"]) <= TOL_STATE
    # and the library's own prefill of the same tokens: both are within the
    # tolerance of the oracle, so they agree with each other within twice it
    out, st_pf, _ = ttcd.block_forward(x, w["beta"], w, p, state_out=True)
    torch.cuda.synchronize()
    assert rel_max(y, out) <= 2 * TOL_OUT
    assert rel_fro(state, st_pf) <= 2 * TOL_STATE


def test_decode_with_state_in(ttcd):
    """A nonzero initial fast weight (state_in) is read by chunk 0 and carried on."""
    shape = DEC_A.with_(T=200)
    inp = make_block_inputs(shape, seed=9)
    g = torch.Generator().manual_seed(1)
    s0 = 0.02 * torch.randn(shape.B, shape.d_model, shape.d_ff, generator=g)
    y, state, _, _, _ = _decode_all(ttcd, shape, inp, state_in=s0.cuda())
    from oracle import ttcd_oracle as orc
    from tests.helpers import np64
    wn = {k: np64(v) for k, v in inp["layers"][0].items()}
    ref = orc.block_forward(np64(inp["x"]), wn["beta"], wn, n_q_heads=shape.n_q_heads,
                            n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, w_S=shape.w_S,
                            w_T=shape.w_T, chunk=shape.chunk, state_in=s0.double().numpy())
    assert rel_max(y, ref["out"]) <= TOL_OUT
    assert rel_fro(state, ref["state_out"]) <= TOL_STATE


def test_graph_decode_matches_eager_decode(ttcd):
    """ttcd_block_decode_next_ex replayed from two CUDA graphs, an ordinary
    step without the chunk commit's launches and a commit step at each chunk's
    last token (the position read from the state on the device), gives the
    eager decode's rows and state bit for bit, across chunk commits, and the
    oracle's."""
    shape = DEC_A.with_(name="dec_graph", T=2 * DEC_A.chunk + 37)
    inp = make_block_inputs(shape, seed=9)
    x, w = to_device(inp)
    p = ttcd.BlockParams.from_shape(shape)
    eager = ttcd.Decoder(w, p)
    graph = ttcd.Decoder(w, p, graph=True)
    ye, yg = [], []
    for t in range(shape.T):
        xt, bt = x[:, t].contiguous(), w["beta"][:, t].contiguous()
        ye.append(eager.step(xt, bt))
        yg.append(graph.step(xt, bt))
    assert eager.check_status() == ttcd.OK and graph.check_status() == ttcd.OK
    assert graph.graphs[False] is not None and graph.graphs[True] is not None
    ye, yg = torch.stack(ye, dim=1), torch.stack(yg, dim=1)
    assert torch.equal(ye, yg)
    assert torch.equal(eager.state_out(), graph.state_out())
    ref = oracle_block(shape, inp)
    assert rel_max(yg, ref["out"]) <= TOL_OUT
