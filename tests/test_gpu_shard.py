"""The sequence-sharded block forward on one GPU: shards run one after another
through the library's four shard phases, each receiving from the shards before
it exactly what a rank would receive (the last rows of the K/V and MLP-input
tails passed down the ranks, and the earlier shards' increment totals), so the
data flow is the multi-rank one without ranks that wait on each other.

Definition: papernotes.org review "Learning What to Remember", 整体框架 (causal
windowed attention, causal short convs, a causal prefix over chunks), so the
concatenated shard outputs and the last shard's state equal the block over the
whole sequence.  Checked against the float64 oracle of the whole sequence
(outputs max|d|/max|ref| <= 1e-2, state relative Frobenius <= 5e-3), against the
unsharded library call, and, bit for bit, the rotated K/V each shard exports
against the unsharded call's (RoPE at the shard's absolute positions).
"""
import pytest
import torch

from tests.helpers import TOL_OUT, TOL_STATE, oracle_block, rel_fro, rel_max, to_device
from ttcd_workloads import BlockShape, make_block_inputs

pytestmark = pytest.mark.gpu

# w_T - 1 = 299 is longer than the middle shard (256 tokens): the last shard's
# K/V halo spans two earlier shards.  The last shard ends in a partial chunk.
SHAPE = BlockShape("shard_bf16", "bf16", B=2, T=1000, d_model=128, n_q_heads=4, n_kv_heads=2,
                   head_dim=64, d_ff=256, w_S=64, w_T=300, chunk=128, conv_k=4)
CASES = [
    (SHAPE, [(0, 384), (384, 640), (640, 1000)]),
    (SHAPE.with_(name="shard_chunk96_k3", B=1, T=700, chunk=96, conv_k=3, w_T=500, w_S=100,
                 head_dim=128, n_q_heads=2, n_kv_heads=1), [(0, 192), (192, 480), (480, 700)]),
]


def _chain(prev_halo, prev_tail, rows, dim):
    """What a rank receives: the last `rows` rows of (its predecessor's halo, tail)."""
    if prev_tail is None:
        return None
    ext = prev_tail if prev_halo is None else torch.cat([prev_halo, prev_tail], dim=dim)
    keep = min(rows, ext.shape[dim])
    return ext.narrow(dim, ext.shape[dim] - keep, keep).contiguous()


@pytest.mark.parametrize("shape,bounds", CASES, ids=lambda v: getattr(v, "name", None))
def test_shards_match_the_whole_sequence(shape, bounds):
    import dual_window_attention_b200 as ttcd
    inp = make_block_inputs(shape, seed=31)
    x, w = to_device(inp)
    p = ttcd.BlockParams.from_shape(shape)
    full_out, full_state, full_ws = ttcd.block_forward(x, w["beta"], w, p, state_out=True)
    assert ttcd.check_device_status(full_ws) == ttcd.OK
    BT = shape.B * shape.T
    dqkv = (shape.n_q_heads + 2 * shape.n_kv_heads) * shape.head_dim
    qkv_full = ttcd.workspace_view(full_ws, p, "qkv", torch.bfloat16, (shape.B, shape.T, dqkv))
    kv_cols = slice(shape.n_q_heads * shape.head_dim, dqkv)

    outs, state, totals = [], None, []
    kv_halo = kv_tail = u_halo = u_tail = None
    for r, (s0, s1) in enumerate(bounds):
        ps = ttcd.BlockParams.from_shape(shape.with_(T=s1 - s0))
        sh = ttcd.Shard(w, ps, s0)
        xs = x[:, s0:s1].contiguous()
        kv_halo = _chain(kv_halo, kv_tail, shape.w_T - 1, 1)
        kv_tail = sh.qkv(xs)
        nt = kv_tail.shape[1]
        assert torch.equal(kv_tail, qkv_full[:, s1 - nt:s1, kv_cols]), f"shard {r} K/V"
        u_halo = _chain(u_halo, u_tail, shape.conv_k - 1, 2)
        u_tail = sh.attend(xs, kv_halo)
        total = sh.mix(w["beta"][:, s0:s1].contiguous(), u_halo)
        state_in = None
        for t in totals:  # the earlier shards' totals, in rank order
            state_in = t.clone() if state_in is None else state_in + t
        out, state = sh.finish(state_in)
        totals.append(total)
        assert sh.check_status() == ttcd.OK
        outs.append(out)
    out = torch.cat(outs, dim=1)
    torch.cuda.synchronize()
    ref = oracle_block(shape, inp)
    assert rel_max(out, ref["out"]) <= TOL_OUT
    assert rel_fro(state, ref["state_out"]) <= TOL_STATE
    # the unsharded call is within the tolerance of the same oracle
    assert rel_max(out, full_out) <= 2 * TOL_OUT
    assert rel_fro(state, full_state) <= 2 * TOL_STATE
    assert out.shape == (shape.B, shape.T, shape.d_model) and BT == out.shape[0] * out.shape[1]
