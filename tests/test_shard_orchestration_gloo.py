"""The orchestration of a sequence-sharded block forward on gloo ranks (CPU).

``sharding.shard_block_forward`` runs one rank's shard through four phases
(QKV; attention with a K/V halo; the MLP up to the shard's increment total,
with the MLP-input halo; the prefix from the earlier shards' totals and the
output), exchanging halos down the ranks and the totals by all-gather between
them.  Here the phases are computed by a stand-in built from the float64
oracle's own steps (the CUDA phases are checked on the GPU in
test_gpu_shard.py), and every rank checks its output rows and its state against
the oracle's block over the whole sequence.  World sizes 2 and 3, with a K/V
halo longer than a shard and a last shard that ends in a partial chunk.

Definition: papernotes.org review "Learning What to Remember", 整体框架 and
关键设计 2-3 (causal windowed attention, causal short convs, causal prefix).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from dual_window_attention_b200.sharding import shard_block_forward, shard_bounds

# shards of 18, 18 and 9 tokens at world 3: the 24-row K/V halo spans two ranks
SHAPE = dict(B=2, T=45, d_model=16, n_q_heads=2, n_kv_heads=1, head_dim=8, d_ff=24, w_S=5,
             w_T=25, chunk=6, conv_k=3)


class _P:
    """The fields of the library's BlockParams that the orchestration reads."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


class OracleShard:
    """The four shard phases from the oracle's steps (float64, torch in and out)."""

    def __init__(self, weights, p, pos0):
        self.w = {k: np.asarray(v, np.float64) for k, v in weights.items()}
        self.p, self.pos0 = p, pos0

    def qkv(self, x):
        from oracle import ttcd_oracle as orc
        p, w = self.p, self.w
        x = x.double().numpy()
        xn = orc.rms_norm(x, w["g_attn"], 1e-6)
        q, k, v = orc.qkv_projection(xn, w["w_qkv"], p.n_q_heads, p.n_kv_heads, p.head_dim)
        pad = lambda a: np.concatenate([np.zeros((a.shape[0], self.pos0) + a.shape[2:]), a], 1)
        self.x = x
        self.q = orc.rope(pad(q), 1e4)[:, self.pos0:]
        self.k = orc.rope(pad(k), 1e4)[:, self.pos0:]
        self.v = v
        kv = np.concatenate([self.k, self.v], axis=2).reshape(x.shape[0], x.shape[1], -1)
        nt = min(p.T, p.w_T - 1)
        return torch.from_numpy(kv[:, p.T - nt:].copy())

    def attend(self, x, kv_halo):
        from oracle import ttcd_oracle as orc
        p, w = self.p, self.w
        B, hd, Hkv, Hq = x.shape[0], p.head_dim, p.n_kv_heads, p.n_q_heads
        nh = 0 if kv_halo is None else kv_halo.shape[1]
        assert nh == min(p.w_T - 1, self.pos0)
        halo = (np.zeros((B, 0, 2 * Hkv, hd)) if nh == 0 else
                kv_halo.double().numpy().reshape(B, nh, 2 * Hkv, hd))
        k_ext = np.concatenate([halo[:, :, :Hkv], self.k], axis=1)
        v_ext = np.concatenate([halo[:, :, Hkv:], self.v], axis=1)
        q_ext = np.concatenate([np.zeros((B, nh, Hq, hd)), self.q], axis=1)
        o_T, o_S, _, _ = orc.dual_window_attention(q_ext, k_ext, v_ext, p.w_S, p.w_T,
                                                   1 / np.sqrt(hd))
        T = p.T
        self.h_T = self.x + o_T[:, nh:].reshape(B, T, -1) @ w["w_o"].T
        self.h_S = self.x + o_S[:, nh:].reshape(B, T, -1) @ w["w_o"].T
        self.u = [orc.rms_norm(h, w["g_mlp"], 1e-6) for h in (self.h_T, self.h_S)]
        n = min(T, p.conv_k - 1)
        return torch.from_numpy(np.stack([u[:, T - n:] for u in self.u]))

    def mix(self, beta, u_halo):
        from oracle import ttcd_oracle as orc
        p, w = self.p, self.w
        nh = 0 if u_halo is None else u_halo.shape[2]
        assert nh == min(p.conv_k - 1, self.pos0)
        Z = [orc.swiglu(u, w["w_gate"], w["w_up"]) for u in self.u]
        zh = [orc.swiglu(u_halo[i].double().numpy(), w["w_gate"], w["w_up"]) if nh else
              np.zeros((Z[0].shape[0], 0, Z[0].shape[2])) for i in range(2)]
        zb_T, zb_S = (orc.causal_depthwise_conv(np.concatenate([zh[i], Z[i]], 1),
                                                w[("conv_T", "conv_S")[i]])[:, nh:]
                      for i in range(2))
        r = orc.value_residual(zb_T, zb_S, w["w_down"], w["w_proj"])
        key = orc.l2_normalize_rows(zb_S, 1e-6)
        self.inc = orc.chunk_increments(r, key, beta.double().numpy(), p.chunk)
        self.Z_S = Z[1]
        return torch.from_numpy(self.inc.sum(axis=1))

    def finish(self, state_in):
        from oracle import ttcd_oracle as orc
        p, w = self.p, self.w
        prefixes, s_out = orc.exclusive_prefix(self.inc, state_in.double().numpy())
        y = np.zeros_like(self.h_S)
        for b in range(y.shape[0]):
            for i in range(prefixes.shape[1]):
                s0, s1 = i * p.chunk, min(p.T, (i + 1) * p.chunk)
                y[b, s0:s1] = self.Z_S[b, s0:s1] @ (w["w_down"] + prefixes[b, i]).T
        return torch.from_numpy(self.h_S + y), torch.from_numpy(s_out)


def _inputs():
    from ttcd_workloads import BlockShape, make_block_inputs
    shape = BlockShape("orchestration", "f32", **SHAPE)
    inp = make_block_inputs(shape, seed=5)
    return shape, inp["x"].double(), {k: v.double() for k, v in inp["layers"][0].items()}


def _rank_main(rank, world, port):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    from oracle import ttcd_oracle as orc
    shape, x, w = _inputs()
    a, e = shard_bounds(shape.T, shape.chunk, world, rank)
    p = _P(**dict(SHAPE, T=e - a))
    out, state = shard_block_forward(x[:, a:e].contiguous(), w["beta"][:, a:e].contiguous(),
                                     {k: v.numpy() for k, v in w.items()}, p, a,
                                     make_shard=OracleShard)
    wn = {k: v.numpy() for k, v in w.items()}
    ref = orc.block_forward(x.numpy(), wn["beta"], wn, n_q_heads=shape.n_q_heads,
                            n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, w_S=shape.w_S,
                            w_T=shape.w_T, chunk=shape.chunk)
    np.testing.assert_allclose(out.numpy(), ref["out"][:, a:e], rtol=0, atol=1e-10)
    if rank == world - 1:
        np.testing.assert_allclose(state.numpy(), ref["state_out"], rtol=0, atol=1e-10)
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_orchestration_equals_the_whole_block(world):
    mp.start_processes(_rank_main, args=(world, _free_port()), nprocs=world,
                       start_method="spawn", join=True)
