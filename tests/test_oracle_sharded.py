"""The sequence-sharded decomposition of the block forward (CPU, gloo ranks).

oracle/ttcd_oracle_sharded.py computes each rank's shard of whole chunks from
its own tokens plus three things from earlier shards: the rotated K/V of the
w_T - 1 tokens before it, the conv_k - 1 rows of Z_T and Z_S before it, and
the sum of the earlier shards' chunk increments as its state_in.  Run on
world-size 2 and 3 gloo process groups, the ranks' outputs, concatenated, and
the last rank's state must equal the unsharded block_forward (the block is
causal, so this is exact up to rounding).  One case makes the last shard's
K/V halo span two earlier shards; the last chunk is partial in every case.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from oracle import ttcd_oracle as orc
from oracle.ttcd_oracle_sharded import shard_forward

B, T, D, F, K = 2, 37, 8, 12, 3           # 8 chunks of 5, the last one of 2 tokens
HQ, HKV, HD, CHUNK = 4, 2, 4, 5


def _case(seed=0):
    rng = np.random.default_rng(seed)
    w = {
        "w_qkv": rng.standard_normal(((HQ + 2 * HKV) * HD, D)) / np.sqrt(D),
        "w_o": rng.standard_normal((D, HQ * HD)) / np.sqrt(HQ * HD),
        "g_attn": 0.5 + rng.random(D),
        "g_mlp": 0.5 + rng.random(D),
        "w_gate": rng.standard_normal((F, D)) / np.sqrt(D),
        "w_up": rng.standard_normal((F, D)) / np.sqrt(D),
        "w_down": rng.standard_normal((D, F)) / np.sqrt(F),
        "w_proj": rng.standard_normal((F, F)) / np.sqrt(F),
        "conv_T": rng.standard_normal((F, K)) * 0.5,
        "conv_S": rng.standard_normal((F, K)) * 0.5,
    }
    x = rng.standard_normal((B, T, D))
    beta = 0.5 / (1 + np.exp(-rng.standard_normal((B, T))))
    state_in = 0.1 * rng.standard_normal((B, D, F))
    return x, beta, w, state_in


def _shards(world):
    """Whole chunks per rank, as even as possible: (start, end) token ranges."""
    n_chunks = (T + CHUNK - 1) // CHUNK
    parts = np.array_split(np.arange(n_chunks), world)
    return [(int(p[0]) * CHUNK, min(T, (int(p[-1]) + 1) * CHUNK)) for p in parts]


class _Solo:
    rank = 0

    @staticmethod
    def all_gather(a):
        return [np.asarray(a)]


class _Gloo:
    def __init__(self, rank, world):
        self.rank, self.world = rank, world

    def all_gather(self, a):
        import torch.distributed as dist
        out = [None] * self.world
        dist.all_gather_object(out, np.asarray(a))
        return out


def _rank_main(rank, world, port, w_T, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    x, beta, w, s0 = _case()
    a, e = _shards(world)[rank]
    out, state = shard_forward(x[:, a:e], beta[:, a:e], w, start=a, ex=_Gloo(rank, world),
                               n_q_heads=HQ, n_kv_heads=HKV, head_dim=HD, w_S=3, w_T=w_T,
                               chunk=CHUNK, state_in=s0)
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), out=out, state=state)
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full(w_T):
    x, beta, w, s0 = _case()
    return orc.block_forward(x, beta, w, n_q_heads=HQ, n_kv_heads=HKV, head_dim=HD, w_S=3,
                             w_T=w_T, chunk=CHUNK, state_in=s0)


@pytest.mark.parametrize("world,w_T", [(2, 12), (3, 20)], ids=["world2_wT12", "world3_wT20"])
def test_sharded_forward_equals_whole_sequence_gloo(world, w_T, tmp_path):
    if world == 3:  # the last shard's K/V halo reaches back over both earlier shards
        (_, _), (a1, e1), (a2, _) = _shards(3)
        assert a2 - (w_T - 1) < a1
    mp.start_processes(_rank_main, args=(world, _free_port(), w_T, str(tmp_path)),
                       nprocs=world, start_method="spawn", join=True)
    res = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    ref = _full(w_T)
    out = np.concatenate([r["out"] for r in res], axis=1)
    np.testing.assert_allclose(out, ref["out"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res[-1]["state"], ref["state_out"], rtol=1e-12, atol=1e-13)


def test_single_shard_is_the_block():
    x, beta, w, s0 = _case()
    out, state = shard_forward(x, beta, w, start=0, ex=_Solo, n_q_heads=HQ, n_kv_heads=HKV,
                               head_dim=HD, w_S=3, w_T=12, chunk=CHUNK, state_in=s0)
    ref = _full(12)
    np.testing.assert_allclose(out, ref["out"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(state, ref["state_out"], rtol=1e-12, atol=1e-13)


def test_shard_must_start_at_a_chunk_boundary():
    x, beta, w, _ = _case()
    with pytest.raises(ValueError):
        shard_forward(x[:, 3:], beta[:, 3:], w, start=3, ex=_Solo, n_q_heads=HQ,
                      n_kv_heads=HKV, head_dim=HD, w_S=3, w_T=12, chunk=CHUNK)
