"""Host-side exchanges of the sequence-sharded block, on gloo ranks (CPU).

dual_window_attention_b200/sharding.py splits a sequence into shards of whole
chunks and moves what a rank needs from the ranks before it: a halo of rows
(the K/V of the w_T - 1 tokens before a shard, or the conv_k - 1 rows of Z) and
the exclusive prefix of the ranks' state totals.  On a world-size-3 gloo group
every rank checks its halo against the slice of the whole sequence that
precedes its shard (including a halo longer than a shard, which spans two
earlier ranks) and its state prefix against the sum of the lower ranks'
totals.  The decomposition these feed is pinned in test_oracle_sharded.py.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from dual_window_attention_b200.sharding import exchange_halo, shard_bounds, state_prefix

T, CHUNK, WORLD = 23, 2, 3


def _global_tensors():
    g = torch.Generator().manual_seed(0)
    k = torch.randn(2, T, 3, 4, generator=g)       # [B, T, Hkv, hd], like the K/V halo
    z = torch.randn(2, T, 5, generator=g)          # [B, T, f], like the conv halo
    totals = torch.randn(WORLD, 2, 4, 6, generator=g)
    s0 = torch.randn(2, 4, 6, generator=g)
    return k, z, totals, s0


def _rank_main(rank, world, port):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    k, z, totals, s0 = _global_tensors()
    a, e = shard_bounds(T, CHUNK, world, rank)
    for rows in (1, 7, 11, 40):               # 11 and 40 reach past one shard of 8
        halo = exchange_halo(k[:, a:e], rows)
        assert torch.equal(halo, k[:, max(0, a - rows):a]), (rank, rows)
    halo = exchange_halo(z[:, a:e], 3)
    assert torch.equal(halo, z[:, max(0, a - 3):a])
    got = state_prefix(totals[rank], state_in=s0)
    ref = s0.clone()
    for j in range(rank):
        ref += totals[j]
    assert torch.equal(got, ref)
    assert torch.equal(state_prefix(totals[rank]), sum((totals[j] for j in range(rank)),
                                                        torch.zeros_like(s0)))
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_halo_and_state_prefix_on_three_gloo_ranks():
    mp.start_processes(_rank_main, args=(WORLD, _free_port()), nprocs=WORLD,
                       start_method="spawn", join=True)


@pytest.mark.parametrize("T_,chunk,world", [(23, 2, 3), (37, 5, 2), (5, 8, 3), (64, 8, 8)])
def test_shard_bounds_cover_the_sequence_in_whole_chunks(T_, chunk, world):
    bounds = [shard_bounds(T_, chunk, world, r) for r in range(world)]
    assert bounds[0][0] == 0 and bounds[-1][1] == T_
    n_chunks = (T_ + chunk - 1) // chunk
    sizes = []
    for (a, e), (a2, _) in zip(bounds, bounds[1:] + [(T_, T_)]):
        assert e == a2 and a <= e and (a % chunk == 0 or a == e == T_)  # empty shards sit at T
        sizes.append((min(e, n_chunks * chunk) - a + chunk - 1) // chunk)
    assert sum(sizes) == n_chunks and max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_bounds(T_, chunk, world, world)
