"""Host-side exchanges of a sequence-sharded block (one rank per GPU).

A sequence-parallel run splits every sequence into contiguous shards of whole
chunks, one per rank, in rank order.  The block is causal, so a rank needs
three things from the ranks before it (papernotes.org review "Learning What
to Remember", 整体框架: windowed attention over earlier tokens, causal short
convs, a causal prefix over chunks):

- the rotated K and V of the w_T - 1 tokens before its first token;
- the conv_k - 1 rows of Z_T and Z_S before its first token;
- the sum of the earlier ranks' chunk increments, which is its state_in.

This module moves those with torch.distributed (NCCL between GPUs, gloo on the
CPU); it does no arithmetic of the method beyond summing the gathered state
totals in rank order.  ``shard_block_forward`` runs one rank's shard through
the library's four shard phases (ttcd_shard_qkv, _attend, _mix, _finish) with
these exchanges between them.  The conv history travels as the earlier
tokens' MLP inputs u (the library recomputes their Z), so no phase waits on a
kernel of another rank that has not started.  Halos are copied into this
rank's own memory (send/recv) before any kernel reads them.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


def shard_bounds(T: int, chunk: int, world: int, rank: int) -> Tuple[int, int]:
    """Token range [start, end) of `rank`: whole chunks, split as evenly as
    possible (the first T_chunks % world ranks take one chunk more); only the
    last rank can end in a partial chunk."""
    if T < 1 or chunk < 1 or not 0 <= rank < world:
        raise ValueError("need T >= 1, chunk >= 1 and 0 <= rank < world")
    n = (T + chunk - 1) // chunk
    base, extra = divmod(n, world)
    c0 = rank * base + min(rank, extra)
    c1 = c0 + base + (1 if rank < extra else 0)
    return min(T, c0 * chunk), min(T, c1 * chunk)


def exchange_halo(local: torch.Tensor, rows: int, dim: int = 1,
                  group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """The `rows` rows (along `dim`) that precede this rank's first row in the
    concatenation of all ranks' `local` tensors in rank order; fewer at the
    start of the sequence.

    The halo passes down the ranks as a chain: rank r receives its halo from
    rank r - 1, then sends rank r + 1 the last `rows` rows of (halo, local), so
    a halo may span several earlier ranks.  Every rank's `local` must have the
    same shape except along `dim`; the row counts travel ahead of the data.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    local = local.contiguous()
    empty_shape = list(local.shape)
    empty_shape[dim] = 0
    halo = local.new_empty(empty_shape)
    if rank > 0:
        n = torch.zeros(1, dtype=torch.int64, device=local.device)
        dist.recv(n, src=_global(rank - 1, group), group=group)
        shape = list(local.shape)
        shape[dim] = int(n.item())
        halo = local.new_empty(shape)
        if halo.numel():
            dist.recv(halo, src=_global(rank - 1, group), group=group)
    if rank < world - 1:
        ext = torch.cat([halo, local], dim=dim)
        keep = min(rows, ext.shape[dim])
        out = ext.narrow(dim, ext.shape[dim] - keep, keep).contiguous()
        n = torch.tensor([keep], dtype=torch.int64, device=local.device)
        dist.send(n, dst=_global(rank + 1, group), group=group)
        if out.numel():
            dist.send(out, dst=_global(rank + 1, group), group=group)
    return halo


def state_prefix(total: torch.Tensor, group: Optional[dist.ProcessGroup] = None,
                 state_in: Optional[torch.Tensor] = None) -> torch.Tensor:
    """state_in + the sum of the lower ranks' `total` (each rank's sum of its
    chunk increments, fp32 [B, d, f]), added in rank order: the exclusive
    prefix over chunks taken over ranks.  One all-gather."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    parts = [torch.empty_like(total) for _ in range(world)]
    dist.all_gather(parts, total.contiguous(), group=group)
    acc = torch.zeros_like(total) if state_in is None else state_in.clone()
    for j in range(rank):
        acc += parts[j]
    return acc


def _global(group_rank: int, group: Optional[dist.ProcessGroup]) -> int:
    return group_rank if group is None else dist.get_global_rank(group, group_rank)


def shard_block_forward(x: torch.Tensor, beta: torch.Tensor, weights, p, pos0: int,
                        group: Optional[dist.ProcessGroup] = None,
                        state_in: Optional[torch.Tensor] = None, make_shard=None):
    """This rank's shard of a sequence-sharded block forward.

    x [B, T, d], beta [B, T]: tokens pos0 .. pos0 + T - 1 of every sequence
    (``shard_bounds`` gives them), ranks holding consecutive shards in rank
    order; p describes this shard (p.T = T).  Returns (out [B, T, d], state
    after this shard [B, d, f]); the last rank's state is the block's state_out.

    ``make_shard(weights, p, pos0)`` builds the object that runs the four
    phases (default: the CUDA library's ``Shard``); every rank takes the same
    exchange steps in the same order.
    """
    if make_shard is None:
        from . import Shard as make_shard
    sh = make_shard(weights, p, pos0)
    kv_tail = sh.qkv(x)
    kv_halo = exchange_halo(kv_tail, p.w_T - 1, dim=1, group=group)
    u_tail = sh.attend(x, kv_halo)
    u_halo = exchange_halo(u_tail, max(p.conv_k - 1, 0), dim=2, group=group)
    total = sh.mix(beta, u_halo)
    s_in = state_prefix(total, group=group, state_in=state_in)
    return sh.finish(s_in)
