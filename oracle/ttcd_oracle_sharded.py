"""Sequence-sharded form of the block forward (test infrastructure only).

TEST INFRASTRUCTURE ONLY, like ``ttcd_oracle``: only ``tests/`` may import it.

A sequence-parallel implementation splits the tokens of each sequence into
contiguous shards of whole chunks, one per rank.  The block is causal, so a
shard needs from the shards before it only:

  - the rotated keys and values of the w_T - 1 tokens before its first token
    (the teacher window's reach; the student window lies inside it), R1;
  - the SwiGLU activations Z_T, Z_S of the conv_k - 1 tokens before it (the
    short convs' reach; no reset at chunk edges), R9;
  - the sum of the earlier shards' chunk increments, which is its state_in:
    the exclusive prefix over chunks (R6) taken over shards first.
    ([REVIEW] 整体框架 and 关键设计 2: a causal prefix over chunks.)

``shard_forward`` computes one rank's part of the block that way, from the
forward oracle's own steps; the only new operations are slicing, concatenation
and the sum of the gathered shard totals.  The exchanges go through
``ex.all_gather(array)``, which returns every rank's array in rank order (a
torch.distributed all-gather, or anything with the same meaning), so the same
function runs on gloo ranks in the tests.  It is pinned by equality with
``block_forward`` on the whole sequence.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from .ttcd_oracle import (causal_depthwise_conv, chunk_increments, dual_window_attention,
                          exclusive_prefix, l2_normalize_rows, qkv_projection, rms_norm, rope,
                          swiglu, value_residual)


def _rope_from(x, theta: float, pos0: int):
    """RoPE at absolute positions pos0 .. pos0 + n - 1: the oracle's rope over a
    sequence padded with pos0 leading rows, keeping the last n rows."""
    pad = np.zeros((x.shape[0], pos0) + x.shape[2:])
    return rope(np.concatenate([pad, x], axis=1), theta)[:, pos0:]


def shard_forward(x, beta, weights: Dict[str, np.ndarray], *, start: int, ex,
                  n_q_heads: int, n_kv_heads: int, head_dim: int, w_S: int, w_T: int,
                  chunk: int, rms_eps: float = 1e-6, l2_eps: float = 1e-6,
                  rope_theta: float = 1e4, softmax_scale: Optional[float] = None,
                  state_in=None):
    """One rank's part of the block forward.

    x [B, n, d], beta [B, n]: tokens start .. start + n - 1 of every sequence;
    start must be a multiple of chunk (shards own whole chunks; only the last
    shard may end in a partial chunk).  Ranks hold consecutive shards in rank
    order.  Returns (out [B, n, d], state after this shard's tokens [B, d, f]);
    the last rank's state is the block's state_out.
    """
    if start % chunk:
        raise ValueError("a shard must start at a chunk boundary")
    x = np.asarray(x, np.float64)
    W = {k: np.asarray(v, np.float64) for k, v in weights.items() if k != "beta"}
    Hq, Hkv, hd = n_q_heads, n_kv_heads, head_dim
    scale = softmax_scale if softmax_scale else 1.0 / np.sqrt(hd)
    B, n, d = x.shape
    f = W["w_down"].shape[1]
    conv_k = W["conv_T"].shape[1]

    # S0 on this shard's tokens, RoPE at their absolute positions
    xn = rms_norm(x, W["g_attn"], rms_eps)
    q, k, v = qkv_projection(xn, W["w_qkv"], Hq, Hkv, hd)
    q = _rope_from(q, rope_theta, start)
    k = _rope_from(k, rope_theta, start)

    # K/V halo: the w_T - 1 tokens before this shard, from the earlier shards
    h0 = max(0, start - (w_T - 1))
    k_seq = np.concatenate(ex.all_gather(k), axis=1)
    v_seq = np.concatenate(ex.all_gather(v), axis=1)
    k_ext, v_ext = k_seq[:, h0:start + n], v_seq[:, h0:start + n]
    halo = start - h0
    # queries of the halo rows are not needed: their outputs are dropped
    q_ext = np.concatenate([np.zeros((B, halo, Hq, hd)), q], axis=1)
    o_T, o_S, _, _ = dual_window_attention(q_ext, k_ext, v_ext, w_S, w_T, scale)
    o_T, o_S = o_T[:, halo:], o_S[:, halo:]

    # o_proj, residual, MLP RMSNorm, SwiGLU with the slow weights
    h_T = x + o_T.reshape(B, n, Hq * hd) @ W["w_o"].T
    h_S = x + o_S.reshape(B, n, Hq * hd) @ W["w_o"].T
    Z_T = swiglu(rms_norm(h_T, W["g_mlp"], rms_eps), W["w_gate"], W["w_up"])
    Z_S = swiglu(rms_norm(h_S, W["g_mlp"], rms_eps), W["w_gate"], W["w_up"])

    # conv halo: the conv_k - 1 rows of Z before this shard
    c0 = max(0, start - (conv_k - 1))
    zt_seq = np.concatenate(ex.all_gather(Z_T), axis=1)
    zs_seq = np.concatenate(ex.all_gather(Z_S), axis=1)
    zb_T = causal_depthwise_conv(np.concatenate([zt_seq[:, c0:start], Z_T], axis=1),
                                 W["conv_T"])[:, start - c0:]
    zb_S = causal_depthwise_conv(np.concatenate([zs_seq[:, c0:start], Z_S], axis=1),
                                 W["conv_S"])[:, start - c0:]

    # value residual, keys, this shard's chunk increments
    r = value_residual(zb_T, zb_S, W["w_down"], W["w_proj"])
    key = l2_normalize_rows(zb_S, l2_eps)
    inc = chunk_increments(r, key, beta, chunk)

    # state_in of this shard: state_in + the earlier shards' totals, in rank order
    totals = ex.all_gather(inc.sum(axis=1))
    rank = ex.rank
    s_in = np.zeros((B, d, f)) if state_in is None else np.array(state_in, np.float64)
    for j in range(rank):
        s_in = s_in + totals[j]
    prefixes, s_out = exclusive_prefix(inc, s_in)

    # read with the fast weight of each chunk
    y = np.zeros((B, n, d))
    for b in range(B):
        for i in range(prefixes.shape[1]):
            s0, s1 = i * chunk, min(n, (i + 1) * chunk)
            y[b, s0:s1] = Z_S[b, s0:s1] @ (W["w_down"] + prefixes[b, i]).T
    return h_S + y, s_out
