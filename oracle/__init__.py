"""CPU float64 oracle of the IP-TTCD block (test infrastructure only).

``ttcd_oracle`` is the forward; ``ttcd_oracle_grad`` is its backward (a
vector-Jacobian product of the same forward) and ``ttcd_oracle_sharded`` its
sequence-sharded decomposition; both are imported explicitly.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
``--impl reference`` legs may import this package.  The CUDA library does not.
"""
from .ttcd_oracle import *  # noqa: F401,F403
from .ttcd_oracle import (block_forward, causal_depthwise_conv, chunk_increments,
                          distillation_loss, dual_window_attention, exclusive_prefix,
                          fastweight_mlp, l2_normalize_rows, qkv_projection, rms_norm,
                          rope, silu, swa_block_forward, swiglu, value_residual, window_mask,
                          windowed_attention, windowed_attention_bruteforce)
