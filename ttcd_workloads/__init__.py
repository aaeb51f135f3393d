"""Seeded synthetic workloads for the IP-TTCD block forward.

This module holds the workload shapes and the seeded input generators that both
the CUDA path (tests, bench) and the CPU oracle consume.  It holds none of the
method's arithmetic: it only draws random numbers and rounds them to the
storage type.

Shapes follow the layer shapes the pages name (Qwen3-0.6B and SmolLM2-360M
continued training at 64K context; GitHub README "TTCD: Test-Time Training via
Context Distillation", section "Continued training (CT) pipeline").  No
dataset, checkpoint or tokenizer is used: every tensor is drawn here.

Recipe (fixed order from one CPU ``torch.Generator`` seeded with ``seed``):

    x ~ N(0, 1)                                   [B, T, d]
    then per layer:
      w_qkv ~ N(0, 1/d)                          [(Hq + 2 Hkv) hd, d]
      w_o   ~ N(0, 1/(Hq hd))                    [d, Hq hd]
      w_gate, w_up ~ N(0, 1/d)                   [f, d]
      w_down ~ N(0, 1/f)                         [d, f]
      w_proj ~ N(0, 1/f)                         [f, f]
      conv_T, conv_S ~ N(0, 0.25)  (variance)    [f, k]
      beta = 0.1 * sigmoid(N(0, 1))              [B, T]
    RMSNorm gains g_attn = g_mlp = 1             [d]

Values are drawn in fp32 and, for bf16 workloads, rounded once to bf16
(round-to-nearest-even); the oracle receives exactly those rounded values.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class BlockShape:
    """Shape and hyper-parameters of one IP-TTCD block (names follow the pages)."""

    name: str
    dtype: str  # "f32" or "bf16": storage/interface type of activations and weights
    B: int
    T: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    d_ff: int
    w_S: int  # student window (keys t-w_S+1 .. t)
    w_T: int  # teacher window (keys t-w_T+1 .. t)
    chunk: int  # fast-weight chunk size C
    conv_k: int  # depthwise causal conv width
    rms_eps: float = 1e-6
    l2_eps: float = 1e-6
    rope_theta: float = 10000.0
    n_layers: int = 1

    @property
    def n_chunks(self) -> int:
        return (self.T + self.chunk - 1) // self.chunk

    @property
    def d_qkv(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    @property
    def softmax_scale(self) -> float:
        return 1.0 / float(self.head_dim) ** 0.5

    def with_(self, **kw) -> "BlockShape":
        return dataclasses.replace(self, **kw)


# The five workloads.  Names state what they are.
TINY_F32 = BlockShape("tiny_fp32_T256", "f32", B=1, T=256, d_model=64, n_q_heads=2,
                      n_kv_heads=1, head_dim=32, d_ff=128, w_S=16, w_T=64, chunk=32,
                      conv_k=4)
SMOLLM2_360M_16K = BlockShape("smollm2_360m_block_T16384", "bf16", B=1, T=16384,
                              d_model=960, n_q_heads=15, n_kv_heads=5, head_dim=64,
                              d_ff=2560, w_S=512, w_T=4096, chunk=512, conv_k=4)
QWEN3_0P6B_64K = BlockShape("qwen3_0.6b_block_T65536", "bf16", B=1, T=65536,
                            d_model=1024, n_q_heads=16, n_kv_heads=8, head_dim=128,
                            d_ff=3072, w_S=512, w_T=8192, chunk=1024, conv_k=4)
# Attention-only sweep at the Qwen3-0.6B head layout.
ATTN_SWEEP_T = 65536
ATTN_SWEEP_W_S = (256, 512, 1024, 2048)
ATTN_SWEEP_W_T = (4096, 8192, 16384)
# 28-layer stack of Qwen3-0.6B-shaped blocks, two batch shapes.
QWEN3_STACK_B1 = QWEN3_0P6B_64K.with_(name="qwen3_0.6b_stack28_B1_T65536", n_layers=28)
QWEN3_STACK_B4 = QWEN3_0P6B_64K.with_(name="qwen3_0.6b_stack28_B4_T16384", B=4, T=16384,
                                      n_layers=28)

ALL_BLOCKS: Dict[str, BlockShape] = {
    s.name: s for s in (TINY_F32, SMOLLM2_360M_16K, QWEN3_0P6B_64K, QWEN3_STACK_B1,
                        QWEN3_STACK_B4)
}


def storage_dtype(shape: BlockShape) -> torch.dtype:
    return torch.float32 if shape.dtype == "f32" else torch.bfloat16


def _normal(g: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def make_layer_weights(shape: BlockShape, g: torch.Generator) -> Dict[str, torch.Tensor]:
    """Draw one layer's weights and beta from ``g`` in the fixed order (fp32 values)."""
    d, f, hd = shape.d_model, shape.d_ff, shape.head_dim
    dq = shape.n_q_heads * hd
    w = {}
    w["w_qkv"] = _normal(g, (shape.d_qkv, d), d ** -0.5)
    w["w_o"] = _normal(g, (d, dq), dq ** -0.5)
    w["w_gate"] = _normal(g, (f, d), d ** -0.5)
    w["w_up"] = _normal(g, (f, d), d ** -0.5)
    w["w_down"] = _normal(g, (d, f), f ** -0.5)
    w["w_proj"] = _normal(g, (f, f), f ** -0.5)
    w["conv_T"] = _normal(g, (f, shape.conv_k), 0.5)
    w["conv_S"] = _normal(g, (f, shape.conv_k), 0.5)
    noise = torch.randn(shape.B, shape.T, generator=g, dtype=torch.float32)
    w["beta"] = 0.1 * torch.sigmoid(noise)
    w["g_attn"] = torch.ones(d, dtype=torch.float32)
    w["g_mlp"] = torch.ones(d, dtype=torch.float32)
    return w


def round_to_storage(t: torch.Tensor, shape: BlockShape, keep_f32: bool = False) -> torch.Tensor:
    if keep_f32 or shape.dtype == "f32":
        return t.float().contiguous()
    return t.to(torch.bfloat16).contiguous()


# beta, gains and conv taps: beta stays fp32 at the interface (a per-token
# coefficient, like the fp32 fast-weight state); conv taps and gains are stored
# in the activation type.
_F32_KEYS = ("beta",)


def make_block_inputs(shape: BlockShape, seed: int = 0) -> Dict[str, object]:
    """Seeded inputs for ``shape``: ``x`` plus a list of per-layer weight dicts.

    Every tensor is on the CPU in its storage type (bf16 or fp32).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = _normal(g, (shape.B, shape.T, shape.d_model), 1.0)
    layers: List[Dict[str, torch.Tensor]] = []
    for _ in range(shape.n_layers):
        w = make_layer_weights(shape, g)
        layers.append({k: round_to_storage(v, shape, keep_f32=(k in _F32_KEYS))
                       for k, v in w.items()})
    return {"x": round_to_storage(x, shape), "layers": layers}


def make_attention_inputs(B: int, T: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                          seed: int = 0, dtype: torch.dtype = torch.bfloat16):
    """Q, K, V ~ N(0, 1) in [B, T, H, hd] layout, rounded to ``dtype``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn(B, T, n_q_heads, head_dim, generator=g, dtype=torch.float32)
    k = torch.randn(B, T, n_kv_heads, head_dim, generator=g, dtype=torch.float32)
    v = torch.randn(B, T, n_kv_heads, head_dim, generator=g, dtype=torch.float32)
    return q.to(dtype).contiguous(), k.to(dtype).contiguous(), v.to(dtype).contiguous()


def make_mlp_inputs(shape: BlockShape, seed: int = 0) -> Dict[str, torch.Tensor]:
    """Inputs of the fast-weight MLP alone: post-norm u_T, u_S, residual h_S, weights, beta.

    u_T = u_S + 0.25 * N(0, 1) so that the teacher and the student differ by a
    fraction of their size, as two attention windows over the same sequence do.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    B, T, d = shape.B, shape.T, shape.d_model
    u_S = _normal(g, (B, T, d), 1.0)
    u_T = u_S + _normal(g, (B, T, d), 0.25)
    h_S = _normal(g, (B, T, d), 1.0)
    w = make_layer_weights(shape, g)
    out = {"u_T": u_T, "u_S": u_S, "h_S": h_S}
    out.update(w)
    return {k: round_to_storage(v, shape, keep_f32=(k in _F32_KEYS)) for k, v in out.items()}
