"""Shared test utilities: error measures and oracle invocation on seeded inputs."""
import numpy as np
import torch

# Tolerances of the block forward: bf16 (and fp32-interface) outputs
# max|d|/max|ref| <= 1e-2; the fp32 fast-weight state relative Frobenius <= 5e-3.
TOL_OUT = 1e-2
TOL_STATE = 5e-3


def np64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().double().numpy() if t.dtype == torch.bfloat16 else \
            t.detach().cpu().double().numpy()
    return np.asarray(t, np.float64)


def rel_max(got, ref) -> float:
    got, ref = np64(got), np64(ref)
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def rel_fro(got, ref) -> float:
    got, ref = np64(got), np64(ref)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))


def oracle_block(shape, inp, layer=0, T=None):
    """Run the oracle block forward on the seeded inputs (optionally a prefix of T tokens)."""
    from oracle import ttcd_oracle as orc
    w = {k: np64(v) for k, v in inp["layers"][layer].items()}
    x = np64(inp["x"])
    beta = w["beta"]
    if T is not None:
        x, beta = x[:, :T], beta[:, :T]
    return orc.block_forward(x, beta, w, n_q_heads=shape.n_q_heads, n_kv_heads=shape.n_kv_heads,
                             head_dim=shape.head_dim, w_S=shape.w_S, w_T=shape.w_T,
                             chunk=shape.chunk, rms_eps=shape.rms_eps, l2_eps=shape.l2_eps,
                             rope_theta=shape.rope_theta)


def to_device(inp, layer=0, device="cuda"):
    w = {k: v.to(device) for k, v in inp["layers"][layer].items()}
    return inp["x"].to(device), w
