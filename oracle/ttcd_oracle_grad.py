"""CPU float64 oracle of the IP-TTCD block backward (a vector-Jacobian product).

TEST INFRASTRUCTURE ONLY, like ``ttcd_oracle``: only ``tests/`` may import it.
It shares no code with the CUDA path; it reuses the forward oracle for the
forward values it differentiates.

What it computes: for any scalar outer loss L whose gradients with respect
to the block's output ``out`` [B, T, d] and final state ``state_out``
[B, d, f] are given (G_out, G_state), the gradients of L with respect to the
block's inputs x, beta, state_in and every weight.  It differentiates the
forward exactly as the forward oracle defines it (readings R1-R13 there), by
the chain rule of each step taken in the reverse of the forward's order:
no fusion and no reordering beyond that.

Readings (sources as in ``ttcd_oracle``):
  G1 The outer gradient flows through every step as written, the write path
     included: R, the keys and beta depend on the slow weights, W_proj and the
     two short convs, and those are trained by the ordinary next-token loss
     ([PODCAST] cue 51; [REVIEW] 关键设计 3 writes the update as a closed-form
     function of them).  The stopgrad of Eq. 4 belongs to the derivation of
     the write rule (the inner loss), not to the outer graph
     ([REVIEW] 关键设计 1, [PODCAST] cue 23).
  G2 The off-policy form stands in the backward too: Z_T and Z_S depend on the
     slow weights only, never on the evolving fast weight ([REVIEW] 关键设计 2).

Pins (tests/test_oracle_grad.py): central finite differences of the forward
oracle along random directions for every input, exact zeros where an input
cannot reach the loss, and reduction to torch autograd of a plain
sliding-window block (library SDPA, rms_norm, silu) when the two windows and
the two convs coincide.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from .ttcd_oracle import block_forward, fastweight_mlp, rms_norm, silu, window_mask

# ---------------------------------------------------------------------------
# One vector-Jacobian product per forward step
# ---------------------------------------------------------------------------


def rms_norm_vjp(x, g, eps: float, dy):
    """y = x r g with r = (mean(x^2) + eps)^(-1/2) over the last axis.

    dx = r (dy g - xhat mean(dy g xhat)), xhat = x r;  dg = sum over rows of dy xhat.
    """
    x = np.asarray(x, np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    xhat = x * r
    dxhat = dy * np.asarray(g, np.float64)
    dx = r * (dxhat - xhat * np.mean(dxhat * xhat, axis=-1, keepdims=True))
    dg = np.sum((dy * xhat).reshape(-1, x.shape[-1]), axis=0)
    return dx, dg


def rope_vjp(dy, theta: float):
    """The rotate-half RoPE is a rotation per pair (x_i, x_{i+hd/2}) by angle
    t theta^(-2i/hd); its transpose rotates the gradient back by the same angle."""
    B, T, H, hd = dy.shape
    half = hd // 2
    inv_freq = theta ** (-(np.arange(half, dtype=np.float64) * 2.0) / hd)
    ang = np.arange(T, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos = np.cos(ang)[None, :, None, :]
    sin = np.sin(ang)[None, :, None, :]
    d1, d2 = dy[..., :half], dy[..., half:]
    return np.concatenate([d1 * cos + d2 * sin, d2 * cos - d1 * sin], axis=-1)


def silu_grad(a):
    s = 1.0 / (1.0 + np.exp(-a))
    return s * (1.0 + a * (1.0 - s))


def swiglu_vjp(u, w_gate, w_up, dZ):
    """Z = silu(a) * b, a = u W_gate^T, b = u W_up^T.  Returns (du, dW_gate, dW_up)."""
    u = np.asarray(u, np.float64)
    wg = np.asarray(w_gate, np.float64)
    wu = np.asarray(w_up, np.float64)
    a = u @ wg.T
    b = u @ wu.T
    da = dZ * b * silu_grad(a)
    db = dZ * silu(a)
    du = da @ wg + db @ wu
    dwg = np.einsum("btf,btd->fd", da, u)
    dwu = np.einsum("btf,btd->fd", db, u)
    return du, dwg, dwu


def causal_depthwise_conv_vjp(z, taps, dzbar):
    """zbar[b, t, c] = sum_m taps[c, m] z[b, t - m, c] (zero before t = 0).

    dz[b, s, c] = sum_m taps[c, m] dzbar[b, s + m, c];
    dtaps[c, m] = sum_{b, t} dzbar[b, t, c] z[b, t - m, c].
    """
    z = np.asarray(z, np.float64)
    taps = np.asarray(taps, np.float64)
    T = z.shape[1]
    dz = np.zeros_like(z)
    dtaps = np.zeros_like(taps)
    for m in range(taps.shape[1]):
        if m >= T:
            break
        dz[:, :T - m, :] += taps[:, m][None, None, :] * dzbar[:, m:, :]
        dtaps[:, m] = np.sum(dzbar[:, m:, :] * z[:, :T - m, :], axis=(0, 1))
    return dz, dtaps


def l2_normalize_rows_vjp(z, eps: float, dk):
    """k = z n^(-1/2), n = ||z||^2 + eps:  dz = n^(-1/2) (dk - k <k, dk>)."""
    z = np.asarray(z, np.float64)
    inv = 1.0 / np.sqrt(np.sum(z * z, axis=-1, keepdims=True) + eps)
    k = z * inv
    return inv * (dk - k * np.sum(k * dk, axis=-1, keepdims=True))


def value_residual_vjp(D, w_down, w_proj, dR):
    """R = (D W_proj^T) W_down^T (reading R12: W_proj first).

    Returns (dD, dW_down, dW_proj)."""
    D = np.asarray(D, np.float64)
    wd = np.asarray(w_down, np.float64)
    wp = np.asarray(w_proj, np.float64)
    E = D @ wp.T
    dE = dR @ wd
    dwd = np.einsum("btd,btf->df", dR, E)
    dD = dE @ wp
    dwp = np.einsum("btf,btg->fg", dE, D)
    return dD, dwd, dwp


def chunk_increments_vjp(r, key, beta, chunk: int, d_inc):
    """Delta W_i = sum_{t in C_i} beta_t r_t k_t^T.

    dr_t = beta_t dDeltaW_i k_t;  dk_t = beta_t dDeltaW_i^T r_t;
    dbeta_t = r_t^T dDeltaW_i k_t.
    """
    r = np.asarray(r, np.float64)
    key = np.asarray(key, np.float64)
    beta = np.asarray(beta, np.float64)
    B, T, _ = r.shape
    dr = np.zeros_like(r)
    dk = np.zeros_like(key)
    dbeta = np.zeros_like(beta)
    for b in range(B):
        for i in range(d_inc.shape[1]):
            s0, s1 = i * chunk, min(T, (i + 1) * chunk)
            G = d_inc[b, i]                       # [d, f]
            rk = key[b, s0:s1] @ G.T              # rows: G k_t, [len, d]
            dr[b, s0:s1] = beta[b, s0:s1, None] * rk
            dk[b, s0:s1] = beta[b, s0:s1, None] * (r[b, s0:s1] @ G)
            dbeta[b, s0:s1] = np.sum(r[b, s0:s1] * rk, axis=-1)
    return dr, dk, dbeta


def exclusive_prefix_vjp(d_prefixes, d_state_out):
    """S_i = S_0 + sum_{j<i} Delta W_j and S_n = S_0 + sum_j Delta W_j (reading R6).

    dDelta W_j = dS_n + sum_{i>j} dS_i;  dS_0 = dS_n + sum_i dS_i."""
    n = d_prefixes.shape[1]
    d_inc = np.zeros_like(d_prefixes)
    acc = np.array(d_state_out, np.float64)
    for i in range(n - 1, -1, -1):
        d_inc[:, i] = acc
        acc = acc + d_prefixes[:, i]
    return d_inc, acc


def windowed_attention_vjp(q, k, v, window: int, scale: float, do):
    """Softmax attention over keys [t - window + 1, t] with GQA (readings R1, R11).

    Per query head: S = scale Q K^T (masked), P = softmax(S), O = P V;
    dP = dO V^T, dS = P (dP - rowsum(dO O)), dQ = scale dS K, dK = scale dS^T Q,
    dV = P^T dO.  Query heads of one KV group add into that group's dK, dV.
    Dense [T, T] per head: small inputs only.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, T, Hq, hd = q.shape
    G = Hq // k.shape[2]
    mask = window_mask(T, window)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            kh = h // G
            s = scale * (q[b, :, h] @ k[b, :, kh].T)
            s = np.where(mask, s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            o = p @ v[b, :, kh]
            dp = do[b, :, h] @ v[b, :, kh].T
            ds = p * (dp - np.sum(do[b, :, h] * o, axis=1, keepdims=True))
            dq[b, :, h] = scale * (ds @ k[b, :, kh])
            dk[b, :, kh] += scale * (ds.T @ q[b, :, h])
            dv[b, :, kh] += p.T @ do[b, :, h]
    return dq, dk, dv


# ---------------------------------------------------------------------------
# Whole block
# ---------------------------------------------------------------------------


def fastweight_mlp_backward(u_T, u_S, beta, w_gate, w_up, w_down, w_proj, conv_T, conv_S,
                            chunk: int, l2_eps: float, d_y, state_in=None,
                            d_state_out=None) -> Dict[str, np.ndarray]:
    """Gradients of L through the forward oracle's ``fastweight_mlp`` (same
    arguments, without h_S), given d_y = dL/dy and d_state_out = dL/d state_out
    (nullable: zero).  Returns a dict keyed "u_T", "u_S", "beta", "state_in",
    "w_gate", "w_up", "w_down", "w_proj", "conv_T", "conv_S".

    The steps of the forward in reverse: the chunked read y_t = (W_down +
    S_i) Z_S[t], the exclusive prefix, the increments, the keys, the value
    residual, the two convs and the two SwiGLU views (readings G1, G2).
    """
    fw = fastweight_mlp(u_T, u_S, beta, w_gate, w_up, w_down, w_proj, conv_T, conv_S, chunk,
                        l2_eps, state_in=state_in, keep_prefixes=True)
    w_down = np.asarray(w_down, np.float64)
    d_y = np.asarray(d_y, np.float64)
    B, T, d = d_y.shape
    f = w_down.shape[1]
    d_state_out = np.zeros((B, d, f)) if d_state_out is None else np.asarray(d_state_out,
                                                                             np.float64)

    # y_t = (W_down + S_i) Z_S[t] for t in chunk i
    dZ_S = np.zeros_like(fw["Z_S"])
    dW_down = np.zeros_like(w_down)
    d_prefixes = np.zeros_like(fw["S_prefix"])
    for b in range(B):
        for i in range(fw["S_prefix"].shape[1]):
            s0, s1 = i * chunk, min(T, (i + 1) * chunk)
            dZ_S[b, s0:s1] = d_y[b, s0:s1] @ (w_down + fw["S_prefix"][b, i])
            g = d_y[b, s0:s1].T @ fw["Z_S"][b, s0:s1]
            dW_down += g
            d_prefixes[b, i] = g

    # exclusive prefix, chunk increments, keys, value residual
    d_inc, d_state_in = exclusive_prefix_vjp(d_prefixes, d_state_out)
    dR, dK, d_beta = chunk_increments_vjp(fw["R"], fw["K"], beta, chunk, d_inc)
    dzb_S = l2_normalize_rows_vjp(fw["zbar_S"], l2_eps, dK)
    dD, dwd, dW_proj = value_residual_vjp(fw["D"], w_down, w_proj, dR)
    dW_down += dwd
    dzb_T = dD                      # D = Zbar_T - Zbar_S
    dzb_S = dzb_S - dD

    # short convs, then SwiGLU of both views with the shared slow weights
    dZ_T, dconv_T = causal_depthwise_conv_vjp(fw["Z_T"], conv_T, dzb_T)
    dz, dconv_S = causal_depthwise_conv_vjp(fw["Z_S"], conv_S, dzb_S)
    dZ_S += dz
    du_T, dW_gate, dW_up = swiglu_vjp(u_T, w_gate, w_up, dZ_T)
    du_S, dwg, dwu = swiglu_vjp(u_S, w_gate, w_up, dZ_S)
    return {"u_T": du_T, "u_S": du_S, "beta": d_beta, "state_in": d_state_in,
            "w_gate": dW_gate + dwg, "w_up": dW_up + dwu, "w_down": dW_down,
            "w_proj": dW_proj, "conv_T": dconv_T, "conv_S": dconv_S}


def block_backward(x, beta, weights: Dict[str, np.ndarray], d_out, *, n_q_heads: int,
                   n_kv_heads: int, head_dim: int, w_S: int, w_T: int, chunk: int,
                   rms_eps: float = 1e-6, l2_eps: float = 1e-6, rope_theta: float = 1e4,
                   softmax_scale: Optional[float] = None, state_in=None,
                   d_state_out=None) -> Dict[str, np.ndarray]:
    """Gradients of L with respect to x, beta, state_in and every weight, given
    d_out = dL/d out and d_state_out = dL/d state_out (nullable: zero).

    The forward is the oracle's ``block_forward`` (same arguments); readings G1, G2.
    Returns a dict keyed like the inputs: "x", "beta", "state_in", "w_qkv",
    "w_o", "g_attn", "g_mlp", "w_gate", "w_up", "w_down", "w_proj", "conv_T",
    "conv_S".
    """
    x = np.asarray(x, np.float64)
    W = {k: np.asarray(v, np.float64) for k, v in weights.items() if k != "beta"}
    Hq, Hkv, hd = n_q_heads, n_kv_heads, head_dim
    scale = softmax_scale if softmax_scale else 1.0 / np.sqrt(hd)
    fw = block_forward(x, beta, weights, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=hd,
                       w_S=w_S, w_T=w_T, chunk=chunk, rms_eps=rms_eps, l2_eps=l2_eps,
                       rope_theta=rope_theta, softmax_scale=softmax_scale,
                       state_in=state_in, keep_prefixes=True)
    B, T, d = x.shape
    f = W["w_down"].shape[1]
    d_out = np.asarray(d_out, np.float64)
    d_state_out = np.zeros((B, d, f)) if d_state_out is None else np.asarray(d_state_out,
                                                                             np.float64)

    # the fast-weight MLP (everything between the MLP inputs u_P and y)
    g = fastweight_mlp_backward(fw["u_T"], fw["u_S"], beta, W["w_gate"], W["w_up"],
                                W["w_down"], W["w_proj"], W["conv_T"], W["conv_S"], chunk,
                                l2_eps, d_out, state_in=state_in, d_state_out=d_state_out)
    d_hS = d_out.copy()             # out = h_S + y
    du_T, du_S, d_beta, d_state_in = g["u_T"], g["u_S"], g["beta"], g["state_in"]
    dW_gate, dW_up, dW_down, dW_proj = g["w_gate"], g["w_up"], g["w_down"], g["w_proj"]
    dconv_T, dconv_S = g["conv_T"], g["conv_S"]

    # MLP RMSNorm (shared gain) of both views
    dh_T, dg_mlp = rms_norm_vjp(fw["h_T"], W["g_mlp"], rms_eps, du_T)
    dh, dg = rms_norm_vjp(fw["h_S"], W["g_mlp"], rms_eps, du_S)
    d_hS += dh
    dg_mlp += dg

    # h_P = x + o_P W_o^T (shared o_proj)
    dx = dh_T + d_hS
    o_T = fw["o_T"].reshape(B, T, Hq * hd)
    o_S = fw["o_S"].reshape(B, T, Hq * hd)
    dW_o = np.einsum("btd,btk->dk", dh_T, o_T) + np.einsum("btd,btk->dk", d_hS, o_S)
    do_T = (dh_T @ W["w_o"]).reshape(B, T, Hq, hd)
    do_S = (d_hS @ W["w_o"]).reshape(B, T, Hq, hd)

    # both windows over the same rotated q, k and v
    dq, dk, dv = windowed_attention_vjp(fw["q"], fw["k"], fw["v"], w_T, scale, do_T)
    dq2, dk2, dv2 = windowed_attention_vjp(fw["q"], fw["k"], fw["v"], w_S, scale, do_S)
    dq += dq2
    dk += dk2
    dv += dv2

    # RoPE, QKV projection, input RMSNorm
    dq = rope_vjp(dq, rope_theta)
    dk = rope_vjp(dk, rope_theta)
    dqkv = np.concatenate([dq.reshape(B, T, Hq * hd), dk.reshape(B, T, Hkv * hd),
                           dv.reshape(B, T, Hkv * hd)], axis=-1)
    xn = rms_norm(x, W["g_attn"], rms_eps)
    dxn = dqkv @ W["w_qkv"]
    dW_qkv = np.einsum("btj,btd->jd", dqkv, xn)
    dx2, dg_attn = rms_norm_vjp(x, W["g_attn"], rms_eps, dxn)
    dx += dx2

    return {"x": dx, "beta": d_beta, "state_in": d_state_in, "w_qkv": dW_qkv, "w_o": dW_o,
            "g_attn": dg_attn, "g_mlp": dg_mlp, "w_gate": dW_gate, "w_up": dW_up,
            "w_down": dW_down, "w_proj": dW_proj, "conv_T": dconv_T, "conv_S": dconv_S}
