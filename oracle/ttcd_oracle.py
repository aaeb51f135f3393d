"""CPU float64 oracle of the IP-TTCD block forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The CUDA library never calls it, and it shares no code with the CUDA
path: the one module both sides use is ``ttcd_workloads`` (seeded random inputs,
no arithmetic of the method).

Every function is the plain definition of one step, written in float64 with
NumPy, with no blocking, fusion or reordering beyond what the definition states
(library matmuls serve as steps).  Sources, cited by page title and section:

[README]  GitHub README "TTCD: Test-Time Training via Context Distillation"
          (github.com/dangxingyu/ttcd), sections "Model configuration" and
          "Fused inference kernels".
[REVIEW]  papernotes.org review "Learning What to Remember: Test-Time Training
          via Context Distillation": section 方法详解 (method: 整体框架 overall
          framework + flowchart A-F), 关键设计 1 (distillation loss, Eq. 4),
          关键设计 2 (in-place fast weight, off-policy approximation),
          关键设计 3 (short convs, W_proj, R_i, K_i, Delta W), 关键设计 4
          (Proposition 1).
[PODCAST] podcast transcript "Test-Time Training via Context Distillation:
          Learning What to Remember", cue numbers (19: sliding window;
          23: Eq. 4 / Eq. 6; 29: Eq. 12 practical update).

Readings where the pages are silent or garbled (each repeated where used):
  R1 window: a window of w keys includes the query itself: keys
     j in [max(0, t-w+1), t]  ([PODCAST] cue 19, "the last w tokens").
  R2 both windows slide per token (not chunk-aligned).
  R3 the student path is the block output; the teacher feeds only R.
  R4 residual sign: teacher minus student ([REVIEW] 关键设计 3; the descent
     direction of Eq. 4).
  R5 beta is a per-token input; Delta W_i = sum_{t in C_i} beta_t r_t k_t^T,
     no 1/|C| factor.
  R6 the chunk prefix is exclusive: chunk i reads sum_{j<i} Delta W_j.
  R7 the fast weight multiplies the raw SwiGLU activation Z_S (not conv'd).
  R8 k_t = zbar_t / sqrt(||zbar_t||^2 + eps_k).
  R9 conv: no bias, zero left padding, no reset at chunk boundaries; tap m
     multiplies position t-m.
  R10 block skeleton: pre-norm RMSNorm -> QKV (no bias) -> RoPE (rotate-half,
     positions 0..T-1) -> dual attention -> shared o_proj + residual ->
     RMSNorm (shared gain) -> SwiGLU; softmax scale 1/sqrt(hd); no QK-norm.
  R11 GQA: query head h reads KV head h // (Hq / Hkv).
  R12 W_proj is applied first: r_t = W_down (W_proj d_t), as written.
  R13 a partial last chunk is allowed; its Delta W counts only in the final state.
  R18 a layer outside the TTT layer set ([README] "Model configuration",
     ttt_layers) is the same skeleton with one sliding window of w_T keys
     (window_size) and the static MLP: no student path, no fast weights.

Parity pins (tests/test_oracle_*.py) tie each function to something other than
itself: brute-force loops, textbook/library special cases, closed forms and
identities.  No page prints a worked numeric example, so absolute values are
pinned by those identities only.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

# ---------------------------------------------------------------------------
# Elementwise and normalisation steps
# ---------------------------------------------------------------------------


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x * (mean(x^2) + eps)^(-1/2) * g.  Reading R10."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)


def rope(x: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding on [B, T, H, hd] at positions 0..T-1.  Reading R10.

    Pair i (i < hd/2) is (x[i], x[i + hd/2]) rotated by angle t * theta^(-2i/hd).
    """
    x = np.asarray(x, dtype=np.float64)
    B, T, H, hd = x.shape
    half = hd // 2
    inv_freq = theta ** (-(np.arange(half, dtype=np.float64) * 2.0) / hd)
    ang = np.arange(T, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos = np.cos(ang)[None, :, None, :]
    sin = np.sin(ang)[None, :, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def swiglu(u: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray) -> np.ndarray:
    """Z = silu(u W_gate^T) * (u W_up^T): the SwiGLU MLP activation with slow weights.

    [REVIEW] 关键设计 2 (SwiGLU MLP whose down-projection is the fast weight).
    """
    u = np.asarray(u, dtype=np.float64)
    return silu(u @ np.asarray(w_gate, np.float64).T) * (u @ np.asarray(w_up, np.float64).T)


def causal_depthwise_conv(z: np.ndarray, taps: np.ndarray) -> np.ndarray:
    """zbar[b, t, c] = sum_m taps[c, m] * z[b, t - m, c], zero for t - m < 0.

    [REVIEW] 关键设计 3 (lightweight depthwise short causal convolutions conv_T,
    conv_S).  Reading R9: no bias, zero left padding, no reset at chunk edges.
    """
    z = np.asarray(z, dtype=np.float64)
    taps = np.asarray(taps, dtype=np.float64)
    T = z.shape[1]
    out = np.zeros_like(z)
    for m in range(taps.shape[1]):
        if m >= T:
            break
        out[:, m:, :] += taps[:, m][None, None, :] * z[:, :T - m, :]
    return out


def l2_normalize_rows(z: np.ndarray, eps: float) -> np.ndarray:
    """k = z / sqrt(||z||^2 + eps) per row.  [REVIEW] 关键设计 3 (K_i = l2-norm(Zbar_S)); R8."""
    z = np.asarray(z, dtype=np.float64)
    return z / np.sqrt(np.sum(z * z, axis=-1, keepdims=True) + eps)


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------


def window_mask(T: int, w: int) -> np.ndarray:
    """Boolean [T, T] mask, True where key j is visible to query t: t-w+1 <= j <= t (R1)."""
    t = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return (j <= t) & (j >= t - w + 1)


def windowed_attention(q, k, v, window: int, scale: float, block: int = 256):
    """Causal sliding-window softmax attention with GQA, blocked over query rows.

    For each query block the dense masked score matrix over the keys the block
    can see is formed and normalised; nothing else is reordered.
    [PODCAST] cue 19 (each token sees the last w tokens); readings R1, R11.

    q [B, T, Hq, hd], k/v [B, T, Hkv, hd] -> (o [B, T, Hq, hd], lse [B, Hq, T]).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, T, Hq, hd = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, T))
    for b in range(B):
        for t0 in range(0, T, block):
            t1 = min(T, t0 + block)
            j0 = max(0, t0 - window + 1)
            tt = np.arange(t0, t1)[:, None]
            jj = np.arange(j0, t1)[None, :]
            mask = (jj <= tt) & (jj >= tt - window + 1)
            qb = q[b, t0:t1].reshape(t1 - t0, Hkv, G, hd).transpose(1, 2, 0, 3)  # [Hkv,G,bt,hd]
            kb = k[b, j0:t1].transpose(1, 0, 2)[:, None]  # [Hkv,1,bj,hd]
            vb = v[b, j0:t1].transpose(1, 0, 2)[:, None]
            s = (qb @ kb.transpose(0, 1, 3, 2)) * scale  # [Hkv,G,bt,bj]
            s = np.where(mask[None, None], s, -np.inf)
            m = np.max(s, axis=-1, keepdims=True)
            p = np.exp(s - m)
            l = np.sum(p, axis=-1, keepdims=True)
            ob = (p @ vb) / l  # [Hkv,G,bt,hd]
            o[b, t0:t1] = ob.transpose(2, 0, 1, 3).reshape(t1 - t0, Hq, hd)
            lse[b, :, t0:t1] = (m + np.log(l))[..., 0].reshape(Hq, t1 - t0)
    return o, lse


def windowed_attention_bruteforce(q, k, v, window: int, scale: float):
    """Per-query loop over the visible keys; tiny inputs only.  Same definition as above."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, T, Hq, hd = q.shape
    G = Hq // k.shape[2]
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, T))
    for b in range(B):
        for h in range(Hq):
            kh = h // G
            for t in range(T):
                keys = range(max(0, t - window + 1), t + 1)
                s = [scale * float(np.dot(q[b, t, h], k[b, j, kh])) for j in keys]
                m = max(s)
                e = [np.exp(x - m) for x in s]
                den = sum(e)
                acc = np.zeros(hd)
                for ej, j in zip(e, keys):
                    acc += ej * v[b, j, kh]
                o[b, t, h] = acc / den
                lse[b, h, t] = m + np.log(den)
    return o, lse


def windowed_attention_row(q, k, v, window: int, scale: float, b: int, t: int, h: int):
    """One output row of the windowed attention: query (b, t, h) against keys
    j in [max(0, t-window+1), t] of KV head h // (Hq/Hkv) (readings R1, R11).
    For sampled checks of long sequences.  Returns (o[b, t, h], lse[b, h, t])."""
    G = q.shape[2] // k.shape[2]
    j0 = max(0, t - window + 1)
    kk = np.asarray(k[b, j0:t + 1, h // G], np.float64)
    vv = np.asarray(v[b, j0:t + 1, h // G], np.float64)
    s = scale * (kk @ np.asarray(q[b, t, h], np.float64))
    m = s.max()
    e = np.exp(s - m)
    return (e[:, None] * vv).sum(0) / e.sum(), m + np.log(e.sum())


def dual_window_attention(q, k, v, w_S: int, w_T: int, scale: float):
    """Teacher (w_T) and student (w_S) sliding-window outputs over the same Q/K/V.

    [README] "Fused inference kernels" (both windowed outputs from one pass
    over K/V); [REVIEW] 整体框架 (long-window teacher, short-window student over
    a shared backbone).  The oracle simply evaluates each window's definition.
    Returns (o_T, o_S, lse_T, lse_S).
    """
    o_T, lse_T = windowed_attention(q, k, v, w_T, scale)
    o_S, lse_S = windowed_attention(q, k, v, w_S, scale)
    return o_T, o_S, lse_T, lse_S


def band_attention(q, k, v, near: int, far: int, scale: float):
    """Causal band attention with GQA: query t attends to keys j with
    t - far <= j <= t - near (clipped at 0), softmax over the band only.

    [README] "Fused inference kernels", lse_dual_attn: the teacher window is
    the student window [t-w_S+1, t] plus a shifted far band [t-w_T+1, t-w_S]
    (near = w_S, far = w_T - 1), and the two partial attentions merge exactly
    through their log-sum-exp.  A row whose band holds no key gets o = 0 and
    lse = -inf (it carries no weight in the merge).  Returns (o, lse).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, T, Hq, hd = q.shape
    G = Hq // k.shape[2]
    o = np.zeros_like(q)
    lse = np.full((B, Hq, T), -np.inf)
    t = np.arange(T)
    j = np.arange(T)
    mask = (j[None, :] <= t[:, None] - near) & (j[None, :] >= t[:, None] - far)
    for b in range(B):
        for h in range(Hq):
            s = scale * (q[b, :, h] @ k[b, :, h // G].T)
            s = np.where(mask, s, -np.inf)
            m = s.max(axis=1)
            rows = np.isfinite(m)
            e = np.exp(s[rows] - m[rows, None])
            den = e.sum(axis=1)
            o[b, rows, h] = (e @ v[b, :, h // G]) / den[:, None]
            lse[b, h, rows] = m[rows] + np.log(den)
    return o, lse


def lse_merge(o1, lse1, o2, lse2):
    """Exact merge of two partial softmax attentions over disjoint key sets:
    o = (o1 e^{lse1} + o2 e^{lse2}) / (e^{lse1} + e^{lse2}), lse = logaddexp.
    o: [B, T, H, hd]; lse: [B, H, T].  [README] "Fused inference kernels"."""
    lse = np.logaddexp(lse1, lse2)
    w1 = np.exp(lse1 - lse).transpose(0, 2, 1)[..., None]
    w2 = np.exp(lse2 - lse).transpose(0, 2, 1)[..., None]
    return w1 * np.asarray(o1, np.float64) + w2 * np.asarray(o2, np.float64), lse


# ---------------------------------------------------------------------------
# Fast-weight MLP (in-place TTCD)
# ---------------------------------------------------------------------------


def value_residual(zbar_T, zbar_S, w_down, w_proj):
    """r_t = W_down^(0) W_proj (zbar_T[t] - zbar_S[t]).

    [REVIEW] 关键设计 3: R_i = W_down^(0) W_proj (Zbar_T - Zbar_S).  Readings R4
    (teacher minus student) and R12 (W_proj applied first, literal order).
    Returns r [B, T, d].
    """
    dlt = np.asarray(zbar_T, np.float64) - np.asarray(zbar_S, np.float64)  # [B,T,f]
    tmp = dlt @ np.asarray(w_proj, np.float64).T  # (W_proj d_t)^T, [B,T,f]
    return tmp @ np.asarray(w_down, np.float64).T  # [B,T,d]


def chunk_increments(r, key, beta, chunk: int):
    """Delta W_i = sum_{t in C_i} beta_t r_t k_t^T for each chunk i, [B, n_chunks, d, f].

    [REVIEW] 关键设计 3 (Delta W_down^(i) = beta_i R_i K_i^T, a low-rank write);
    [PODCAST] cue 29 (write scaled by a learned coefficient).  Readings R5, R13.
    """
    r = np.asarray(r, np.float64)
    key = np.asarray(key, np.float64)
    beta = np.asarray(beta, np.float64)
    B, T, d = r.shape
    f = key.shape[-1]
    n = (T + chunk - 1) // chunk
    out = np.zeros((B, n, d, f))
    for b in range(B):
        for i in range(n):
            s0, s1 = i * chunk, min(T, (i + 1) * chunk)
            out[b, i] = (r[b, s0:s1] * beta[b, s0:s1, None]).T @ key[b, s0:s1]
    return out


def exclusive_prefix(increments, state_in=None):
    """S_0 = state_in (or 0), S_{i+1} = S_i + Delta W_i.  Returns (S_0..S_{n-1}, S_n).

    [REVIEW] 整体框架 / 关键设计 2 (causal prefix scan over chunks); reading R6.
    """
    inc = np.asarray(increments, np.float64)
    B, n, d, f = inc.shape
    s = np.zeros((B, d, f)) if state_in is None else np.array(state_in, np.float64)
    prefixes = np.zeros_like(inc)
    for i in range(n):
        prefixes[:, i] = s
        s = s + inc[:, i]
    return prefixes, s


def fastweight_mlp(u_T, u_S, beta, w_gate, w_up, w_down, w_proj, conv_T, conv_S,
                   chunk: int, l2_eps: float, h_S=None, state_in=None,
                   keep_prefixes: bool = True) -> Dict[str, np.ndarray]:
    """The in-place fast-weight MLP of one IP-TTCD block (off-policy form).

    Steps (flowchart C-F of [REVIEW] 方法详解; [REVIEW] 关键设计 2 and 3;
    [PODCAST] cue 29):
      Z_P  = SwiGLU(u_P) with slow weights W^(0)              (off-policy)
      Zb_P = conv_P(Z_P)                                      (short causal convs)
      r_t  = W_down W_proj (Zb_T - Zb_S)[t]                   (value residual)
      k_t  = l2norm(Zb_S[t]) ; Delta W_i = sum beta_t r_t k_t^T
      S_i  = state_in + sum_{j<i} Delta W_j                   (exclusive prefix)
      y_t  = (W_down + S_{i(t)}) Z_S[t]                       (R7)
      out  = h_S + y  when h_S is given.
    """
    Z_T = swiglu(u_T, w_gate, w_up)
    Z_S = swiglu(u_S, w_gate, w_up)
    zb_T = causal_depthwise_conv(Z_T, conv_T)
    zb_S = causal_depthwise_conv(Z_S, conv_S)
    r = value_residual(zb_T, zb_S, w_down, w_proj)
    key = l2_normalize_rows(zb_S, l2_eps)
    inc = chunk_increments(r, key, beta, chunk)
    prefixes, state_out = exclusive_prefix(inc, state_in)
    B, T, f = Z_S.shape
    w_down = np.asarray(w_down, np.float64)
    y = np.zeros((B, T, w_down.shape[0]))
    for b in range(B):
        for i in range(prefixes.shape[1]):
            s0, s1 = i * chunk, min(T, (i + 1) * chunk)
            y[b, s0:s1] = Z_S[b, s0:s1] @ (w_down + prefixes[b, i]).T
    res = {"Z_T": Z_T, "Z_S": Z_S, "zbar_T": zb_T, "zbar_S": zb_S, "D": zb_T - zb_S,
           "R": r, "K": key, "dW": inc, "state_out": state_out, "y": y}
    if keep_prefixes:
        res["S_prefix"] = prefixes
    if h_S is not None:
        res["out"] = np.asarray(h_S, np.float64) + y
    return res


# ---------------------------------------------------------------------------
# Whole block
# ---------------------------------------------------------------------------


def qkv_projection(xn, w_qkv, Hq: int, Hkv: int, hd: int):
    """Shared Q/K/V of both windows from the normalised input (reading R10)."""
    qkv = np.asarray(xn, np.float64) @ np.asarray(w_qkv, np.float64).T
    B, T, _ = qkv.shape
    q = qkv[..., :Hq * hd].reshape(B, T, Hq, hd)
    k = qkv[..., Hq * hd:(Hq + Hkv) * hd].reshape(B, T, Hkv, hd)
    v = qkv[..., (Hq + Hkv) * hd:].reshape(B, T, Hkv, hd)
    return q, k, v


def block_forward(x, beta, weights: Dict[str, np.ndarray], *, n_q_heads: int,
                  n_kv_heads: int, head_dim: int, w_S: int, w_T: int, chunk: int,
                  rms_eps: float = 1e-6, l2_eps: float = 1e-6, rope_theta: float = 1e4,
                  softmax_scale: Optional[float] = None, state_in=None,
                  keep_prefixes: bool = False) -> Dict[str, np.ndarray]:
    """Forward pass of one IP-TTCD block; returns every intermediate and ``out``.

    [REVIEW] 整体框架 + flowchart A-F; [README] "Model configuration"
    (window_size = teacher window w_T, student window w_S); readings R1-R13.
    """
    x = np.asarray(x, np.float64)
    Hq, Hkv, hd = n_q_heads, n_kv_heads, head_dim
    scale = softmax_scale if softmax_scale else 1.0 / np.sqrt(hd)
    xn = rms_norm(x, weights["g_attn"], rms_eps)
    q, k, v = qkv_projection(xn, weights["w_qkv"], Hq, Hkv, hd)
    q = rope(q, rope_theta)
    k = rope(k, rope_theta)
    o_T, o_S, lse_T, lse_S = dual_window_attention(q, k, v, w_S, w_T, scale)
    B, T = x.shape[:2]
    w_o = np.asarray(weights["w_o"], np.float64)
    h_T = x + o_T.reshape(B, T, Hq * hd) @ w_o.T
    h_S = x + o_S.reshape(B, T, Hq * hd) @ w_o.T
    u_T = rms_norm(h_T, weights["g_mlp"], rms_eps)
    u_S = rms_norm(h_S, weights["g_mlp"], rms_eps)
    mlp = fastweight_mlp(u_T, u_S, beta, weights["w_gate"], weights["w_up"],
                         weights["w_down"], weights["w_proj"], weights["conv_T"],
                         weights["conv_S"], chunk, l2_eps, h_S=h_S, state_in=state_in,
                         keep_prefixes=keep_prefixes)
    res = {"q": q, "k": k, "v": v, "o_T": o_T, "o_S": o_S, "lse_T": lse_T, "lse_S": lse_S,
           "h_T": h_T, "h_S": h_S, "u_T": u_T, "u_S": u_S}
    res.update(mlp)
    return res


def swa_block_forward(x, weights: Dict[str, np.ndarray], *, n_q_heads: int, n_kv_heads: int,
                      head_dim: int, window: int, rms_eps: float = 1e-6,
                      rope_theta: float = 1e4,
                      softmax_scale: Optional[float] = None) -> Dict[str, np.ndarray]:
    """Forward pass of a plain sliding-window block: a layer outside the TTT
    layer set ([README] "Model configuration": ttt_layers, window_size; reading
    R18; skeleton R10, R11).

      h = x + SWA_window(RoPE(q), RoPE(k), v) W_o^T,  q,k,v = RMSNorm(x) W_qkv^T
      out = h + W_down SwiGLU(RMSNorm(h))
    """
    x = np.asarray(x, np.float64)
    Hq, Hkv, hd = n_q_heads, n_kv_heads, head_dim
    sm_scale = softmax_scale if softmax_scale else 1.0 / np.sqrt(float(hd))
    xn = rms_norm(x, weights["g_attn"], rms_eps)
    q, k, v = qkv_projection(xn, weights["w_qkv"], Hq, Hkv, hd)
    q, k = rope(q, rope_theta), rope(k, rope_theta)
    o, lse = windowed_attention(q, k, v, window, sm_scale)
    B, T = x.shape[:2]
    h = x + o.reshape(B, T, Hq * hd) @ np.asarray(weights["w_o"], np.float64).T
    u = rms_norm(h, weights["g_mlp"], rms_eps)
    z = swiglu(u, weights["w_gate"], weights["w_up"])
    out = h + z @ np.asarray(weights["w_down"], np.float64).T
    return {"q": q, "k": k, "v": v, "o": o, "lse": lse, "h": h, "u": u, "z": z, "out": out}


# ---------------------------------------------------------------------------
# Objective used to check the write rule (not part of the forward pass)
# ---------------------------------------------------------------------------


def distillation_loss(w_down, z_S_chunk, y_T_const):
    """L_i = (1/|C_i|) sum_t 1/2 ||W_down z_S[t] - stopgrad(y_T[t])||^2.

    [REVIEW] 关键设计 1 (Eq. 4, the LaTeX on the page is garbled; reassembled
    with [PODCAST] cue 23: half a squared error, teacher detached).  The
    teacher output enters as a constant, which is what stopgrad means for a
    derivative with respect to W_down.
    """
    y_S = np.asarray(z_S_chunk, np.float64) @ np.asarray(w_down, np.float64).T
    diff = y_S - np.asarray(y_T_const, np.float64)
    return 0.5 * float(np.sum(diff * diff)) / diff.shape[0]
