"""Pins for the oracle's whole block (CPU only).

The block skeleton (pre-norm, QKV, RoPE, o_proj, residual, RMSNorm, SwiGLU) is
not spelled out on the pages; with equal windows and equal convolutions the
IP-TTCD block must reduce to a plain sliding-window transformer block, which is
written here independently with torch float64 library routines.
"""
import numpy as np
import pytest
import torch

from oracle import ttcd_oracle as orc
from ttcd_workloads import TINY_F32, make_block_inputs


def _np(t):
    return t.double().numpy()


def _block(shape, inp, layer=0, **over):
    w = {k: _np(v) for k, v in inp["layers"][layer].items()}
    w.update(over)
    return orc.block_forward(_np(inp["x"]), w["beta"], w, n_q_heads=shape.n_q_heads,
                             n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim,
                             w_S=shape.w_S, w_T=shape.w_T, chunk=shape.chunk,
                             rms_eps=shape.rms_eps, l2_eps=shape.l2_eps,
                             rope_theta=shape.rope_theta)


def _plain_swa_block(x, w, shape, window):
    """Plain pre-norm sliding-window transformer block, torch float64."""
    x = torch.from_numpy(x)
    B, T, d = x.shape
    Hq, Hkv, hd = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    W = {k: torch.from_numpy(np.asarray(v, np.float64)) for k, v in w.items()}
    xn = torch.nn.functional.rms_norm(x, (d,), W["g_attn"], eps=shape.rms_eps)
    qkv = xn @ W["w_qkv"].T
    q = qkv[..., :Hq * hd].reshape(B, T, Hq, hd)
    k = qkv[..., Hq * hd:(Hq + Hkv) * hd].reshape(B, T, Hkv, hd)
    v = qkv[..., (Hq + Hkv) * hd:].reshape(B, T, Hkv, hd)
    half = hd // 2
    ang = torch.outer(torch.arange(T, dtype=torch.float64),
                      shape.rope_theta ** (-2.0 * torch.arange(half, dtype=torch.float64) / hd))
    rot = torch.polar(torch.ones_like(ang), ang)[None, :, None, :]

    def rope(t):
        z = torch.complex(t[..., :half], t[..., half:]) * rot
        return torch.cat([z.real, z.imag], -1)

    q, k = rope(q), rope(k)
    i = torch.arange(T)
    mask = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - window)
    G = Hq // Hkv
    o = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), k.repeat_interleave(G, 2).transpose(1, 2),
        v.repeat_interleave(G, 2).transpose(1, 2), attn_mask=mask)
    h = x + o.transpose(1, 2).reshape(B, T, Hq * hd) @ W["w_o"].T
    u = torch.nn.functional.rms_norm(h, (d,), W["g_mlp"], eps=shape.rms_eps)
    z = torch.nn.functional.silu(u @ W["w_gate"].T) * (u @ W["w_up"].T)
    return (h + z @ W["w_down"].T).numpy()


def test_equal_windows_reduce_to_plain_swa_block():
    shape = TINY_F32.with_(w_S=48, w_T=48)
    inp = make_block_inputs(shape, seed=0)
    w = {k: _np(v) for k, v in inp["layers"][0].items()}
    res = _block(shape, inp, conv_T=w["conv_S"])
    assert np.all(res["R"] == 0)
    ref = _plain_swa_block(_np(inp["x"]), w, shape, 48)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-11)


def test_distinct_norm_gains_reduce_to_plain_swa_block():
    """The same reduction with random, different gains for the two RMSNorms:
    the attention norm takes g_attn, the MLP norm g_mlp (both views share it)."""
    shape = TINY_F32.with_(w_S=40, w_T=40)
    inp = make_block_inputs(shape, seed=2)
    w = {k: _np(v) for k, v in inp["layers"][0].items()}
    rng = np.random.default_rng(9)
    w["g_attn"] = 0.5 + rng.random(shape.d_model)
    w["g_mlp"] = 0.5 + rng.random(shape.d_model)
    w["conv_T"] = w["conv_S"]
    res = _block(shape, inp, **{k: w[k] for k in ("g_attn", "g_mlp", "conv_T")})
    ref = _plain_swa_block(_np(inp["x"]), w, shape, 40)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-11)


def test_student_path_is_block_output_with_static_mlp_when_beta_zero():
    shape = TINY_F32
    inp = make_block_inputs(shape, seed=0)
    w = {k: _np(v) for k, v in inp["layers"][0].items()}
    res = _block(shape, inp, beta=np.zeros((1, shape.T)))
    ref = _plain_swa_block(_np(inp["x"]), w, shape, shape.w_S)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-11)


def _swa(shape, inp, window, layer=0):
    w = {k: _np(v) for k, v in inp["layers"][layer].items()}
    return orc.swa_block_forward(_np(inp["x"]), w, n_q_heads=shape.n_q_heads,
                                 n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim,
                                 window=window, rms_eps=shape.rms_eps,
                                 rope_theta=shape.rope_theta)


@pytest.mark.parametrize("window", [1, 16, 64, 300])
def test_plain_swa_block_matches_torch_built_block(window):
    """The oracle's plain sliding-window block (a layer outside the TTT layer
    set) against the block written with torch float64 library routines, with
    distinct norm gains."""
    shape = TINY_F32
    inp = make_block_inputs(shape, seed=4)
    rng = np.random.default_rng(5)
    inp["layers"][0]["g_attn"] = torch.from_numpy(0.5 + rng.random(shape.d_model))
    inp["layers"][0]["g_mlp"] = torch.from_numpy(0.5 + rng.random(shape.d_model))
    w = {k: _np(v) for k, v in inp["layers"][0].items()}
    res = _swa(shape, inp, window)
    ref = _plain_swa_block(_np(inp["x"]), w, shape, window)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-11)


def test_plain_swa_block_is_the_ttcd_block_with_one_window_and_no_update():
    """With w_S = w_T and beta = 0 the IP-TTCD block's student output is the plain
    block of window w_T, whatever the conv taps and W_proj."""
    shape = TINY_F32.with_(w_S=64, w_T=64)
    inp = make_block_inputs(shape, seed=6)
    res = _block(shape, inp, beta=np.zeros((1, shape.T)))
    np.testing.assert_allclose(_swa(shape, inp, 64)["out"], res["out"], rtol=1e-10, atol=1e-11)


def test_block_attention_matches_bruteforce_on_tiny_workload():
    shape = TINY_F32
    inp = make_block_inputs(shape, seed=0)
    res = _block(shape, inp)
    for key, w in (("o_T", shape.w_T), ("o_S", shape.w_S)):
        ob, _ = orc.windowed_attention_bruteforce(res["q"], res["k"], res["v"], w,
                                                  shape.softmax_scale)
        np.testing.assert_allclose(res[key], ob, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("T_prefix", [1, 31, 32, 100, 255])
def test_block_is_causal_prefix_invariant(T_prefix):
    """Outputs at positions < T' depend only on inputs at positions < T'."""
    shape = TINY_F32
    inp = make_block_inputs(shape, seed=0)
    full = _block(shape, inp)
    short = dict(inp)
    short["x"] = inp["x"][:, :T_prefix]
    short["layers"] = [dict(inp["layers"][0], beta=inp["layers"][0]["beta"][:, :T_prefix])]
    part = _block(shape.with_(T=T_prefix), short)
    np.testing.assert_allclose(part["out"], full["out"][:, :T_prefix], rtol=1e-11, atol=1e-12)
