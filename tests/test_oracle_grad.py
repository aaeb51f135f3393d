"""Pins for the oracle's block backward (CPU only).

The backward (oracle/ttcd_oracle_grad.py) is the chain rule of the forward
oracle's steps, readings G1-G2: the outer gradient flows through every step as
written, the write path included (podcast transcript "Test-Time Training via
Context Distillation", cue 51: W_proj, the short convs and the write gate are
trained by the next-token loss).  It is pinned by:

- central finite differences of the forward oracle (itself pinned by the other
  test_oracle_*.py files) along a random direction, for every input and weight;
- exact zeros: with beta = 0 and no state gradient, nothing reaches W_proj or
  the two convs, whose only route to the loss is the fast-weight write;
- reduction: with equal windows and equal convs the block is a plain
  sliding-window block (D = R = 0), so the gradients of every shared input
  equal torch autograd through a plain block built from library SDPA,
  rms_norm and silu;
- single steps against library autograd: the windowed GQA attention (SDPA
  with a band mask), the causal depthwise conv (conv1d), RMSNorm and SwiGLU.
"""
import numpy as np
import pytest
import torch

from oracle import ttcd_oracle as orc
from oracle.ttcd_oracle_grad import block_backward

B, T, D, F, K = 2, 21, 8, 12, 3          # 21 tokens: four chunks of 5 and a ragged one
HQ, HKV, HD = 4, 2, 4
SHAPE = dict(n_q_heads=HQ, n_kv_heads=HKV, head_dim=HD, w_S=3, w_T=7, chunk=5)
NAMES = ["x", "beta", "state_in", "w_qkv", "w_o", "g_attn", "g_mlp", "w_gate", "w_up",
         "w_down", "w_proj", "conv_T", "conv_S"]
WEIGHTS = NAMES[3:]


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
    g_out = rng.standard_normal((B, T, D))
    g_state = rng.standard_normal((B, D, F))
    return x, beta, w, state_in, g_out, g_state


def _loss(args, g_out, g_state, shape):
    w = {k: args[k] for k in WEIGHTS}
    r = orc.block_forward(args["x"], args["beta"], w, state_in=args["state_in"], **shape)
    loss = np.sum(g_out * r["out"])
    if g_state is not None:
        loss += np.sum(g_state * r["state_out"])
    return loss


@pytest.mark.parametrize("with_state", [True, False], ids=["state", "no_state"])
@pytest.mark.parametrize("name", NAMES)
def test_directional_derivative_matches_central_difference(name, with_state):
    x, beta, w, s0, g_out, g_state = _case()
    if not with_state:
        g_state = None
    grads = block_backward(x, beta, w, g_out, state_in=s0, d_state_out=g_state, **SHAPE)
    args = {"x": x, "beta": beta, "state_in": s0, **w}
    v = np.random.default_rng(100 + NAMES.index(name)).standard_normal(args[name].shape)
    eps = 1e-6

    def at(delta):
        a = dict(args)
        a[name] = args[name] + delta * v
        return _loss(a, g_out, g_state, SHAPE)

    fd = (at(eps) - at(-eps)) / (2 * eps)
    an = float(np.sum(grads[name] * v))
    assert grads[name].shape == args[name].shape
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (fd, an)


def test_write_path_weights_get_no_gradient_without_writes():
    x, beta, w, s0, g_out, _ = _case(1)
    g = block_backward(x, np.zeros_like(beta), w, g_out, state_in=s0, **SHAPE)
    for name in ("w_proj", "conv_T", "conv_S"):
        assert np.all(g[name] == 0), name
    assert np.any(g["beta"] != 0)  # a write would still change later chunks


def _plain_block_torch(t, window):
    """Plain pre-norm sliding-window block (torch float64, differentiable)."""
    x = t["x"]
    b, n, d = x.shape
    xn = torch.nn.functional.rms_norm(x, (d,), t["g_attn"], eps=1e-6)
    qkv = xn @ t["w_qkv"].T
    q = qkv[..., :HQ * HD].reshape(b, n, HQ, HD)
    k = qkv[..., HQ * HD:(HQ + HKV) * HD].reshape(b, n, HKV, HD)
    v = qkv[..., (HQ + HKV) * HD:].reshape(b, n, HKV, HD)
    half = HD // 2
    ang = torch.outer(torch.arange(n, dtype=torch.float64),
                      1e4 ** (-2.0 * torch.arange(half, dtype=torch.float64) / HD))
    rot = torch.polar(torch.ones_like(ang), ang)[None, :, None, :]

    def rope(z):
        c = torch.complex(z[..., :half], z[..., half:]) * rot
        return torch.cat([c.real, c.imag], -1)

    q, k = rope(q), rope(k)
    i = torch.arange(n)
    mask = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - window)
    G = HQ // HKV
    o = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), k.repeat_interleave(G, 2).transpose(1, 2),
        v.repeat_interleave(G, 2).transpose(1, 2), attn_mask=mask)
    h = x + o.transpose(1, 2).reshape(b, n, HQ * HD) @ t["w_o"].T
    u = torch.nn.functional.rms_norm(h, (d,), t["g_mlp"], eps=1e-6)
    z = torch.nn.functional.silu(u @ t["w_gate"].T) * (u @ t["w_up"].T)
    return h + z @ t["w_down"].T


def test_equal_windows_and_convs_reduce_to_plain_block_autograd():
    x, beta, w, _, g_out, _ = _case(2)
    w["conv_T"] = w["conv_S"].copy()
    shape = dict(SHAPE, w_S=7, w_T=7)
    g = block_backward(x, beta, w, g_out, **shape)
    shared = ["x", "w_qkv", "w_o", "g_attn", "g_mlp", "w_gate", "w_up", "w_down"]
    t = {k: torch.tensor(x if k == "x" else w[k], requires_grad=True) for k in shared}
    out = _plain_block_torch(t, 7)
    np.testing.assert_allclose(out.detach().numpy(), orc.block_forward(
        x, beta, w, **shape)["out"], rtol=1e-12, atol=1e-12)
    (out * torch.from_numpy(g_out)).sum().backward()
    for k in shared:
        np.testing.assert_allclose(g[k], t[k].grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=k)


# ------------------------------------------------ single steps against library autograd

def _autograd(fn, *arrays, grad_out):
    ts = [torch.tensor(a, requires_grad=True) for a in arrays]
    (fn(*ts) * torch.from_numpy(grad_out)).sum().backward()
    return [t.grad.numpy() for t in ts]


@pytest.mark.parametrize("window", [1, 5, 40])
def test_attention_vjp_matches_sdpa_autograd(window):
    from oracle.ttcd_oracle_grad import windowed_attention_vjp
    rng = np.random.default_rng(window)
    b, n, hq, hkv, hd = 2, 33, 6, 2, 8
    q, k, v = (rng.standard_normal((b, n, h, hd)) for h in (hq, hkv, hkv))
    do = rng.standard_normal((b, n, hq, hd))
    scale = 1.0 / np.sqrt(hd)
    i = torch.arange(n)
    mask = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - window)

    def sdpa(qt, kt, vt):
        g = hq // hkv
        o = torch.nn.functional.scaled_dot_product_attention(
            qt.transpose(1, 2), kt.repeat_interleave(g, 2).transpose(1, 2),
            vt.repeat_interleave(g, 2).transpose(1, 2), attn_mask=mask, scale=scale)
        return o.transpose(1, 2)

    ref = _autograd(sdpa, q, k, v, grad_out=do)
    got = windowed_attention_vjp(q, k, v, window, scale, do)
    for r, g_ in zip(ref, got):
        np.testing.assert_allclose(g_, r, rtol=1e-10, atol=1e-12)


def test_conv_vjp_matches_conv1d_autograd():
    from oracle.ttcd_oracle_grad import causal_depthwise_conv_vjp
    rng = np.random.default_rng(4)
    b, n, f, k = 2, 17, 5, 4
    z, taps, dzbar = rng.standard_normal((b, n, f)), rng.standard_normal((f, k)), \
        rng.standard_normal((b, n, f))

    def conv(zt, wt):  # causal depthwise conv: tap m multiplies t - m
        x = torch.nn.functional.pad(zt.transpose(1, 2), (k - 1, 0))
        return torch.nn.functional.conv1d(x, wt.flip(-1)[:, None, :], groups=f).transpose(1, 2)

    ref = _autograd(conv, z, taps, grad_out=dzbar)
    got = causal_depthwise_conv_vjp(z, taps, dzbar)
    for r, g_ in zip(ref, got):
        np.testing.assert_allclose(g_, r, rtol=1e-12, atol=1e-13)


def test_rmsnorm_and_swiglu_vjps_match_autograd():
    from oracle.ttcd_oracle_grad import rms_norm_vjp, swiglu_vjp
    rng = np.random.default_rng(5)
    x, g, dy = rng.standard_normal((3, 4, 9)), 0.5 + rng.random(9), rng.standard_normal((3, 4, 9))
    ref = _autograd(lambda xt, gt: torch.nn.functional.rms_norm(xt, (9,), gt, eps=1e-6),
                    x, g, grad_out=dy)
    got = rms_norm_vjp(x, g, 1e-6, dy)
    for r, g_ in zip(ref, got):
        np.testing.assert_allclose(g_, r, rtol=1e-12, atol=1e-13)
    u, wg, wu = rng.standard_normal((2, 5, 6)), rng.standard_normal((7, 6)), \
        rng.standard_normal((7, 6))
    dz = rng.standard_normal((2, 5, 7))
    ref = _autograd(lambda ut, a, b: torch.nn.functional.silu(ut @ a.T) * (ut @ b.T),
                    u, wg, wu, grad_out=dz)
    got = swiglu_vjp(u, wg, wu, dz)
    for r, g_ in zip(ref, got):
        np.testing.assert_allclose(g_, r, rtol=1e-12, atol=1e-13)


# ------------------------------------------------ the fast-weight MLP on its own

MLP_NAMES = ["u_T", "u_S", "beta", "state_in", "w_gate", "w_up", "w_down", "w_proj", "conv_T",
             "conv_S"]


def _mlp_case(seed=0):
    x, beta, w, s0, g_out, g_state = _case(seed)
    rng = np.random.default_rng(seed + 50)
    args = {"u_T": rng.standard_normal((B, T, D)), "u_S": rng.standard_normal((B, T, D)),
            "beta": beta, "state_in": s0,
            **{k: w[k] for k in ("w_gate", "w_up", "w_down", "w_proj", "conv_T", "conv_S")}}
    return args, g_out, g_state


def _mlp_loss(a, g_y, g_state):
    r = orc.fastweight_mlp(a["u_T"], a["u_S"], a["beta"], a["w_gate"], a["w_up"], a["w_down"],
                           a["w_proj"], a["conv_T"], a["conv_S"], SHAPE["chunk"], 1e-6,
                           state_in=a["state_in"])
    loss = np.sum(g_y * r["y"])
    if g_state is not None:
        loss += np.sum(g_state * r["state_out"])
    return loss


@pytest.mark.parametrize("with_state", [True, False], ids=["state", "no_state"])
@pytest.mark.parametrize("name", MLP_NAMES)
def test_mlp_backward_matches_central_difference(name, with_state):
    """fastweight_mlp_backward against central differences of fastweight_mlp
    (the review's 关键设计 2-3 forward) along a random direction."""
    from oracle.ttcd_oracle_grad import fastweight_mlp_backward
    args, g_y, g_state = _mlp_case()
    if not with_state:
        g_state = None
    grads = fastweight_mlp_backward(
        args["u_T"], args["u_S"], args["beta"], args["w_gate"], args["w_up"], args["w_down"],
        args["w_proj"], args["conv_T"], args["conv_S"], SHAPE["chunk"], 1e-6, g_y,
        state_in=args["state_in"], d_state_out=g_state)
    v = np.random.default_rng(200 + MLP_NAMES.index(name)).standard_normal(args[name].shape)
    eps = 1e-6

    def at(delta):
        a = dict(args)
        a[name] = args[name] + delta * v
        return _mlp_loss(a, g_y, g_state)

    fd = (at(eps) - at(-eps)) / (2 * eps)
    an = float(np.sum(grads[name] * v))
    assert grads[name].shape == args[name].shape
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (fd, an)
