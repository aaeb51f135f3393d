"""Pins for the oracle's elementwise steps and fast-weight MLP (CPU only).

Sources: papernotes.org review "Learning What to Remember: Test-Time Training
via Context Distillation" (方法详解, 关键设计 1-4) and the podcast transcript
(cues 23, 27, 29).  Each test checks the oracle against a library routine, a
closed form, an independent sequential form, or an identity the pages state.
"""
import numpy as np
import pytest
import torch

from oracle import ttcd_oracle as orc

RNG = np.random.default_rng(1234)


def _r(*shape):
    return RNG.standard_normal(shape)


# ----------------------------------------------------------------- elementwise


def test_rms_norm_matches_torch():
    x = _r(3, 5, 17)
    g = _r(17)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (17,), torch.from_numpy(g), eps=1e-6)
    np.testing.assert_allclose(orc.rms_norm(x, g, 1e-6), ref.numpy(), rtol=1e-13)


def test_rms_norm_unit_rms_and_scale_invariance():
    x = _r(4, 64)
    y = orc.rms_norm(x, np.ones(64), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, -1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(orc.rms_norm(7.5 * x, np.ones(64), 0.0), y, rtol=1e-13)


@pytest.mark.parametrize("hd", [2, 8, 32, 128])
def test_rope_is_complex_rotation(hd):
    """Pair (x_i, x_{i+hd/2}) as x_i + i x_{i+hd/2}, multiplied by exp(i t theta^(-2i/hd))."""
    B, T, H = 2, 11, 3
    x = _r(B, T, H, hd)
    out = orc.rope(x, 10000.0)
    half = hd // 2
    z = x[..., :half] + 1j * x[..., half:]
    ang = np.outer(np.arange(T), 10000.0 ** (-2.0 * np.arange(half) / hd))
    zr = z * np.exp(1j * ang)[None, :, None, :]
    np.testing.assert_allclose(out[..., :half], zr.real, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out[..., half:], zr.imag, rtol=1e-12, atol=1e-12)


def test_rope_relative_position():
    hd, T = 16, 40
    qv, kv = _r(hd), _r(hd)
    q = orc.rope(np.broadcast_to(qv, (1, T, 1, hd)).copy(), 10000.0)[0, :, 0]
    k = orc.rope(np.broadcast_to(kv, (1, T, 1, hd)).copy(), 10000.0)[0, :, 0]
    np.testing.assert_array_equal(q[0], qv)  # position 0 is the identity
    for shift in (1, 7, 20):
        np.testing.assert_allclose(q[10] @ k[3], q[10 + shift] @ k[3 + shift], rtol=1e-10)


def test_swiglu_matches_torch():
    u, wg, wu = _r(2, 9, 12), _r(20, 12), _r(20, 12)
    tu = torch.from_numpy(u)
    ref = torch.nn.functional.silu(tu @ torch.from_numpy(wg).T) * (tu @ torch.from_numpy(wu).T)
    np.testing.assert_allclose(orc.swiglu(u, wg, wu), ref.numpy(), rtol=1e-13)


@pytest.mark.parametrize("k", [1, 2, 4, 8])
def test_causal_conv_matches_torch_conv1d(k):
    B, T, f = 2, 19, 6
    z, taps = _r(B, T, f), _r(f, k)
    # conv1d is a correlation: weight index (k-1-m) meets input t-m after left padding k-1.
    ref = torch.nn.functional.conv1d(
        torch.nn.functional.pad(torch.from_numpy(z).transpose(1, 2), (k - 1, 0)),
        torch.from_numpy(taps[:, ::-1].copy())[:, None, :], groups=f).transpose(1, 2)
    np.testing.assert_allclose(orc.causal_depthwise_conv(z, taps), ref.numpy(), rtol=1e-12,
                               atol=1e-14)


def test_causal_conv_identity_and_shift():
    z = _r(1, 10, 3)
    ident = np.zeros((3, 4))
    ident[:, 0] = 1.0
    np.testing.assert_array_equal(orc.causal_depthwise_conv(z, ident), z)
    shift = np.zeros((3, 4))
    shift[:, 2] = 1.0
    out = orc.causal_depthwise_conv(z, shift)
    np.testing.assert_array_equal(out[:, 2:], z[:, :-2])
    np.testing.assert_array_equal(out[:, :2], 0.0)


def test_l2_normalize_rows():
    z = _r(3, 7, 11)
    k = orc.l2_normalize_rows(z, 0.0)
    np.testing.assert_allclose(np.linalg.norm(k, axis=-1), 1.0, rtol=1e-14)
    ref = torch.nn.functional.normalize(torch.from_numpy(z), dim=-1)
    np.testing.assert_allclose(k, ref.numpy(), rtol=1e-13)
    zero = np.zeros((1, 2, 5))
    np.testing.assert_array_equal(orc.l2_normalize_rows(zero, 1e-6), 0.0)


# ----------------------------------------------------------------- fast weights


def _mlp_case(B=2, T=70, d=6, f=10, k=4, seed=0):
    rng = np.random.default_rng(seed)
    w = dict(w_gate=rng.standard_normal((f, d)) / np.sqrt(d),
             w_up=rng.standard_normal((f, d)) / np.sqrt(d),
             w_down=rng.standard_normal((d, f)) / np.sqrt(f),
             w_proj=rng.standard_normal((f, f)) / np.sqrt(f),
             conv_T=rng.standard_normal((f, k)) * 0.5,
             conv_S=rng.standard_normal((f, k)) * 0.5)
    u_S = rng.standard_normal((B, T, d))
    u_T = u_S + 0.3 * rng.standard_normal((B, T, d))
    beta = 0.1 / (1 + np.exp(-rng.standard_normal((B, T))))
    h_S = rng.standard_normal((B, T, d))
    return u_T, u_S, beta, h_S, w


def _run(u_T, u_S, beta, h_S, w, chunk, **kw):
    return orc.fastweight_mlp(u_T, u_S, beta, w["w_gate"], w["w_up"], w["w_down"], w["w_proj"],
                              w["conv_T"], w["conv_S"], chunk, 1e-6, h_S=h_S, **kw)


def test_equal_views_and_convs_give_no_write_and_plain_mlp():
    u_T, u_S, beta, h_S, w = _mlp_case()
    w["conv_T"] = w["conv_S"].copy()
    res = _run(u_S, u_S, beta, h_S, w, chunk=16)
    assert np.all(res["D"] == 0) and np.all(res["R"] == 0) and np.all(res["dW"] == 0)
    tu = torch.from_numpy(u_S)
    z = torch.nn.functional.silu(tu @ torch.from_numpy(w["w_gate"]).T) * (tu @ torch.from_numpy(w["w_up"]).T)
    plain = torch.from_numpy(h_S) + z @ torch.from_numpy(w["w_down"]).T
    np.testing.assert_allclose(res["out"], plain.numpy(), rtol=1e-12, atol=1e-12)


def test_beta_zero_is_static_mlp():
    u_T, u_S, beta, h_S, w = _mlp_case()
    res = _run(u_T, u_S, np.zeros_like(beta), h_S, w, chunk=16)
    np.testing.assert_allclose(res["y"], orc.swiglu(u_S, w["w_gate"], w["w_up"]) @ w["w_down"].T,
                               rtol=1e-12, atol=1e-13)
    assert np.all(res["state_out"] == 0)


def test_zero_student_conv_gives_zero_keys_and_no_write():
    u_T, u_S, beta, h_S, w = _mlp_case()
    w["conv_S"] = np.zeros_like(w["conv_S"])
    res = _run(u_T, u_S, beta, h_S, w, chunk=16)
    assert np.all(res["K"] == 0) and np.all(res["dW"] == 0) and np.all(res["state_out"] == 0)


def test_identity_convs_and_proj_give_down_projected_difference():
    u_T, u_S, beta, h_S, w = _mlp_case()
    ident = np.zeros_like(w["conv_T"])
    ident[:, 0] = 1.0
    w.update(conv_T=ident, conv_S=ident.copy(), w_proj=np.eye(w["w_proj"].shape[0]))
    res = _run(u_T, u_S, beta, h_S, w, chunk=16)
    ref = (orc.swiglu(u_T, w["w_gate"], w["w_up"]) - orc.swiglu(u_S, w["w_gate"], w["w_up"])) @ w["w_down"].T
    np.testing.assert_allclose(res["R"], ref, rtol=1e-12, atol=1e-13)


def test_value_residual_basis_probe():
    """r is linear in the difference d_t = zbar_T - zbar_S; a unit difference e_j
    gives column j of the map, W_down (W_proj e_j) = W_down @ W_proj[:, j] (R12),
    and the opposite difference gives its negative (R4)."""
    rng = np.random.default_rng(5)
    d, f = 3, 7
    w_down, w_proj = rng.standard_normal((d, f)), rng.standard_normal((f, f))
    eye = np.eye(f)[None]  # token j carries e_j
    zero = np.zeros_like(eye)
    r = orc.value_residual(eye, zero, w_down, w_proj)[0]
    for j in range(f):
        np.testing.assert_allclose(r[j], w_down @ w_proj[:, j], rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(orc.value_residual(zero, eye, w_down, w_proj)[0], -r)


@pytest.mark.parametrize("chunk", [1, 7, 16, 70, 100])
def test_parallel_prefix_equals_sequential_recurrence(chunk):
    """Off-policy parallel form == chunk-by-chunk loop with frozen activations."""
    u_T, u_S, beta, h_S, w = _mlp_case()
    state_in = 0.01 * RNG.standard_normal((2, 6, 10))
    res = _run(u_T, u_S, beta, h_S, w, chunk=chunk, state_in=state_in)
    zs, r, key = res["Z_S"], res["R"], res["K"]
    B, T, _ = zs.shape
    for b in range(B):
        W = w["w_down"] + state_in[b]
        for s0 in range(0, T, chunk):
            s1 = min(T, s0 + chunk)
            for t in range(s0, s1):  # read with the weight as it stood before this chunk
                np.testing.assert_allclose(res["y"][b, t], W @ zs[b, t], rtol=1e-11, atol=1e-12)
            for t in range(s0, s1):  # then write this chunk's rank-one terms
                W = W + beta[b, t] * np.outer(r[b, t], key[b, t])
        np.testing.assert_allclose(res["state_out"][b], W - w["w_down"], rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("s", [0, 15, 16, 40, 69])
def test_chunk_mask_probe(s):
    """A write at token s is read exactly by the tokens of later chunks."""
    chunk = 16
    u_T, u_S, _, h_S, w = _mlp_case(B=1)
    T = u_T.shape[1]
    base = _run(u_T, u_S, np.zeros((1, T)), h_S, w, chunk=chunk)
    beta = np.zeros((1, T))
    beta[0, s] = 0.5
    pert = _run(u_T, u_S, beta, h_S, w, chunk=chunk)
    changed = np.any(pert["out"][0] != base["out"][0], axis=-1)
    t = np.arange(T)
    np.testing.assert_array_equal(changed, t // chunk > s // chunk)


def test_write_is_negative_gradient_of_distillation_loss():
    """Eq. 4 -> Eq. 6: with identity convs, W_proj = I, raw keys and beta = 1/|C_i|,
    the chunk write equals minus the gradient of the distillation loss."""
    rng = np.random.default_rng(7)
    C, d, f = 9, 5, 8
    w_down = rng.standard_normal((d, f))
    z_T, z_S = rng.standard_normal((C, f)), rng.standard_normal((C, f))
    r = orc.value_residual(z_T[None], z_S[None], w_down, np.eye(f))
    dW = orc.chunk_increments(r, z_S[None], np.full((1, C), 1.0 / C), C)[0, 0]
    y_T = z_T @ w_down.T  # teacher output, detached
    grad = np.zeros_like(w_down)
    eps = 1e-6
    for a in range(d):
        for c in range(f):
            wp, wm = w_down.copy(), w_down.copy()
            wp[a, c] += eps
            wm[a, c] -= eps
            grad[a, c] = (orc.distillation_loss(wp, z_S, y_T) - orc.distillation_loss(wm, z_S, y_T)) / (2 * eps)
    np.testing.assert_allclose(dW, -grad, rtol=1e-7, atol=1e-8)


def test_proposition_one_single_orthogonal_write():
    """One write at q1 moves the student output at a later q2 by eta*c_gap*c_align
    along the teacher output (equality for a single orthogonal write)."""
    rng = np.random.default_rng(3)
    d, f, C, eta = 4, 6, 4, 0.7
    w_down = rng.standard_normal((d, f))
    basis = np.linalg.qr(rng.standard_normal((f, f)))[0].T  # orthonormal rows
    T = 2 * C
    z_S = np.zeros((1, T, f))
    q1, q2 = 1, C + 2
    z_S[0, q1] = basis[0]                       # unit student activation at q1
    c_align = 0.6
    z_S[0, q2] = c_align * basis[0] + 0.8 * basis[1]
    z_T = z_S.copy()
    z_T[0, q1] = basis[0] + 0.9 * basis[2] - 0.3 * basis[0]
    r = orc.value_residual(z_T, z_S, w_down, np.eye(f))
    key = orc.l2_normalize_rows(z_S, 1e-300)  # unit rows stay exact, zero rows stay 0
    beta = np.zeros((1, T))
    beta[0, q1] = eta
    prefixes, _ = orc.exclusive_prefix(orc.chunk_increments(r, key, beta, C))
    y_T_q1 = w_down @ z_T[0, q1]
    y_S_q1 = w_down @ z_S[0, q1]
    c_gap = float(y_T_q1 @ (y_T_q1 - y_S_q1))
    dy_q2 = prefixes[0, q2 // C] @ z_S[0, q2]
    np.testing.assert_allclose(float(y_T_q1 @ dy_q2), eta * c_gap * c_align, rtol=1e-12)
    assert np.all(prefixes[0, 0] == 0)  # q1's own chunk does not see the write
