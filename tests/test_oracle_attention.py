"""Pins for the oracle's attention (CPU only).

Each test ties the blocked float64 oracle to something other than itself:
per-token brute-force loops, a textbook library routine (torch SDPA in
float64), closed forms of degenerate windows, the log-sum-exp combination
identity of the LSE dual-attention variant (GitHub README "TTCD", section
"Fused inference kernels", lse_dual_attn), and index-mask probes.
"""
import numpy as np
import pytest
import torch

from oracle import ttcd_oracle as orc
from ttcd_workloads import TINY_F32, make_attention_inputs


def _rand_qkv(B, T, Hq, Hkv, hd, seed):
    q, k, v = make_attention_inputs(B, T, Hq, Hkv, hd, seed=seed, dtype=torch.float32)
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


@pytest.mark.parametrize("B,T,Hq,Hkv,hd,w", [
    (1, 256, 2, 1, 32, 16),   # tiny workload, student window
    (1, 256, 2, 1, 32, 64),   # tiny workload, teacher window
    (2, 37, 3, 1, 8, 5),      # odd sizes, ragged block tail, batch 2
    (1, 70, 4, 2, 16, 70),    # window == T
    (1, 300, 2, 2, 4, 129),   # window crosses a 256-row query block
])
def test_blocked_matches_bruteforce(B, T, Hq, Hkv, hd, w):
    q, k, v = _rand_qkv(B, T, Hq, Hkv, hd, seed=T + w)
    scale = hd ** -0.5
    o, lse = orc.windowed_attention(q, k, v, w, scale)
    ob, lseb = orc.windowed_attention_bruteforce(q, k, v, w, scale)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lseb, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("w", [50, 64, 1000])
def test_window_at_least_T_is_full_causal_sdpa(w):
    B, T, Hq, Hkv, hd = 2, 50, 4, 2, 16
    q, k, v = _rand_qkv(B, T, Hq, Hkv, hd, seed=3)
    o, _ = orc.windowed_attention(q, k, v, w, hd ** -0.5)
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    tv = torch.from_numpy(v).repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-10, atol=1e-12)


def test_window_one_returns_own_value():
    B, T, Hq, Hkv, hd = 1, 40, 4, 2, 8
    q, k, v = _rand_qkv(B, T, Hq, Hkv, hd, seed=5)
    o, lse = orc.windowed_attention(q, k, v, 1, 0.3)
    for h in range(Hq):
        np.testing.assert_array_equal(o[:, :, h], v[:, :, h // 2])
        np.testing.assert_allclose(lse[:, h], 0.3 * np.sum(q[:, :, h] * k[:, :, h // 2], -1),
                                   rtol=1e-13)


def test_gqa_head_mapping():
    B, T, Hq, Hkv, hd = 1, 33, 6, 2, 8
    q, k, v = _rand_qkv(B, T, Hq, Hkv, hd, seed=9)
    o, _ = orc.windowed_attention(q, k, v, 7, 0.5)
    for h in range(Hq):
        oh, _ = orc.windowed_attention_bruteforce(q[:, :, h:h + 1], k[:, :, h // 3:h // 3 + 1],
                                                  v[:, :, h // 3:h // 3 + 1], 7, 0.5)
        np.testing.assert_allclose(o[:, :, h], oh[:, :, 0], rtol=1e-12, atol=1e-13)


def test_lse_combination_identity():
    """Teacher = student band + far band, merged through their log-sum-exp."""
    B, T, Hq, Hkv, hd, wS, wT = 1, 90, 2, 1, 8, 7, 30
    q, k, v = _rand_qkv(B, T, Hq, Hkv, hd, seed=11)
    scale = hd ** -0.5
    oT, oS, lT, lS = orc.dual_window_attention(q, k, v, wS, wT, scale)
    for h in range(Hq):
        for t in range(T):
            far = list(range(max(0, t - wT + 1), max(0, t - wS + 1)))
            if not far:
                np.testing.assert_allclose(oT[0, t, h], oS[0, t, h], rtol=1e-12, atol=1e-14)
                continue
            s = np.array([scale * q[0, t, h] @ k[0, j, 0] for j in far])
            lfar = np.log(np.sum(np.exp(s - s.max()))) + s.max()
            ofar = (np.exp(s - lfar)[:, None] * v[0, far, 0]).sum(0)
            merged = np.logaddexp(lS[0, h, t], lfar)
            np.testing.assert_allclose(lT[0, h, t], merged, rtol=1e-12)
            comb = np.exp(lS[0, h, t] - merged) * oS[0, t, h] + np.exp(lfar - merged) * ofar
            np.testing.assert_allclose(oT[0, t, h], comb, rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("w", [1, 16, 64, 300])
def test_mask_probe_lse_counts_keys(w):
    """Q = 0 gives equal scores, so exp(lse[t]) is the number of visible keys."""
    B, T, hd = 1, 256, 8
    q = np.zeros((B, T, 1, hd))
    _, k, v = _rand_qkv(B, T, 1, 1, hd, seed=1)
    _, lse = orc.windowed_attention(q, k, v, w, 1.0)
    counts = np.minimum(np.arange(T) + 1, w)
    np.testing.assert_allclose(np.exp(lse[0, 0]), counts, rtol=1e-13)


@pytest.mark.parametrize("w", [1, 16, 64])
def test_mask_probe_one_hot_value(w):
    """V one-hot at key j: O[t] is nonzero exactly when j is in t's window."""
    T, hd = 128, 4
    q = np.zeros((1, T, 1, hd))
    k = np.zeros((1, T, 1, hd))
    for j in (0, 5, 63, 64, 127):
        v = np.zeros((1, T, 1, hd))
        v[0, j, 0, 0] = 1.0
        o, _ = orc.windowed_attention(q, k, v, w, 1.0)
        seen = o[0, :, 0, 0] != 0
        t = np.arange(T)
        np.testing.assert_array_equal(seen, (j <= t) & (j >= t - w + 1))
        np.testing.assert_allclose(o[0, seen, 0, 0], 1.0 / np.minimum(t[seen] + 1, w), rtol=1e-14)


def test_tiny_workload_dual_windows_bruteforce():
    s = TINY_F32
    q, k, v = _rand_qkv(s.B, s.T, s.n_q_heads, s.n_kv_heads, s.head_dim, seed=0)
    oT, oS, lT, lS = orc.dual_window_attention(q, k, v, s.w_S, s.w_T, s.softmax_scale)
    bT, blT = orc.windowed_attention_bruteforce(q, k, v, s.w_T, s.softmax_scale)
    bS, blS = orc.windowed_attention_bruteforce(q, k, v, s.w_S, s.softmax_scale)
    np.testing.assert_allclose(oT, bT, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(oS, bS, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lT, blT, rtol=1e-12)
    np.testing.assert_allclose(lS, blS, rtol=1e-12)


def test_single_row_matches_bruteforce():
    """The row-at-a-time form used for sampled checks of long sequences equals
    the per-query loop on every row of a small GQA case (2 sequences, ragged
    windows, rows before and after the window fills)."""
    g = np.random.default_rng(7)
    B, T, Hq, Hkv, hd, w = 2, 40, 6, 2, 8, 13
    q, k, v = (g.standard_normal((B, T, H, hd)) for H in (Hq, Hkv, Hkv))
    o, lse = orc.windowed_attention_bruteforce(q, k, v, w, 0.3)
    for b in range(B):
        for t in (0, 1, 12, 13, 39):
            for h in range(Hq):
                orow, l = orc.windowed_attention_row(q, k, v, w, 0.3, b, t, h)
                np.testing.assert_allclose(orow, o[b, t, h], rtol=1e-12, atol=1e-12)
                assert abs(l - lse[b, h, t]) < 1e-12


def test_band_attention_special_cases():
    """near = 0, far = w - 1 is the sliding window of w keys; a band that lies
    before the sequence start is empty (o = 0, lse = -inf)."""
    q, k, v = _rand_qkv(1, 50, 4, 2, 8, seed=21)
    for w in (1, 7, 50):
        o, lse = orc.band_attention(q, k, v, 0, w - 1, 0.4)
        ow, lsew = orc.windowed_attention(q, k, v, w, 0.4)
        np.testing.assert_allclose(o, ow, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, lsew, rtol=1e-12, atol=1e-12)
    o, lse = orc.band_attention(q, k, v, 10, 20, 0.4)
    assert np.all(o[:, :10] == 0) and np.all(np.isneginf(lse[:, :, :10]))
    assert np.all(np.isfinite(lse[:, :, 10:]))


def test_far_band_matches_per_query_loop_and_merges_to_teacher():
    """The oracle's far band [t-w_T+1, t-w_S] against an explicit per-query
    loop, and lse_merge(student window, far band) against the teacher window."""
    B, T, Hq, Hkv, hd, wS, wT = 2, 70, 4, 2, 8, 9, 33
    q, k, v = _rand_qkv(B, T, Hq, Hkv, hd, seed=5)
    scale = hd ** -0.5
    of, lf = orc.band_attention(q, k, v, wS, wT - 1, scale)
    for b in range(B):
        for h in range(Hq):
            for t in range(T):
                keys = list(range(max(0, t - wT + 1), t - wS + 1))
                if not keys:
                    assert np.isneginf(lf[b, h, t]) and np.all(of[b, t, h] == 0)
                    continue
                s = np.array([scale * q[b, t, h] @ k[b, j, h // 2] for j in keys])
                e = np.exp(s - s.max())
                np.testing.assert_allclose(of[b, t, h], (e[:, None] * v[b, keys, h // 2]).sum(0) / e.sum(),
                                           rtol=1e-12, atol=1e-13)
                np.testing.assert_allclose(lf[b, h, t], s.max() + np.log(e.sum()), rtol=1e-12)
    oT, oS, lT, lS = orc.dual_window_attention(q, k, v, wS, wT, scale)
    om, lm = orc.lse_merge(oS, lS, of, lf)
    np.testing.assert_allclose(om, oT, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lm, lT, rtol=1e-12)
