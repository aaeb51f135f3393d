"""GPU parity of the fused dual-window attention against the float64 oracle.

Definition: GitHub README "TTCD", section "Fused inference kernels"; podcast
cue 19 (a window of w keys ends at the query).  Tolerance for bf16 outputs:
max|d| / max|ref| <= 1e-2; index masks bit-exact.
"""
import numpy as np
import pytest
import torch

from oracle import ttcd_oracle as orc
from tests.helpers import TOL_OUT, np64, rel_max
from ttcd_workloads import make_attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ttcd():
    import dual_window_attention_b200 as m
    m.load_library()
    return m


CASES = [
    # B, T, Hq, Hkv, hd, w_S, w_T
    (1, 256, 2, 1, 32, 16, 64),        # tiny workload head layout
    (1, 1000, 4, 2, 64, 100, 300),     # ragged T, windows not multiples of the tile
    (2, 700, 4, 1, 128, 128, 512),     # batch 2, tile-aligned windows, GQA 4:1
    (1, 640, 3, 3, 128, 1, 1000),      # student window 1, teacher window > T
    (1, 513, 2, 2, 64, 200, 200),      # equal windows
    (1, 300, 6, 2, 32, 33, 129),       # hd 32, GQA 3:1
]


@pytest.mark.parametrize("B,T,Hq,Hkv,hd,wS,wT", CASES)
def test_dual_window_attention_parity(ttcd, B, T, Hq, Hkv, hd, wS, wT):
    q, k, v = make_attention_inputs(B, T, Hq, Hkv, hd, seed=T + hd)
    o_T, o_S, lse_T, lse_S = ttcd.dual_window_attn(q.cuda(), k.cuda(), v.cuda(), wS, wT, lse=True)
    torch.cuda.synchronize()
    assert ttcd.get_device_error()[0] == ttcd.OK
    rT, rS, rlT, rlS = orc.dual_window_attention(np64(q), np64(k), np64(v), wS, wT, hd ** -0.5)
    assert rel_max(o_T, rT) <= TOL_OUT
    assert rel_max(o_S, rS) <= TOL_OUT
    np.testing.assert_allclose(np64(lse_T), rlT, atol=2e-3, rtol=0)
    np.testing.assert_allclose(np64(lse_S), rlS, atol=2e-3, rtol=0)


@pytest.mark.parametrize("w", [1, 16, 100, 128, 300])
def test_mask_probe_key_counts_bit_exact(ttcd, w):
    """Q = 0: every visible key gets weight 1, so exp(lse[t]) counts the window exactly."""
    B, T, H, hd = 1, 600, 1, 64
    q = torch.zeros(B, T, H, hd, dtype=torch.bfloat16, device="cuda")
    _, k, v = make_attention_inputs(B, T, H, H, hd, seed=1)
    _, _, lse_T, lse_S = ttcd.dual_window_attn(q, k.cuda(), v.cuda(), w, max(w, 200), lse=True)
    counts_S = np.minimum(np.arange(T) + 1, w)
    counts_T = np.minimum(np.arange(T) + 1, max(w, 200))
    np.testing.assert_array_equal(np.rint(np.exp(np64(lse_S)[0, 0])), counts_S)
    np.testing.assert_array_equal(np.rint(np.exp(np64(lse_T)[0, 0])), counts_T)


@pytest.mark.parametrize("j", [0, 5, 127, 128, 255, 400])
def test_mask_probe_one_hot_value_bit_exact(ttcd, j):
    """V one-hot at key j: o[t] is nonzero exactly for the queries whose window holds j."""
    B, T, H, hd, wS, wT = 1, 512, 1, 64, 37, 160
    q = torch.zeros(B, T, H, hd, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros_like(q)
    v = torch.zeros_like(q)
    v[0, j, 0, 0] = 1.0
    o_T, o_S, _, _ = ttcd.dual_window_attn(q, k, v, wS, wT)
    t = np.arange(T)
    for o, w in ((o_S, wS), (o_T, wT)):
        seen = np64(o)[0, :, 0, 0] != 0
        np.testing.assert_array_equal(seen, (j <= t) & (j >= t - w + 1))


@pytest.fixture(scope="module")
def sweep_inputs():
    """Q, K, V ~ N(0, 1) at the Qwen3-0.6B head layout, T = 65536 (the attention sweep)."""
    from ttcd_workloads import ATTN_SWEEP_T
    q, k, v = make_attention_inputs(1, ATTN_SWEEP_T, 16, 8, 128, seed=0)
    return (q, k, v), (q.cuda(), k.cuda(), v.cuda()), (np64(q), np64(k), np64(v))


def _sampled_rows_error(o_dev, qkv64, w, rows, rng):
    """max|d| / max|ref| of sampled rows (two random heads per row) against the oracle's
    row-at-a-time windowed attention."""
    qn, kn, vn = qkv64
    got = np64(o_dev)
    Hq, hd = qn.shape[2], qn.shape[3]
    err = refmax = 0.0
    for t in rows:
        for h in rng.choice(Hq, 2, replace=False):
            ref, _ = orc.windowed_attention_row(qn, kn, vn, w, hd ** -0.5, 0, int(t), int(h))
            err = max(err, float(np.max(np.abs(got[0, t, h] - ref))))
            refmax = max(refmax, float(np.max(np.abs(ref))))
    return err / refmax


def _rows(T, w_S, w_T, rng):
    edges = [0, 1, 127, 128, w_S - 1, w_S, w_T - 1, w_T, T - 1]
    return np.unique(np.concatenate([[e for e in edges if 0 <= e < T], rng.integers(0, T, 24)]))


def test_full_size_sampled_rows(ttcd, sweep_inputs):
    """T = 65536, 16/8 heads, hd 128, w_S 512, w_T 8192 (the block's windows): sampled
    rows of both outputs against the oracle."""
    _, (q, k, v), qkv64 = sweep_inputs
    o_T, o_S, _, _ = ttcd.dual_window_attn(q, k, v, 512, 8192)
    torch.cuda.synchronize()
    assert ttcd.get_device_error()[0] == ttcd.OK
    rng = np.random.default_rng(0)
    rows = _rows(q.shape[1], 512, 8192, rng)
    assert _sampled_rows_error(o_T, qkv64, 8192, rows, rng) <= TOL_OUT
    assert _sampled_rows_error(o_S, qkv64, 512, rows, rng) <= TOL_OUT
    assert torch.isfinite(o_T).all() and torch.isfinite(o_S).all()


@pytest.mark.parametrize("w_T", [4096, 8192, 16384])
@pytest.mark.parametrize("w_S", [256, 512, 1024, 2048])
def test_window_sweep_full_size_sampled_rows(ttcd, sweep_inputs, w_S, w_T):
    """The attention sweep at T = 65536 (w_S in {256..2048} x w_T in {4096..16384}):
    sampled rows, including the rows where either window fills, against the oracle."""
    _, (q, k, v), qkv64 = sweep_inputs
    o_T, o_S, _, _ = ttcd.dual_window_attn(q, k, v, w_S, w_T)
    torch.cuda.synchronize()
    assert ttcd.get_device_error()[0] == ttcd.OK
    rng = np.random.default_rng(w_S + w_T)
    rows = _rows(q.shape[1], w_S, w_T, rng)
    assert _sampled_rows_error(o_T, qkv64, w_T, rows, rng) <= TOL_OUT
    assert _sampled_rows_error(o_S, qkv64, w_S, rows, rng) <= TOL_OUT
    assert torch.isfinite(o_T).all() and torch.isfinite(o_S).all()


# ---------------------------------------------------------------------- LSE combination form
@pytest.mark.parametrize("B,T,Hq,Hkv,hd,wS,wT", CASES)
def test_lse_combination_parity(ttcd, B, T, Hq, Hkv, hd, wS, wT):
    """ttcd_dual_window_attn_lse (student window + far band merged through the
    log-sum-exp; README "Fused inference kernels", lse_dual_attn) against the
    oracle: both windows, the far band, and every lse; an empty far band is
    exactly o = 0, lse = -inf."""
    q, k, v = make_attention_inputs(B, T, Hq, Hkv, hd, seed=T + hd)
    o_T, o_S, o_far, lse_T, lse_S, lse_far = ttcd.dual_window_attn_lse(q.cuda(), k.cuda(),
                                                                       v.cuda(), wS, wT)
    torch.cuda.synchronize()
    assert ttcd.get_device_error()[0] == ttcd.OK
    qn, kn, vn = np64(q), np64(k), np64(v)
    scale = hd ** -0.5
    rT, rS, rlT, rlS = orc.dual_window_attention(qn, kn, vn, wS, wT, scale)
    rF, rlF = orc.band_attention(qn, kn, vn, wS, wT - 1, scale)
    assert rel_max(o_T, rT) <= TOL_OUT
    assert rel_max(o_S, rS) <= TOL_OUT
    empty = np.isneginf(rlF)
    lf = np64(lse_far)
    assert np.array_equal(np.isneginf(lf), empty)
    np.testing.assert_allclose(lf[~empty], rlF[~empty], atol=2e-3, rtol=0)
    of = np64(o_far)
    assert np.all(of.transpose(0, 2, 1, 3)[empty] == 0)
    if (~empty).any():
        assert rel_max(of.transpose(0, 2, 1, 3)[~empty], rF.transpose(0, 2, 1, 3)[~empty]) <= TOL_OUT
    np.testing.assert_allclose(np64(lse_T), rlT, atol=2e-3, rtol=0)
    np.testing.assert_allclose(np64(lse_S), rlS, atol=2e-3, rtol=0)
    # the two implementations agree with each other
    f_T, f_S, _, _ = ttcd.dual_window_attn(q.cuda(), k.cuda(), v.cuda(), wS, wT)
    assert rel_max(o_T, f_T) <= TOL_OUT and torch.equal(o_S, f_S)


def test_lse_combination_full_size(ttcd, sweep_inputs):
    """T = 65536, Qwen3 heads, 512/8192: the LSE form against the fused form and,
    on sampled rows, against the oracle."""
    _, (q, k, v), qkv64 = sweep_inputs
    o_T, o_S, o_far, _, _, lse_far = ttcd.dual_window_attn_lse(q, k, v, 512, 8192)
    f_T, f_S, _, _ = ttcd.dual_window_attn(q, k, v, 512, 8192)
    torch.cuda.synchronize()
    assert ttcd.get_device_error()[0] == ttcd.OK
    assert rel_max(o_T, f_T) <= TOL_OUT and torch.equal(o_S, f_S)
    rng = np.random.default_rng(3)
    rows = _rows(q.shape[1], 512, 8192, rng)
    assert _sampled_rows_error(o_T, qkv64, 8192, rows, rng) <= TOL_OUT
    assert torch.isneginf(lse_far[:, :, :512]).all() and (o_far[:, :512] == 0).all()
    assert torch.isfinite(lse_far[:, :, 512:]).all()
