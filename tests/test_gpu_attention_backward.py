"""GPU parity of ttcd_dual_window_attn_backward against the float64 oracle's
windowed_attention_vjp (pinned against library SDPA autograd in
test_oracle_grad.py), summed over the two windows.

papernotes.org review "Learning What to Remember", 局限与展望 (training runs both
attention windows); podcast cue 19 (a window of w keys ends at the query).

Tolerance: dq, dk, dv within relative Frobenius 1e-2 of the oracle's.  The
kernel rebuilds P from the forward's log-sum-exp and rounds P and dS to bf16
(relative 2^-9 each, about 2.3e-3 rms), and its delta = rowsum(dO o) uses the
forward's bf16 o (another 2^-9 relative per element); the products dV = P^T dO,
dK = dS^T Q, dQ = dS K carry one or two such roundings, about 3e-3 rms, and the
bound leaves a factor 3 for the cancellation in dP - delta.
"""
import numpy as np
import pytest
import torch

from oracle.ttcd_oracle_grad import windowed_attention_vjp
from tests.helpers import np64, rel_fro
from ttcd_workloads import make_attention_inputs

pytestmark = pytest.mark.gpu

TOL_GRAD = 1e-2

CASES = [
    # B, T, Hq, Hkv, hd, w_S, w_T
    (2, 700, 4, 2, 64, 40, 300),       # ragged T, windows not multiples of the tile
    (1, 520, 4, 1, 128, 128, 256),     # tile-aligned windows, GQA 4:1
    (1, 333, 2, 2, 128, 1, 1000),      # student window 1, teacher window > T
    (1, 400, 2, 1, 64, 150, 150),      # equal windows
    (2, 260, 6, 3, 128, 77, 129),      # GQA 2:1, three KV heads
]


@pytest.fixture(scope="module")
def ttcd():
    import dual_window_attention_b200 as m
    m.load_library()
    return m


@pytest.mark.parametrize("B,T,Hq,Hkv,hd,wS,wT", CASES)
def test_attention_backward_parity(ttcd, B, T, Hq, Hkv, hd, wS, wT):
    q, k, v = make_attention_inputs(B, T, Hq, Hkv, hd, seed=T + 7 * hd)
    g = torch.Generator().manual_seed(T)
    do_T = torch.randn(B, T, Hq, hd, generator=g).to(torch.bfloat16)
    do_S = torch.randn(B, T, Hq, hd, generator=g).to(torch.bfloat16)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o_T, o_S, lse_T, lse_S = ttcd.dual_window_attn(qc, kc, vc, wS, wT, lse=True)
    dq, dk, dv, ws = ttcd.dual_window_attn_backward(qc, kc, vc, o_T, o_S, lse_T, lse_S,
                                                   do_T.cuda(), do_S.cuda(), wS, wT)
    torch.cuda.synchronize()
    assert ttcd.check_device_status(ws) == ttcd.OK
    scale = 1.0 / np.sqrt(hd)
    rq, rk, rv = windowed_attention_vjp(np64(q), np64(k), np64(v), wT, scale, np64(do_T))
    sq, sk, sv = windowed_attention_vjp(np64(q), np64(k), np64(v), wS, scale, np64(do_S))
    errs = {"dq": rel_fro(dq, rq + sq), "dk": rel_fro(dk, rk + sk), "dv": rel_fro(dv, rv + sv)}
    print(f"\nB{B} T{T} Hq{Hq} Hkv{Hkv} hd{hd} w {wS}/{wT}: " +
          ", ".join(f"{n} {e:.2e}" for n, e in errs.items()))
    for n, e in errs.items():
        assert e <= TOL_GRAD, (n, e)
