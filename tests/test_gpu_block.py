"""GPU parity of ttcd_block_forward (and each stage's intermediate) against the
float64 oracle on seeded synthetic inputs.

Block definition: papernotes.org review "Learning What to Remember", 方法详解
(flowchart A-F) and 关键设计 2-3.  Tolerances: outputs max|d|/max|ref| <= 1e-2,
fp32 fast-weight state relative Frobenius <= 5e-3.
"""
import numpy as np
import pytest
import torch

from tests.helpers import TOL_OUT, TOL_STATE, np64, oracle_block, rel_fro, rel_max, to_device
from ttcd_workloads import (QWEN3_0P6B_64K, SMOLLM2_360M_16K, TINY_F32, BlockShape,
                            make_block_inputs)

pytestmark = pytest.mark.gpu

SMALL_BF16 = BlockShape("small_bf16_ragged", "bf16", B=2, T=1000, d_model=128, n_q_heads=4,
                        n_kv_heads=2, head_dim=64, d_ff=256, w_S=64, w_T=256, chunk=128,
                        conv_k=4)
SMALL_BF16_C96 = SMALL_BF16.with_(name="small_bf16_chunk96", B=1, T=777, chunk=96, conv_k=3,
                                  head_dim=128, n_q_heads=2, n_kv_heads=1, w_S=100, w_T=500)


@pytest.fixture(scope="module")
def ttcd():
    import dual_window_attention_b200 as m
    m.load_library()
    return m


def _run(ttcd, shape, inp, layer=0):
    p = ttcd.BlockParams.from_shape(shape)
    x, w = to_device(inp, layer)
    out, state, ws = ttcd.block_forward(x, w["beta"], w, p, state_out=True)
    assert ttcd.check_device_status(ws) == ttcd.OK
    return p, out, state, ws


def _stage_checks(ttcd, p, ws, ref, shape, weights=None):
    BT, d, f = shape.B * shape.T, shape.d_model, shape.d_ff
    Hq, Hkv, hd = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    view = lambda n, dt, sh: np64(ttcd.workspace_view(ws, p, n, dt, sh))
    bf, f32 = torch.bfloat16, torch.float32
    op = f32 if shape.dtype == "f32" else bf  # operand type of o, u, D, Kt, Rt, Wall
    qkv = view("qkv", bf, (BT, (Hq + 2 * Hkv) * hd))
    checks = {
        "q": (qkv[:, :Hq * hd], ref["q"].reshape(BT, -1)),
        "k": (qkv[:, Hq * hd:(Hq + Hkv) * hd], ref["k"].reshape(BT, -1)),
        "v": (qkv[:, (Hq + Hkv) * hd:], ref["v"].reshape(BT, -1)),
        "o_T": (view("o", op, (2, BT, Hq * hd))[0], ref["o_T"].reshape(BT, -1)),
        "o_S": (view("o", op, (2, BT, Hq * hd))[1], ref["o_S"].reshape(BT, -1)),
        "h_S": (view("h", f32, (BT, d)), ref["h_S"].reshape(BT, -1)),
        "hg_T": (view("u", op, (2, BT, d))[0], ref["h_T"].reshape(BT, -1)),  # gains are 1
    }
    if op == f32:  # fp32 operands: Z_T, Z_S stored in fp32
        checks["Z_T"] = (view("Z", f32, (2, BT, f))[0], ref["Z_T"].reshape(BT, -1))
        checks["Z_S"] = (view("Z", f32, (2, BT, f))[1], ref["Z_S"].reshape(BT, -1))
    else:  # bf16: Z stays on chip; the fused epilogue writes Z_S, D and the keys
        Nc, Cp = shape.n_chunks, (shape.chunk + 63) // 64 * 64
        t = np.arange(shape.T)
        pidx = ((np.arange(shape.B)[:, None] * Nc + t // shape.chunk) * Cp + t % shape.chunk).ravel()
        P = shape.B * Nc * Cp
        checks["Z_S"] = (view("Zs16", bf, (BT, f)), ref["Z_S"].reshape(BT, -1))
        checks["D"] = (view("D", bf, (P, f))[pidx], ref["D"].reshape(BT, -1))
        checks["Kp"] = (view("Kp", bf, (P, f))[pidx], ref["zbar_S"].reshape(BT, -1))
        if weights is not None:  # M = W_down W_proj, with W_proj an MN-major GEMM operand
            checks["M"] = (view("M", bf, (d, f)), np64(weights["w_down"]) @ np64(weights["w_proj"]))
    errs = {k: rel_max(g, r) for k, (g, r) in checks.items()}
    bad = {k: e for k, e in errs.items() if e > TOL_OUT}
    assert not bad, bad
    return errs


@pytest.mark.parametrize("shape", [TINY_F32, SMALL_BF16, SMALL_BF16_C96], ids=lambda s: s.name)
def test_block_forward_parity_small(ttcd, shape):
    inp = make_block_inputs(shape, seed=0)
    p, out, state, ws = _run(ttcd, shape, inp)
    ref = oracle_block(shape, inp)
    errs = _stage_checks(ttcd, p, ws, ref, shape, inp["layers"][0])
    e_out, e_state = rel_max(out, ref["out"]), rel_fro(state, ref["state_out"])
    print(f"\n{shape.name}: out max-rel {e_out:.2e}, state rel-Frobenius {e_state:.2e}, "
          + ", ".join(f"{k} {v:.1e}" for k, v in errs.items()))
    assert e_out <= TOL_OUT
    assert e_state <= TOL_STATE


def test_block_forward_parity_smollm2_shape(ttcd):
    """SmolLM2-360M-shaped block at T = 16384, full oracle comparison."""
    shape = SMOLLM2_360M_16K
    inp = make_block_inputs(shape, seed=0)
    p, out, state, ws = _run(ttcd, shape, inp)
    ref = oracle_block(shape, inp)
    e_out, e_state = rel_max(out, ref["out"]), rel_fro(state, ref["state_out"])
    print(f"\n{shape.name}: out max-rel {e_out:.2e}, state rel-Frobenius {e_state:.2e}")
    assert e_out <= TOL_OUT
    assert e_state <= TOL_STATE


def test_block_forward_qwen3_shape_prefix(ttcd):
    """Qwen3-0.6B-shaped block at T = 65536.  The block is causal, so its first
    T' outputs equal the oracle run on the first T' tokens.  T' = 10 chunks + a
    ragged tail of 300: past the 8192-key teacher window, so the last 2349
    compared rows attend over a full window and read a 10-chunk prefix.  The
    state of the prefix is checked on a separate T' run."""
    shape = QWEN3_0P6B_64K
    inp = make_block_inputs(shape, seed=0)
    p, out, state, ws = _run(ttcd, shape, inp)
    Tp = 10 * shape.chunk + 300
    ref = oracle_block(shape, inp, T=Tp)
    assert rel_max(out[:, :Tp], ref["out"]) <= TOL_OUT
    assert torch.isfinite(out).all() and torch.isfinite(state).all()
    # the prefix run through the library: its state matches the oracle's prefix state
    short = dict(inp)
    short["x"] = inp["x"][:, :Tp].contiguous()
    short["layers"] = [dict(inp["layers"][0], beta=inp["layers"][0]["beta"][:, :Tp].contiguous())]
    _, out_p, state_p, _ = _run(ttcd, shape.with_(T=Tp), short)
    e_out, e_state = rel_max(out_p, ref["out"]), rel_fro(state_p, ref["state_out"])
    print(f"\nqwen3 block prefix T={Tp}: out max-rel {e_out:.2e}, state rel-Frobenius {e_state:.2e}")
    assert e_out <= TOL_OUT
    assert e_state <= TOL_STATE
    assert torch.equal(out_p, out[:, :Tp])


def test_equal_windows_and_convs_write_nothing(ttcd):
    """w_S = w_T with conv_T = conv_S gives D = 0, so the state stays exactly zero."""
    shape = SMALL_BF16.with_(w_S=256, w_T=256)
    inp = make_block_inputs(shape, seed=1)
    inp["layers"][0]["conv_T"] = inp["layers"][0]["conv_S"].clone()
    p, out, state, ws = _run(ttcd, shape, inp)
    assert torch.count_nonzero(state).item() == 0
    ref = oracle_block(shape, inp)
    assert rel_max(out, ref["out"]) <= TOL_OUT


def test_beta_zero_is_static_mlp(ttcd):
    shape = SMALL_BF16
    inp = make_block_inputs(shape, seed=2)
    inp["layers"][0]["beta"] = torch.zeros_like(inp["layers"][0]["beta"])
    p, out, state, ws = _run(ttcd, shape, inp)
    assert torch.count_nonzero(state).item() == 0
    ref = oracle_block(shape, inp)
    assert rel_max(out, ref["out"]) <= TOL_OUT


@pytest.mark.parametrize("s", [0, 127, 128, 900])
def test_chunk_mask_probe_bit_exact(ttcd, s):
    """beta one-hot at token s: outputs change exactly in the chunks after chunk(s)."""
    shape = SMALL_BF16.with_(B=1)
    inp = make_block_inputs(shape, seed=3)
    inp["layers"][0]["beta"] = torch.zeros_like(inp["layers"][0]["beta"])
    _, base, _, _ = _run(ttcd, shape, inp)
    inp["layers"][0]["beta"][0, s] = 0.5
    _, pert, _, _ = _run(ttcd, shape, inp)
    changed = (pert != base).any(-1)[0].cpu().numpy()
    t = np.arange(shape.T)
    np.testing.assert_array_equal(changed, t // shape.chunk > s // shape.chunk)
