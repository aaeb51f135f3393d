"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, validates arguments on the host, and answers size queries."""
import ctypes
import os
import re

import pytest

import dual_window_attention_b200 as ttcd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ttcd.h")


@pytest.fixture(scope="module")
def lib():
    from dual_window_attention_b200 import build
    build.build()
    return ttcd.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ttcd_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_three_entry_points():
    names = declared_functions()
    for n in ("ttcd_dual_window_attn", "ttcd_dual_window_attn_lse", "ttcd_fastweight_mlp",
              "ttcd_block_forward"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n


def _params(**kw):
    base = dict(B=1, T=256, d_model=64, n_q_heads=2, n_kv_heads=1, head_dim=32, d_ff=128,
                w_S=16, w_T=64, chunk=32, conv_k=4, dtype=ttcd.F32)
    base.update(kw)
    return ttcd.BlockParams(**base)


def test_status_strings(lib):
    assert ttcd.status_string(ttcd.OK) == "ok"
    assert "timed out" in ttcd.status_string(ttcd.ERR_TIMEOUT)
    assert ttcd.version().startswith("ttcd")


def test_workspace_sizes(lib):
    p = _params()
    assert ttcd.block_forward_workspace_size(p) > ttcd.fastweight_mlp_workspace_size(p) > 0
    for bad in (dict(head_dim=48), dict(w_S=65), dict(n_kv_heads=3), dict(conv_k=9),
                dict(chunk=0), dict(T=0), dict(d_model=96), dict(dtype=7)):
        assert ttcd.block_forward_workspace_size(_params(**bad)) == 0, bad


def test_workspace_offsets_are_ordered_and_aligned(lib):
    p = _params()
    names = ["status", "wqkv_g", "rstd_in", "qkv", "o", "h", "u", "Z", "Zs16", "D", "Kp", "ssq",
             "R", "Wall"]
    offs = [ttcd.workspace_offset(p, n) for n in names]
    assert offs[0] == 0  # the status word opens every workspace
    assert all(o % 1024 == 0 for o in offs)
    assert offs == sorted(offs)
    with pytest.raises(ttcd.TTCDError):
        ttcd.workspace_offset(p, "nope")


def test_short_bf16_problems_take_the_fp32_operand_route(lib):
    """bf16 with T < chunk runs on fp32 copies: its workspace holds fp32 operands
    and the widened inputs, weights and output, so it is larger than the bf16
    workspace of a one-chunk problem, and its intermediates are fp32."""
    short = _params(dtype=ttcd.BF16, T=31, chunk=32)
    one_chunk = _params(dtype=ttcd.BF16, T=32, chunk=32)
    f32_short = _params(dtype=ttcd.F32, T=31, chunk=32)
    assert ttcd.block_forward_workspace_size(short) > ttcd.block_forward_workspace_size(one_chunk)
    assert ttcd.block_forward_workspace_size(short) > ttcd.block_forward_workspace_size(f32_short)
    assert ttcd.fastweight_mlp_workspace_size(short) > ttcd.fastweight_mlp_workspace_size(one_chunk)
    # "u" holds 2 B T d elements: fp32 on the wide route, bf16 otherwise
    for p, elem in ((short, 4), (one_chunk, 2)):
        span = ttcd.workspace_offset(p, "Z") - ttcd.workspace_offset(p, "u")
        need = 2 * p.B * p.T * p.d_model * elem
        assert need <= span < need + 1024, (p.T, span, need)


def test_check_device_status_validates_on_host(lib):
    assert lib.ttcd_check_device_status(None, None) == ttcd.ERR_INVALID_ARG
    assert lib.ttcd_check_device_status(ctypes.c_void_p((1 << 20) + 4), None) == ttcd.ERR_INVALID_ARG
    assert lib.ttcd_test_bounded_wait(0, None, None) == ttcd.ERR_INVALID_ARG
    assert lib.ttcd_test_bounded_wait(1000, ctypes.c_void_p((1 << 20) + 8), None) == ttcd.ERR_INVALID_ARG


def test_profiled_entry_validates_events_on_host(lib):
    fake = 1 << 20
    p = _params().c()
    w = ttcd._Weights(*([fake] * 10))
    need = lib.ttcd_block_forward_workspace_size(ctypes.byref(p))
    f = lib.ttcd_block_forward_profiled
    ev = (ctypes.c_void_p * 17)(*([fake] * 17))
    args = (fake, fake, ctypes.byref(w), ctypes.byref(p), None, fake, fake, need, None)
    assert f(*args, ev, 17) == ttcd.ERR_INVALID_ARG  # at most 16 events
    assert f(*args, None, 3) == ttcd.ERR_INVALID_ARG
    assert f(*args, (ctypes.c_void_p * 2)(fake, None), 2) == ttcd.ERR_INVALID_ARG
    assert f(*args, ev, -1) == ttcd.ERR_INVALID_ARG


def test_attention_rejects_bad_arguments_on_host(lib):
    fake = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: validation fails first
    f = lib.ttcd_dual_window_attn
    # null pointer
    assert f(None, fake, fake, fake, fake, None, None, 1, 256, 2, 1, 32, 16, 64, 0.0, ttcd.BF16, None) == ttcd.ERR_INVALID_ARG
    # misaligned pointer
    assert f(ctypes.c_void_p((1 << 20) + 2), fake, fake, fake, fake, None, None, 1, 256, 2, 1, 32, 16, 64, 0.0, ttcd.BF16, None) == ttcd.ERR_INVALID_ARG
    # w_S > w_T, Hq % Hkv, bad sizes
    assert f(fake, fake, fake, fake, fake, None, None, 1, 256, 2, 1, 32, 65, 64, 0.0, ttcd.BF16, None) == ttcd.ERR_INVALID_ARG
    assert f(fake, fake, fake, fake, fake, None, None, 1, 256, 3, 2, 32, 16, 64, 0.0, ttcd.BF16, None) == ttcd.ERR_INVALID_ARG
    assert f(fake, fake, fake, fake, fake, None, None, 0, 256, 2, 1, 32, 16, 64, 0.0, ttcd.BF16, None) == ttcd.ERR_INVALID_ARG
    # unsupported head_dim / dtype
    assert f(fake, fake, fake, fake, fake, None, None, 1, 256, 2, 1, 48, 16, 64, 0.0, ttcd.BF16, None) == ttcd.ERR_UNSUPPORTED
    assert f(fake, fake, fake, fake, fake, None, None, 1, 256, 2, 1, 32, 16, 64, 0.0, ttcd.F32, None) == ttcd.ERR_UNSUPPORTED


def test_block_and_mlp_reject_bad_arguments_on_host(lib):
    fake = 1 << 20
    p = _params().c()
    w = ttcd._Weights(*([fake] * 10))
    wnull = ttcd._Weights(*([fake] * 9 + [0]))
    ws_need = lib.ttcd_block_forward_workspace_size(ctypes.byref(p))
    bf = lib.ttcd_block_forward
    assert bf(None, fake, ctypes.byref(w), ctypes.byref(p), None, fake, fake, ws_need, None) == ttcd.ERR_INVALID_ARG
    assert bf(fake, fake, ctypes.byref(wnull), ctypes.byref(p), None, fake, fake, ws_need, None) == ttcd.ERR_INVALID_ARG
    assert bf(fake, fake, ctypes.byref(w), ctypes.byref(p), None, fake, fake, ws_need - 1, None) == ttcd.ERR_WORKSPACE
    bad = _params(head_dim=48).c()
    assert bf(fake, fake, ctypes.byref(w), ctypes.byref(bad), None, fake, fake, ws_need, None) == ttcd.ERR_UNSUPPORTED
    mf = lib.ttcd_fastweight_mlp
    need = lib.ttcd_fastweight_mlp_workspace_size(ctypes.byref(p))
    assert mf(fake, fake, None, fake, ctypes.byref(w), ctypes.byref(p), None, None, fake, fake, need - 1, None) == ttcd.ERR_WORKSPACE
    assert mf(fake, None, None, fake, ctypes.byref(w), ctypes.byref(p), None, None, fake, fake, need, None) == ttcd.ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 128, 2, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ttcd.dual_window_attn(q, q[:, :, :1].contiguous(), q[:, :, :1].contiguous(), 16, 64)


def test_lse_form_rejects_bad_arguments_on_host(lib):
    fake = ctypes.c_void_p(1 << 20)
    f = lib.ttcd_dual_window_attn_lse
    ok_args = [fake] * 9
    assert f(*([None] + ok_args[1:]), 1, 256, 2, 1, 32, 16, 64, 0.0, ttcd.BF16, None) == ttcd.ERR_INVALID_ARG
    # lse_S and lse_far are required (the merge reads them)
    assert f(*(ok_args[:7] + [None, fake]), 1, 256, 2, 1, 32, 16, 64, 0.0, ttcd.BF16, None) == ttcd.ERR_INVALID_ARG
    assert f(*ok_args, 1, 256, 2, 1, 32, 65, 64, 0.0, ttcd.BF16, None) == ttcd.ERR_INVALID_ARG
    assert f(*ok_args, 1, 256, 2, 1, 48, 16, 64, 0.0, ttcd.BF16, None) == ttcd.ERR_UNSUPPORTED
    assert f(*ok_args, 1, 256, 2, 1, 32, 16, 64, 0.0, ttcd.F32, None) == ttcd.ERR_UNSUPPORTED


def test_decode_sizes_and_host_checks(lib):
    p = _params(dtype=ttcd.BF16).c()
    n_state = lib.ttcd_decode_state_size(ctypes.byref(p))
    n_ws = lib.ttcd_decode_workspace_size(ctypes.byref(p))
    assert n_state > 0 and n_ws > 0
    # decode is bf16 only; more than 8 query heads per KV head are not supported
    assert lib.ttcd_decode_state_size(ctypes.byref(_params(dtype=ttcd.F32).c())) == 0
    assert lib.ttcd_decode_state_size(ctypes.byref(_params(dtype=ttcd.BF16, n_q_heads=16, n_kv_heads=1).c())) == 0
    fake = 1 << 20
    w = ttcd._Weights(*([fake] * 10))
    dec = lib.ttcd_block_decode
    beta = ctypes.c_void_p(fake)
    # negative position, null input, short state, short workspace
    assert dec(fake, beta, -1, ctypes.byref(w), ctypes.byref(p), fake, n_state, fake, fake, n_ws, None) == ttcd.ERR_INVALID_ARG
    assert dec(None, beta, 0, ctypes.byref(w), ctypes.byref(p), fake, n_state, fake, fake, n_ws, None) == ttcd.ERR_INVALID_ARG
    assert dec(fake, beta, 0, ctypes.byref(w), ctypes.byref(p), fake, n_state - 1, fake, fake, n_ws, None) == ttcd.ERR_WORKSPACE
    assert dec(fake, beta, 0, ctypes.byref(w), ctypes.byref(p), fake, n_state, fake, fake, n_ws - 1, None) == ttcd.ERR_WORKSPACE
    rd = lib.ttcd_decode_state_read
    assert rd(ctypes.byref(p), -1, fake, n_state, fake, None) == ttcd.ERR_INVALID_ARG
    assert rd(ctypes.byref(p), 3, fake, n_state - 1, fake, None) == ttcd.ERR_WORKSPACE
    # the device-position form takes the same checks, without t
    nxt = lib.ttcd_block_decode_next
    assert nxt(None, beta, ctypes.byref(w), ctypes.byref(p), fake, n_state, fake, fake, n_ws, None) == ttcd.ERR_INVALID_ARG
    assert nxt(fake, beta, ctypes.byref(w), ctypes.byref(p), fake, n_state - 1, fake, fake, n_ws, None) == ttcd.ERR_WORKSPACE
    assert nxt(fake, beta, ctypes.byref(w), ctypes.byref(p), fake, n_state, fake, fake, n_ws - 1, None) == ttcd.ERR_WORKSPACE


def test_backward_sizes_and_host_checks(lib):
    """The three backward entry points: bf16 only, hd 64 or 128 for the
    attention and the block, and every pointer and size checked on the host."""
    p = _params(dtype=ttcd.BF16, head_dim=64, d_model=128, d_ff=256)
    pc = p.c()
    n_mlp = lib.ttcd_fastweight_mlp_backward_workspace_size(ctypes.byref(pc))
    n_blk = lib.ttcd_block_backward_workspace_size(ctypes.byref(pc))
    assert n_blk > n_mlp > ttcd.fastweight_mlp_workspace_size(p) > 0
    assert lib.ttcd_fastweight_mlp_backward_workspace_size(ctypes.byref(_params(dtype=ttcd.F32).c())) == 0
    assert lib.ttcd_block_backward_workspace_size(ctypes.byref(_params(dtype=ttcd.BF16).c())) == 0  # hd 32
    n_att = lib.ttcd_dual_window_attn_backward_workspace_size(1, 256, 2)
    assert n_att >= ttcd.STATUS_BYTES + 4 * 2 * 256 * 4
    assert lib.ttcd_dual_window_attn_backward_workspace_size(0, 256, 2) == 0
    fake = 1 << 20
    w = ttcd._Weights(*([fake] * 10))
    g = ttcd._MlpGrads(*([fake] * 6))
    mlp = lib.ttcd_fastweight_mlp_backward
    args = [fake, fake, fake, ctypes.byref(w), ctypes.byref(pc), None, fake, None, fake, fake, fake,
            None, ctypes.byref(g), fake, n_mlp, None]
    bad = list(args); bad[6] = None                   # no d_y
    assert mlp(*bad) == ttcd.ERR_INVALID_ARG
    bad = list(args); bad[12] = None                  # no gradient table
    assert mlp(*bad) == ttcd.ERR_INVALID_ARG
    bad = list(args); bad[14] = n_mlp - 1             # short workspace
    assert mlp(*bad) == ttcd.ERR_WORKSPACE
    bg = ttcd._BlockGrads(*([fake] * 10))
    blk = lib.ttcd_block_backward
    args = [fake, fake, ctypes.byref(w), ctypes.byref(pc), None, fake, None, fake, fake, None,
            ctypes.byref(bg), fake, n_blk, None]
    bad = list(args); bad[5] = None                   # no d_out
    assert blk(*bad) == ttcd.ERR_INVALID_ARG
    bad = list(args); bad[12] = n_blk - 1
    assert blk(*bad) == ttcd.ERR_WORKSPACE
    att = lib.ttcd_dual_window_attn_backward
    a = [fake] * 12 + [1, 256, 2, 1, 64, 16, 64, 0.0, fake, n_att, None]
    bad = list(a); bad[16] = 32                       # hd 32
    assert att(*bad) == ttcd.ERR_UNSUPPORTED
    bad = list(a); bad[17], bad[18] = 65, 64          # w_S > w_T
    assert att(*bad) == ttcd.ERR_INVALID_ARG
    bad = list(a); bad[9] = None                      # no dq
    assert att(*bad) == ttcd.ERR_INVALID_ARG
    bad = list(a); bad[21] = n_att - 1
    assert att(*bad) == ttcd.ERR_WORKSPACE


def test_attention_timeline_is_compiled_out_of_the_library(lib):
    """The clock64 timeline of the attention kernel exists only in the separate
    instrumented build; the library reports it as unsupported, touching no GPU."""
    buf = (ctypes.c_longlong * 2048)()
    assert lib.ttcd_attn_timeline_read(buf, 2048) == ttcd.ERR_UNSUPPORTED


def test_plain_block_rejects_bad_arguments_on_host(lib):
    """ttcd_swa_block_forward validates on the host; it needs none of the fast-weight
    pointers (w_proj, conv_T, conv_S may be null)."""
    fake = 1 << 20
    p = _params().c()
    w_plain = ttcd._Weights(*([fake] * 7 + [0, 0, 0]))  # w_proj, conv_T, conv_S null
    need = lib.ttcd_swa_block_forward_workspace_size(ctypes.byref(p))
    assert need > 0
    sb = lib.ttcd_swa_block_forward
    assert sb(None, ctypes.byref(w_plain), ctypes.byref(p), fake, fake, need, None) == ttcd.ERR_INVALID_ARG
    assert sb(fake, ctypes.byref(w_plain), ctypes.byref(p), fake, fake, need - 1, None) == ttcd.ERR_WORKSPACE
    w_no_down = ttcd._Weights(*([fake] * 6 + [0, 0, 0, 0]))
    assert sb(fake, ctypes.byref(w_no_down), ctypes.byref(p), fake, fake, need, None) == ttcd.ERR_INVALID_ARG
    bad = _params(head_dim=48).c()
    assert lib.ttcd_swa_block_forward_workspace_size(ctypes.byref(bad)) == 0
    assert sb(fake, ctypes.byref(w_plain), ctypes.byref(bad), fake, fake, need, None) == ttcd.ERR_UNSUPPORTED
