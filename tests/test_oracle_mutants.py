"""The oracle's pins catch plausible mistakes (CPU only).

Each mutant below plants one plausible mistake in a temporary copy of the
oracle: a dropped term, a flipped sign, an off-by-one window edge, a transposed
or swapped operand, an inclusive prefix, a wrong GQA head. The forward mutants
change ``ttcd_oracle.py``, the backward mutants ``ttcd_oracle_grad.py`` and the
sharding mutants ``ttcd_oracle_sharded.py`` (whose pins,
``test_oracle_sharded.py``, run for those and for the unmutated copy).
For each one the oracle's own pin tests (``test_oracle_attention.py``,
``test_oracle_mlp.py``, ``test_oracle_block.py``, ``test_oracle_grad.py``) run
against the copy, and at least one of them must fail. The unmutated copy must pass, which shows that the harness runs the pins
at all.

The mistakes stay on the CPU, in the copy; the CUDA path is not involved.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["test_oracle_attention.py", "test_oracle_mlp.py", "test_oracle_block.py",
             "test_oracle_grad.py"]

# (name, exact text in the oracle, replacement). The text must occur exactly once.
MUTANTS = [
    # RMSNorm
    ("rmsnorm_no_gain", "return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)",
     "return x / np.sqrt(ms + eps)"),
    ("rmsnorm_mean_abs", "ms = np.mean(x * x, axis=-1, keepdims=True)",
     "ms = np.mean(np.abs(x), axis=-1, keepdims=True)"),
    ("rmsnorm_eps_outside_sqrt", "return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)",
     "return x / (np.sqrt(ms) + eps) * np.asarray(g, dtype=np.float64)"),
    # plain sliding-window block (a layer outside the TTT layer set)
    ("swa_block_no_mlp_residual", "out = h + z @ np.asarray(weights[\"w_down\"], np.float64).T",
     "out = z @ np.asarray(weights[\"w_down\"], np.float64).T"),
    ("swa_block_rope_on_q_only", "q, k = rope(q, rope_theta), rope(k, rope_theta)",
     "q = rope(q, rope_theta)"),
    ("swa_block_mlp_norm_uses_attn_gain", 'u = rms_norm(h, weights["g_mlp"], rms_eps)',
     'u = rms_norm(h, weights["g_attn"], rms_eps)'),
    ("mlp_norm_uses_attn_gain",
     'u_T = rms_norm(h_T, weights["g_mlp"], rms_eps)\n    u_S = rms_norm(h_S, weights["g_mlp"], rms_eps)',
     'u_T = rms_norm(h_T, weights["g_attn"], rms_eps)\n    u_S = rms_norm(h_S, weights["g_attn"], rms_eps)'),
    # RoPE
    ("rope_sign", "x1 * cos - x2 * sin, x2 * cos + x1 * sin", "x1 * cos + x2 * sin, x2 * cos - x1 * sin"),
    ("rope_freq_exponent", "* 2.0) / hd)", ") / hd)"),
    ("rope_positions_from_one", "ang = np.arange(T, dtype=np.float64)[:, None]",
     "ang = (np.arange(T, dtype=np.float64) + 1.0)[:, None]"),
    ("rope_on_q_only", "k = rope(k, rope_theta)", "k = k"),
    # SwiGLU
    ("silu_sign", "return x / (1.0 + np.exp(-x))", "return x / (1.0 + np.exp(x))"),
    ("swiglu_gate_up_swapped",
     "silu(u @ np.asarray(w_gate, np.float64).T) * (u @ np.asarray(w_up, np.float64).T)",
     "silu(u @ np.asarray(w_up, np.float64).T) * (u @ np.asarray(w_gate, np.float64).T)"),
    # causal convolution
    ("conv_taps_reversed", "out[:, m:, :] += taps[:, m][None, None, :]",
     "out[:, m:, :] += taps[:, taps.shape[1] - 1 - m][None, None, :]"),
    ("conv_anticausal", "out[:, m:, :] += taps[:, m][None, None, :] * z[:, :T - m, :]",
     "out[:, :T - m, :] += taps[:, m][None, None, :] * z[:, m:, :]"),
    # key normalisation
    ("l2norm_no_sqrt", "return z / np.sqrt(np.sum(z * z, axis=-1, keepdims=True) + eps)",
     "return z / (np.sum(z * z, axis=-1, keepdims=True) + eps)"),
    ("l2norm_eps_dropped", "return z / np.sqrt(np.sum(z * z, axis=-1, keepdims=True) + eps)",
     "return z / np.sqrt(np.sum(z * z, axis=-1, keepdims=True))"),
    ("key_from_teacher", "key = l2_normalize_rows(zb_S, l2_eps)", "key = l2_normalize_rows(zb_T, l2_eps)"),
    # attention
    ("window_one_too_wide", "mask = (jj <= tt) & (jj >= tt - window + 1)",
     "mask = (jj <= tt) & (jj >= tt - window)"),
    ("window_excludes_self", "mask = (jj <= tt) & (jj >= tt - window + 1)",
     "mask = (jj < tt) | ((jj == tt) & (tt == 0))"),
    ("lse_drops_max", "lse[b, :, t0:t1] = (m + np.log(l))", "lse[b, :, t0:t1] = (np.log(l))"),
    ("attention_unnormalised", "ob = (p @ vb) / l", "ob = (p @ vb)"),
    ("gqa_head_modulo", "qb = q[b, t0:t1].reshape(t1 - t0, Hkv, G, hd).transpose(1, 2, 0, 3)",
     "qb = q[b, t0:t1].reshape(t1 - t0, G, Hkv, hd).transpose(2, 1, 0, 3)"),
    ("row_gqa_head_modulo",
     "kk = np.asarray(k[b, j0:t + 1, h // G], np.float64)\n    vv = np.asarray(v[b, j0:t + 1, h // G], np.float64)",
     "kk = np.asarray(k[b, j0:t + 1, h % k.shape[2]], np.float64)\n"
     "    vv = np.asarray(v[b, j0:t + 1, h % k.shape[2]], np.float64)"),
    ("softmax_scale_1_over_hd", "scale = softmax_scale if softmax_scale else 1.0 / np.sqrt(hd)",
     "scale = softmax_scale if softmax_scale else 1.0 / hd"),
    ("band_near_edge", "mask = (j[None, :] <= t[:, None] - near)", "mask = (j[None, :] <= t[:, None] - near + 1)"),
    ("band_far_edge", "& (j[None, :] >= t[:, None] - far)", "& (j[None, :] > t[:, None] - far)"),
    ("lse_merge_weight", "w2 = np.exp(lse2 - lse)", "w2 = np.exp(lse2 - lse1)"),
    # block wiring
    ("qkv_k_v_swapped",
     "k = qkv[..., Hq * hd:(Hq + Hkv) * hd].reshape(B, T, Hkv, hd)\n    v = qkv[..., (Hq + Hkv) * hd:].reshape(B, T, Hkv, hd)",
     "v = qkv[..., Hq * hd:(Hq + Hkv) * hd].reshape(B, T, Hkv, hd)\n    k = qkv[..., (Hq + Hkv) * hd:].reshape(B, T, Hkv, hd)"),
    # block wiring
    ("student_residual_dropped", "h_S = x + o_S.reshape(B, T, Hq * hd) @ w_o.T",
     "h_S = o_S.reshape(B, T, Hq * hd) @ w_o.T"),
    ("output_from_teacher_path", "chunk, l2_eps, h_S=h_S, state_in=state_in",
     "chunk, l2_eps, h_S=h_T, state_in=state_in"),
    ("o_proj_transposed", "h_T = x + o_T.reshape(B, T, Hq * hd) @ w_o.T",
     "h_T = x + o_T.reshape(B, T, Hq * hd) @ w_o"),
    # fast-weight write and read
    ("residual_sign", "dlt = np.asarray(zbar_T, np.float64) - np.asarray(zbar_S, np.float64)",
     "dlt = np.asarray(zbar_S, np.float64) - np.asarray(zbar_T, np.float64)"),
    ("w_proj_transposed", "tmp = dlt @ np.asarray(w_proj, np.float64).T",
     "tmp = dlt @ np.asarray(w_proj, np.float64)"),
    ("w_down_dropped_from_residual", "return tmp @ np.asarray(w_down, np.float64).T",
     "return tmp[..., :np.asarray(w_down).shape[0]]"),
    ("beta_dropped", "out[b, i] = (r[b, s0:s1] * beta[b, s0:s1, None]).T @ key[b, s0:s1]",
     "out[b, i] = r[b, s0:s1].T @ key[b, s0:s1]"),
    ("beta_squared", "out[b, i] = (r[b, s0:s1] * beta[b, s0:s1, None]).T @ key[b, s0:s1]",
     "out[b, i] = (r[b, s0:s1] * beta[b, s0:s1, None] ** 2).T @ key[b, s0:s1]"),
    ("inclusive_prefix", "prefixes[:, i] = s\n        s = s + inc[:, i]",
     "s = s + inc[:, i]\n        prefixes[:, i] = s"),
    ("prefix_starts_at_first_increment", "prefixes[:, i] = s\n        s = s + inc[:, i]",
     "prefixes[:, i] = s + (inc[:, 0] if i == 0 else 0)\n        s = s + inc[:, i]"),
    ("state_in_ignored",
     "s = np.zeros((B, d, f)) if state_in is None else np.array(state_in, np.float64)",
     "s = np.zeros((B, d, f))"),
    ("fast_weight_subtracted", "y[b, s0:s1] = Z_S[b, s0:s1] @ (w_down + prefixes[b, i]).T",
     "y[b, s0:s1] = Z_S[b, s0:s1] @ (w_down - prefixes[b, i]).T"),
    ("read_uses_conv_activation", "y[b, s0:s1] = Z_S[b, s0:s1] @ (w_down + prefixes[b, i]).T",
     "y[b, s0:s1] = zb_S[b, s0:s1] @ (w_down + prefixes[b, i]).T"),
    ("read_ignores_fast_weight", "y[b, s0:s1] = Z_S[b, s0:s1] @ (w_down + prefixes[b, i]).T",
     "y[b, s0:s1] = Z_S[b, s0:s1] @ w_down.T"),
    ("chunk_edge_off_by_one", "s0, s1 = i * chunk, min(T, (i + 1) * chunk)\n            out[b, i]",
     "s0, s1 = i * chunk, min(T, (i + 1) * chunk + 1)\n            out[b, i]"),
]


# Mistakes in the backward oracle: (name, exact text in ttcd_oracle_grad.py, replacement).
GRAD_MUTANTS = [
    ("vjp_rmsnorm_no_projection",
     "dx = r * (dxhat - xhat * np.mean(dxhat * xhat, axis=-1, keepdims=True))", "dx = r * dxhat"),
    ("vjp_rope_forward_rotation", "d1 * cos + d2 * sin, d2 * cos - d1 * sin",
     "d1 * cos - d2 * sin, d2 * cos + d1 * sin"),
    ("vjp_silu_derivative", "return s * (1.0 + a * (1.0 - s))", "return s * (1.0 - s)"),
    ("vjp_swiglu_gate_up_swapped", "du = da @ wg + db @ wu", "du = da @ wu + db @ wg"),
    ("vjp_conv_wrong_shift", "dz[:, :T - m, :] += taps[:, m][None, None, :] * dzbar[:, m:, :]",
     "dz[:, m:, :] += taps[:, m][None, None, :] * dzbar[:, :T - m, :]"),
    ("vjp_l2norm_no_projection", "return inv * (dk - k * np.sum(k * dk, axis=-1, keepdims=True))",
     "return inv * dk"),
    ("vjp_w_proj_transposed", "dD = dE @ wp", "dD = dE @ wp.T"),
    ("vjp_beta_dropped", "dr[b, s0:s1] = beta[b, s0:s1, None] * rk", "dr[b, s0:s1] = rk"),
    ("vjp_prefix_inclusive", "d_inc[:, i] = acc\n        acc = acc + d_prefixes[:, i]",
     "acc = acc + d_prefixes[:, i]\n        d_inc[:, i] = acc"),
    ("vjp_softmax_no_rowsum",
     "ds = p * (dp - np.sum(do[b, :, h] * o, axis=1, keepdims=True))", "ds = p * dp"),
    ("vjp_dk_unscaled", "dk[b, :, kh] += scale * (ds.T @ q[b, :, h])", "dk[b, :, kh] += ds.T @ q[b, :, h]"),
    ("vjp_residual_sign", "dzb_S = dzb_S - dD", "dzb_S = dzb_S + dD"),
    ("vjp_read_ignores_fast_weight",
     'dZ_S[b, s0:s1] = d_y[b, s0:s1] @ (w_down + fw["S_prefix"][b, i])',
     'dZ_S[b, s0:s1] = d_y[b, s0:s1] @ w_down'),
    ("vjp_teacher_path_dropped_from_x", "dx = dh_T + d_hS", "dx = d_hS"),
    ("vjp_student_window_as_teacher",
     'windowed_attention_vjp(fw["q"], fw["k"], fw["v"], w_S, scale, do_S)',
     'windowed_attention_vjp(fw["q"], fw["k"], fw["v"], w_T, scale, do_S)'),
]
# Mistakes in the sequence-sharded form (ttcd_oracle_sharded.py).
SHARD_MUTANTS = [
    ("shard_kv_halo_one_short", "h0 = max(0, start - (w_T - 1))", "h0 = max(0, start - (w_T - 2))"),
    ("shard_conv_halo_one_short", "c0 = max(0, start - (conv_k - 1))",
     "c0 = max(0, start - (conv_k - 2))"),
    ("shard_state_prefix_inclusive", "for j in range(rank):", "for j in range(rank + 1):"),
    ("shard_rope_from_zero", "q = _rope_from(q, rope_theta, start)\n    k = _rope_from(k, rope_theta, start)",
     "q = _rope_from(q, rope_theta, 0)\n    k = _rope_from(k, rope_theta, 0)"),
]
ALL_MUTANTS = [(n, "ttcd_oracle.py", o, r) for n, o, r in MUTANTS] + \
              [(n, "ttcd_oracle_grad.py", o, r) for n, o, r in GRAD_MUTANTS] + \
              [(n, "ttcd_oracle_sharded.py", o, r) for n, o, r in SHARD_MUTANTS]
# the sharded pins spawn gloo ranks; they run for the unmutated copy and the sharded mutants
SHARD_PIN = "test_oracle_sharded.py"


def _make_tree(dst: str, name: str, target: str, old: str, new: str) -> None:
    """A copy of the oracle, the workload generators and the pin tests, with one mistake."""
    shutil.copytree(os.path.join(ROOT, "ttcd_workloads"), os.path.join(dst, "ttcd_workloads"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(os.path.join(dst, "tests"))
    for f in ["conftest.py", "helpers.py", *PIN_FILES, SHARD_PIN]:
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests"))
    if name == "unmutated":
        return
    path = os.path.join(dst, "oracle", target)
    src = open(path).read()
    assert src.count(old) == 1, f"mutant {name}: text found {src.count(old)} times"
    with open(path, "w") as f:
        f.write(src.replace(old, new))


def _run_pins(dst: str, sharded: bool) -> int:
    env = dict(os.environ, OMP_NUM_THREADS="1", MKL_NUM_THREADS="1", PYTHONDONTWRITEBYTECODE="1")
    files = PIN_FILES + ([SHARD_PIN] if sharded else [])
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           *[os.path.join("tests", f) for f in files]]
    return subprocess.run(cmd, cwd=dst, env=env, stdout=subprocess.DEVNULL,
                          stderr=subprocess.DEVNULL, timeout=600).returncode


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    cases = [("unmutated", "", "", "")] + ALL_MUTANTS
    dirs = {}
    for name, target, old, new in cases:
        d = str(tmp_path_factory.mktemp(name))
        _make_tree(d, name, target, old, new)
        dirs[name] = d
    sharded = {name: name == "unmutated" or target == "ttcd_oracle_sharded.py"
               for name, target, _, _ in cases}
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        rcs = dict(zip(dirs, ex.map(lambda n: _run_pins(dirs[n], sharded[n]), dirs)))
    return rcs


def test_unmutated_copy_passes_its_pins(outcomes):
    assert outcomes["unmutated"] == 0


@pytest.mark.parametrize("name", [m[0] for m in ALL_MUTANTS])
def test_pins_catch_mutant(outcomes, name):
    # pytest exits 1 when a test failed; 2-5 would mean the copy did not even run
    assert outcomes[name] == 1, f"no pin fails for the planted mistake {name!r} (rc {outcomes[name]})"
