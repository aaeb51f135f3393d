"""IP-TTCD block forward on B200 (sm_100a): thin Python binding over libttcd.so.

The binding only marshals arguments: device memory comes from PyTorch, every
step of the computation runs in the library's CUDA kernels.  There is no CPU
fallback; if the library is missing or a tensor is not on a CUDA device the
call raises.

    import dual_window_attention_b200 as ttcd
    o_T, o_S, lse_T, lse_S = ttcd.dual_window_attn(q, k, v, w_S=512, w_T=8192)
    out, state = ttcd.block_forward(x, beta, weights, params)
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Dict, Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libttcd.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(6)
F32, BF16 = 0, 1


class TTCDError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class _Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("d_model", ctypes.c_int),
                ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("d_ff", ctypes.c_int), ("w_S", ctypes.c_int),
                ("w_T", ctypes.c_int), ("chunk", ctypes.c_int), ("conv_k", ctypes.c_int),
                ("rms_eps", ctypes.c_float), ("l2_eps", ctypes.c_float),
                ("rope_theta", ctypes.c_float), ("softmax_scale", ctypes.c_float),
                ("dtype", ctypes.c_int)]


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_qkv", "w_o", "g_attn", "g_mlp", "w_gate",
                                               "w_up", "w_down", "w_proj", "conv_T", "conv_S")]


WEIGHT_NAMES = tuple(n for n, _ in _Weights._fields_)


class _BlockGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_NAMES]


class _MlpGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_gate", "w_up", "w_down", "w_proj", "conv_T",
                                               "conv_S")]

_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libttcd.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"CUDA library {path} is missing: build it with "
                          "`python -m dual_window_attention_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    P, W = ctypes.POINTER(_Params), ctypes.POINTER(_Weights)
    lib.ttcd_dual_window_attn.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp]
    lib.ttcd_dual_window_attn_lse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i,
                                              i, f, i, vp]
    lib.ttcd_decode_state_size.argtypes = [P]
    lib.ttcd_decode_state_size.restype = sz
    lib.ttcd_decode_workspace_size.argtypes = [P]
    lib.ttcd_decode_workspace_size.restype = sz
    lib.ttcd_decode_state_init.argtypes = [W, P, vp, vp, sz, vp, sz, vp]
    lib.ttcd_block_decode.argtypes = [vp, vp, i, W, P, vp, sz, vp, vp, sz, vp]
    lib.ttcd_block_decode_next.argtypes = [vp, vp, W, P, vp, sz, vp, vp, sz, vp]
    lib.ttcd_block_decode_next_ex.argtypes = [vp, vp, W, P, vp, sz, vp, vp, sz, i, vp]
    lib.ttcd_decode_state_read.argtypes = [P, i, vp, sz, vp, vp]
    lib.ttcd_fastweight_mlp.argtypes = [vp, vp, vp, vp, W, P, vp, vp, vp, vp, sz, vp]
    lib.ttcd_block_forward.argtypes = [vp, vp, W, P, vp, vp, vp, sz, vp]
    lib.ttcd_swa_block_forward.argtypes = [vp, W, P, vp, vp, sz, vp]
    lib.ttcd_swa_block_forward_workspace_size.argtypes = [P]
    lib.ttcd_swa_block_forward_workspace_size.restype = sz
    lib.ttcd_block_forward_profiled.argtypes = [vp, vp, W, P, vp, vp, vp, sz, vp,
                                                ctypes.POINTER(ctypes.c_void_p), i]
    lib.ttcd_check_device_status.argtypes = [vp, vp]
    lib.ttcd_fastweight_mlp_workspace_size.argtypes = [P]
    lib.ttcd_fastweight_mlp_workspace_size.restype = sz
    lib.ttcd_block_forward_workspace_size.argtypes = [P]
    lib.ttcd_block_forward_workspace_size.restype = sz
    lib.ttcd_block_workspace_offset.argtypes = [P, ctypes.c_char_p, ctypes.POINTER(sz)]
    lib.ttcd_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), vp]
    lib.ttcd_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.ttcd_set_wait_timeout_ns.restype = None
    lib.ttcd_test_bounded_wait.argtypes = [ctypes.c_uint64, vp, vp]
    lib.ttcd_test_exp2_poly.argtypes = [vp, vp, i, vp]
    lib.ttcd_test_exp2_poly.restype = i
    lib.ttcd_attn_timeline_read.argtypes = [ctypes.POINTER(ctypes.c_longlong), sz]
    lib.ttcd_attn_timeline_read.restype = i
    lib.ttcd_status_string.argtypes = [i]
    lib.ttcd_status_string.restype = ctypes.c_char_p
    lib.ttcd_version.restype = ctypes.c_char_p
    lib.ttcd_kernel_launch_count.argtypes = []
    lib.ttcd_kernel_launch_count.restype = ctypes.c_ulonglong
    ll = ctypes.c_longlong
    lib.ttcd_shard_workspace_size.argtypes = [P]
    lib.ttcd_shard_workspace_size.restype = sz
    lib.ttcd_shard_qkv.argtypes = [vp, W, P, ll, vp, vp, sz, vp]
    lib.ttcd_shard_attend.argtypes = [vp, vp, W, P, ll, vp, vp, sz, vp]
    lib.ttcd_shard_mix.argtypes = [vp, vp, W, P, ll, vp, vp, sz, vp]
    lib.ttcd_shard_finish.argtypes = [W, P, ll, vp, vp, vp, vp, sz, vp]
    lib.ttcd_dual_window_attn_backward_workspace_size.argtypes = [i, i, i]
    lib.ttcd_dual_window_attn_backward_workspace_size.restype = sz
    lib.ttcd_dual_window_attn_backward.argtypes = [vp] * 12 + [i] * 7 + [f, vp, sz, vp]
    lib.ttcd_block_backward_workspace_size.argtypes = [P]
    lib.ttcd_block_backward_workspace_size.restype = sz
    lib.ttcd_block_backward.argtypes = [vp, vp, W, P, vp, vp, vp, vp, vp, vp,
                                        ctypes.POINTER(_BlockGrads), vp, sz, vp]
    lib.ttcd_fastweight_mlp_backward_workspace_size.argtypes = [P]
    lib.ttcd_fastweight_mlp_backward_workspace_size.restype = sz
    lib.ttcd_fastweight_mlp_backward.argtypes = [vp, vp, vp, W, P, vp, vp, vp, vp, vp, vp, vp,
                                                 ctypes.POINTER(_MlpGrads), vp, sz, vp]
    lib.ttcd_fastweight_mlp_noalloc.argtypes = [vp, vp, vp, vp, W, P, vp, vp, vp, vp]
    lib.ttcd_fastweight_mlp_noalloc.restype = i
    lib.ttcd_fastweight_mlp_noalloc_capacity.argtypes = []
    lib.ttcd_fastweight_mlp_noalloc_capacity.restype = sz
    for fn in ("ttcd_dual_window_attn", "ttcd_dual_window_attn_lse", "ttcd_fastweight_mlp",
               "ttcd_block_forward", "ttcd_block_forward_profiled", "ttcd_block_workspace_offset",
               "ttcd_get_device_error", "ttcd_check_device_status", "ttcd_test_bounded_wait",
               "ttcd_decode_state_init", "ttcd_block_decode", "ttcd_decode_state_read",
               "ttcd_block_decode_next", "ttcd_block_decode_next_ex", "ttcd_fastweight_mlp_backward",
               "ttcd_dual_window_attn_backward", "ttcd_block_backward",
               "ttcd_shard_qkv", "ttcd_shard_attend", "ttcd_shard_mix", "ttcd_shard_finish"):
        getattr(lib, fn).restype = i
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().ttcd_status_string(status).decode()


def version() -> str:
    return load_library().ttcd_version().decode()


def _check(status: int, what: str) -> None:
    if status != OK:
        raise TTCDError(status, what)


@dataclasses.dataclass
class BlockParams:
    """Mirror of ttcd_block_params (names follow the pages: w_T, w_S, chunk C)."""

    B: int
    T: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    d_ff: int
    w_S: int
    w_T: int
    chunk: int
    conv_k: int = 4
    rms_eps: float = 1e-6
    l2_eps: float = 1e-6
    rope_theta: float = 10000.0
    softmax_scale: float = 0.0
    dtype: int = BF16

    def c(self) -> _Params:
        return _Params(*[getattr(self, f) for f, _ in _Params._fields_])

    @classmethod
    def from_shape(cls, shape) -> "BlockParams":
        return cls(B=shape.B, T=shape.T, d_model=shape.d_model, n_q_heads=shape.n_q_heads,
                   n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, d_ff=shape.d_ff,
                   w_S=shape.w_S, w_T=shape.w_T, chunk=shape.chunk, conv_k=shape.conv_k,
                   rms_eps=shape.rms_eps, l2_eps=shape.l2_eps, rope_theta=shape.rope_theta,
                   dtype=F32 if shape.dtype == "f32" else BF16)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == F32 else torch.bfloat16


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libttcd takes CUDA tensors only (no CPU path)")
    if not t.is_contiguous():
        raise ValueError("libttcd takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _weights(w: Dict[str, torch.Tensor]) -> _Weights:
    return _Weights(*[_ptr(w.get(n)) for n in WEIGHT_NAMES])


def dual_window_attn(q, k, v, w_S: int, w_T: int, scale: float = 0.0, o_T=None, o_S=None,
                     lse: bool = False, stream=None):
    """Fused dual-window attention; returns (o_T, o_S, lse_T, lse_S) (lse None unless asked)."""
    lib = load_library()
    B, T, Hq, hd = q.shape
    Hkv = k.shape[2]
    o_T = torch.empty_like(q) if o_T is None else o_T
    o_S = torch.empty_like(q) if o_S is None else o_S
    lse_T = lse_S = None
    if lse:
        lse_T = torch.empty(B, Hq, T, device=q.device, dtype=torch.float32)
        lse_S = torch.empty_like(lse_T)
    dt = BF16 if q.dtype == torch.bfloat16 else F32
    st = lib.ttcd_dual_window_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o_T), _ptr(o_S), _ptr(lse_T),
                                   _ptr(lse_S), B, T, Hq, Hkv, hd, w_S, w_T, scale, dt,
                                   _stream(stream))
    _check(st, "ttcd_dual_window_attn")
    return o_T, o_S, lse_T, lse_S


def dual_window_attn_backward(q, k, v, o_T, o_S, lse_T, lse_S, do_T, do_S, w_S: int, w_T: int,
                              scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
                              stream=None):
    """Vector-Jacobian product of ``dual_window_attn`` (bf16, hd 64 or 128):
    (dq, dk, dv) in fp32 for output gradients do_T, do_S, given the forward's
    o_T, o_S, lse_T, lse_S.  Returns (dq, dk, dv, workspace)."""
    lib = load_library()
    B, T, Hq, hd = q.shape
    Hkv = k.shape[2]
    need = int(lib.ttcd_dual_window_attn_backward_workspace_size(B, T, Hq))
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    dq = torch.empty(B, T, Hq, hd, device=q.device, dtype=torch.float32)
    dk = torch.empty(B, T, Hkv, hd, device=q.device, dtype=torch.float32)
    dv = torch.empty_like(dk)
    st = lib.ttcd_dual_window_attn_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o_T), _ptr(o_S), _ptr(lse_T), _ptr(lse_S), _ptr(do_T),
        _ptr(do_S), _ptr(dq), _ptr(dk), _ptr(dv), B, T, Hq, Hkv, hd, w_S, w_T, scale,
        _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "ttcd_dual_window_attn_backward")
    return dq, dk, dv, workspace


def dual_window_attn_lse(q, k, v, w_S: int, w_T: int, scale: float = 0.0, stream=None):
    """Dual-window attention by LSE combination (student window + far band).

    Returns (o_T, o_S, o_far, lse_T, lse_S, lse_far)."""
    lib = load_library()
    B, T, Hq, hd = q.shape
    Hkv = k.shape[2]
    o_T, o_S, o_far = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    lse_T = torch.empty(B, Hq, T, device=q.device, dtype=torch.float32)
    lse_S, lse_far = torch.empty_like(lse_T), torch.empty_like(lse_T)
    dt = BF16 if q.dtype == torch.bfloat16 else F32
    st = lib.ttcd_dual_window_attn_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(o_T), _ptr(o_S),
                                       _ptr(o_far), _ptr(lse_T), _ptr(lse_S), _ptr(lse_far), B, T,
                                       Hq, Hkv, hd, w_S, w_T, scale, dt, _stream(stream))
    _check(st, "ttcd_dual_window_attn_lse")
    return o_T, o_S, o_far, lse_T, lse_S, lse_far


def block_forward_workspace_size(p: BlockParams) -> int:
    pc = p.c()
    return load_library().ttcd_block_forward_workspace_size(ctypes.byref(pc))


def fastweight_mlp_workspace_size(p: BlockParams) -> int:
    pc = p.c()
    return load_library().ttcd_fastweight_mlp_workspace_size(ctypes.byref(pc))


def workspace_offset(p: BlockParams, name: str) -> int:
    pc = p.c()
    off = ctypes.c_size_t(0)
    _check(load_library().ttcd_block_workspace_offset(ctypes.byref(pc), name.encode(),
                                                      ctypes.byref(off)), "workspace_offset")
    return off.value


def workspace_view(ws: torch.Tensor, p: BlockParams, name: str, dtype: torch.dtype, shape):
    """View of a named intermediate inside a block_forward workspace (uint8 tensor)."""
    off = workspace_offset(p, name)
    n = 1
    for s in shape:
        n *= s
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype).view(*shape)


STATUS_BYTES = 256  # TTCD_STATUS_BYTES: the status word's region at the start of a workspace


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A workspace with its status region cleared (the library reads and clears
    the status word; it never initialises it)."""
    ws = torch.empty(max(nbytes, STATUS_BYTES), dtype=torch.uint8, device=device)
    ws[:STATUS_BYTES].zero_()
    return ws


def block_forward(x, beta, weights: Dict[str, torch.Tensor], p: BlockParams, out=None,
                  state_out: bool = False, workspace: Optional[torch.Tensor] = None,
                  stream=None, events=None) -> Tuple[torch.Tensor, Optional[torch.Tensor], torch.Tensor]:
    """One IP-TTCD block forward.  Returns (out, state_out or None, workspace).

    ``events``: optional torch.cuda.Event objects recorded at the stage boundaries
    of this call (ttcd_block_forward_profiled).  Timeouts are recorded in the
    workspace's status word: read them with ``check_device_status(workspace)``."""
    lib = load_library()
    need = block_forward_workspace_size(p)
    if need == 0:
        raise TTCDError(ERR_INVALID_ARG, "ttcd_block_forward_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, x.device)
    out = torch.empty_like(x) if out is None else out
    st_t = (torch.empty(p.B, p.d_model, p.d_ff, device=x.device, dtype=torch.float32)
            if state_out else None)
    pc, wc = p.c(), _weights(weights)
    if events:
        for e in events:  # torch creates the underlying CUDA event on first record
            if not e.cuda_event:
                e.record()
        arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        st = lib.ttcd_block_forward_profiled(_ptr(x), _ptr(beta), ctypes.byref(wc),
                                             ctypes.byref(pc), _ptr(st_t), _ptr(out),
                                             _ptr(workspace), workspace.numel(), _stream(stream),
                                             arr, len(events))
        _check(st, "ttcd_block_forward_profiled")
    else:
        st = lib.ttcd_block_forward(_ptr(x), _ptr(beta), ctypes.byref(wc), ctypes.byref(pc),
                                    _ptr(st_t), _ptr(out), _ptr(workspace), workspace.numel(),
                                    _stream(stream))
        _check(st, "ttcd_block_forward")
    return out, st_t, workspace


def swa_block_forward_workspace_size(p: BlockParams) -> int:
    return int(load_library().ttcd_swa_block_forward_workspace_size(ctypes.byref(p.c())))


def swa_block_forward(x, weights: Dict[str, torch.Tensor], p: BlockParams, out=None,
                      workspace: Optional[torch.Tensor] = None,
                      stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One plain sliding-window block (window p.w_T, static MLP): a layer outside
    the TTT layer set.  Returns (out, workspace)."""
    lib = load_library()
    need = swa_block_forward_workspace_size(p)
    if need == 0:
        raise TTCDError(ERR_INVALID_ARG, "ttcd_swa_block_forward_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, x.device)
    out = torch.empty_like(x) if out is None else out
    pc, wc = p.c(), _weights(weights)
    st = lib.ttcd_swa_block_forward(_ptr(x), ctypes.byref(wc), ctypes.byref(pc), _ptr(out),
                                    _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "ttcd_swa_block_forward")
    return out, workspace


def block_stack_forward(x, layers, p: BlockParams, workspace: Optional[torch.Tensor] = None,
                        stream=None, on_layer=None, ttt_layers=None) -> torch.Tensor:
    """A stack of blocks: layer l's output is layer l+1's input.

    ``layers`` is a list of weight dicts (the keys block_forward takes plus each
    layer's per-token ``beta``).  ``ttt_layers`` (an iterable of layer indices,
    default all) names the IP-TTCD blocks; the other layers are plain
    sliding-window blocks (swa_block_forward: window p.w_T, static MLP; their
    beta, w_proj and conv taps are not read).  One workspace serves every layer
    and two activation buffers alternate, so nothing is allocated per layer.
    ``on_layer(l, out)``, if given, sees each layer's output before the buffer is
    reused.  Returns the last layer's output (a fresh tensor, not ``x``)."""
    ttt = set(range(len(layers))) if ttt_layers is None else set(ttt_layers)
    need = max(block_forward_workspace_size(p), swa_block_forward_workspace_size(p))
    if need == 0:
        raise TTCDError(ERR_INVALID_ARG, "ttcd_block_forward_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, x.device)
    bufs = (torch.empty_like(x), torch.empty_like(x))
    cur = x
    for l, w in enumerate(layers):
        out = bufs[l & 1]
        if l in ttt:
            block_forward(cur, w["beta"], w, p, out=out, workspace=workspace, stream=stream)
        else:
            swa_block_forward(cur, w, p, out=out, workspace=workspace, stream=stream)
        if on_layer is not None:
            on_layer(l, out)
        cur = out
    return cur


class Decoder:
    """Token-by-token decode of one block for a batch of B sequences in lockstep.

    Holds the decode state (K/V ring cache, conv history, the current chunk's
    rows, the fast weight) and a step workspace, both allocated once.
    ``step(x_t, beta_t)`` takes x_t [B, d] bf16 and beta_t [B] fp32 of the next
    position and returns y_t [B, d]; ``state_out()`` is the fast-weight state
    after the tokens so far (partial chunk included).

    ``graph=True``: the steps use ttcd_block_decode_next_ex (the position lives
    in the state); token 0 runs eagerly, then two steps are captured in CUDA
    graphs with fixed input and output buffers: an ordinary step without the
    chunk commit's launches, replayed for every later token, and a commit step,
    replayed at the last token of each chunk (the host's position decides)."""

    def __init__(self, weights: Dict[str, torch.Tensor], p: BlockParams, state_in=None,
                 device="cuda", stream=None, graph: bool = False):
        self.lib = load_library()
        self.p, self.pc, self.wc = p, p.c(), _weights(weights)
        self.weights = weights  # keep the tensors alive
        self.stream = stream
        n_state = self.lib.ttcd_decode_state_size(ctypes.byref(self.pc))
        n_ws = self.lib.ttcd_decode_workspace_size(ctypes.byref(self.pc))
        if n_state == 0 or n_ws == 0:
            raise TTCDError(ERR_UNSUPPORTED, "ttcd_decode_state_size")
        self.state = alloc_workspace(n_state, device)
        self.ws = alloc_workspace(n_ws, device)
        _check(self.lib.ttcd_decode_state_init(ctypes.byref(self.wc), ctypes.byref(self.pc),
                                               _ptr(state_in), _ptr(self.state),
                                               self.state.numel(), _ptr(self.ws), self.ws.numel(),
                                               _stream(stream)), "ttcd_decode_state_init")
        self.t = 0
        self.use_graph, self.warm = graph, False
        # captured steps: key True = with the chunk commit, False = without
        self.graphs = {True: None, False: None}
        self.graph_launches = {True: 0, False: 0}  # kernels per replay of each
        self.replayed_launches = 0  # kernels launched by all replays so far
        if graph:
            self.x_buf = torch.empty(p.B, p.d_model, device=device, dtype=torch.bfloat16)
            self.b_buf = torch.empty(p.B, device=device, dtype=torch.float32)
            self.y_buf = torch.empty_like(self.x_buf)

    def _next(self, commit: bool = True):
        _check(self.lib.ttcd_block_decode_next_ex(_ptr(self.x_buf), _ptr(self.b_buf),
                                                  ctypes.byref(self.wc), ctypes.byref(self.pc),
                                                  _ptr(self.state), self.state.numel(),
                                                  _ptr(self.y_buf), _ptr(self.ws),
                                                  self.ws.numel(), int(commit), _stream(None)),
               "ttcd_block_decode_next_ex")

    def seek(self, t: int):
        """Sets the next position to t (host count and, in graph mode, the
        state's device position: an int64 at byte 8 of the state)."""
        self.t = t
        if self.use_graph:
            self.state[8:16].copy_(torch.tensor([t], dtype=torch.int64).view(torch.uint8))

    def step(self, x_t, beta_t, y=None):
        """In graph mode x_t, beta_t and y may be x_buf, b_buf and y_buf
        themselves (no copies)."""
        if self.use_graph:
            if x_t.data_ptr() != self.x_buf.data_ptr():
                self.x_buf.copy_(x_t)
            if beta_t.data_ptr() != self.b_buf.data_ptr():
                self.b_buf.copy_(beta_t)
            if not self.warm:
                self._next()  # eager: also loads every kernel before the captures
                self.warm = True
            else:
                commit = self.t % self.p.chunk == self.p.chunk - 1
                if self.graphs[commit] is None:
                    torch.cuda.synchronize()
                    n0 = kernel_launch_count()
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        self._next(commit)
                    self.graphs[commit] = g
                    self.graph_launches[commit] = kernel_launch_count() - n0
                self.graphs[commit].replay()
                self.replayed_launches += self.graph_launches[commit]
            self.t += 1
            if y is not None and y.data_ptr() == self.y_buf.data_ptr():
                return y
            return self.y_buf.clone() if y is None else y.copy_(self.y_buf)
        y = torch.empty_like(x_t) if y is None else y
        _check(self.lib.ttcd_block_decode(_ptr(x_t), _ptr(beta_t), self.t, ctypes.byref(self.wc),
                                          ctypes.byref(self.pc), _ptr(self.state),
                                          self.state.numel(), _ptr(y), _ptr(self.ws),
                                          self.ws.numel(), _stream(self.stream)),
               "ttcd_block_decode")
        self.t += 1
        return y

    def check_status(self) -> int:
        """Status of the decode calls so far (reads and clears the state's word)."""
        return check_device_status(self.state, self.stream)

    def state_out(self):
        out = torch.empty(self.p.B, self.p.d_model, self.p.d_ff, device=self.state.device,
                          dtype=torch.float32)
        _check(self.lib.ttcd_decode_state_read(ctypes.byref(self.pc), self.t, _ptr(self.state),
                                               self.state.numel(), _ptr(out),
                                               _stream(self.stream)), "ttcd_decode_state_read")
        return out


class Shard:
    """One shard of a sequence-sharded block forward: tokens pos0 .. pos0 + p.T - 1
    of each of the p.B sequences (pos0 a multiple of p.chunk), bf16.

    The four phases run in order on one workspace; between them the caller
    passes on what the next shard needs (see ``sharding.shard_block_forward``):

        kv_tail = sh.qkv(x)                      # rotated K/V of the last tokens
        u_tail = sh.attend(x, kv_halo)           # normalised MLP inputs of the last tokens
        total = sh.mix(beta, u_halo)             # sum of this shard's chunk increments
        out, state = sh.finish(state_in)         # state_in = earlier shards' totals

    kv rows are [2, Hkv, hd] (K heads then V heads) per token."""

    def __init__(self, weights: Dict[str, torch.Tensor], p: BlockParams, pos0: int,
                 device="cuda", stream=None):
        self.lib = load_library()
        self.p, self.pc, self.wc, self.pos0 = p, p.c(), _weights(weights), int(pos0)
        self.weights = weights
        self.stream = stream
        self.device = torch.device(device)
        n = self.lib.ttcd_shard_workspace_size(ctypes.byref(self.pc))
        if n == 0:
            raise TTCDError(ERR_INVALID_ARG, "ttcd_shard_workspace_size")
        self.ws = alloc_workspace(n, device)
        self.n_halo = min(p.w_T - 1, self.pos0)
        self.kv_width = 2 * p.n_kv_heads * p.head_dim

    def _ws(self):
        return _ptr(self.ws), self.ws.numel(), _stream(self.stream)

    def qkv(self, x):
        p = self.p
        kv_tail = torch.empty(p.B, min(p.T, p.w_T - 1), self.kv_width, device=self.device,
                              dtype=torch.bfloat16)
        _check(self.lib.ttcd_shard_qkv(_ptr(x), ctypes.byref(self.wc), ctypes.byref(self.pc),
                                       self.pos0, _ptr(kv_tail), *self._ws()), "ttcd_shard_qkv")
        return kv_tail

    def attend(self, x, kv_halo):
        p = self.p
        if kv_halo is not None and kv_halo.shape[1] != self.n_halo:
            raise ValueError(f"K/V halo of {kv_halo.shape[1]} rows, need {self.n_halo}")
        if self.n_halo == 0:
            kv_halo = None
        u_tail = torch.empty(2, p.B, min(p.T, max(p.conv_k - 1, 0)), p.d_model,
                             device=self.device, dtype=torch.bfloat16)
        _check(self.lib.ttcd_shard_attend(_ptr(x), _ptr(kv_halo), ctypes.byref(self.wc),
                                          ctypes.byref(self.pc), self.pos0,
                                          _ptr(u_tail) if u_tail.numel() else None,
                                          *self._ws()), "ttcd_shard_attend")
        return u_tail

    def mix(self, beta, u_halo):
        p = self.p
        nh = min(p.conv_k - 1, self.pos0)
        if nh > 0 and (u_halo is None or u_halo.shape[2] != nh):
            raise ValueError(f"MLP-input halo of {None if u_halo is None else u_halo.shape[2]} "
                             f"rows, need {nh}")
        total = torch.empty(p.B, p.d_model, p.d_ff, device=self.device, dtype=torch.float32)
        _check(self.lib.ttcd_shard_mix(_ptr(beta), _ptr(u_halo) if nh > 0 else None,
                                       ctypes.byref(self.wc), ctypes.byref(self.pc), self.pos0,
                                       _ptr(total), *self._ws()), "ttcd_shard_mix")
        return total

    def finish(self, state_in=None, state_out: bool = True):
        p = self.p
        out = torch.empty(p.B, p.T, p.d_model, device=self.device, dtype=torch.bfloat16)
        st = (torch.empty(p.B, p.d_model, p.d_ff, device=self.device, dtype=torch.float32)
              if state_out else None)
        _check(self.lib.ttcd_shard_finish(ctypes.byref(self.wc), ctypes.byref(self.pc),
                                          self.pos0, _ptr(state_in), _ptr(st), _ptr(out),
                                          *self._ws()), "ttcd_shard_finish")
        return out, st

    def check_status(self) -> int:
        return check_device_status(self.ws, self.stream)


def fastweight_mlp(u_T, u_S, beta, weights: Dict[str, torch.Tensor], p: BlockParams, h_S=None,
                   state_in=None, state_out: bool = False, y=None,
                   workspace: Optional[torch.Tensor] = None, stream=None):
    """In-place fast-weight MLP.  Returns (y, state_out or None, workspace)."""
    lib = load_library()
    need = fastweight_mlp_workspace_size(p)
    if need == 0:
        raise TTCDError(ERR_INVALID_ARG, "ttcd_fastweight_mlp_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, u_T.device)
    y = torch.empty_like(u_S) if y is None else y
    st_t = (torch.empty(p.B, p.d_model, p.d_ff, device=u_T.device, dtype=torch.float32)
            if state_out else None)
    pc, wc = p.c(), _weights(weights)
    st = lib.ttcd_fastweight_mlp(_ptr(u_T), _ptr(u_S), _ptr(h_S), _ptr(beta), ctypes.byref(wc),
                                 ctypes.byref(pc), _ptr(state_in), _ptr(st_t), _ptr(y),
                                 _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "ttcd_fastweight_mlp")
    return y, st_t, workspace


def block_backward(x, beta, weights: Dict[str, torch.Tensor], p: BlockParams, d_out,
                   state_in=None, d_state_out=None, workspace: Optional[torch.Tensor] = None,
                   stream=None):
    """Vector-Jacobian product of ``block_forward`` (bf16, hd 64 or 128): the
    gradients of a loss with dL/dout = d_out and dL/dstate_out = d_state_out (or
    zero) with respect to x, beta, state_in and the ten weights, all fp32.
    Returns (grads dict keyed "x", "beta", "state_in" and the weight names;
    workspace)."""
    lib = load_library()
    need = int(lib.ttcd_block_backward_workspace_size(ctypes.byref(p.c())))
    if need == 0:
        raise TTCDError(ERR_UNSUPPORTED, "ttcd_block_backward_workspace_size")
    dev = x.device
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    f32 = dict(device=dev, dtype=torch.float32)
    g = {"x": torch.empty(p.B, p.T, p.d_model, **f32), "beta": torch.empty(p.B, p.T, **f32),
         "state_in": torch.empty(p.B, p.d_model, p.d_ff, **f32)}
    for n in WEIGHT_NAMES:
        g[n] = torch.empty(weights[n].shape, **f32)
    gc = _BlockGrads(*[_ptr(g[n]) for n in WEIGHT_NAMES])
    pc, wc = p.c(), _weights(weights)
    st = lib.ttcd_block_backward(_ptr(x), _ptr(beta), ctypes.byref(wc), ctypes.byref(pc),
                                 _ptr(state_in), _ptr(d_out), _ptr(d_state_out), _ptr(g["x"]),
                                 _ptr(g["beta"]), _ptr(g["state_in"]), ctypes.byref(gc),
                                 _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "ttcd_block_backward")
    return g, workspace


def fastweight_mlp_backward(u_T, u_S, beta, weights: Dict[str, torch.Tensor], p: BlockParams,
                            d_y, state_in=None, d_state_out=None,
                            workspace: Optional[torch.Tensor] = None, stream=None):
    """Vector-Jacobian product of ``fastweight_mlp`` (bf16): the gradients of a
    loss with dL/dy = d_y and dL/dstate_out = d_state_out (or zero) with respect
    to u_T, u_S, beta, state_in and the MLP weights, all fp32.  Returns
    (grads dict keyed "u_T", "u_S", "beta", "state_in", "w_gate", "w_up",
    "w_down", "w_proj", "conv_T", "conv_S"; workspace)."""
    lib = load_library()
    need = int(lib.ttcd_fastweight_mlp_backward_workspace_size(ctypes.byref(p.c())))
    if need == 0:
        raise TTCDError(ERR_UNSUPPORTED, "ttcd_fastweight_mlp_backward_workspace_size")
    dev = u_T.device
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    f32 = dict(device=dev, dtype=torch.float32)
    B, T, d, f, k = p.B, p.T, p.d_model, p.d_ff, p.conv_k
    g = {"u_T": torch.empty(B, T, d, **f32), "u_S": torch.empty(B, T, d, **f32),
         "beta": torch.empty(B, T, **f32), "state_in": torch.empty(B, d, f, **f32),
         "w_gate": torch.empty(f, d, **f32), "w_up": torch.empty(f, d, **f32),
         "w_down": torch.empty(d, f, **f32), "w_proj": torch.empty(f, f, **f32),
         "conv_T": torch.empty(f, k, **f32), "conv_S": torch.empty(f, k, **f32)}
    gc = _MlpGrads(*[_ptr(g[n]) for n, _ in _MlpGrads._fields_])
    pc, wc = p.c(), _weights(weights)
    st = lib.ttcd_fastweight_mlp_backward(
        _ptr(u_T), _ptr(u_S), _ptr(beta), ctypes.byref(wc), ctypes.byref(pc), _ptr(state_in),
        _ptr(d_y), _ptr(d_state_out), _ptr(g["u_T"]), _ptr(g["u_S"]), _ptr(g["beta"]),
        _ptr(g["state_in"]), ctypes.byref(gc), _ptr(workspace), workspace.numel(),
        _stream(stream))
    _check(st, "ttcd_fastweight_mlp_backward")
    return g, workspace


def fastweight_mlp_noalloc(u_T, u_S, beta, weights: Dict[str, torch.Tensor], p: BlockParams,
                           h_S=None, state_in=None, state_out=None, y=None, stream=None):
    """ttcd_fastweight_mlp without a workspace: for callers that cannot allocate scratch.

    The library's scratch is its fixed 32 MiB device array; larger problems are
    rejected.  The outputs are ordinary tensors: ``y`` ([B, T, d], the type of
    u) and ``state_out`` (fp32 [B, d, f], or True to have one allocated) are
    the caller's when given, and this wrapper allocates ``y`` when it is None
    (a caller that may not allocate passes its own).  Calls that overlap on the
    GPU race on the shared array.  Returns (y, state_out or None).
    """
    lib = load_library()
    if y is None:
        y = torch.empty_like(u_S)
    if state_out is True:
        state_out = torch.empty(p.B, p.d_model, p.d_ff, device=u_S.device, dtype=torch.float32)
    elif state_out is False:
        state_out = None
    pc, wc = p.c(), _weights(weights)
    st = lib.ttcd_fastweight_mlp_noalloc(_ptr(u_T), _ptr(u_S), _ptr(h_S), _ptr(beta),
                                         ctypes.byref(wc), ctypes.byref(pc), _ptr(state_in),
                                         _ptr(state_out), _ptr(y), _stream(stream))
    _check(st, "ttcd_fastweight_mlp_noalloc")
    return y, state_out


def check_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Status of the calls that used this workspace (or decode state) since the
    last check: OK or ERR_TIMEOUT.  Reads and clears its status word; synchronises."""
    return load_library().ttcd_check_device_status(_ptr(workspace), _stream(stream))


def get_device_error(stream=None) -> Tuple[int, int]:
    """(status, raw flags) of the per-device status word of the entry points
    without a workspace (attention, the MLP without scratch); clears it.
    Synchronises."""
    flags = ctypes.c_uint32(0)
    st = load_library().ttcd_get_device_error(ctypes.byref(flags), _stream(stream))
    return st, flags.value


def set_wait_timeout_ns(ns: int) -> None:
    load_library().ttcd_set_wait_timeout_ns(ns)


def kernel_launch_count() -> int:
    return int(load_library().ttcd_kernel_launch_count())


def test_bounded_wait(timeout_ns: int, status: Optional[torch.Tensor] = None, stream=None) -> int:
    """Self-test of the bounded waits: a wait that nothing ends gives up after
    ``timeout_ns`` and records a timeout in ``status`` (a workspace or decode
    state) or, when None, in the per-device word."""
    return load_library().ttcd_test_bounded_wait(timeout_ns, _ptr(status), _stream(stream))


def attn_timeline_read():
    """The instrumented attention kernel's clock64 marks of its last launch as a
    [2 heads, 128 visits, 8 marks] int64 tensor (libttcd_timeline.so only; the
    normal library raises TTCDError with status unsupported)."""
    n = 2 * 128 * 8
    buf = (ctypes.c_longlong * n)()
    _check(load_library().ttcd_attn_timeline_read(buf, n), "ttcd_attn_timeline_read")
    return torch.tensor(list(buf), dtype=torch.int64).view(2, 128, 8)


def test_exp2_poly(x: torch.Tensor, stream=None) -> torch.Tensor:
    """The attention kernel's FMA-pipe 2^x evaluated at x (fp32 CUDA tensor)."""
    y = torch.empty_like(x)
    _check(load_library().ttcd_test_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)),
           "ttcd_test_exp2_poly")
    return y
