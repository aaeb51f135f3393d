/*
 * ttcd.h — C ABI of libttcd: the forward pass of one IP-TTCD block
 * (In-Place Test-Time Context Distillation) on NVIDIA B200 (sm_100a).
 *
 * Sources of the definitions (cited by page title and section):
 *   [README]  GitHub README "TTCD: Test-Time Training via Context Distillation",
 *             sections "Model configuration" and "Fused inference kernels".
 *   [REVIEW]  papernotes.org review "Learning What to Remember: Test-Time
 *             Training via Context Distillation", section 方法详解 (overall
 *             framework, flowchart A-F) and 关键设计 2-3 (in-place fast weight,
 *             off-policy approximation, short convs, W_proj, R_i, K_i, Delta W).
 *   [PODCAST] podcast transcript "Test-Time Training via Context Distillation:
 *             Learning What to Remember", cues 19 (sliding window) and 29
 *             (practical update).
 *
 * Conventions for every entry point:
 *   - Every pointer argument named as a tensor is a DEVICE pointer, owned by the
 *     caller; the library never allocates or frees device memory.  Scratch
 *     space comes only from the caller's `workspace` (size from the matching
 *     *_workspace_size query).  Parameter structs are HOST pointers, read during
 *     the call only.
 *   - Layouts are dense row-major with the last index fastest: activations
 *     [B, T, ...], weights in the `[out, in]` Linear convention (y = x W^T).
 *   - Every device pointer must be 16-byte aligned; each tensor's innermost
 *     extent times its element size must be a multiple of 16 bytes.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and keep no state between calls: everything a call writes is in
 *     the caller's buffers.  Calls on different workspaces may run concurrently
 *     on different streams or host threads.  Process-wide settings are only the
 *     wait bound (ttcd_set_wait_timeout_ns) and a diagnostic launch counter.
 *   - Arguments are validated on the host before any launch; a bad argument
 *     returns TTCD_ERR_INVALID_ARG or TTCD_ERR_UNSUPPORTED and launches nothing.
 *     A launch failure returns TTCD_ERR_CUDA.
 *   - Every device-side wait is bounded.  One that gives up records
 *     TTCD_ERR_TIMEOUT in the call's status word and the kernel returns; no
 *     entry point aborts, traps or throws.  The status word is the first 4 bytes
 *     of the call's workspace (block forward, fast-weight MLP) or decode state:
 *     it accumulates over calls until ttcd_check_device_status() reads and
 *     clears it, so zero the first TTCD_STATUS_BYTES bytes of a new workspace
 *     before its first use (ttcd_decode_state_init clears a decode state).
 *     Entry points without a workspace (the two attention calls and
 *     ttcd_fastweight_mlp_noalloc) record into one status word per device,
 *     shared by all their callers and read by ttcd_get_device_error().
 */
#ifndef TTCD_H_
#define TTCD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTCD_OK = 0,
  TTCD_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, inconsistent sizes   */
  TTCD_ERR_UNSUPPORTED = 2,  /* valid but not implemented (head_dim, dtype)    */
  TTCD_ERR_CUDA = 3,         /* a CUDA runtime/driver call or launch failed    */
  TTCD_ERR_TIMEOUT = 4,      /* a bounded device wait gave up                  */
  TTCD_ERR_WORKSPACE = 5     /* workspace smaller than the size query returned */
} ttcd_status;

typedef enum { TTCD_F32 = 0, TTCD_BF16 = 1 } ttcd_dtype;

/* Bytes at the start of every workspace and decode state that hold its status
 * word (the rest of the region is reserved). */
#define TTCD_STATUS_BYTES 256

/* Shape and hyper-parameters of one block.  Names follow the pages:
 * window_size = teacher window w_T, student window w_S, fast-weight chunk C,
 * conv width ([README] "Model configuration"). */
typedef struct {
  int B;              /* sequences in the batch                                */
  int T;              /* tokens per sequence                                   */
  int d_model;        /* d, a multiple of 64                                   */
  int n_q_heads;      /* Hq                                                    */
  int n_kv_heads;     /* Hkv, Hq % Hkv == 0; query head h reads KV head h/(Hq/Hkv) */
  int head_dim;       /* hd in {32, 64, 128}; (Hq + 2 Hkv) hd a multiple of 64 */
  int d_ff;           /* f                                                     */
  int w_S;            /* student window, 1 <= w_S <= w_T                       */
  int w_T;            /* teacher window                                        */
  int chunk;          /* C >= 1; a partial last chunk is allowed               */
  int conv_k;         /* depthwise conv width, 1..8                            */
  float rms_eps;      /* RMSNorm epsilon (1e-6)                                */
  float l2_eps;       /* key normalisation epsilon (1e-6)                      */
  float rope_theta;   /* RoPE base (1e4)                                       */
  float softmax_scale;/* 0 => 1/sqrt(head_dim)                                 */
  ttcd_dtype dtype;   /* type of x, weights and out (beta/state are fp32)      */
} ttcd_block_params;

/* Slow weights W^(0) of one block, device pointers in params.dtype.
 * w_qkv rows: Hq*hd query rows, then Hkv*hd key rows, then Hkv*hd value rows. */
typedef struct {
  const void* w_qkv;  /* [(Hq + 2 Hkv) hd, d]                                  */
  const void* w_o;    /* [d, Hq hd]   shared by teacher and student            */
  const void* g_attn; /* [d]          input RMSNorm gain                       */
  const void* g_mlp;  /* [d]          MLP RMSNorm gain (shared by both paths)  */
  const void* w_gate; /* [f, d]                                                */
  const void* w_up;   /* [f, d]                                                */
  const void* w_down; /* [d, f]       W_down^(0), the in-place fast weight's base */
  const void* w_proj; /* [f, f]       learned projection of the value residual */
  const void* conv_T; /* [f, k]       teacher conv taps, tap m multiplies t-m  */
  const void* conv_S; /* [f, k]       student conv taps                        */
} ttcd_block_weights;

/*
 * ttcd_dual_window_attn — fused dual-window causal sliding-window attention.
 *
 * Defines ([README] "Fused inference kernels", fused_dual_attn; [REVIEW]
 * 方法详解 overall framework; [PODCAST] cue 19): for every query t and head h,
 *   o_W[t,h] = sum_{j in win_W(t)} softmax_j(scale * q[t,h].k[j,g]) v[j,g],
 *   win_W(t) = { j : max(0, t-W+1) <= j <= t },  g = h / (Hq/Hkv),
 * for W = w_T (teacher, o_T) and W = w_S (student, o_S), computed in one pass
 * over K/V that reuses each Q.K^T tile for both windows.
 *   q          [B, T, Hq, hd]  bf16, device
 *   k, v       [B, T, Hkv, hd] bf16, device
 *   o_T, o_S   [B, T, Hq, hd]  bf16, device, written
 *   lse_T/lse_S [B, Hq, T] fp32 natural-log log-sum-exp, device, nullable
 *   scale      softmax scale; 0 => 1/sqrt(hd)
 *   dtype      must be TTCD_BF16 (TTCD_F32 -> TTCD_ERR_UNSUPPORTED)
 * Errors: hd not in {32,64,128}, Hq % Hkv != 0, w_S < 1, w_S > w_T, B or T < 1,
 * null/misaligned pointers -> TTCD_ERR_INVALID_ARG / TTCD_ERR_UNSUPPORTED.
 */
ttcd_status ttcd_dual_window_attn(const void* q, const void* k, const void* v, void* o_T,
                                  void* o_S, float* lse_T, float* lse_S, int B, int T, int Hq,
                                  int Hkv, int hd, int w_S, int w_T, float scale,
                                  ttcd_dtype dtype, void* stream);

/*
 * ttcd_dual_window_attn_lse — the same two outputs by LSE combination.
 *
 * Defines ([README] "Fused inference kernels", lse_dual_attn): the teacher
 * window is the student window plus the shifted far band
 *   far(t) = { j : max(0, t-w_T+1) <= j <= t-w_S },
 * attended separately and merged exactly through the log-sum-exps:
 *   o_T = (o_S e^{lse_S} + o_far e^{lse_far}) / (e^{lse_S} + e^{lse_far}),
 *   lse_T = log(e^{lse_S} + e^{lse_far}).
 * A row whose far band is empty (t < w_S, or w_S = w_T) gets o_far = 0 and
 * lse_far = -inf, and then o_T = o_S.  A second implementation of
 * ttcd_dual_window_attn (one pass over K/V; the accumulator restarts at the
 * student edge) followed by an elementwise merge.
 *   q, k, v, o_T, o_S, scale, dtype, errors: as ttcd_dual_window_attn
 *   o_far      [B, T, Hq, hd]  bf16, device, written (far-band attention)
 *   lse_S, lse_far [B, Hq, T] fp32, device, written (required: the merge reads them)
 *   lse_T      [B, Hq, T] fp32, device, nullable
 */
ttcd_status ttcd_dual_window_attn_lse(const void* q, const void* k, const void* v, void* o_T,
                                      void* o_S, void* o_far, float* lse_T, float* lse_S,
                                      float* lse_far, int B, int T, int Hq, int Hkv, int hd,
                                      int w_S, int w_T, float scale, ttcd_dtype dtype,
                                      void* stream);

/* Workspace bytes of ttcd_dual_window_attn_backward (status word, and per
 * window the [B, Hq, T] row dot products and base-2 log-sum-exps, padded to a
 * multiple of 128 tokens, fp32); 0 for invalid sizes. */
size_t ttcd_dual_window_attn_backward_workspace_size(int B, int T, int Hq);

/*
 * ttcd_dual_window_attn_backward — vector-Jacobian product of ttcd_dual_window_attn.
 *
 * For a scalar loss L with dL/do_T = do_T and dL/do_S = do_S, the gradients
 * with respect to q, k and v, both windows together ([REVIEW] 局限与展望:
 * training differentiates both attention windows; each window is the softmax
 * attention of ttcd_dual_window_attn):
 *   per window P: dV += P^T dO_P,  dS = P (dO_P V^T - rowsum(dO_P o_P)) scale,
 *                 dK += dS^T Q,  dQ += dS K   (query heads of a group add into
 *                 their KV head).
 * P is rebuilt from the forward's log-sum-exp, so the call takes the forward's
 * o_T, o_S, lse_T and lse_S (from ttcd_dual_window_attn with both lse outputs).
 *   q, k, v        [B, T, H, hd] bf16, device (as the forward)
 *   o_T, o_S       [B, T, Hq, hd] bf16, device (the forward's outputs)
 *   lse_T, lse_S   [B, Hq, T] fp32, device (the forward's log-sum-exps)
 *   do_T, do_S     [B, T, Hq, hd] bf16, device
 *   dq             [B, T, Hq, hd] fp32, device, written
 *   dk, dv         [B, T, Hkv, hd] fp32, device, written
 *   hd             64 or 128 (32: TTCD_ERR_UNSUPPORTED)
 *   workspace      >= ttcd_dual_window_attn_backward_workspace_size(B, T, Hq) bytes,
 *                  device, 16-byte aligned; status word first
 * Precision: bf16 tensor-core operands (q, k, v, dO and the rebuilt P and dS
 * rounded to bf16), fp32 accumulation; dq sums the key tiles' contributions
 * with fp32 reductions in L2, so its low bits depend on their order.
 */
ttcd_status ttcd_dual_window_attn_backward(const void* q, const void* k, const void* v,
                                           const void* o_T, const void* o_S, const float* lse_T,
                                           const float* lse_S, const void* do_T,
                                           const void* do_S, float* dq, float* dk, float* dv,
                                           int B, int T, int Hq, int Hkv, int hd, int w_S,
                                           int w_T, float scale, void* workspace,
                                           size_t ws_bytes, void* stream);

/*
 * ttcd_fastweight_mlp — the in-place fast-weight MLP of one block (off-policy).
 *
 * Defines ([REVIEW] 关键设计 2 and 3, flowchart C-F; [PODCAST] cue 29):
 *   Z_P   = silu(u_P W_gate^T) * (u_P W_up^T)            P in {T, S}, slow weights
 *   Zb_P  = conv_P(Z_P)   causal depthwise, tap m multiplies t-m, zero history
 *   r_t   = W_down W_proj (Zb_T - Zb_S)[t]               value residual
 *   k_t   = Zb_S[t] / sqrt(||Zb_S[t]||^2 + l2_eps)       key
 *   dW_i  = sum_{t in chunk i} beta_t r_t k_t^T          [d, f]
 *   S_0   = state_in (or 0),  S_{i+1} = S_i + dW_i       fp32 exclusive prefix
 *   y_t   = h_S[t] + (W_down + S_{i(t)}) Z_S[t]          (h_S term if non-null)
 *   state_out = S_{n_chunks} (includes a partial last chunk)
 *   u_T, u_S   [B, T, d] post-RMSNorm activations, params.dtype, device
 *   h_S        [B, T, d] params.dtype, device, nullable (residual added to y)
 *   beta       [B, T] fp32, device
 *   state_in   [B, d, f] fp32, device, nullable;  state_out likewise
 *   y          [B, T, d] params.dtype, device, written
 *   workspace  >= ttcd_fastweight_mlp_workspace_size(p) bytes, device, 16-byte aligned;
 *              its first TTCD_STATUS_BYTES bytes hold the call's status word
 * Precision: TTCD_BF16 contracts bf16 operands with fp32 accumulation, except
 * when T < chunk: a state written by fewer than `chunk` tokens does not average
 * out the bf16 rounding of u, D, M, R and k', so such calls widen the inputs and
 * weights exactly to fp32 in the workspace and contract them as tf32 (fp32
 * accumulation); y is rounded to bf16 once.  TTCD_F32 always uses tf32.
 */
ttcd_status ttcd_fastweight_mlp(const void* u_T, const void* u_S, const void* h_S,
                                const float* beta, const ttcd_block_weights* w,
                                const ttcd_block_params* p, const float* state_in,
                                float* state_out, void* y, void* workspace, size_t ws_bytes,
                                void* stream);

/* fp32 gradients of the fast-weight MLP's weights (device, written, not accumulated). */
typedef struct {
  float* w_gate; /* [d_ff, d_model] */
  float* w_up;   /* [d_ff, d_model] */
  float* w_down; /* [d_model, d_ff] */
  float* w_proj; /* [d_ff, d_ff] */
  float* conv_T; /* [d_ff, conv_k] */
  float* conv_S; /* [d_ff, conv_k] */
} ttcd_mlp_grads;

/* Workspace bytes of ttcd_fastweight_mlp_backward; 0 when p is invalid or not TTCD_BF16. */
size_t ttcd_fastweight_mlp_backward_workspace_size(const ttcd_block_params* p);

/*
 * ttcd_fastweight_mlp_backward — vector-Jacobian product of ttcd_fastweight_mlp.
 *
 * For a scalar loss L with dL/dy = d_y and dL/dstate_out = d_state_out, the
 * gradients of L with respect to u_T, u_S, beta, state_in and the six MLP
 * weights, by the chain rule of the steps listed at ttcd_fastweight_mlp taken in
 * reverse ([REVIEW] 关键设计 2-3; the write path is differentiated too: W_proj,
 * the two convs and beta reach the loss only through the fast-weight writes;
 * [REVIEW] 局限与展望 on training cost).  The forward's intermediates are
 * recomputed in the workspace, so the call takes the forward's inputs.
 *   u_T, u_S, beta, w, p, state_in: as ttcd_fastweight_mlp (TTCD_BF16 only)
 *   d_y          [B, T, d] bf16, device
 *   d_state_out  [B, d, f] fp32, device, nullable (zero)
 *   du_T, du_S   [B, T, d] fp32, device, written
 *   d_beta       [B, T] fp32, device, written
 *   d_state_in   [B, d, f] fp32, device, nullable, written
 *   grads        the weight gradients (all six pointers required)
 *   workspace    >= ttcd_fastweight_mlp_backward_workspace_size(p) bytes, device,
 *                16-byte aligned; status word first, as for the forward
 * Precision: bf16 GEMM operands (u, dy, Z_S, the per-chunk G_i and W_i, the
 * row gradients dRt, s dRt and [da | db], dM), fp32 accumulation, fp32
 * element-wise steps and outputs.
 * Errors: TTCD_ERR_UNSUPPORTED for TTCD_F32; otherwise as ttcd_fastweight_mlp.
 */
ttcd_status ttcd_fastweight_mlp_backward(const void* u_T, const void* u_S, const float* beta,
                                         const ttcd_block_weights* w, const ttcd_block_params* p,
                                         const float* state_in, const void* d_y,
                                         const float* d_state_out, float* du_T, float* du_S,
                                         float* d_beta, float* d_state_in,
                                         const ttcd_mlp_grads* grads, void* workspace,
                                         size_t ws_bytes, void* stream);

/*
 * ttcd_block_forward — forward pass of one IP-TTCD block (student path output).
 *
 * Defines ([REVIEW] 方法详解 overall framework + flowchart A-F; readings of the
 * unstated skeleton: pre-norm, no biases, rotate-half RoPE at positions 0..T-1):
 *   xn = RMSNorm(x; g_attn);  q,k,v = xn W_qkv^T;  q,k = RoPE(q,k)
 *   o_T, o_S = ttcd_dual_window_attn(q, k, v)
 *   h_P = x + o_P W_o^T;  u_P = RMSNorm(h_P; g_mlp)
 *   out = ttcd_fastweight_mlp(u_T, u_S, h_S, beta, ...)
 *   x, out     [B, T, d] params.dtype, device
 *   beta       [B, T] fp32, device
 *   state_out  [B, d, f] fp32, device, nullable (final fast-weight state)
 *   workspace  >= ttcd_block_forward_workspace_size(p) bytes, device, 16-byte aligned;
 *              its first TTCD_STATUS_BYTES bytes hold the call's status word
 * The workspace holds every intermediate after the call; their byte offsets
 * are returned by ttcd_block_workspace_offset().  The input RMSNorm is applied
 * as a row scale 1/rms(x) in the QKV epilogue with its gain folded into a copy
 * of W_qkv (xn W_qkv^T = (x (W_qkv diag g_attn)^T) / rms(x)).  Precision as
 * ttcd_fastweight_mlp: TTCD_BF16 with T < chunk runs the whole block on fp32
 * copies (tf32 MMAs; q, k, v stay bf16).
 */
ttcd_status ttcd_block_forward(const void* x, const float* beta, const ttcd_block_weights* w,
                               const ttcd_block_params* p, float* state_out, void* out,
                               void* workspace, size_t ws_bytes, void* stream);

/*
 * ttcd_swa_block_forward — one plain sliding-window transformer block: a layer
 * of an IP-TTCD model that is not in its TTT layer set (GitHub README "TTCD",
 * "Model configuration": ttt_layers picks the layers that learn at test time;
 * window_size is the attention window of every layer, the teacher window).
 * It has no student path and no fast weights:
 *   xn = RMSNorm(x; g_attn);  q,k,v = xn W_qkv^T;  q,k = RoPE(q,k)
 *   h = x + SWA_{w_T}(q, k, v) W_o^T     (keys [t - w_T + 1, t], GQA)
 *   out = h + W_down (silu(u W_gate^T) * (u W_up^T)),  u = RMSNorm(h; g_mlp)
 * Arguments and layouts as ttcd_block_forward; params.w_S, chunk, conv_k,
 * l2_eps and the weights w_proj, conv_T, conv_S are not read (they may be
 * null).  workspace >= ttcd_swa_block_forward_workspace_size(p) bytes, 16-byte
 * aligned, status word first.  Precision: bf16 operands (TTCD_BF16, at every
 * T) or fp32 with tf32 MMAs (TTCD_F32); q, k, v and the attention are bf16;
 * fp32 accumulation and residual.  Errors as ttcd_block_forward.
 */
ttcd_status ttcd_swa_block_forward(const void* x, const ttcd_block_weights* w,
                                   const ttcd_block_params* p, void* out, void* workspace,
                                   size_t ws_bytes, void* stream);
size_t ttcd_swa_block_forward_workspace_size(const ttcd_block_params* p);

/* fp32 gradients of the block's weights (device, written, not accumulated);
 * fields in the order and shapes of ttcd_block_weights. */
typedef struct {
  float* w_qkv;  /* [(Hq + 2 Hkv) hd, d] */
  float* w_o;    /* [d, Hq hd] */
  float* g_attn; /* [d] */
  float* g_mlp;  /* [d] */
  float* w_gate; /* [f, d] */
  float* w_up;   /* [f, d] */
  float* w_down; /* [d, f] */
  float* w_proj; /* [f, f] */
  float* conv_T; /* [f, conv_k] */
  float* conv_S; /* [f, conv_k] */
} ttcd_block_grads;

/* Workspace bytes of ttcd_block_backward; 0 when p is invalid, not TTCD_BF16
 * or head_dim is not 64 or 128. */
size_t ttcd_block_backward_workspace_size(const ttcd_block_params* p);

/*
 * ttcd_block_backward — vector-Jacobian product of ttcd_block_forward.
 *
 * For a scalar loss L with dL/dout = d_out and dL/dstate_out = d_state_out,
 * the gradients of L with respect to x, beta, state_in and every weight: the
 * chain rule of the steps listed at ttcd_block_forward in reverse ([REVIEW]
 * 方法详解 flowchart A-F, 关键设计 2-3; training differentiates the whole block,
 * [REVIEW] 局限与展望).  The forward is recomputed in the workspace.
 *   x, beta, w, p, state_in: as ttcd_block_forward (TTCD_BF16, hd 64 or 128)
 *   d_out        [B, T, d] bf16, device
 *   d_state_out  [B, d, f] fp32, device, nullable (zero)
 *   dx           [B, T, d] fp32, device, written
 *   d_beta       [B, T] fp32, device, written
 *   d_state_in   [B, d, f] fp32, device, nullable, written
 *   grads        the ten weight gradients (all required)
 *   workspace    >= ttcd_block_backward_workspace_size(p) bytes, device, 16-byte
 *                aligned; status word first
 * Precision: as ttcd_fastweight_mlp_backward and ttcd_dual_window_attn_backward;
 * the RMSNorm backward steps are fp32.
 * Errors: TTCD_ERR_UNSUPPORTED for TTCD_F32, head_dim 32 or d_model > 12288.
 */
ttcd_status ttcd_block_backward(const void* x, const float* beta, const ttcd_block_weights* w,
                                const ttcd_block_params* p, const float* state_in,
                                const void* d_out, const float* d_state_out, float* dx,
                                float* d_beta, float* d_state_in, const ttcd_block_grads* grads,
                                void* workspace, size_t ws_bytes, void* stream);

/*
 * ttcd_block_forward_profiled — ttcd_block_forward that also records the
 * caller's CUDA events (cudaEvent_t handles, owned by the caller) on `stream`
 * at its stage boundaries, for per-stage timing.  Not part of the method.
 *   events[k] is recorded at boundary k: 0 start, 1 after the rotary table, the
 *   input RMS row scales and the gain-scaled W_qkv, 2 after QKV+RoPE, 3 after
 *   attention, 4 after o_proj (with the MLP RMSNorm statistics), 5 after
 *   gate/up+SwiGLU (with bf16 operands, the convs, D and the keys are in the
 *   same kernel), 6 after the key scales (fp32 operands: the conv/residual/key
 *   kernel and the key scales), 7 after M = W_down W_proj,
 *   8 after R, 9 after the chunk scan, 10 after the output GEMM.  Boundaries at
 *   or beyond n_events are skipped; 0 <= n_events <= 16; events[0..n_events-1]
 *   must be non-null.  The events belong to this call only.
 */
ttcd_status ttcd_block_forward_profiled(const void* x, const float* beta,
                                        const ttcd_block_weights* w, const ttcd_block_params* p,
                                        float* state_out, void* out, void* workspace,
                                        size_t ws_bytes, void* stream, void* const* events,
                                        int n_events);

/*
 * Sequence-sharded block forward: the four phases of one shard.
 *
 * A sequence-parallel run splits every sequence into contiguous shards of whole
 * chunks, one per rank (GPU), in rank order; only the last shard may end in a
 * partial chunk.  The block is causal (windowed attention over earlier tokens,
 * causal short convs, a causal prefix over chunks: [REVIEW] 整体框架 and
 * 关键设计 2-3; [README] "Model configuration" names flame's context
 * parallelism for long-context training), so a shard needs three things from
 * the shards before it, exchanged by the caller between the phases:
 *   - the rotated K and V of the n_halo = min(w_T - 1, pos0) tokens before it
 *     (the teacher window's reach);
 *   - the MLP inputs u_P = RMSNorm(h_P; g_mlp) of the min(conv_k - 1, pos0)
 *     tokens before it, from which it recomputes their Z_T, Z_S (the short
 *     convs' history);
 *   - the sum of the earlier shards' chunk increments (plus the block's
 *     state_in), its state_in: the exclusive prefix over chunks taken over
 *     shards first.
 * Each phase exports what the next shard needs from this one; a halo may span
 * several earlier shards, so the caller passes on the last rows of (halo it
 * received, tail this shard exported).  Run on shards in any order subject to
 * those exchanges, and concatenated, the shards' outputs are the rows of
 * ttcd_block_forward over the whole sequence and the last shard's state_out is
 * its state_out.
 *
 * Every phase of one shard takes the same p (p->T = this shard's tokens; p->dtype
 * TTCD_BF16), pos0 (the absolute position of its first token, a multiple of
 * p->chunk) and workspace (>= ttcd_shard_workspace_size(p) bytes, 16-byte
 * aligned, status word first), which carries the shard's intermediates from
 * phase to phase.  kv rows are [2, Hkv, hd] bf16 (K heads, then V heads).
 *
 * ttcd_shard_qkv: input RMSNorm, QKV, RoPE at positions pos0 .. pos0 + T - 1.
 *   x [B, T, d] bf16;  kv_tail [B, min(T, w_T - 1), 2 Hkv hd] bf16, written
 *   (nullable): the rotated K, V of this shard's last min(T, w_T - 1) tokens.
 * ttcd_shard_attend: dual-window attention of the shard's queries over
 *   (K/V halo, own K/V), o_proj for both paths with the residual, MLP RMSNorm.
 *   kv_halo [B, n_halo, 2 Hkv hd] bf16 (required when n_halo > 0);
 *   u_tail [2, B, min(T, conv_k - 1), d] bf16, written (nullable): the
 *   normalised MLP inputs of the shard's last tokens, teacher then student.
 * ttcd_shard_mix: the fast-weight MLP up to the chunk increments, and their sum.
 *   beta [B, T] fp32;  u_halo [2, B, min(conv_k - 1, pos0), d] bf16 (required
 *   when pos0 > 0 and conv_k > 1);  total [B, d, f] fp32, written: the sum of
 *   this shard's chunk increments Delta W_i.
 * ttcd_shard_finish: the fp32 prefix from state_in over the shard's chunks and
 *   the output y = h_S + (W_down + S_i) Z_S.
 *   state_in [B, d, f] fp32 (nullable: zero);  state_out [B, d, f] fp32
 *   (nullable): the state after this shard;  out [B, T, d] bf16, written.
 * Errors as ttcd_block_forward; pos0 < 0 or not a multiple of chunk ->
 * TTCD_ERR_INVALID_ARG; TTCD_F32 -> TTCD_ERR_UNSUPPORTED.  Precision: bf16
 * operands at every T (the fp32-operand route of short problems is not taken).
 */
size_t ttcd_shard_workspace_size(const ttcd_block_params* p);
ttcd_status ttcd_shard_qkv(const void* x, const ttcd_block_weights* w, const ttcd_block_params* p,
                           long long pos0, void* kv_tail, void* workspace, size_t ws_bytes,
                           void* stream);
ttcd_status ttcd_shard_attend(const void* x, const void* kv_halo, const ttcd_block_weights* w,
                              const ttcd_block_params* p, long long pos0, void* u_tail,
                              void* workspace, size_t ws_bytes, void* stream);
ttcd_status ttcd_shard_mix(const float* beta, const void* u_halo, const ttcd_block_weights* w,
                           const ttcd_block_params* p, long long pos0, float* total,
                           void* workspace, size_t ws_bytes, void* stream);
ttcd_status ttcd_shard_finish(const ttcd_block_weights* w, const ttcd_block_params* p,
                              long long pos0, const float* state_in, float* state_out, void* out,
                              void* workspace, size_t ws_bytes, void* stream);

/*
 * ttcd_fastweight_mlp_noalloc — ttcd_fastweight_mlp for callers that cannot
 * provide scratch memory.  The paper has no counterpart; this is a deployment
 * convenience.
 *
 * Who needs it: callers whose device memory is owned entirely by a host
 * framework's pool with no way to borrow a workspace from it, and callers in
 * latency-critical loops that may not call cudaMalloc (it can synchronise the
 * device).  Same arguments and result as ttcd_fastweight_mlp, without the
 * workspace pair: the scratch is a fixed 32 MiB array compiled into the library
 * (held by every GPU that loads the library until the process exits).  The
 * library allocates nothing for it.
 *   - Problems whose ttcd_fastweight_mlp_workspace_size exceeds
 *     ttcd_fastweight_mlp_noalloc_capacity() (32 MiB) are rejected with
 *     TTCD_ERR_WORKSPACE before anything is launched.
 *   - The first call on each device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (every byte a call reads is written earlier in the same call, so
 *     nothing needs clearing).  Calls whose kernels overlap on the GPU (other
 *     streams, other host threads) race on it: serialise them.
 *   - With no workspace to hold a status word, a wait that gives up is recorded
 *     in the per-device word read by ttcd_get_device_error().
 */
ttcd_status ttcd_fastweight_mlp_noalloc(const void* u_T, const void* u_S, const void* h_S,
                                        const float* beta, const ttcd_block_weights* w,
                                        const ttcd_block_params* p, const float* state_in,
                                        float* state_out, void* y, void* stream);

/* Bytes of the fixed scratch array used by ttcd_fastweight_mlp_noalloc. */
size_t ttcd_fastweight_mlp_noalloc_capacity(void);

/*
 * Decode: the block one token at a time, with carried state.
 *
 * Defines the same function as ttcd_block_forward, evaluated incrementally:
 * the block is causal (windowed attention over earlier tokens, causal convs,
 * an exclusive prefix over chunks), so the output for token t depends only
 * on tokens 0..t.  A sequence of ttcd_block_decode calls at t = 0, 1, ..., T-1
 * therefore returns the rows of ttcd_block_forward's output, and
 * ttcd_decode_state_read after token T-1 returns its state_out.  ([REVIEW]
 * 方法详解 and 关键设计 2: the fast weight of chunk i is W_down + the sum of
 * the earlier chunks' Delta W; [PODCAST] cue 61: decode is not measured on the
 * pages.)
 *
 * The state (caller-owned device memory, ttcd_decode_state_size bytes,
 * 16-byte aligned, layout internal to the library) holds the status word of
 * every decode call in its first TTCD_STATUS_BYTES bytes and, per sequence:
 *   - the K/V cache of the last w_T tokens (ring buffer, bf16);
 *   - the last conv_k-1 rows of Z_T and Z_S (conv history, fp32);
 *   - r_t and k'_t of the current chunk's tokens (bf16);
 *   - the fast weight S (fp32 [d, f]) and W_down + S (bf16), updated when a
 *     chunk ends, and M = W_down W_proj.
 * The batch is B sequences decoded in lockstep (all at position t).
 *
 * ttcd_decode_state_init: clears the state and sets S = state_in (nullable:
 *   zero), W_down + S and M; call before t = 0 and whenever the weights change.
 * ttcd_block_decode: one token.
 *   x_t     [B, d] bf16, device;  beta_t [B] fp32, device;  t >= 0, increasing
 *           by one per call from 0;  y [B, d] bf16, device, written.
 *   workspace >= ttcd_decode_workspace_size(p) bytes (per-step scratch).
 *   At the last token of a chunk (t % chunk == chunk-1) the chunk's Delta W is
 *   added to S before the call returns.
 * ttcd_decode_state_read: the fast-weight state after tokens 0..t_next-1,
 *   including the tokens of a partial chunk (as ttcd_block_forward's
 *   state_out): state_out [B, d, f] fp32, device.
 * Only TTCD_BF16 is supported (TTCD_F32 -> TTCD_ERR_UNSUPPORTED); p->T is not
 * used.  Other errors as ttcd_block_forward.
 */
size_t ttcd_decode_state_size(const ttcd_block_params* p);
size_t ttcd_decode_workspace_size(const ttcd_block_params* p);
ttcd_status ttcd_decode_state_init(const ttcd_block_weights* w, const ttcd_block_params* p,
                                   const float* state_in, void* state, size_t state_bytes,
                                   void* workspace, size_t ws_bytes, void* stream);
ttcd_status ttcd_block_decode(const void* x_t, const float* beta_t, int t,
                              const ttcd_block_weights* w, const ttcd_block_params* p,
                              void* state, size_t state_bytes, void* y, void* workspace,
                              size_t ws_bytes, void* stream);
ttcd_status ttcd_decode_state_read(const ttcd_block_params* p, int t_next, void* state,
                                   size_t state_bytes, float* state_out, void* stream);

/*
 * ttcd_block_decode_next — ttcd_block_decode at the state's own position.
 *
 * The decode state keeps a position counter, an int64 at byte offset 8 of the
 * state (0 after ttcd_decode_state_init; a caller may write it on the device
 * to start elsewhere); this call decodes that position and advances it by one.  Every kernel reads
 * the position from the state, and the chunk commit is launched at every step
 * and acts only at the last token of a chunk, so no launch argument depends on
 * the position: one call can be captured in a CUDA graph and replayed for
 * every later token (the graph's x_t, beta_t and y buffers stay fixed).  Make
 * the first call on a device outside a capture.  Arguments and errors as
 * ttcd_block_decode without t; use either this call or ttcd_block_decode on one
 * state, not both (ttcd_decode_state_read still takes the next position).
 */
ttcd_status ttcd_block_decode_next(const void* x_t, const float* beta_t,
                                   const ttcd_block_weights* w, const ttcd_block_params* p,
                                   void* state, size_t state_bytes, void* y, void* workspace,
                                   size_t ws_bytes, void* stream);

/*
 * ttcd_block_decode_next_ex — ttcd_block_decode_next with the chunk commit
 * optional.  commit != 0: as ttcd_block_decode_next.  commit == 0: the step
 * omits the chunk commit's launches (the chunk scan that adds the chunk's
 * Delta W to the state, and the W_down + S refresh), which act only at the
 * last token of a chunk; the caller must pass commit != 0 at every position
 * p with p % chunk == chunk - 1, or the chunk's Delta W is lost.  This lets a
 * caller capture two CUDA graphs, an ordinary step and a commit step, and
 * replay the ordinary one for chunk - 1 of every chunk tokens.  Arguments
 * and errors otherwise as ttcd_block_decode_next.
 */
ttcd_status ttcd_block_decode_next_ex(const void* x_t, const float* beta_t,
                                      const ttcd_block_weights* w, const ttcd_block_params* p,
                                      void* state, size_t state_bytes, void* y, void* workspace,
                                      size_t ws_bytes, int commit, void* stream);

/* Workspace bytes needed by each entry point; 0 if the parameters are invalid. */
size_t ttcd_fastweight_mlp_workspace_size(const ttcd_block_params* p);
size_t ttcd_block_forward_workspace_size(const ttcd_block_params* p);

/*
 * Byte offset inside the block_forward workspace of a named intermediate, for
 * inspection after a call (same layout for ttcd_fastweight_mlp where named).
 * Names and layouts (row-major):
 *   (E = bf16 for TTCD_BF16 with T >= chunk, fp32 for TTCD_F32 and for
 *   TTCD_BF16 with T < chunk; q, k, v are always bf16)
 *   "status"  uint32 status word (TTCD_STATUS_BYTES reserved)
 *   "wqkv_g"  E [(Hq + 2 Hkv) hd, d]  W_qkv diag(g_attn)
 *   "rstd_in" fp32 [B*T]  1/rms of each input row
 *   "qkv"  bf16 [B*T, (Hq + 2 Hkv) hd]: q heads (rotated), k heads (rotated), v heads
 *   "o"    E [2, B*T, Hq*hd]      (o_T rows, then o_S rows)
 *   "h"    fp32 [B*T, d] (student residual h_S)
 *   "u"    E [2, B*T, d] (block: h * g_mlp; the MLP RMSNorm's 1/rms is applied as a
 *          row scale from "hssq" fp32 [ceil(d/256), 2*B*T] partial sums of h^2)
 *   "Z"    fp32 [2, B*T, f] (E = fp32 only: with bf16 operands Z never leaves the chip)
 *   "Zs16" bf16 [B*T, f]  Z_S, the output GEMM's operand (E = bf16 only)
 *   "D"    E [P, f]               "Kp" E [P, f] (unnormalised keys)
 *   "ssq"  fp32 [n, P]: per-token partial sums of Kp^2 over column blocks of 128
 *          (E = bf16) or 64 (E = fp32) columns, n = ceil(f / block)
 *   "R"    E [P, d] (value residual times beta_t / ||Zbar_S[t]||)
 *   "Wall" E [B*n_chunks, d, f]   (W_down + S_i per chunk)
 * where P = B * n_chunks * Cp, Cp = chunk rounded up to 64, and token t of
 * sequence b sits at padded index (b*n_chunks + t/C)*Cp + t%C.
 * Returns TTCD_ERR_INVALID_ARG for an unknown name or invalid params.
 */
ttcd_status ttcd_block_workspace_offset(const ttcd_block_params* p, const char* name,
                                        size_t* offset);

/*
 * ttcd_check_device_status — reads and clears the status word of a workspace
 * (ttcd_block_forward, ttcd_fastweight_mlp) or of a decode state, after all
 * work queued on `stream` (synchronises `stream`).  Returns TTCD_ERR_TIMEOUT if
 * a device wait of a call that used this workspace gave up since the last
 * check, TTCD_OK otherwise; TTCD_ERR_INVALID_ARG for a null or misaligned
 * pointer.  Only calls on this workspace are reported: other callers' timeouts
 * are in their own workspaces.
 */
ttcd_status ttcd_check_device_status(void* workspace, void* stream);

/* Reads and clears the per-device status word of the entry points without a
 * workspace (the attention calls, ttcd_fastweight_mlp_noalloc, and
 * ttcd_test_bounded_wait with no status region), on the current device
 * (synchronises `stream`).  *flags receives the raw bits; returns
 * TTCD_ERR_TIMEOUT if a wait gave up since the last read, TTCD_OK otherwise.
 * Callers of those entry points share this word. */
ttcd_status ttcd_get_device_error(uint32_t* flags, void* stream);

/* Bound in nanoseconds on every device-side wait (default 2e9 = 2 s). */
void ttcd_set_wait_timeout_ns(uint64_t ns);

/*
 * ttcd_test_bounded_wait — failure-detection self-test.  Launches one CTA that
 * waits on an mbarrier nothing ever arrives at, bounded by `timeout_ns`; the
 * wait gives up, records TTCD_ERR_TIMEOUT in the status word at `status` (a
 * workspace or decode state, 16-byte aligned; null: the per-device word) and
 * the kernel returns normally.  The paper has no counterpart; this exists so a
 * test can check the timeout path without hanging a GPU.
 */
ttcd_status ttcd_test_bounded_wait(uint64_t timeout_ns, void* status, void* stream);

/*
 * ttcd_test_exp2_poly — evaluates, for a test, the 2^x that the attention
 * kernel computes on the FMA pipe for one exponential pair in four: a cubic in
 * the fractional part (coefficients fitted to 2^f on [-0.5, 0.5] by
 * Lawson-reweighted least squares on Chebyshev nodes, relative error 1.01e-4)
 * scaled by the integer part through the exponent field; inputs below -126 are
 * clamped.  x, y: n fp32 values, device, 4-byte aligned; y written.  The paper
 * has no counterpart; it exists so the polynomial can be checked against 2^x.
 */
ttcd_status ttcd_test_exp2_poly(const float* x, float* y, int n, void* stream);

/*
 * ttcd_attn_timeline_read — diagnostic.  In a library built with
 * -DTTCD_ATTN_TIMELINE=1 (`python -m dual_window_attention_b200.build
 * --attn-timeline`, a separate libttcd_timeline.so) the fused attention kernel
 * records, for the CTA with blockIdx.x == 0, clock64 values at the phase
 * boundaries of every visit: [head 2][visit 128][mark 8] int64, marks 0 S ready,
 * 1 S in registers, 2 row maximum, 3 rescale check, 4 P published, 5 PV issued,
 * 6 next QK issued (7 unused, 0 where not reached).  Copies the 2048 values of
 * the last launch to host `out` (n >= 2048) and clears them.  Synchronous.
 * Returns TTCD_ERR_UNSUPPORTED in the normal build.  The paper has no
 * counterpart; it exists to reproduce the attention kernel's timing diagnosis.
 */
ttcd_status ttcd_attn_timeline_read(long long* out, size_t n);

/* Number of kernels this library has launched since it was loaded (process-wide
 * diagnostic counter, atomic). */
unsigned long long ttcd_kernel_launch_count(void);

const char* ttcd_status_string(ttcd_status s);

/* Library version string, e.g. "ttcd 0.2 sm_100a". */
const char* ttcd_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TTCD_H_ */
