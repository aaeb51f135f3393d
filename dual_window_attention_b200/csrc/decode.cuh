// Decode: one token per sequence through the IP-TTCD block, with carried state.
//
// The block is causal (papernotes.org review "Learning What to Remember",
// 方法详解: windowed attention over earlier tokens, causal short convs, an
// exclusive prefix over chunks), so token t needs only: the K/V of the last
// w_T tokens, the last conv_k-1 rows of Z_T and Z_S, the r_t and k'_t of the
// current chunk (its Delta W is formed when the chunk ends), and the fast
// weight of the current chunk, W_down + S.  These kernels are the
// memory-bound per-token steps; the dense products run on the tcgen05 GEMM
// and the chunk commit on the chunk-scan kernel.
#pragma once
#include "gemm.cuh"

namespace ttcd {

// 16-byte global -> shared copy that bypasses L1 (both addresses 16-byte aligned);
// completion by cp_async_wait_all in the issuing thread, then a block barrier.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

constexpr int DEC_KC = 256;       // keys per attention split
constexpr int DEC_THREADS = 256;  // attention split block
constexpr int DEC_MAXG = 8;       // query heads per KV head handled by one block

// Position of the token being decoded: the kernels take it as an argument, or,
// when `pos` is set, read it from device memory (the decode state's own
// counter), so that a step's launches have no argument that changes from token
// to token and the step can be captured once in a CUDA graph and replayed.
__device__ __forceinline__ int dec_pos(int t, const long long* pos) {
  return pos ? static_cast<int>(*pos) : t;
}

// q and k rotated at position t (rotate-half RoPE, angle t * theta^(-2i/hd) in
// double precision), k and v appended to the ring caches at slot t % W.
// qkv [B, (Hq + 2 Hkv) hd] fp32 -> q_rot [B, Hq, hd] bf16; kc, vc [B, W, Hkv, hd].
// grid (B, Hq + 2 Hkv), block hd / 2.
__global__ void decode_rope_cache_kernel(const float* __restrict__ qkv,
                                         __nv_bfloat16* __restrict__ q_rot,
                                         __nv_bfloat16* __restrict__ kc,
                                         __nv_bfloat16* __restrict__ vc, int Hq, int Hkv, int hd,
                                         int t, int W, double theta,
                                         const long long* pos = nullptr) {
  t = dec_pos(t, pos);
  const int b = blockIdx.x, head = blockIdx.y, i = threadIdx.x;
  const int half = hd / 2;
  const float* src = qkv + static_cast<long long>(b) * (Hq + 2 * Hkv) * hd +
                     static_cast<long long>(head) * hd;
  const long long slot = t % W;
  if (head < Hq + Hkv) {
    double s, c;
    sincos(static_cast<double>(t) * pow(theta, -2.0 * i / hd), &s, &c);
    const float cf = static_cast<float>(c), sf = static_cast<float>(s);
    const float a = src[i], bb = src[i + half];
    __nv_bfloat16* dst = head < Hq
                             ? q_rot + (static_cast<long long>(b) * Hq + head) * hd
                             : kc + ((b * static_cast<long long>(W) + slot) * Hkv + (head - Hq)) * hd;
    dst[i] = __float2bfloat16_rn(a * cf - bb * sf);
    dst[i + half] = __float2bfloat16_rn(bb * cf + a * sf);
  } else {
    __nv_bfloat16* dst =
        vc + ((b * static_cast<long long>(W) + slot) * Hkv + (head - Hq - Hkv)) * hd;
    dst[i] = __float2bfloat16_rn(src[i]);
    dst[i + half] = __float2bfloat16_rn(src[i + half]);
  }
}

// Shared memory of one attention split: the split's K rows, then its V rows,
// at a pitch of HD * 2 + 16 bytes (a quarter warp reading 16 bytes from each
// of 8 consecutive rows, or 8 consecutive 16-byte pieces of one row, meets
// no bank twice), the group's q in fp32 and the two windows' scores.
template <int HD>
constexpr int dec_pitch() { return HD * 2 + 16; }
// The row tile, also the scratch of the final key-group sums (fp32, two
// windows, DEC_THREADS / (HD / 8) groups).
template <int HD>
constexpr int dec_tile_bytes() {
  return DEC_KC * dec_pitch<HD>() > (DEC_THREADS / (HD / 8)) * 2 * HD * 4
             ? DEC_KC * dec_pitch<HD>()
             : (DEC_THREADS / (HD / 8)) * 2 * HD * 4;
}
template <int HD>
constexpr int dec_attn_smem_bytes(int G) {
  return dec_tile_bytes<HD>() + G * HD * 4 + 2 * G * DEC_KC * 4;
}

// Both windows of one KV head's query heads over one split of DEC_KC keys of
// the teacher range [max(0, t-w_T+1), t]; the student window is its last w_S
// keys.  The block copies the split's K rows into shared memory with all
// copies in flight at once, forms the scores, starts the same copy of the V
// rows over the K rows, and runs the softmax while they arrive.  Partial
// results (log2-domain max, sum, unnormalised output) per (b, h, window,
// split): pm, pl [B, Hq, 2, nsplit], po [B, Hq, 2, nsplit, HD].
// GM >= Hq / Hkv bounds the query heads per KV head (the register arrays).
// grid (B * Hkv, nsplit), block DEC_THREADS, dynamic shared memory
// dec_attn_smem_bytes<HD>(Hq / Hkv).
template <int HD, int GM>
__global__ void __launch_bounds__(DEC_THREADS)
    decode_attn_partial_kernel(const __nv_bfloat16* __restrict__ q_rot,
                               const __nv_bfloat16* __restrict__ kc,
                               const __nv_bfloat16* __restrict__ vc, float* __restrict__ pm,
                               float* __restrict__ pl, float* __restrict__ po, int Hq, int Hkv,
                               int W, int t, int w_S, int w_T, float scale_log2, int nsplit,
                               const long long* pos = nullptr) {
  t = dec_pos(t, pos);
  constexpr int PITCH = dec_pitch<HD>();
  constexpr int TPR = HD / 8;              // 16-byte pieces per row
  constexpr int RPP = DEC_THREADS / TPR;   // rows per pass of the block
  static_assert(DEC_THREADS % TPR == 0 && RPP * 2 * HD * 4 <= dec_tile_bytes<HD>(),
                "the key-group reduction must fit the row tile");
  extern __shared__ __align__(16) unsigned char dsm[];
  unsigned char* tile = dsm;
  const int b = blockIdx.x / Hkv, g = blockIdx.x % Hkv, sp = blockIdx.y;
  const int G = Hq / Hkv;
  float* qs = reinterpret_cast<float*>(dsm + dec_tile_bytes<HD>());  // [G][HD]
  float* ps = qs + G * HD;                                      // [2][G][DEC_KC]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j_lo = max(0, t - w_T + 1);
  const int j0 = j_lo + sp * DEC_KC;
  const int n = max(0, min(t - j0 + 1, DEC_KC));  // keys of this split
  const int s_lo = max(0, t - w_S + 1) - j0;      // first student key index (may be <0 or >=n)
  // this thread's 16-byte piece of every RPP-th row: rows r0, r0 + RPP, ...
  const int piece = tid % TPR, r0 = tid / TPR;
  const long long row_stride = static_cast<long long>(Hkv) * HD;  // elements between ring slots
  const long long head_base = (static_cast<long long>(b) * W * Hkv + g) * HD + piece * 8;
  auto copy_rows = [&](const __nv_bfloat16* cache) {
    int slot = (j0 + r0) % W;
    for (int r = r0; r < n; r += RPP) {
      cp_async16(tile + r * PITCH + piece * 16, cache + head_base + slot * row_stride);
      slot += RPP;
      if (slot >= W) slot -= W;
    }
  };
  copy_rows(kc);
  for (int e = tid; e < G * HD; e += DEC_THREADS)
    qs[e] = __bfloat162float(q_rot[(static_cast<long long>(b) * Hq + g * G) * HD + e]);
  cp_async_wait_all();
  __syncthreads();
  // scores (log2 domain), one key row per thread at a time
  for (int kk = tid; kk < n; kk += DEC_THREADS) {
    const uint4* krow = reinterpret_cast<const uint4*>(tile + kk * PITCH);
    // even and odd columns summed apart, two per packed FMA
    float2 acc[GM];
#pragma unroll
    for (int hh = 0; hh < GM; ++hh) acc[hh] = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int c8 = 0; c8 < HD / 8; ++c8) {
      const uint4 u = krow[c8];
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 k2 = make_float2(bf16lo_to_f32(w4[q]), bf16hi_to_f32(w4[q]));
#pragma unroll
        for (int hh = 0; hh < GM; ++hh)
          if (hh < G)
            acc[hh] = __ffma2_rn(*reinterpret_cast<const float2*>(&qs[hh * HD + c8 * 8 + 2 * q]),
                                 k2, acc[hh]);
      }
    }
#pragma unroll
    for (int hh = 0; hh < GM; ++hh)
      if (hh < G) ps[hh * DEC_KC + kk] = (acc[hh].x + acc[hh].y) * scale_log2;
  }
  __syncthreads();
  copy_rows(vc);  // V over K, in flight during the softmax
  // per (head, window): maximum, probabilities, sum (one warp per pair)
  float* pT = ps;                 // [G][DEC_KC]: teacher scores, then probabilities
  float* pS = ps + G * DEC_KC;    // [G][DEC_KC]: student probabilities
  for (int pr = warp; pr < 2 * G; pr += DEC_THREADS / 32) {
    const int hh = pr >> 1, win = pr & 1;  // win 0: teacher, 1: student
    const int k_first = win ? max(s_lo, 0) : 0;
    float m = -INFINITY;
    for (int kk = k_first + lane; kk < n; kk += 32) m = fmaxf(m, pT[hh * DEC_KC + kk]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int kk = lane; kk < DEC_KC; kk += 32) {
      const float p = (kk >= k_first && kk < n) ? exp2f(pT[hh * DEC_KC + kk] - m) : 0.f;
      if (win) pS[hh * DEC_KC + kk] = p;
      l += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      const long long pi = ((static_cast<long long>(b) * Hq + g * G + hh) * 2 + win) * nsplit + sp;
      pm[pi] = m;
      pl[pi] = l;
    }
  }
  __syncthreads();
  // teacher probabilities in place of the scores
  for (int pr = warp; pr < G; pr += DEC_THREADS / 32) {
    const long long pi = ((static_cast<long long>(b) * Hq + g * G + pr) * 2) * nsplit + sp;
    const float m = pm[pi];
    for (int kk = lane; kk < DEC_KC; kk += 32)
      pT[pr * DEC_KC + kk] = kk < n ? exp2f(pT[pr * DEC_KC + kk] - m) : 0.f;
  }
  cp_async_wait_all();
  __syncthreads();
  // P.V from shared memory: TPR threads cover a row (8 columns each), RPP key
  // groups take every RPP-th key, and the groups are summed through shared
  // memory (reusing the row tile).
  {
    const int dg = piece, kg = r0;
    float2 aT2[GM][4], aS2[GM][4];  // column pairs, two per packed FMA
#pragma unroll
    for (int hh = 0; hh < GM; ++hh)
#pragma unroll
      for (int e = 0; e < 4; ++e) aT2[hh][e] = aS2[hh][e] = make_float2(0.f, 0.f);
#pragma unroll 2
    for (int kk = kg; kk < n; kk += RPP) {
      const uint4 u = *reinterpret_cast<const uint4*>(tile + kk * PITCH + dg * 16);
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
      float2 vv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) vv[q] = make_float2(bf16lo_to_f32(w4[q]), bf16hi_to_f32(w4[q]));
#pragma unroll
      for (int hh = 0; hh < GM; ++hh)
        if (hh < G) {
          const float wT = pT[hh * DEC_KC + kk], wS = pS[hh * DEC_KC + kk];
          const float2 wT2 = make_float2(wT, wT), wS2 = make_float2(wS, wS);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            aT2[hh][e] = __ffma2_rn(wT2, vv[e], aT2[hh][e]);
            aS2[hh][e] = __ffma2_rn(wS2, vv[e], aS2[hh][e]);
          }
        }
    }
    float aT[GM][8], aS[GM][8];
#pragma unroll
    for (int hh = 0; hh < GM; ++hh)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        aT[hh][2 * e] = aT2[hh][e].x;
        aT[hh][2 * e + 1] = aT2[hh][e].y;
        aS[hh][2 * e] = aS2[hh][e].x;
        aS[hh][2 * e + 1] = aS2[hh][e].y;
      }
    // Sum the key groups one head at a time (RPP * 2 * HD floats fit the tile).
    float* red = reinterpret_cast<float*>(tile);
#pragma unroll
    for (int hh = 0; hh < GM; ++hh) {
      if (hh >= G) break;  // G is the same for the whole block
      __syncthreads();
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        red[(kg * 2 + 0) * HD + dg * 8 + e] = aT[hh][e];
        red[(kg * 2 + 1) * HD + dg * 8 + e] = aS[hh][e];
      }
      __syncthreads();
      for (int o = tid; o < 2 * HD; o += DEC_THREADS) {
        const int win = o / HD, d = o % HD;
        float acc = 0.f;
        for (int q = 0; q < RPP; ++q) acc += red[(q * 2 + win) * HD + d];
        const long long base =
            (((static_cast<long long>(b) * Hq + g * G + hh) * 2) + win) * nsplit + sp;
        po[base * HD + d] = acc;
      }
    }
  }
}
// Merge the splits: o = sum_s po_s 2^(pm_s - m) / sum_s pl_s 2^(pm_s - m).
// o [2, B, Hq * HD] bf16 (teacher rows, then student rows).  grid B * Hq * 2, block HD.
template <int HD>
__global__ void decode_attn_combine_kernel(const float* __restrict__ pm,
                                           const float* __restrict__ pl,
                                           const float* __restrict__ po,
                                           __nv_bfloat16* __restrict__ o, int B, int Hq,
                                           int nsplit) {
  const int r = blockIdx.x;  // ((b * Hq + h) * 2 + win)
  const int win = r & 1, bh = r >> 1;
  const int b = bh / Hq, h = bh % Hq;
  const int d = threadIdx.x;
  float m = -INFINITY;
  for (int s = 0; s < nsplit; ++s) m = fmaxf(m, pm[static_cast<long long>(r) * nsplit + s]);
  float l = 0.f, acc = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const long long pi = static_cast<long long>(r) * nsplit + s;
    const float w = pm[pi] == -INFINITY ? 0.f : exp2f(pm[pi] - m);
    l += pl[pi] * w;
    acc += po[pi * HD + d] * w;
  }
  o[((static_cast<long long>(win) * B + b) * Hq + h) * HD + d] = __float2bfloat16_rn(acc / l);
}

// h_P = x + hp_P for both paths (rows 0..B-1 teacher, B..2B-1 student), the
// student's h kept in fp32, and u_P = RMSNorm(h_P; g) in bf16.  grid 2B, block 256.
__global__ void decode_residual_norm_kernel(const __nv_bfloat16* __restrict__ x,
                                            const float* __restrict__ hp,
                                            const __nv_bfloat16* __restrict__ g,
                                            __nv_bfloat16* __restrict__ u,
                                            float* __restrict__ hS, int B, int d, float eps) {
  __shared__ float red[8];
  const int r = blockIdx.x, b = r % B;
  float ss = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float h = __bfloat162float(x[static_cast<long long>(b) * d + c]) +
                    hp[static_cast<long long>(r) * d + c];
    ss += h * h;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += red[w];
  const float rstd = rsqrtf(tot / d + eps);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float h = __bfloat162float(x[static_cast<long long>(b) * d + c]) +
                    hp[static_cast<long long>(r) * d + c];
    u[static_cast<long long>(r) * d + c] =
        __float2bfloat16_rn(h * rstd * __bfloat162float(g[c]));
    if (r >= B) hS[static_cast<long long>(b) * d + c] = h;
  }
}

// One token of the short causal convs, the residual difference and the key:
//   zbar_P = sum_m taps_P[c, m] Z_P[t-m]   (history rows t-1..t-k+1, zero before 0)
//   D = zbar_T - zbar_S;  k' = zbar_S (unnormalised) into the chunk buffer row t % C;
//   Z_S also as the bf16 output operand; per-block partial sums of zbar_S^2.
// Z [2B, f] fp32 (teacher rows first); hist [2, B, H, f] fp32 ring (slot = position % H).
// grid (cdiv(f, 256), B), block 256; ssq_part [B, gridDim.x].
__global__ void decode_conv_kernel(const float* __restrict__ Z,
                                   const __nv_bfloat16* __restrict__ tapT,
                                   const __nv_bfloat16* __restrict__ tapS,
                                   float* __restrict__ hist, __nv_bfloat16* __restrict__ D,
                                   __nv_bfloat16* __restrict__ Kc, __nv_bfloat16* __restrict__ Zs16,
                                   float* __restrict__ ssq_part, int B, int f, int k, int t, int C,
                                   int Cp, const long long* pos = nullptr) {
  t = dec_pos(t, pos);
  __shared__ float red[8];
  const int b = blockIdx.y;
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int H = k > 1 ? k - 1 : 1;
  float ss = 0.f;
  if (c < f) {
    float* hT = hist + static_cast<long long>(b) * H * f;
    float* hSb = hist + (static_cast<long long>(B) + b) * H * f;
    const float zt = Z[static_cast<long long>(b) * f + c];
    const float zs = Z[(static_cast<long long>(B) + b) * f + c];
    float bT = __bfloat162float(tapT[static_cast<long long>(c) * k]) * zt;
    float bS = __bfloat162float(tapS[static_cast<long long>(c) * k]) * zs;
    for (int m = 1; m < k; ++m) {
      if (t - m < 0) break;
      const long long slot = (t - m) % H;
      bT += __bfloat162float(tapT[static_cast<long long>(c) * k + m]) * hT[slot * f + c];
      bS += __bfloat162float(tapS[static_cast<long long>(c) * k + m]) * hSb[slot * f + c];
    }
    if (k > 1) {  // position t replaces position t-H, which no later token needs
      hT[static_cast<long long>(t % H) * f + c] = zt;
      hSb[static_cast<long long>(t % H) * f + c] = zs;
    }
    D[static_cast<long long>(b) * f + c] = __float2bfloat16_rn(bT - bS);
    Kc[(static_cast<long long>(b) * Cp + t % C) * f + c] = __float2bfloat16_rn(bS);
    Zs16[static_cast<long long>(b) * f + c] = __float2bfloat16_rn(zs);
    ss = bS * bS;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += red[w];
    ssq_part[static_cast<long long>(b) * gridDim.x + blockIdx.x] = tot;
  }
}

// beta_t[b] / sqrt(||zbar_S||^2 + eps) from the conv kernel's partial sums,
// added in a fixed order (lane-strided, then a butterfly): every lane of the
// calling warp returns the same value.
__device__ __forceinline__ float dec_key_scale(const float* __restrict__ ssq_part, int n_part,
                                               const float* __restrict__ beta, float eps, int b,
                                               int lane) {
  float s = 0.f;
  for (int i = lane; i < n_part; i += 32) s += ssq_part[static_cast<long long>(b) * n_part + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return beta[b] / sqrtf(s + eps);
}

// kscale[b] = dec_key_scale(b).  grid B, block 32.
__global__ void decode_kscale_kernel(const float* __restrict__ ssq_part, int n_part,
                                     const float* __restrict__ beta, float* __restrict__ kscale,
                                     float eps) {
  const float k = dec_key_scale(ssq_part, n_part, beta, eps, blockIdx.x, threadIdx.x);
  if (threadIdx.x == 0) kscale[blockIdx.x] = k;
}

// Epilogue arguments of the key-row GEMV (EPI 2): the key scale from the conv
// kernel's partial sums, and the destination row of the current chunk slot
// (row (pos ? *pos : t) % C of each sequence's Cp-row block).
struct DecKeyRowEpi {
  const float* ssq_part;
  int n_part;
  const float* beta;
  float eps;
  const long long* pos;
  int t;
  int C;
  int Cp;
};

// Y[r, n] = epi(W[n, :] . X[r, :]) for R <= DEC_GEMV_ROWS input rows: the
// dense products of a decode step, whose few rows would leave a 128-row tensor
// core tile nearly empty.  One warp per weight row n streams W[n] once (16-byte
// loads) against every input row (from L1).  Epilogues: 0 fp32 store;
// 1 silu(W[n].x) * (W2[n].x) (SwiGLU, fp32); 2 bf16 store scaled by the key
// scale of row r into its chunk-slot row (kr).
// grid cdiv(N, 8), block 256.
constexpr int DEC_GEMV_ROWS = 16;   // rows one GEMV launch can take
constexpr int DEC_GEMV_SWITCH = 8;  // up to this many rows the GEMV beats a 128-row GEMM tile (B200, measured)
// The products with B rows (QKV, and r over the long K = d_ff) take the GEMV
// up to this many rows; their few-CTA GEMM grids lose to it until then (B200,
// measured per B with the CUDA graph).
constexpr int DEC_GEMV_SWITCH_B = 6;
template <int EPI>
__global__ void decode_gemv_kernel(const __nv_bfloat16* __restrict__ Wm,
                                   const __nv_bfloat16* __restrict__ W2,
                                   const __nv_bfloat16* __restrict__ X, void* __restrict__ Y,
                                   int R, int N, int K, long long ldy,
                                   DecKeyRowEpi kr = DecKeyRowEpi{}) {
  const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (n >= N) return;
  constexpr int NW = EPI == 1 ? 2 : 1;
  const int slot_row = EPI == 2 ? static_cast<int>((kr.pos ? *kr.pos : kr.t) % kr.C) : 0;
  float acc[NW][DEC_GEMV_ROWS];
#pragma unroll
  for (int q = 0; q < NW; ++q)
#pragma unroll
    for (int r = 0; r < DEC_GEMV_ROWS; ++r) acc[q][r] = 0.f;
  const uint4* w1 = reinterpret_cast<const uint4*>(Wm + static_cast<long long>(n) * K);
  const uint4* w2 = EPI == 1 ? reinterpret_cast<const uint4*>(W2 + static_cast<long long>(n) * K) : w1;
  for (int c8 = lane; c8 < K / 8; c8 += 32) {
    float wv[NW][8];
#pragma unroll
    for (int q = 0; q < NW; ++q) {
      const uint4 u = q ? w2[c8] : w1[c8];
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        wv[q][2 * e] = bf16lo_to_f32(w4[e]);
        wv[q][2 * e + 1] = bf16hi_to_f32(w4[e]);
      }
    }
#pragma unroll
    for (int r = 0; r < DEC_GEMV_ROWS; ++r) {
      if (r >= R) break;
      const uint4 xu = reinterpret_cast<const uint4*>(X + static_cast<long long>(r) * K)[c8];
      const uint32_t x4[4] = {xu.x, xu.y, xu.z, xu.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = bf16lo_to_f32(x4[e]), x1 = bf16hi_to_f32(x4[e]);
#pragma unroll
        for (int q = 0; q < NW; ++q) acc[q][r] += wv[q][2 * e] * x0 + wv[q][2 * e + 1] * x1;
      }
    }
  }
#pragma unroll
  for (int r = 0; r < DEC_GEMV_ROWS; ++r) {
    if (r >= R) break;
#pragma unroll
    for (int q = 0; q < NW; ++q)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[q][r] += __shfl_xor_sync(0xffffffffu, acc[q][r], o);
    if (lane == 0) {
      if (EPI == 0) {
        static_cast<float*>(Y)[r * ldy + n] = acc[0][r];
      } else if (EPI == 1) {
        const float gg = acc[0][r];
        static_cast<float*>(Y)[r * ldy + n] = gg / (1.0f + __expf(-gg)) * acc[NW - 1][r];
      }
    }
    if (EPI == 2) {  // whole warp: the key scale's butterfly
      const float ks = dec_key_scale(kr.ssq_part, kr.n_part, kr.beta, kr.eps, r, lane);
      if (lane == 0)
        static_cast<__nv_bfloat16*>(Y)[(static_cast<long long>(r) * kr.Cp + slot_row) * ldy + n] =
            __float2bfloat16_rn(acc[0][r] * ks);
    }
  }
}

// rows [B, d] -> dst rows b * Cp + row (the current chunk slot of each sequence)
// With `pos` set, row = *pos % C.
__global__ void decode_row_copy_kernel(const __nv_bfloat16* __restrict__ src,
                                       __nv_bfloat16* __restrict__ dst, int B, int d, int Cp,
                                       int row, const long long* pos = nullptr, int C = 1) {
  if (pos) row = static_cast<int>(*pos % C);
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<long long>(B) * d) return;
  const long long b = i / d, c = i % d;
  dst[(b * Cp + row) * d + c] = src[i];
}

// y[b, i] = hS[b, i] + sum_c Weff[b, i, c] Zs[b, c]: the fast-weight read with
// the current chunk's weight W_down + S.  One warp per output row.
// grid (cdiv(d, 8), B), block 256.
__global__ void decode_out_kernel(const __nv_bfloat16* __restrict__ Weff,
                                  const __nv_bfloat16* __restrict__ Zs,
                                  const float* __restrict__ hS, __nv_bfloat16* __restrict__ y,
                                  int d, int f) {
  const int b = blockIdx.y;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= d) return;
  const uint4* wr = reinterpret_cast<const uint4*>(Weff + (static_cast<long long>(b) * d + i) * f);
  const uint4* zr = reinterpret_cast<const uint4*>(Zs + static_cast<long long>(b) * f);
  float acc = 0.f;
  for (int c8 = lane; c8 < f / 8; c8 += 32) {
    const uint4 a = wr[c8], z = zr[c8];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, zw[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      acc += bf16lo_to_f32(aw[q]) * bf16lo_to_f32(zw[q]) + bf16hi_to_f32(aw[q]) * bf16hi_to_f32(zw[q]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0)
    y[static_cast<long long>(b) * d + i] = __float2bfloat16_rn(hS[static_cast<long long>(b) * d + i] + acc);
}

// Weff[b] = bf16(W_down + S[b]), 4 elements per thread and step.  With `commit_pos`
// set it acts only at the last token of a chunk (*commit_pos % C == C - 1).
__global__ void decode_weff_kernel(const __nv_bfloat16* __restrict__ w_down,
                                   const float* __restrict__ S, __nv_bfloat16* __restrict__ Weff,
                                   long long df, long long n4,
                                   const long long* commit_pos = nullptr, int C = 1) {
  if (commit_pos && *commit_pos % C != C - 1) return;
  // grid-stride over a small fixed grid: in a replayed decode step the launch
  // usually only checks the position and exits
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long e = i * 4, w = e % df;
    const float4 s = *reinterpret_cast<const float4*>(S + e);
    const uint2 wd = *reinterpret_cast<const uint2*>(w_down + w);
    uint2 out;
    out.x = pack_bf16x2(bf16lo_to_f32(wd.x) + s.x, bf16hi_to_f32(wd.x) + s.y);
    out.y = pack_bf16x2(bf16lo_to_f32(wd.y) + s.z, bf16hi_to_f32(wd.y) + s.w);
    *reinterpret_cast<uint2*>(Weff + e) = out;
  }
}

// Advances the decode state's position counter by one token (the last launch
// of a step that reads the position from device memory).
__global__ void decode_advance_kernel(long long* __restrict__ pos) { *pos += 1; }

}  // namespace ttcd
