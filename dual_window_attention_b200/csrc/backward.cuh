// Backward of the in-place fast-weight MLP (sm_100a): GEMM epilogues and the
// memory-bound steps between the GEMMs.
//
// papernotes.org review "Learning What to Remember", 关键设计 2-3 and 局限与展望
// (training runs the whole block, the write path included): the chain rule of
//   Z_P = silu(u_P W_gate^T) * (u_P W_up^T),  Zbar_P = conv_P(Z_P),
//   D = Zbar_T - Zbar_S,  r_t = M D_t (M = W_down W_proj),
//   s_t = beta_t / n_t,  n_t = (|Zbar_S[t]|^2 + eps)^(1/2),
//   Delta W_i = sum_{t in C_i} s_t r_t Zbar_S[t]^T,  S_{i+1} = S_i + Delta W_i,
//   y_t = (W_down + S_{i(t)}) Z_S[t],
// taken in the reverse of that order.  With G_i = dL/dDelta W_i (the reverse
// prefix of the per-chunk dL/dS_i = sum_{t in C_i} dy_t Z_S[t]^T):
//   dRt_t = G_i Zbar_S[t]                 (gradient of the scaled row s_t r_t)
//   E_t   = M^T dRt_t,  dD_t = s_t E_t,  ds_t = D_t . E_t  (= r_t . dRt_t)
//   dbeta_t = ds_t / n_t,  dZbar_S[t] = G_i^T (s_t r_t) - ds_t beta_t / n_t^3 Zbar_S[t] - dD_t
//   dM = sum_t s_t dRt_t D_t^T,  dW_down += dM W_proj^T,  dW_proj = W_down^T dM.
// Rows of the chunk-padded buffers follow the forward's layout: sequence b,
// chunk i, row j at (b Nc + i) Cp + j, pad rows zero.
#pragma once
#include "elementwise.cuh"
#include "gemm.cuh"

namespace ttcd {

// out_u[row] = bf16(acc), out_s[row] = bf16(acc * scale[row]); columns < N (a
// multiple of 64).  Direct stores.
struct EpiStoreScaledPair {
  static constexpr bool kStaged = false;
  static constexpr bool kCollective = false;
  __nv_bfloat16* out_u;
  __nv_bfloat16* out_s;
  long long ldo;
  int N;
  const float* scale;
  __device__ float pre(const TileCtx& c, int r) const {
    return r < c.valid_rows ? __ldg(scale + c.row0 + r) : 0.f;
  }
  template <int BN>
  __device__ void run(const TileCtx& c, uint32_t taddr, int r, EpiStage&, float sc) const {
    const bool ok = r < c.valid_rows;
    const long long row = c.row0 + r;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      const int col = c.tn * BN + cc;
      if (col >= N) break;
      float v[32];
      tmem_ld32f(taddr + cc, v);
      if (!ok) continue;
      store_bf16x32(out_u + row * ldo + col, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= sc;
      store_bf16x32(out_s + row * ldo + col, v);
    }
  }
};

// acc = E = dRt M (fp32).  dD[row] = scale[row] * E (fp32 [rows, N]) and
// part[tn][row] = sum over this tile's columns of D[row, col] * E[row, col]
// (D bf16 [rows, N]); fixed summation order.
struct EpiBwdE {
  static constexpr bool kStaged = false;
  static constexpr bool kCollective = false;
  float* dD;
  const __nv_bfloat16* D;
  float* part;
  long long rows;
  int N;
  const float* scale;
  __device__ float pre(const TileCtx& c, int r) const {
    return r < c.valid_rows ? __ldg(scale + c.row0 + r) : 0.f;
  }
  template <int BN>
  __device__ void run(const TileCtx& c, uint32_t taddr, int r, EpiStage&, float sc) const {
    const bool ok = r < c.valid_rows;
    const long long row = c.row0 + r;
    float dot = 0.f;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      const int col = c.tn * BN + cc;
      if (col >= N) break;
      float v[32];
      tmem_ld32f(taddr + cc, v);
      if (!ok) continue;
      float dv[32];
      load_x32(D + row * N + col, dv);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        dot = fmaf(dv[i], v[i], dot);
        v[i] *= sc;
      }
      store_f32x32(dD + row * N + col, v);
    }
    if (ok) part[static_cast<long long>(c.tn) * rows + row] = dot;
  }
};

// out[row] = acc + coef[row] * X[row] - Y[row]  (X bf16, Y and out fp32, all
// [rows, N]).
struct EpiBwdZbS {
  static constexpr bool kStaged = false;
  static constexpr bool kCollective = false;
  float* out;
  const __nv_bfloat16* X;
  const float* Y;
  int N;
  const float* coef;
  __device__ float pre(const TileCtx& c, int r) const {
    return r < c.valid_rows ? __ldg(coef + c.row0 + r) : 0.f;
  }
  template <int BN>
  __device__ void run(const TileCtx& c, uint32_t taddr, int r, EpiStage&, float cf) const {
    const bool ok = r < c.valid_rows;
    const long long row = c.row0 + r;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      const int col = c.tn * BN + cc;
      if (col >= N) break;
      float v[32];
      tmem_ld32f(taddr + cc, v);
      if (!ok) continue;
      float x[32], y[32];
      load_x32(X + row * N + col, x);
      load_x32(Y + row * N + col, y);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] += fmaf(cf, x[i], -y[i]);
      store_f32x32(out + row * N + col, v);
    }
  }
};

// Gate/up recomputed (accumulator columns [0, BN/2) a = u W_gate^T, [BN/2, BN)
// b = u W_up^T for output columns tn*BN/2 + [0, BN/2)), with dz = dZ[row, col]:
//   da = dz b silu'(a),  db = dz silu(a),  Z = silu(a) b,
// silu'(a) = sigma(a) (1 + a (1 - sigma(a))).  dab[row] = [da | db] (bf16, row
// length 2N), z[row] = Z (bf16, row length N).
struct EpiSwiGLUBwd {
  static constexpr bool kStaged = false;
  static constexpr bool kCollective = false;
  const float* dZ;
  __nv_bfloat16* dab;
  __nv_bfloat16* z;
  int N;
  __device__ float pre(const TileCtx&, int) const { return 1.f; }
  template <int BN>
  __device__ void run(const TileCtx& c, uint32_t taddr, int r, EpiStage&, float) const {
    const bool ok = r < c.valid_rows;
    const long long row = c.row0 + r;
#pragma unroll 1
    for (int cc = 0; cc < BN / 2; cc += 32) {
      const int col = c.tn * (BN / 2) + cc;
      if (col >= N) break;
      float a[32], b[32];
      tmem_ld32f(taddr + cc, a);
      tmem_ld32f(taddr + BN / 2 + cc, b);
      if (!ok) continue;
      float dz[32], zz[32];
      load_x32(dZ + row * N + col, dz);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float sg = __fdividef(1.0f, 1.0f + __expf(-a[i]));
        const float si = a[i] * sg;
        zz[i] = si * b[i];
        const float da = dz[i] * b[i] * sg * fmaf(a[i], 1.0f - sg, 1.0f);
        b[i] = dz[i] * si;
        a[i] = da;
      }
      __nv_bfloat16* drow = dab + row * (2ll * N);
      store_bf16x32(drow + col, a);
      store_bf16x32(drow + N + col, b);
      store_bf16x32(z + row * N + col, zz);
    }
  }
};

// dst[(b Nc + i) Cp + j] = src[b T + i C + j] for tokens of the sequence, zero
// on pad rows; 8 elements (16 bytes) per thread, ncols a multiple of 8.
template <class E>
__global__ void chunk_pad_rows_kernel(const E* __restrict__ src, E* __restrict__ dst, int ncols,
                                      int T, int C, int Cp, int Nc, long long P) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int per_row = ncols / (16 / static_cast<int>(sizeof(E)));
  if (idx >= P * per_row) return;
  const long long p = idx / per_row;
  const int q = static_cast<int>(idx % per_row);
  const long long seq = static_cast<long long>(Nc) * Cp;
  const int b = static_cast<int>(p / seq);
  const long long rem = p % seq;
  const int i = static_cast<int>(rem / Cp), j = static_cast<int>(rem % Cp);
  const int t = i * C + j;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (j < C && t < T)
    v = __ldg(reinterpret_cast<const uint4*>(src + (static_cast<long long>(b) * T + t) * ncols) + q);
  reinterpret_cast<uint4*>(dst + p * ncols)[q] = v;
}

// Per padded row: ds = sum of the E epilogue's partial dots, n = (ssq + eps)^(1/2);
// d_beta[b, t] = ds / n and coef = -ds beta / n^3 (zero on pad rows).
__global__ void key_backward_kernel(const float* __restrict__ epart, int n_epart,
                                    const float* __restrict__ ssq_part, int n_ssq,
                                    const float* __restrict__ beta, float* __restrict__ d_beta,
                                    float* __restrict__ coef, int T, int C, int Cp, int Nc,
                                    long long P, float eps) {
  const long long p = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (p >= P) return;
  const long long seq = static_cast<long long>(Nc) * Cp;
  const int b = static_cast<int>(p / seq);
  const long long rem = p % seq;
  const int i = static_cast<int>(rem / Cp), j = static_cast<int>(rem % Cp);
  const int t = i * C + j;
  if (!(j < C && t < T)) {
    coef[p] = 0.f;
    return;
  }
  float ds = 0.f, ssq = 0.f;
  for (int q = 0; q < n_epart; ++q) ds += epart[static_cast<long long>(q) * P + p];
  for (int q = 0; q < n_ssq; ++q) ssq += ssq_part[static_cast<long long>(q) * P + p];
  const float inv = rsqrtf(ssq + eps);
  const long long bt = static_cast<long long>(b) * T + t;
  d_beta[bt] = ds * inv;
  coef[p] = -ds * beta[bt] * inv * inv * inv;
}

// Backward of the causal depthwise convs (tap m multiplies t - m, so the
// transpose reads t + m) and the sum with the read path's dZ_S:
//   dZ[path, b, s, c] = sum_{m < k, s + m < T} w_path[c, m] dZbar_path[b, s + m, c]
//                       (+ dZs_read[b, s, c] for the student path),
// dZbar_* in the chunk-padded layout, dZ [2, B, T, f] fp32 (teacher first).
// Thread = (path, sequence, 4 columns, CONV_BWD_ROWS consecutive tokens): it
// slides a window of k dZbar rows down its tokens (one 16-byte load per row)
// and takes its taps from the forward's bf16 table [path][f/8][KMAX][8]; the
// padded row index advances without divisions.
constexpr int CONV_BWD_ROWS = 16;

template <int KMAX>
__global__ void __launch_bounds__(256) conv_backward_kernel(
    const float* __restrict__ dzb_T, const float* __restrict__ dzb_S,
    const float* __restrict__ dzs_read, const __nv_bfloat16* __restrict__ taps,
    float* __restrict__ dZ, int B, int T, int f, int k, int C, int Cp, int Nc) {
  const int f4 = f / 4;
  const int nrb = (T + CONV_BWD_ROWS - 1) / CONV_BWD_ROWS;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= 2ll * B * nrb * f4) return;
  const int c4 = static_cast<int>(idx % f4);
  const long long rest = idx / f4;
  const int rb = static_cast<int>(rest % nrb);
  const int b = static_cast<int>((rest / nrb) % B);
  const int path = static_cast<int>(rest / (static_cast<long long>(nrb) * B));
  const int c0 = 4 * c4;
  const float* dzb = path ? dzb_S : dzb_T;
  // taps of the 4 columns: 8 bf16 of tap m hold columns 8 (c0 / 8) .. + 7
  float w[KMAX][4];
  {
    const uint4* tp = reinterpret_cast<const uint4*>(taps) +
                      (static_cast<long long>(path) * (f / 8) + c0 / 8) * KMAX;
    const int half = (c0 / 4) & 1;
#pragma unroll
    for (int m = 0; m < KMAX; ++m) {
      const uint4 u = __ldg(tp + m);
      const uint32_t a = half ? u.z : u.x, bb = half ? u.w : u.y;
      w[m][0] = bf16lo_to_f32(a);
      w[m][1] = bf16hi_to_f32(a);
      w[m][2] = bf16lo_to_f32(bb);
      w[m][3] = bf16hi_to_f32(bb);
    }
  }
  const int s0 = rb * CONV_BWD_ROWS;
  const int s1 = min(T, s0 + CONV_BWD_ROWS);
  // window: win[m] = dZbar row s + m (zero past T); rows up to s + KMAX - 1 are
  // held (their taps are zero when m >= k), so every index is static
  float4 win[KMAX];
  int ci = s0 / C, cj = s0 % C;  // chunk and row within it of the next row to load
  auto next_row = [&]() {
    const long long pr = (static_cast<long long>(b) * Nc + ci) * Cp + cj;
    if (++cj == C) { cj = 0; ++ci; }
    return __ldg(reinterpret_cast<const float4*>(dzb + pr * f + c0));
  };
#pragma unroll
  for (int m = 0; m < KMAX - 1; ++m)
    win[m + 1] = s0 + m < T ? next_row() : make_float4(0.f, 0.f, 0.f, 0.f);
  const long long BT = static_cast<long long>(B) * T;
  for (int s = s0; s < s1; ++s) {
#pragma unroll
    for (int m = 0; m < KMAX - 1; ++m) win[m] = win[m + 1];
    win[KMAX - 1] = s + KMAX - 1 < T ? next_row() : make_float4(0.f, 0.f, 0.f, 0.f);
    const long long bt = static_cast<long long>(b) * T + s;
    float4 acc = path ? __ldg(reinterpret_cast<const float4*>(dzs_read + bt * f + c0))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m = 0; m < KMAX; ++m) {
      if (m >= k) break;
      acc.x = fmaf(w[m][0], win[m].x, acc.x);
      acc.y = fmaf(w[m][1], win[m].y, acc.y);
      acc.z = fmaf(w[m][2], win[m].z, acc.z);
      acc.w = fmaf(w[m][3], win[m].w, acc.w);
    }
    reinterpret_cast<float4*>(dZ + (path * BT + bt) * f)[c4] = acc;
  }
}

constexpr int TAP_SPLITS = 128;  // most token splits of the tap gradient (partials per split)
constexpr int TAP_THREADS = 128;

__device__ __forceinline__ void bf16x4_to_f32(uint2 u, float (&v)[4]) {
  v[0] = bf16lo_to_f32(u.x);
  v[1] = bf16hi_to_f32(u.x);
  v[2] = bf16lo_to_f32(u.y);
  v[3] = bf16hi_to_f32(u.y);
}

// part[split][path][c][m] = sum over the split's tokens (b, t), t >= m, of
// dZbar_path[b, t, c] Z_path[b, t - m, c].  Thread = (path, 4 columns, split):
// it walks its contiguous tokens keeping the last k rows of Z in registers
// (packed bf16) and a ring of the next TAP_AHEAD tokens' Z (8 bytes) and dZbar
// (16 bytes) in flight while it accumulates the current one.  The host picks
// nsplit <= TAP_SPLITS so that the grid fits one wave.  Z [2, B, T, f] bf16,
// dZbar chunk-padded fp32.
constexpr int TAP_AHEAD = 4;
template <int KMAX>
__global__ void __launch_bounds__(TAP_THREADS, KMAX <= 4 ? 6 : 4) conv_tap_grad_kernel(
    const float* __restrict__ dzb_T, const float* __restrict__ dzb_S,
    const __nv_bfloat16* __restrict__ z, float* __restrict__ part, int B, int T, int f, int k,
    int C, int Cp, int Nc, int nsplit) {
  const int f4 = f / 4;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= 2 * f4 * nsplit) return;
  const int c4 = idx % f4;
  const int split = (idx / f4) % nsplit;
  const int path = idx / (f4 * nsplit);
  const long long BT = static_cast<long long>(B) * T;
  const long long per = (BT + nsplit - 1) / nsplit;
  const long long r0 = split * per, r1 = min(BT, r0 + per);
  const float* dzb = (path ? dzb_S : dzb_T) + c4 * 4;
  const __nv_bfloat16* zp = z + path * BT * f + c4 * 4;
  float acc[KMAX][4];
#pragma unroll
  for (int m = 0; m < KMAX; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;
  uint2 zw[KMAX];  // zw[m] = Z row t - m, 4 bf16
#pragma unroll
  for (int m = 0; m < KMAX; ++m) zw[m] = make_uint2(0u, 0u);
  if (r0 < r1) {
    int t = static_cast<int>(r0 % T);  // position of the token being summed
    // the k - 1 rows before the split's first token (same sequence only)
#pragma unroll
    for (int m = 1; m < KMAX; ++m)
      if (m < k && t - m >= 0) zw[m] = __ldg(reinterpret_cast<const uint2*>(zp + (r0 - m) * f));
    // load cursor: the next token to fetch, as (sequence, chunk, row in chunk)
    long long lr = r0;
    int lb = static_cast<int>(r0 / T), lci = t / C, lcj = t % C, lt = t;
    uint2 zr[TAP_AHEAD];
    float4 gr[TAP_AHEAD];
    auto fetch = [&](uint2& zd, float4& gd) {
      zd = __ldg(reinterpret_cast<const uint2*>(zp + lr * f));
      gd = __ldg(reinterpret_cast<const float4*>(
          dzb + ((static_cast<long long>(lb) * Nc + lci) * Cp + lcj) * f));
      ++lr;
      ++lt;
      if (++lcj == C) { lcj = 0; ++lci; }
      if (lt == T) { lt = 0; ++lb; lci = 0; lcj = 0; }
    };
#pragma unroll
    for (int j = 0; j < TAP_AHEAD; ++j)
      if (lr < r1) fetch(zr[j], gr[j]);
    for (long long bt = r0; bt < r1; bt += TAP_AHEAD) {
#pragma unroll
      for (int j = 0; j < TAP_AHEAD; ++j) {
        if (bt + j < r1) {
          if (t == 0) {  // a sequence starts: the window restarts from zeros
#pragma unroll
            for (int m = 1; m < KMAX; ++m) zw[m] = make_uint2(0u, 0u);
          }
          zw[0] = zr[j];
          const float g[4] = {gr[j].x, gr[j].y, gr[j].z, gr[j].w};
          if (lr < r1) fetch(zr[j], gr[j]);  // refill the slot TAP_AHEAD tokens ahead
#pragma unroll
          for (int m = 0; m < KMAX; ++m) {
            float zf[4];
            bf16x4_to_f32(zw[m], zf);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[m][i] = fmaf(g[i], zf[i], acc[m][i]);
          }
          // shift the window: row t becomes t - 1 for the next token
#pragma unroll
          for (int m = KMAX - 1; m > 0; --m) zw[m] = zw[m - 1];
          if (++t == T) t = 0;
        }
      }
    }
  }
  float* dst = part + ((static_cast<long long>(split) * 2 + path) * f + c4 * 4) * k;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int m = 0; m < KMAX; ++m)
      if (m < k) dst[i * k + m] = acc[m][i];
}

// out[path][c][m] = sum over the nsplit splits of part[split][path][c][m].
__global__ void conv_tap_reduce_kernel(const float* __restrict__ part, float* __restrict__ out_T,
                                       float* __restrict__ out_S, int f, int k, int nsplit) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= 2 * f * k) return;
  const int path = idx / (f * k), e = idx % (f * k);
  float s = 0.f;
  for (int q = 0; q < nsplit; ++q) s += part[(static_cast<long long>(q) * 2 + path) * f * k + e];
  (path ? out_S : out_T)[e] = s;
}

// dW_down = part + sum_b (d_state_in[b] - d_state_out[b])  (d_state_out nullable):
// the read path's sum_t dy_t Z_S[t]^T is the reverse prefix's total less its start.
__global__ void dw_down_combine_kernel(const float* __restrict__ part,
                                       const float* __restrict__ d_state_in,
                                       const float* __restrict__ d_state_out,
                                       float* __restrict__ out, int B, long long n) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float s = part[i];
  for (int b = 0; b < B; ++b) {
    s += d_state_in[b * n + i];
    if (d_state_out) s -= d_state_out[b * n + i];
  }
  out[i] = s;
}

// ------------------------------------------------------------ block backward
// Backward of y = x r g, r = (mean(x^2) + eps)^(-1/2) (the block's RMSNorms):
//   dx = r (a - xhat mean(a xhat)),  a = dy g,  xhat = x r;  dg = sum_rows dy xhat.
// One warp per row (grid-stride); dg accumulates per block in shared memory
// and leaves as one partial row per block, gpart [gridDim.x, d].

// The MLP RMSNorm of both paths (rows t and BT + t of h and du), with the
// residual of the output (out = h_S + y, so d_out reaches h_S directly):
//   dh_T = vjp(h_T, du_T),  dh_S = vjp(h_S, du_S) + d_out
//   dh16 rows t, BT + t = bf16(dh_T), bf16(dh_S);  dx[t] = dh_T + dh_S  (x -> h_P)
__global__ void __launch_bounds__(256) mlp_norm_backward_kernel(
    const float* __restrict__ h, const float* __restrict__ du, const __nv_bfloat16* __restrict__ g,
    const __nv_bfloat16* __restrict__ d_out, __nv_bfloat16* __restrict__ dh16,
    float* __restrict__ dx, float* __restrict__ gpart, long long BT, int d, float eps) {
  extern __shared__ float gsum[];  // [d]
  for (int c = threadIdx.x; c < d; c += blockDim.x) gsum[c] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long t = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
       t < BT; t += nw) {
    float rr[2], mm[2];
    // pass 1: r and mean(a xhat) of both rows
#pragma unroll
    for (int path = 0; path < 2; ++path) {
      const long long row = path * BT + t;
      float ss = 0.f, ax = 0.f;
      for (int c = lane * 8; c < d; c += 256) {
        float x[8], dy[8], gv[8];
        ld8f(h + row * d + c, x);
        ld8f(du + row * d + c, dy);
        ld8f(g + c, gv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          ss = fmaf(x[i], x[i], ss);
          ax = fmaf(dy[i] * gv[i], x[i], ax);
        }
      }
      ss = warp_sum(ss);
      ax = warp_sum(ax);
      rr[path] = rsqrtf(ss / d + eps);
      mm[path] = ax * rr[path] / d;  // mean(a xhat) = r mean(a x)
    }
    // pass 2: dh of both rows, dx = dh_T + dh_S, dg
    for (int c = lane * 8; c < d; c += 256) {
      float gv[8], dh[2][8];
      ld8f(g + c, gv);
#pragma unroll
      for (int path = 0; path < 2; ++path) {
        const long long row = path * BT + t;
        float x[8], dy[8];
        ld8f(h + row * d + c, x);
        ld8f(du + row * d + c, dy);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float xh = x[i] * rr[path];
          dh[path][i] = rr[path] * (dy[i] * gv[i] - xh * mm[path]);
          atomicAdd(&gsum[c + i], dy[i] * xh);
        }
      }
      float res[8], sum[8];
      ld8f(d_out + t * d + c, res);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        dh[1][i] += res[i];
        sum[i] = dh[0][i] + dh[1][i];
      }
      st8f(dh16 + t * d + c, dh[0]);
      st8f(dh16 + (BT + t) * d + c, dh[1]);
      st8f(dx + t * d + c, sum);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += blockDim.x)
    gpart[static_cast<long long>(blockIdx.x) * d + c] = gsum[c];
}

// The input RMSNorm: dx[t] += vjp(x[t], dxn[t]) (x bf16), dg partials.
__global__ void __launch_bounds__(256) input_norm_backward_kernel(
    const __nv_bfloat16* __restrict__ x, const float* __restrict__ dxn,
    const __nv_bfloat16* __restrict__ g, float* __restrict__ dx, float* __restrict__ gpart,
    long long BT, int d, float eps) {
  extern __shared__ float gsum[];  // [d]
  for (int c = threadIdx.x; c < d; c += blockDim.x) gsum[c] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long t = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
       t < BT; t += nw) {
    float ss = 0.f, ax = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
      float xv[8], dy[8], gv[8];
      ld8f(x + t * d + c, xv);
      ld8f(dxn + t * d + c, dy);
      ld8f(g + c, gv);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ss = fmaf(xv[i], xv[i], ss);
        ax = fmaf(dy[i] * gv[i], xv[i], ax);
      }
    }
    ss = warp_sum(ss);
    ax = warp_sum(ax);
    const float r = rsqrtf(ss / d + eps);
    const float mm = ax * r / d;
    for (int c = lane * 8; c < d; c += 256) {
      float xv[8], dy[8], gv[8], o[8];
      ld8f(x + t * d + c, xv);
      ld8f(dxn + t * d + c, dy);
      ld8f(g + c, gv);
      ld8f(dx + t * d + c, o);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float xh = xv[i] * r;
        o[i] += r * (dy[i] * gv[i] - xh * mm);
        atomicAdd(&gsum[c + i], dy[i] * xh);
      }
      st8f(dx + t * d + c, o);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += blockDim.x)
    gpart[static_cast<long long>(blockIdx.x) * d + c] = gsum[c];
}

// out[c] = sum over the rows of part [n, d] (fixed order).
__global__ void column_sum_kernel(const float* __restrict__ part, float* __restrict__ out, int n,
                                  int d) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= d) return;
  float s = 0.f;
  for (int i = 0; i < n; ++i) s += part[static_cast<long long>(i) * d + c];
  out[c] = s;
}

// RoPE backward and packing of the Q/K/V gradients into one bf16 row per token:
// dqkv[bt] = [R^T dq (Hq heads) | R^T dk (Hkv heads) | dv (Hkv heads)], where
// R^T turns the pair (d_i, d_{i+hd/2}) at position t by -angle:
// (d_i c + d_{i+hd/2} s, d_{i+hd/2} c - d_i s); cs [hd/2][T] half2 (cos, sin),
// the forward's table.  One thread per (token, head, pair); the V heads copy.
__global__ void rope_backward_pack_kernel(const float* __restrict__ dq, const float* __restrict__ dk,
                                          const float* __restrict__ dv,
                                          const __half2* __restrict__ cs,
                                          __nv_bfloat16* __restrict__ dqkv, long long BT, int T,
                                          int Hq, int Hkv, int hd) {
  const int half = hd / 2;
  const int heads = Hq + 2 * Hkv;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= BT * heads * half) return;
  const int i = static_cast<int>(idx % half);
  const int hh = static_cast<int>((idx / half) % heads);
  const long long bt = idx / (static_cast<long long>(half) * heads);
  const int t = static_cast<int>(bt % T);
  const long long ld = static_cast<long long>(heads) * hd;
  __nv_bfloat16* out = dqkv + bt * ld + static_cast<long long>(hh) * hd;
  const float* src;
  if (hh < Hq) src = dq + (bt * Hq + hh) * hd;
  else if (hh < Hq + Hkv) src = dk + (bt * Hkv + (hh - Hq)) * hd;
  else src = dv + (bt * Hkv + (hh - Hq - Hkv)) * hd;
  const float a = src[i], b = src[i + half];
  if (hh < Hq + Hkv) {
    const float2 e = __half22float2(cs[static_cast<long long>(i) * T + t]);
    out[i] = __float2bfloat16_rn(a * e.x + b * e.y);
    out[i + half] = __float2bfloat16_rn(b * e.x - a * e.y);
  } else {
    out[i] = __float2bfloat16_rn(a);
    out[i + half] = __float2bfloat16_rn(b);
  }
}

}  // namespace ttcd
