// Memory-bound kernels of the block: RMSNorm, rotary table, the fused
// short-conv / residual-difference / key kernel, key scales, casts, transpose.
#pragma once
#include "ptx.cuh"

namespace ttcd {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ void store8(__nv_bfloat16* dst, const float (&v)[8]) {
  uint4 w;
  w.x = pack_bf16x2(v[0], v[1]);
  w.y = pack_bf16x2(v[2], v[3]);
  w.z = pack_bf16x2(v[4], v[5]);
  w.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(dst) = w;
}
__device__ __forceinline__ void store8(float* dst, const float (&v)[8]) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* dst, float a, float b, float c, float d) {
  uint2 w;
  w.x = pack_bf16x2(a, b);
  w.y = pack_bf16x2(c, d);
  *reinterpret_cast<uint2*>(dst) = w;
}
__device__ __forceinline__ void store4(float* dst, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(dst) = make_float4(a, b, c, d);
}
template <class E>
__device__ __forceinline__ E from_f32(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ float from_f32<float>(float v) {
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// out[r, :] = bf16(in[r, :] * (mean(in[r,:]^2) + eps)^(-1/2) * g).  One warp per row.
// RMSNorm as the block's pre-norm (papernotes.org review, 方法详解: the shared
// backbone; the pages leave the skeleton unstated, a pre-norm decoder layer is
// the plain reading).
// One warp per row; rows up to RMS_CACHE * 256 columns stay in registers
// between the sum of squares and the scaling (one pass over HBM), longer rows
// are read again.
constexpr int RMS_CACHE = 4;
template <class InT, class GT, class OutT>
__global__ void rmsnorm_kernel(const InT* __restrict__ in, const GT* __restrict__ g,
                               OutT* __restrict__ out, long long rows, int d, float eps) {
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const InT* x = in + row * d;
  float xv[RMS_CACHE][8];
  float ss = 0.f;
#pragma unroll
  for (int q = 0; q < RMS_CACHE; ++q) {
    const int c = lane * 8 + q * 256;
    if (c < d) {
      ld8f(x + c, xv[q]);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss += xv[q][i] * xv[q][i];
    }
  }
  for (int c = lane * 8 + RMS_CACHE * 256; c < d; c += 256) {
    float v[8];
    ld8f(x + c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss += v[i] * v[i];
  }
  ss = warp_sum(ss);
  const float rs = rsqrtf(ss / d + eps);
  OutT* y = out + row * d;
#pragma unroll
  for (int q = 0; q < RMS_CACHE; ++q) {
    const int c = lane * 8 + q * 256;
    if (c < d) {
      float gv[8];
      ld8f(g + c, gv);
#pragma unroll
      for (int i = 0; i < 8; ++i) xv[q][i] *= rs * gv[i];
      store8(y + c, xv[q]);
    }
  }
  for (int c = lane * 8 + RMS_CACHE * 256; c < d; c += 256) {
    float v[8], gv[8];
    ld8f(x + c, v);
    ld8f(g + c, gv);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= rs * gv[i];
    store8(y + c, v);
  }
}

// rstd[r] = (mean(in[r, :]^2) + eps)^(-1/2): the input RMSNorm as a per-row
// scale, applied in the QKV GEMM epilogue (the block's pre-norm; papernotes.org
// review, 方法详解, shared backbone; the skeleton is a reading, see the oracle).
// One warp per row, 16-byte loads, d a multiple of 8.
template <class InT>
__global__ void rms_rowscale_kernel(const InT* __restrict__ in, float* __restrict__ rstd,
                                    long long rows, int d, float eps) {
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const InT* x = in + row * d;
  float ss = 0.f;
  for (int c = lane * 8; c < d; c += 256) {
    float v[8];
    ld8f(x + c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss += v[i] * v[i];
  }
  ss = warp_sum(ss);
  if (lane == 0) rstd[row] = rsqrtf(ss / d + eps);
}

// out[r, c] = w[r, c] * g[c] for a row-major [rows, cols] weight, 8 elements per
// thread (cols a multiple of 8): the RMSNorm gain folded into the next GEMM's
// weight, (x * g) W^T = x (W diag g)^T.  n8 = rows * cols / 8.
template <class E>
__global__ void scale_cols_kernel(const E* __restrict__ w, const E* __restrict__ g,
                                  E* __restrict__ out, long long n8, int cols) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const long long e0 = i * 8;
  const int c = static_cast<int>(e0 % cols);
  float v[8], gv[8];
  ld8f(w + e0, v);
  ld8f(g + c, gv);
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] *= gv[k];
  store8(out + e0, v);
}

// out[i] = OutT(in[i]), grid-stride (bf16 <-> fp32 conversions of interface tensors).
template <class InT, class OutT>
__global__ void cast_kernel(const InT* __restrict__ in, OutT* __restrict__ out, long long n) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += stride)
    out[i] = from_f32<OutT>(to_f32(in[i]));
}

// cs[i][t] = (cos, sin)((pos0 + t) * theta^(-2i/hd)) for every frequency
// i < hd/2 and position t < T, frequency-major [hd/2][T]: one thread per entry,
// the angle and its sincos in double precision, rounded once to half precision
// (11-bit significands, far below the bf16 rounding of q and k).  A warp
// writes 32 consecutive positions of one frequency (128 contiguous bytes).
// pos0: absolute position of row 0 (a sequence shard starts past 0);
// log2_theta = log2 of the RoPE base, so theta^(-2i/hd) = 2^(-(2i/hd) log2 theta).
__global__ void rope_table_kernel(__half2* __restrict__ cs, int T, int hd, double log2_theta,
                                  long long pos0 = 0) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int half = hd / 2;
  if (idx >= static_cast<long long>(half) * T) return;
  const int i = static_cast<int>(idx / T);
  const int t = static_cast<int>(idx % T);
  const double a = exp2(-2.0 * i / hd * log2_theta);
  double s, c;
  sincos(static_cast<double>(pos0 + t) * a, &s, &c);
  cs[idx] = __floats2half2_rn(static_cast<float>(c), static_cast<float>(s));
}

// Fused short causal convolutions, residual difference and student keys.
// papernotes.org review, 关键设计 3: Zbar_P = conv_P(Z_P) (depthwise, causal),
// D = Zbar_T - Zbar_S, K = l2-norm(Zbar_S).  The per-row norm needs the whole
// d_ff row, so this kernel writes Zbar_S unnormalised (Kp) and the squares of
// its 64-channel slice into ssq_part[channel block][p]; the scale
// beta_t / ||.|| is applied to the value residual instead (Delta W = sum
// beta r k^T is linear in that scale).
//
// Z     fp32 [2, BT, f]: teacher rows then student rows
// taps  [f, k] (tap m multiplies t - m), TapT = bf16 or fp32
// D, Kp E [P, f]         Zs16 E [BT, f] (nullable)        ssq_part fp32 [f/64, P]
// Padded index p = (b*Nc + i)*Cp + j holds token t = i*C + j when j < C and t < T;
// other p get D = 0 and Kp = 0.
// Block: 64 channels x 64 padded positions (inside one chunk: Cp is a multiple
// of 64), 256 threads; thread (cq, tg) owns channels 4cq..4cq+3 of positions
// 4tg..4tg+3 and slides a k-row window over them in registers.  A warp's loads
// and stores cover two 256-byte (fp32) or 128-byte (bf16) row segments.
// Blocks of one position tile run back to back over the channel blocks, so
// concurrently running blocks read whole rows of Z.
constexpr int CONV_TP = 64, CONV_TC = 64;
template <class TapT, class E, int CONV_MAXK>  // conv width k <= CONV_MAXK
__global__ void __launch_bounds__(256, CONV_MAXK <= 4 ? 3 : 1)
    conv_residual_key_kernel(const float* __restrict__ Z, const TapT* __restrict__ tapT,
                             const TapT* __restrict__ tapS, E* __restrict__ D,
                             E* __restrict__ Kp, E* __restrict__ Zs16,
                             float* __restrict__ ssq_part, int T, int f, int k, int C, int Cp,
                             int Nc, long long BT, long long P) {
  const int cblk = blockIdx.x;
  const long long p0 = static_cast<long long>(blockIdx.y) * CONV_TP;
  const int c0 = cblk * CONV_TC;
  const int tid = threadIdx.x;
  const int cq = tid & 15, tg = tid >> 4;
  const int c = c0 + 4 * cq;
  const long long seq_len_p = static_cast<long long>(Nc) * Cp;
  const int b = static_cast<int>(p0 / seq_len_p);
  const long long rem0 = p0 % seq_len_p;
  const int ci = static_cast<int>(rem0 / Cp), j0 = static_cast<int>(rem0 % Cp);
  const int tc0 = ci * C;                       // first token of this chunk
  const int len = min(C, T - tc0);              // tokens of this chunk
  const long long rowT0 = static_cast<long long>(b) * T;

  float wT[CONV_MAXK][4], wS[CONV_MAXK][4];
#pragma unroll
  for (int m = 0; m < CONV_MAXK; ++m)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      wT[m][e] = m < k ? to_f32(tapT[static_cast<long long>(c + e) * k + m]) : 0.f;
      wS[m][e] = m < k ? to_f32(tapS[static_cast<long long>(c + e) * k + m]) : 0.f;
    }
  // history: rows t-1 .. t-(k-1) of both paths for the first of this thread's positions
  const int jfirst = j0 + 4 * tg;
  float4 hT[CONV_MAXK - 1], hS[CONV_MAXK - 1];  // hT[m-1] = Z_T row (t - m)
#pragma unroll
  for (int m = 1; m < CONV_MAXK; ++m) {
    hT[m - 1] = make_float4(0.f, 0.f, 0.f, 0.f);
    hS[m - 1] = hT[m - 1];
    const int t = tc0 + jfirst - m;
    if (m < k && t >= 0 && jfirst < len) {
      hT[m - 1] = *reinterpret_cast<const float4*>(Z + (rowT0 + t) * f + c);
      hS[m - 1] = *reinterpret_cast<const float4*>(Z + (BT + rowT0 + t) * f + c);
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = jfirst + q;
    const long long p = p0 + 4 * tg + q;
    const bool valid = j < len;
    float4 zt = make_float4(0.f, 0.f, 0.f, 0.f), zs = zt;
    if (valid) {
      zt = *reinterpret_cast<const float4*>(Z + (rowT0 + tc0 + j) * f + c);
      zs = *reinterpret_cast<const float4*>(Z + (BT + rowT0 + tc0 + j) * f + c);
    }
    float bT[4] = {wT[0][0] * zt.x, wT[0][1] * zt.y, wT[0][2] * zt.z, wT[0][3] * zt.w};
    float bS[4] = {wS[0][0] * zs.x, wS[0][1] * zs.y, wS[0][2] * zs.z, wS[0][3] * zs.w};
#pragma unroll
    for (int m = 1; m < CONV_MAXK; ++m) {
      bT[0] += wT[m][0] * hT[m - 1].x; bS[0] += wS[m][0] * hS[m - 1].x;
      bT[1] += wT[m][1] * hT[m - 1].y; bS[1] += wS[m][1] * hS[m - 1].y;
      bT[2] += wT[m][2] * hT[m - 1].z; bS[2] += wS[m][2] * hS[m - 1].z;
      bT[3] += wT[m][3] * hT[m - 1].w; bS[3] += wS[m][3] * hS[m - 1].w;
    }
    if (!valid) {
#pragma unroll
      for (int e = 0; e < 4; ++e) bT[e] = bS[e] = 0.f;
    }
    store4(D + p * f + c, bT[0] - bS[0], bT[1] - bS[1], bT[2] - bS[2], bT[3] - bS[3]);
    store4(Kp + p * f + c, bS[0], bS[1], bS[2], bS[3]);
    if (valid && Zs16) store4(Zs16 + (rowT0 + tc0 + j) * f + c, zs.x, zs.y, zs.z, zs.w);
    float sq = bS[0] * bS[0] + bS[1] * bS[1] + bS[2] * bS[2] + bS[3] * bS[3];
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (cq == 0) ssq_part[static_cast<long long>(cblk) * P + p] = sq;
    // slide the window
#pragma unroll
    for (int m = CONV_MAXK - 2; m > 0; --m) {
      hT[m] = hT[m - 1];
      hS[m] = hS[m - 1];
    }
    hT[0] = zt;
    hS[0] = zs;
  }
}

// Zeroes the padding rows of the chunk-padded [P, f] buffers D and Kp (padded
// index p = (b*Nc + i)*Cp + j with j at or past chunk i's token count), which
// the fused gate/up epilogue does not write: the chunk-scan GEMM contracts over
// whole 64-token blocks, so those rows must hold zeros.  One thread per 8
// columns of a row (f a multiple of 8).
template <class E>
__global__ void pad_rows_zero_kernel(E* __restrict__ D, E* __restrict__ Kp, int f, int T, int C,
                                     int Cp, int Nc, long long P) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int per_row = f / 8;
  const long long p = idx / per_row;
  if (p >= P) return;
  const long long rem = p % (static_cast<long long>(Nc) * Cp);
  const int i = static_cast<int>(rem / Cp), j = static_cast<int>(rem % Cp);
  if (j < min(C, T - i * C)) return;
  const int c = static_cast<int>(idx % per_row) * 8;
  const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  store8(D + p * f + c, z);
  store8(Kp + p * f + c, z);
}

// out[path][b][j][:] = u[row][:] * rstd[row], row = path*BT + b*T + T - n + j,
// for j < n: the MLP inputs u_P = RMSNorm(h_P) of the last n tokens of every
// sequence (u holds h * g_mlp, rstd the row scales), which a sequence shard
// hands to the next one as the history of its short convs.  One thread per 8
// columns; out is [2, B, n, d].
template <class E>
__global__ void u_tail_kernel(const E* __restrict__ u, const float* __restrict__ rstd,
                              E* __restrict__ out, int B, int T, int d, int n, long long BT) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int per_row = d / 8;
  const long long r = idx / per_row;
  if (r >= 2ll * B * n) return;
  const int c = static_cast<int>(idx % per_row) * 8;
  const int j = static_cast<int>(r % n);
  const long long pb = r / n;
  const int b = static_cast<int>(pb % B), path = static_cast<int>(pb / B);
  const long long row = path * BT + static_cast<long long>(b) * T + T - n + j;
  float v[8];
  ld8f(u + row * d + c, v);
  const float s = rstd[row];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] *= s;
  store8(out + r * d + c, v);
}

// kscale[p] = beta[b, t] / sqrt(ssq[p] + eps) for real tokens, 0 for padding, where
// ssq[p] = sum over channel blocks (in order) of ssq_part[blk][p].
__global__ void key_scale_kernel(const float* __restrict__ ssq_part, int n_part,
                                 const float* __restrict__ beta, float* __restrict__ kscale,
                                 int T, int C, int Cp, int Nc, long long P, float eps) {
  const long long p = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (p >= P) return;
  float ssq = 0.f;
  for (int i = 0; i < n_part; ++i) ssq += ssq_part[static_cast<long long>(i) * P + p];
  const long long seq_len_p = static_cast<long long>(Nc) * Cp;
  const int b = static_cast<int>(p / seq_len_p);
  const long long rem = p % seq_len_p;
  const int i = static_cast<int>(rem / Cp), j = static_cast<int>(rem % Cp);
  const int t = i * C + j;
  const bool valid = j < C && t < T;
  kscale[p] = valid ? beta[static_cast<long long>(b) * T + t] * rsqrtf(ssq + eps) : 0.f;
}

// rstd[row] = (sum over tiles of ssq[tile][row] / d + eps)^(-1/2): the MLP
// RMSNorm's row scale from the partial sums the o_proj epilogue wrote.
// rows r0 .. rows-1 of the [n_part, rows] partial sums (r0 > 0: a later part only)
__global__ void rms_rstd_kernel(const float* __restrict__ ssq, int n_part, long long rows,
                                float inv_d, float eps, float* __restrict__ rstd,
                                long long r0 = 0) {
  const long long r = r0 + static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  float sum = 0.f;
  for (int i = 0; i < n_part; ++i) sum += ssq[i * rows + r];
  rstd[r] = rsqrtf(sum * inv_d + eps);
}

template <class InT>
__global__ void cast_to_bf16_kernel(const InT* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                    long long n) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) out[i] = __float2bfloat16_rn(to_f32(in[i]));
}

// out[c, r] = in[r, c] for an [R, Cn] matrix.
template <class InT, class OutT>
__global__ void transpose_kernel(const InT* __restrict__ in, OutT* __restrict__ out, int R,
                                 int Cn) {
  __shared__ float tile[32][33];
  const int bx = blockIdx.x * 32, by = blockIdx.y * 32;
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int r = by + y, c = bx + threadIdx.x;
    if (r < R && c < Cn) tile[y][threadIdx.x] = to_f32(in[static_cast<long long>(r) * Cn + c]);
  }
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int c = bx + y, r = by + threadIdx.x;
    if (r < R && c < Cn) out[static_cast<long long>(c) * R + r] = from_f32<OutT>(tile[threadIdx.x][y]);
  }
}

}  // namespace ttcd
