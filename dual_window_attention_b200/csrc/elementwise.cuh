// Memory-bound kernels of the block: RMSNorm, rotary table, the fused
// short-conv / residual-difference / key kernel, key scales, casts, transpose.
#pragma once
#include "ptx.cuh"

namespace ttcd {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// out[r, :] = bf16(in[r, :] * (mean(in[r,:]^2) + eps)^(-1/2) * g).  One warp per row.
// RMSNorm as the block's pre-norm (papernotes.org review, 方法详解: the shared
// backbone; the pages leave the skeleton unstated, a pre-norm decoder layer is
// the plain reading).
template <class InT, class GT>
__global__ void rmsnorm_kernel(const InT* __restrict__ in, const GT* __restrict__ g,
                               __nv_bfloat16* __restrict__ out, long long rows, int d, float eps) {
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const InT* x = in + row * d;
  float ss = 0.f;
  for (int c = lane * 8; c < d; c += 256) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v = to_f32(x[c + i]);
      ss += v * v;
    }
  }
  ss = warp_sum(ss);
  const float rs = rsqrtf(ss / d + eps);
  __nv_bfloat16* y = out + row * d;
  for (int c = lane * 8; c < d; c += 256) {
    uint4 w;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = to_f32(x[c + i]) * rs * to_f32(g[c + i]);
    w.x = pack_bf16x2(v[0], v[1]);
    w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]);
    w.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(y + c) = w;
  }
}

// cs[t][i] = (cos, sin)(t * theta^(-2i/hd)), evaluated in double precision.
__global__ void rope_table_kernel(float2* __restrict__ cs, int T, int hd, double theta) {
  const int half = hd / 2;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(T) * half) return;
  const int t = static_cast<int>(idx / half);
  const int i = static_cast<int>(idx % half);
  const double inv = pow(theta, -2.0 * i / hd);
  double s, c;
  sincos(static_cast<double>(t) * inv, &s, &c);
  cs[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

// Fused short causal convolutions, residual difference and student keys.
// papernotes.org review, 关键设计 3: Zbar_P = conv_P(Z_P) (depthwise, causal),
// D = Zbar_T - Zbar_S, K = l2-norm(Zbar_S).  The per-row norm needs the whole
// d_ff row, so this kernel writes Zbar_S unnormalised (transposed, Kt) and adds
// its squares into ssq_part[channel block][p]; the scale beta_t / ||.|| is applied to the value
// residual instead (Delta W = sum beta r k^T is linear in that scale).
//
// Z     fp32 [2, BT, f]: teacher rows then student rows
// taps  [f, k] (tap m multiplies t - m), TapT = bf16 or fp32
// D     bf16 [P, f]      Kt bf16 [f, P]     Zs16 bf16 [BT, f]    ssq_part fp32 [f/64, P]
// Padded index p = (b*Nc + i)*Cp + j holds token t = i*C + j when j < C and t < T;
// other p get D = 0 and Kt = 0.
// Block: 64 padded positions x 64 channels, 256 threads (thread = one position,
// 16 channels).
constexpr int CONV_TP = 64, CONV_TC = 64;
template <class TapT>
__global__ void __launch_bounds__(256)
    conv_residual_key_kernel(const float* __restrict__ Z, const TapT* __restrict__ tapT,
                             const TapT* __restrict__ tapS, __nv_bfloat16* __restrict__ D,
                             __nv_bfloat16* __restrict__ Kt, __nv_bfloat16* __restrict__ Zs16,
                             float* __restrict__ ssq_part, int T, int f, int k, int C, int Cp,
                             int Nc, long long BT, long long P) {
  __shared__ __nv_bfloat16 tileK[CONV_TC][CONV_TP + 8];
  __shared__ float sq_part[4][CONV_TP];
  const long long p0 = static_cast<long long>(blockIdx.x) * CONV_TP;
  const int c0 = blockIdx.y * CONV_TC;
  const int tp = threadIdx.x & 63;   // position within tile
  const int cg = threadIdx.x >> 6;   // 16-channel group
  const long long p = p0 + tp;
  const long long seq_len_p = static_cast<long long>(Nc) * Cp;
  const int b = static_cast<int>(p / seq_len_p);
  const long long rem = p % seq_len_p;
  const int i = static_cast<int>(rem / Cp), j = static_cast<int>(rem % Cp);
  const int t = i * C + j;
  const bool valid = p < P && j < C && t < T;
  const int cbase = c0 + cg * 16;
  float zbS[16];
  float sq = 0.f;
  if (valid) {
    float zbT[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) { zbT[c] = 0.f; zbS[c] = 0.f; }
    const long long rowT = static_cast<long long>(b) * T + t;
    for (int m = 0; m < k; ++m) {
      if (t - m < 0) break;
      const float* zt = Z + (rowT - m) * f + cbase;
      const float* zs = Z + (BT + rowT - m) * f + cbase;
#pragma unroll
      for (int c4 = 0; c4 < 16; c4 += 4) {
        const float4 a = *reinterpret_cast<const float4*>(zt + c4);
        const float4 s = *reinterpret_cast<const float4*>(zs + c4);
        const float wa[4] = {a.x, a.y, a.z, a.w};
        const float ws[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = cbase + c4 + e;
          zbT[c4 + e] += to_f32(tapT[c * k + m]) * wa[e];
          zbS[c4 + e] += to_f32(tapS[c * k + m]) * ws[e];
        }
      }
      if (m == 0) {
        uint4 w0, w1;
        w0.x = pack_bf16x2(zs[0], zs[1]);   w0.y = pack_bf16x2(zs[2], zs[3]);
        w0.z = pack_bf16x2(zs[4], zs[5]);   w0.w = pack_bf16x2(zs[6], zs[7]);
        w1.x = pack_bf16x2(zs[8], zs[9]);   w1.y = pack_bf16x2(zs[10], zs[11]);
        w1.z = pack_bf16x2(zs[12], zs[13]); w1.w = pack_bf16x2(zs[14], zs[15]);
        uint4* dz = reinterpret_cast<uint4*>(Zs16 + rowT * f + cbase);
        dz[0] = w0;
        dz[1] = w1;
      }
    }
    uint4 w0, w1;
    float dd[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      dd[c] = zbT[c] - zbS[c];
      sq += zbS[c] * zbS[c];
    }
    w0.x = pack_bf16x2(dd[0], dd[1]);   w0.y = pack_bf16x2(dd[2], dd[3]);
    w0.z = pack_bf16x2(dd[4], dd[5]);   w0.w = pack_bf16x2(dd[6], dd[7]);
    w1.x = pack_bf16x2(dd[8], dd[9]);   w1.y = pack_bf16x2(dd[10], dd[11]);
    w1.z = pack_bf16x2(dd[12], dd[13]); w1.w = pack_bf16x2(dd[14], dd[15]);
    uint4* dD = reinterpret_cast<uint4*>(D + p * f + cbase);
    dD[0] = w0;
    dD[1] = w1;
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c) zbS[c] = 0.f;
    if (p < P) {
      uint4* dD = reinterpret_cast<uint4*>(D + p * f + cbase);
      dD[0] = make_uint4(0, 0, 0, 0);
      dD[1] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int c = 0; c < 16; ++c) tileK[cg * 16 + c][tp] = __float2bfloat16_rn(zbS[c]);
  sq_part[cg][tp] = sq;
  __syncthreads();
  // Deterministic per-(channel block, position) partial sums; summed in order later.
  if (cg == 0 && p < P)
    ssq_part[static_cast<long long>(blockIdx.y) * P + p] =
        ((sq_part[0][tp] + sq_part[1][tp]) + sq_part[2][tp]) + sq_part[3][tp];
  // Transposed store: each warp writes rows of Kt (64 positions = 128 bytes).
  for (int r = threadIdx.x >> 3; r < CONV_TC; r += 32) {
    const int seg = threadIdx.x & 7;  // 8 x 16 bytes per row
    const long long pp = p0 + seg * 8;
    if (pp < P) {
      const uint4 w = *reinterpret_cast<const uint4*>(&tileK[r][seg * 8]);
      *reinterpret_cast<uint4*>(Kt + static_cast<long long>(c0 + r) * P + pp) = w;
    }
  }
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

template <class InT>
__global__ void cast_to_bf16_kernel(const InT* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                    long long n) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) out[i] = __float2bfloat16_rn(to_f32(in[i]));
}

// out[c, r] = in[r, c] for an [R, Cn] matrix.
template <class InT>
__global__ void transpose_to_bf16_kernel(const InT* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                         int R, int Cn) {
  __shared__ float tile[32][33];
  const int bx = blockIdx.x * 32, by = blockIdx.y * 32;
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int r = by + y, c = bx + threadIdx.x;
    if (r < R && c < Cn) tile[y][threadIdx.x] = to_f32(in[static_cast<long long>(r) * Cn + c]);
  }
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int c = bx + y, r = by + threadIdx.x;
    if (r < R && c < Cn) out[static_cast<long long>(c) * R + r] = __float2bfloat16_rn(tile[threadIdx.x][y]);
  }
}

}  // namespace ttcd
