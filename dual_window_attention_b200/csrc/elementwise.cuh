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
template <class InT, class GT, class OutT>
__global__ void rmsnorm_kernel(const InT* __restrict__ in, const GT* __restrict__ g,
                               OutT* __restrict__ out, long long rows, int d, float eps) {
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
  OutT* y = out + row * d;
  for (int c = lane * 8; c < d; c += 256) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = to_f32(x[c + i]) * rs * to_f32(g[c + i]);
    store8(y + c, v);
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
// d_ff row, so this kernel writes Zbar_S unnormalised (transposed, Kt) and the
// squares of its 64-channel slice into ssq_part[channel block][p]; the scale
// beta_t / ||.|| is applied to the value residual instead (Delta W = sum beta r
// k^T is linear in that scale).
//
// Z     fp32 [2, BT, f]: teacher rows then student rows
// taps  [f, k] (tap m multiplies t - m), TapT = bf16 or fp32
// D     bf16 [P, f]      Kt bf16 [f, P]     Zs16 bf16 [BT, f]    ssq_part fp32 [f/64, P]
// Padded index p = (b*Nc + i)*Cp + j holds token t = i*C + j when j < C and t < T;
// other p get D = 0 and Kt = 0.
// Block: 64 padded positions (inside one chunk, since Cp is a multiple of 64) x
// 64 channels, 256 threads.  The Z rows t0-(k-1) .. t0+63 of both paths are
// staged in shared memory with coalesced 16-byte loads (16 threads per 256-byte
// row); thread (cq, tr) then owns channels 4cq..4cq+3 of positions tr + 16 i.
constexpr int CONV_TP = 64, CONV_TC = 64, CONV_MAXK = 8;
template <class TapT, class E>
__global__ void __launch_bounds__(256)
    conv_residual_key_kernel(const float* __restrict__ Z, const TapT* __restrict__ tapT,
                             const TapT* __restrict__ tapS, E* __restrict__ D,
                             E* __restrict__ Kt, E* __restrict__ Zs16,
                             float* __restrict__ ssq_part, int T, int f, int k, int C, int Cp,
                             int Nc, long long BT, long long P) {
  constexpr int ROWS = CONV_TP + CONV_MAXK - 1;
  __shared__ __align__(16) float zT[ROWS][CONV_TC];
  __shared__ __align__(16) float zS[ROWS][CONV_TC];
  __shared__ float taps[2][CONV_MAXK][CONV_TC];
  // The key tile (token-major fp32, odd row stride of 65 words so that both its
  // row writes and its column reads spread over the banks) reuses zT's storage
  // once the convolutions are done.
  constexpr int KSTRIDE = CONV_TC + 1;
  float* tileK = &zT[0][0];
  static_assert(sizeof(zT) >= sizeof(float) * KSTRIDE * CONV_TP, "key tile must fit in zT");
  const long long p0 = static_cast<long long>(blockIdx.x) * CONV_TP;
  const int c0 = blockIdx.y * CONV_TC;
  const long long seq_len_p = static_cast<long long>(Nc) * Cp;
  const int b = static_cast<int>(p0 / seq_len_p);
  const long long rem0 = p0 % seq_len_p;
  const int ci = static_cast<int>(rem0 / Cp), j0 = static_cast<int>(rem0 % Cp);
  const int t0 = ci * C + j0;               // token of position p0 (if valid)
  const int n_valid = max(0, min(CONV_TP, min(C - j0, T - t0)));
  const long long rowT0 = static_cast<long long>(b) * T;
  const int tid = threadIdx.x;

  for (int i = tid; i < 2 * CONV_MAXK * CONV_TC; i += 256) {
    const int path = i / (CONV_MAXK * CONV_TC), m = (i / CONV_TC) % CONV_MAXK, c = i % CONV_TC;
    const TapT* tp = path ? tapS : tapT;
    taps[path][m][c] = m < k ? to_f32(tp[static_cast<long long>(c0 + c) * k + m]) : 0.f;
  }
  // Stage rows t0-(k-1) .. t0+n_valid-1 (missing rows are zero).
  const int halo = k - 1;
  for (int i = tid; i < (n_valid + halo) * 16; i += 256) {
    const int rr = i >> 4, cq = i & 15;
    const int t = t0 - halo + rr;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), s = a;
    if (t >= 0) {
      a = *reinterpret_cast<const float4*>(Z + (rowT0 + t) * f + c0 + 4 * cq);
      s = *reinterpret_cast<const float4*>(Z + (BT + rowT0 + t) * f + c0 + 4 * cq);
    }
    *reinterpret_cast<float4*>(&zT[CONV_MAXK - 1 - halo + rr][4 * cq]) = a;
    *reinterpret_cast<float4*>(&zS[CONV_MAXK - 1 - halo + rr][4 * cq]) = s;
  }
  __syncthreads();

  const int cq = tid & 15, tr = tid >> 4;
  float keys[CONV_TP / 16][4];
#pragma unroll
  for (int it = 0; it < CONV_TP / 16; ++it) {
    const int jj = tr + 16 * it;  // position within the tile
    const long long p = p0 + jj;
    const bool valid = jj < n_valid;
    float zbT[4] = {0.f, 0.f, 0.f, 0.f}, zbS[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) {
      for (int m = 0; m < k; ++m) {
        const int row = CONV_MAXK - 1 + jj - m;
        const float4 a = *reinterpret_cast<const float4*>(&zT[row][4 * cq]);
        const float4 s = *reinterpret_cast<const float4*>(&zS[row][4 * cq]);
        zbT[0] += taps[0][m][4 * cq + 0] * a.x; zbS[0] += taps[1][m][4 * cq + 0] * s.x;
        zbT[1] += taps[0][m][4 * cq + 1] * a.y; zbS[1] += taps[1][m][4 * cq + 1] * s.y;
        zbT[2] += taps[0][m][4 * cq + 2] * a.z; zbS[2] += taps[1][m][4 * cq + 2] * s.z;
        zbT[3] += taps[0][m][4 * cq + 3] * a.w; zbS[3] += taps[1][m][4 * cq + 3] * s.w;
      }
    }
    // D (zeros at padding) and the bf16 copy of Z_S, 8 bytes per thread, 128 bytes per row.
    store4(D + p * f + c0 + 4 * cq, zbT[0] - zbS[0], zbT[1] - zbS[1], zbT[2] - zbS[2],
           zbT[3] - zbS[3]);
    if (valid && Zs16) {
      const float4 s = *reinterpret_cast<const float4*>(&zS[CONV_MAXK - 1 + jj][4 * cq]);
      store4(Zs16 + (rowT0 + t0 + jj) * f + c0 + 4 * cq, s.x, s.y, s.z, s.w);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) keys[it][e] = zbS[e];
    // squares of this 64-channel slice, reduced over the 16 threads of the row
    float sq = zbS[0] * zbS[0] + zbS[1] * zbS[1] + zbS[2] * zbS[2] + zbS[3] * zbS[3];
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (cq == 0) ssq_part[static_cast<long long>(blockIdx.y) * P + p] = sq;
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < CONV_TP / 16; ++it)
#pragma unroll
    for (int e = 0; e < 4; ++e) tileK[(tr + 16 * it) * KSTRIDE + 4 * cq + e] = keys[it][e];
  __syncthreads();
  // Transposed store of the keys: each row of Kt (one channel) gets 64 positions
  // in 16-byte segments; consecutive threads write consecutive segments.
  constexpr int SEG_E = 16 / sizeof(E), SEGS = CONV_TP / SEG_E;
  for (int i = tid; i < CONV_TC * SEGS; i += 256) {
    const int r = i / SEGS, seg = i % SEGS;
    __align__(16) E vals[SEG_E];
#pragma unroll
    for (int j = 0; j < SEG_E; ++j) vals[j] = from_f32<E>(tileK[(seg * SEG_E + j) * KSTRIDE + r]);
    *reinterpret_cast<uint4*>(Kt + static_cast<long long>(c0 + r) * P + p0 + seg * SEG_E) =
        *reinterpret_cast<const uint4*>(vals);
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
