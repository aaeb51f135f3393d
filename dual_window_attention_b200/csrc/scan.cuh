// Chunked fast-weight increments with an on-chip exclusive prefix scan (sm_100a).
//
// papernotes.org review "Learning What to Remember", 关键设计 2 and 3:
//   Delta W_i = beta_i R_i K_i^T (low-rank, one per chunk), accumulated by a
//   causal prefix scan over chunks; README "Model configuration"
//   (ttt_force_grouped_scan: the fused scan path).
//
// One CTA owns a 128 x 128 tile (rows of d, columns of f) of one sequence's
// d x f state.  It walks the chunks in order.  For chunk i the tensor cores
// form Delta W_i = R[chunk i]^T . Kp[chunk i] (contraction over the chunk's
// padded tokens; R [P, d] and Kp [P, f] are token-major, so both operands are
// MN-major tiles: boxes of BK MN-elements x BK tokens, 128-byte swizzled) in
// one of two TMEM accumulators, while the epilogue
// warps fold the previous chunk into the fp32 running state S (a third TMEM
// region) and emit W_{i+1} = bf16(W_down + S_{i+1}) for the output GEMM.
// Chunk 0 reads W_0 = bf16(W_down + state_in).  The last state is written to
// state_out in fp32.
#pragma once
#include "gemm.cuh"

namespace ttcd {

template <class E>
struct ScanArgs {
  int d, f, Nc, Cp;
  const E* w_down;        // [d, f]
  const float* state_in;  // [B, d, f] nullable
  float* state_out;       // [B, d, f] nullable
  E* w_all;               // [B*Nc, d, f]
  int tiles_m, tiles_n;
};

// MN = true: R [P, d] and Kp [P, f] token-major, read as MN-major operands
// (bf16).  MN = false: their transposes Rt [d, P] and Kt [f, P], read as
// K-major operands (used for tf32, whose operands stay K-major).
template <class E, int STAGES, bool MN>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    fastweight_scan_kernel(const __grid_constant__ CUtensorMap mapR,
                           const __grid_constant__ CUtensorMap mapK, const ScanArgs<E> a,
                           const DevStatus st) {
  constexpr int BN = 128;
  constexpr int BK = ElemTraits<E>::BK;          // tokens per k-block == MN elements per box
  constexpr int BOX_BYTES = BK * BK * static_cast<int>(sizeof(E));
  constexpr int A_BYTES = GEMM_BM * 128, B_BYTES = BN * 128;  // 16 KB each either way
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr int KSTEP_BYTES = (32 / static_cast<int>(sizeof(E))) * 128;  // tokens per MMA x 128 B
  constexpr uint32_t IDESC = idesc_f32acc(GEMM_BM, BN, ElemTraits<E>::FMT, MN, MN);
  constexpr uint32_t COL_STATE = 256;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tn = blockIdx.x % a.tiles_n;
  const int tm = (blockIdx.x / a.tiles_n) % a.tiles_m;
  const int b = blockIdx.x / (a.tiles_n * a.tiles_m);
  const int m0 = tm * GEMM_BM, n0 = tn * BN;
  const int kpc = a.Cp / BK;  // k-blocks per chunk
  const long long P = static_cast<long long>(gridDim.x / (a.tiles_n * a.tiles_m)) * a.Nc * a.Cp;
  (void)P;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&accf[s], 1); mbar_init(&acce[s], 128); }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_map(&mapR);
    tma_prefetch_map(&mapK);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int i = 0; i < a.Nc && ok; ++i) {
        for (int kb = 0; kb < kpc; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, st, abort)) { ok = false; break; }
          uint8_t* sa = smem + s * STAGE_BYTES;
          const int y = (b * a.Nc + i) * a.Cp + kb * BK;  // first token of the k-block
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          if constexpr (MN) {
#pragma unroll
            for (int q = 0; q < GEMM_BM / BK; ++q)
              tma_load_2d(sa + q * BOX_BYTES, &mapR, &full[s], m0 + q * BK, y);
#pragma unroll
            for (int q = 0; q < BN / BK; ++q)
              tma_load_2d(sa + A_BYTES + q * BOX_BYTES, &mapK, &full[s], n0 + q * BK, y);
          } else {
            tma_load_2d(sa, &mapR, &full[s], y, m0);
            tma_load_2d(sa + A_BYTES, &mapK, &full[s], y, n0);
          }
        }
      }
      volatile int no_abort = 0;
      for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
        mbar_wait(&full[j % STAGES], (j / STAGES) & 1, st, &no_abort);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int i = 0; i < a.Nc && ok; ++i) {
        const int ab = i & 1;
        if (!mbar_wait(&acce[ab], ((i >> 1) & 1) ^ 1, st, abort)) break;
        tc_fence_after();
        for (int kb = 0; kb < kpc; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, st, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * STAGE_BYTES), sb = sa + A_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t da = MN ? sdesc_sw128(sa + k * KSTEP_BYTES, BOX_BYTES, 1024)
                                   : sdesc_sw128(sa + k * 32, 16, 1024);
            const uint64_t db = MN ? sdesc_sw128(sb + k * KSTEP_BYTES, BOX_BYTES, 1024)
                                   : sdesc_sw128(sb + k * 32, 16, 1024);
            mma_ss<E>(tmem + ab * BN, da, db, IDESC, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&accf[ab]);
      }
      mma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, st, &no_abort);
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int row = m0 + r;
    const bool row_ok = row < a.d;
    const uint32_t laddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const long long dfs = static_cast<long long>(a.d) * a.f;
    // S_0 = state_in (or 0); W_0 = bf16(W_down + S_0).
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      const int col = n0 + cc;
      float s[32];
      if (row_ok && col < a.f && a.state_in) {
        load_x32(a.state_in + b * dfs + static_cast<long long>(row) * a.f + col, s);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) s[e] = 0.f;
      }
      uint32_t u[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(s[e]);
      tmem_st32(laddr + COL_STATE + cc, u);
      if (row_ok && col < a.f) {
        float w[32];
        load_x32(a.w_down + static_cast<long long>(row) * a.f + col, w);
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] += s[e];
        store_x32(a.w_all + (static_cast<long long>(b) * a.Nc) * dfs +
                      static_cast<long long>(row) * a.f + col, w);
      }
    }
    tmem_st_wait();
    for (int i = 0; i < a.Nc; ++i) {
      const int ab = i & 1;
      if (!mbar_wait(&accf[ab], (i >> 1) & 1, st, abort)) break;
      tc_fence_after();
      const bool last = i + 1 == a.Nc;
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += 32) {
        const int col = n0 + cc;
        uint32_t dw[32], sv[32];
        tmem_ld32(laddr + ab * BN + cc, dw);
        tmem_ld32(laddr + COL_STATE + cc, sv);
        tmem_ld_wait();
        float s[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          s[e] = __uint_as_float(sv[e]) + __uint_as_float(dw[e]);
          sv[e] = __float_as_uint(s[e]);
        }
        tmem_st32(laddr + COL_STATE + cc, sv);
        if (row_ok && col < a.f) {
          if (!last) {
            float w[32];
            load_x32(a.w_down + static_cast<long long>(row) * a.f + col, w);
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] += s[e];
            store_x32(a.w_all + (static_cast<long long>(b) * a.Nc + i + 1) * dfs +
                          static_cast<long long>(row) * a.f + col, w);
          } else if (a.state_out) {
            store_f32x32(a.state_out + b * dfs + static_cast<long long>(row) * a.f + col, s);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&acce[ab]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ttcd
