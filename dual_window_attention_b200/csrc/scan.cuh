// Chunked fast-weight increments with an on-chip exclusive prefix scan (sm_100a).
//
// papernotes.org review "Learning What to Remember", 关键设计 2 and 3:
//   Delta W_i = beta_i R_i K_i^T (low-rank, one per chunk), accumulated by a
//   causal prefix scan over chunks; README "Model configuration"
//   (ttt_force_grouped_scan: the fused scan path).
//
// One CTA owns a 128 x 192 tile (rows of d, columns of f) of one sequence's
// d x f state and walks the chunks in order.  For chunk i the tensor cores form
// Delta W_i = R[chunk i]^T . Kp[chunk i] (contraction over the chunk's padded
// tokens) in one of two TMEM accumulators (2 x 192 columns), while eight
// epilogue warps fold the previous chunk into the fp32 running state S, which
// they keep in registers (each thread: one row, 96 columns), and emit
// W_{i+1} = W_down + S_{i+1} for the output GEMM.  Chunk 0 reads
// W_0 = W_down + state_in; the last state goes to state_out in fp32.  N = 192
// (not 256) gives 128 tiles at the Qwen3 shape, so most SMs get one.
// MN = true: R [P, d] and Kp [P, f] token-major, read as MN-major operands
// (bf16, boxes of 64 MN-elements x 64 tokens).  MN = false: their transposes
// Rt [d, P] and Kt [f, P], read as K-major operands (tf32).
// Warps: 0 TMA, 1 TMEM + MMA, 2-3 idle, 4-11 epilogue (setmaxnreg 56 / 224).
#pragma once
#include "gemm.cuh"

namespace ttcd {

template <class E>
struct ScanArgs {
  int d, f, Nc, Cp;
  const E* w_down;        // [d, f]
  const float* state_in;  // [B, d, f] nullable
  float* state_out;       // [B, d, f] nullable
  E* w_all;               // [B*Nc, d, f], nullable (state only)
  int tiles_m, tiles_n;
  // Decode commit from a graph: when set, the kernel acts only at the last
  // token of a chunk (*commit_pos % commit_C == commit_C - 1) and otherwise
  // returns at once (every thread of every block alike, before any set-up).
  const long long* commit_pos;
  int commit_C;
  // Walk the chunks last to first (step j reads chunk Nc-1-j and w_all entries
  // are written at the chunk they belong to): with w_down null this is the
  // backward of the exclusive prefix, w_all[i] = state_in + sum_{j>i} Delta_j.
  bool reverse;
};

constexpr int SCAN_BN = 192;
constexpr int SCAN_THREADS = 384;

template <class E, int STAGES, bool MN>
__global__ void __launch_bounds__(SCAN_THREADS, 1)
    fastweight_scan_kernel(const __grid_constant__ CUtensorMap mapR,
                           const __grid_constant__ CUtensorMap mapK, const ScanArgs<E> a,
                           const DevStatus st) {
  constexpr int BN = SCAN_BN;
  constexpr int BK = ElemTraits<E>::BK;  // tokens per k-block == MN elements per box
  constexpr int BOX_BYTES = BK * BK * static_cast<int>(sizeof(E));
  constexpr int A_BYTES = GEMM_BM * 128, B_BYTES = BN * 128;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr int KSTEP_BYTES = (32 / static_cast<int>(sizeof(E))) * 128;  // tokens per MMA x 128 B
  constexpr uint32_t IDESC = idesc_f32acc(GEMM_BM, BN, ElemTraits<E>::FMT, MN, MN);

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

  if (a.commit_pos && *a.commit_pos % a.commit_C != a.commit_C - 1) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tn = blockIdx.x % a.tiles_n;
  const int tm = (blockIdx.x / a.tiles_n) % a.tiles_m;
  const int b = blockIdx.x / (a.tiles_n * a.tiles_m);
  const int m0 = tm * GEMM_BM, n0 = tn * BN;
  const int kpc = a.Cp / BK;  // k-blocks per chunk

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&accf[s], 1); mbar_init(&acce[s], 256); }
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

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (warp == 0 && lane == 0) {
      int it = 0;
      bool ok = true;
      for (int i = 0; i < a.Nc && ok; ++i) {
        for (int kb = 0; kb < kpc; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, st, abort)) { ok = false; break; }
          uint8_t* sa = smem + s * STAGE_BYTES;
          const int ci = a.reverse ? a.Nc - 1 - i : i;
          const int y = (b * a.Nc + ci) * a.Cp + kb * BK;  // first token of the k-block
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
    } else if (warp == 1) {
      // MMA issuer: the whole warp walks the loop, one elected lane issues.
      constexpr uint32_t HI = sdesc_hi_sw128(1024);
      const uint32_t lo0 = sdesc_lo(smem_u32(smem), MN ? BOX_BYTES : 16);
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, st, abort));
      };
      int it = 0;
      bool ok = true;
      for (int i = 0; i < a.Nc && ok; ++i) {
        const int ab = i & 1;
        if (!wait(&acce[ab], ((i >> 1) & 1) ^ 1)) break;
        tc_fence_after();
        for (int kb = 0; kb < kpc; ++kb, ++it) {
          const int s = it % STAGES;
          if (!wait(&full[s], (it / STAGES) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_lo = lo0 + ((s * STAGE_BYTES) >> 4);
          const uint32_t b_lo = a_lo + (A_BYTES >> 4);
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t off = (MN ? k * KSTEP_BYTES : k * 32) >> 4;
              mma_ss_lh<E>(tmem + ab * BN, a_lo + off, HI, b_lo + off, HI, IDESC,
                           (kb | k) != 0 ? 1u : 0u);
            }
            mma_commit(&empty[s]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) mma_commit(&accf[ab]);
        __syncwarp();
      }
      if (elect_one()) mma_commit(drain);
      __syncwarp();
      volatile int no_abort = 0;
      mbar_wait(drain, 0, st, &no_abort);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
    const int q = warp & 3;              // TMEM lane quarter
    const int half = (warp - 4) >> 2;    // column half of the tile
    const int row = m0 + q * 32 + lane;
    const bool row_ok = row < a.d;
    constexpr int HC = SCAN_BN / 2;     // state columns per thread
    const int c0 = n0 + half * HC;       // first state column of this thread
    const uint32_t laddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + half * HC;
    const long long dfs = static_cast<long long>(a.d) * a.f;
    const E* wrow = a.w_down ? a.w_down + static_cast<long long>(row) * a.f : nullptr;
    auto w_index = [&](int j) {  // w_all entry of step j
      return static_cast<long long>(b) * a.Nc + (a.reverse ? a.Nc - 1 - j : j);
    };
    float S[HC];
    // S_0 = state_in (or 0); W_0 = W_down + S_0 (W_down null: 0).
#pragma unroll
    for (int cc = 0; cc < HC; cc += 32) {
      const int col = c0 + cc;
      float s32[32];
      if (row_ok && col < a.f && a.state_in) {
        load_x32(a.state_in + b * dfs + static_cast<long long>(row) * a.f + col, s32);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) s32[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) S[cc + e] = s32[e];
      if (row_ok && col < a.f && a.w_all) {
        float w[32];
        if (wrow) {
          load_x32(wrow + col, w);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) w[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] += s32[e];
        store_x32(a.w_all + w_index(0) * dfs + static_cast<long long>(row) * a.f + col, w);
      }
    }
    for (int i = 0; i < a.Nc; ++i) {
      const int ab = i & 1;
      if (!mbar_wait(&accf[ab], (i >> 1) & 1, st, abort)) break;
      tc_fence_after();
      const bool last = i + 1 == a.Nc;
#pragma unroll
      for (int cc = 0; cc < HC; cc += 32) {
        float dw[32];
        tmem_ld32f(laddr + ab * BN + cc, dw);
#pragma unroll
        for (int e = 0; e < 32; ++e) S[cc + e] += dw[e];
      }
      // The accumulator is free as soon as it has been read.
      tc_fence_before();
      mbar_arrive(&acce[ab]);
#pragma unroll
      for (int cc = 0; cc < HC; cc += 32) {
        const int col = c0 + cc;
        if (!row_ok || col >= a.f) continue;
        float v[32];
        if (!last) {
          if (!a.w_all) continue;
          if (wrow) {
            load_x32(wrow + col, v);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0.f;
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] += S[cc + e];
          store_x32(a.w_all + w_index(i + 1) * dfs + static_cast<long long>(row) * a.f + col, v);
        } else if (a.state_out) {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = S[cc + e];
          store_f32x32(a.state_out + b * dfs + static_cast<long long>(row) * a.f + col, v);
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ttcd
