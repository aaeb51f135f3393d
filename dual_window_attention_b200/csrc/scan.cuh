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
//
// PAIR = true (bf16, token-major operands): a cluster of two CTAs shares one
// 256 x 192 tile through M = 256 MMAs (tcgen05 .cta_group::2).  Each CTA loads
// its own 128 rows of R and its half of the tile's key columns (96, as two
// 64-column boxes whose last 32 columns the MMA does not read), so each
// k-block moves 32 KB into each SM instead of 40 KB.  Rank 0 waits for both
// CTAs' bytes on its own full barriers, issues the MMAs and commits them to
// both CTAs' stage and accumulator barriers; each CTA's epilogue folds its own
// 128 rows and releases the accumulator on rank 0's barrier.  Both CTAs end at
// a cluster barrier, so neither leaves while the other's MMAs or arrivals can
// still touch its shared memory.
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

// Rows of d per tile (per pair of CTAs when PAIR).
template <bool PAIR>
constexpr int scan_tile_rows() {
  return PAIR ? 2 * GEMM_BM : GEMM_BM;
}
// Key columns a CTA loads per k-block: all 192, or in a pair two boxes of 64
// for its 96.
template <bool PAIR>
constexpr int scan_b_cols() {
  return PAIR ? 128 : SCAN_BN;
}
template <class E, bool PAIR>
constexpr int scan_stage_bytes() {
  return GEMM_BM * 128 + scan_b_cols<PAIR>() * 128;
}
// bf16 W entries leave through shared memory: per epilogue warp 32 rows of 96
// columns (192 bytes) at a 208-byte pitch, so that both the row-per-thread
// writes and the row-contiguous reads are free of bank conflicts.
constexpr int SCAN_WROW = 208;
template <class E>
constexpr int scan_wstage_bytes() {
  return sizeof(E) == 2 ? 8 * 32 * SCAN_WROW : 0;
}
template <class E, int STAGES, bool PAIR>
constexpr int scan_smem_bytes() {
  return 1024 + STAGES * scan_stage_bytes<E, PAIR>() + scan_wstage_bytes<E>() + 256;
}

template <class E, int STAGES, bool MN, bool PAIR = false>
__global__ void __launch_bounds__(SCAN_THREADS, 1)
    fastweight_scan_kernel(const __grid_constant__ CUtensorMap mapR,
                           const __grid_constant__ CUtensorMap mapK, const ScanArgs<E> a,
                           const DevStatus st) {
  static_assert(!PAIR || (MN && sizeof(E) == 2), "CTA pairs take bf16 token-major operands");
  constexpr int BN = SCAN_BN;
  constexpr int BK = ElemTraits<E>::BK;  // tokens per k-block == MN elements per box
  constexpr int BOX_BYTES = BK * BK * static_cast<int>(sizeof(E));
  constexpr int B_COLS = PAIR ? BN / 2 : BN;  // key columns of the tile this CTA holds
  constexpr int A_BYTES = GEMM_BM * 128, B_BYTES = scan_b_cols<PAIR>() * 128;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static_assert(STAGE_BYTES == scan_stage_bytes<E, PAIR>(), "stage size");
  constexpr int KSTEP_BYTES = (32 / static_cast<int>(sizeof(E))) * 128;  // tokens per MMA x 128 B
  constexpr uint32_t IDESC =
      idesc_f32acc(scan_tile_rows<PAIR>(), BN, ElemTraits<E>::FMT, MN, MN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* wstage = smem + STAGES * STAGE_BYTES;  // bf16: W entry staging rows
  uint64_t* full = reinterpret_cast<uint64_t*>(wstage + scan_wstage_bytes<E>());
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (!PAIR && a.commit_pos && *a.commit_pos % a.commit_C != a.commit_C - 1) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int tile = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int tn = tile % a.tiles_n;
  const int tm = (tile / a.tiles_n) % a.tiles_m;
  const int b = tile / (a.tiles_n * a.tiles_m);
  const int m0 = tm * scan_tile_rows<PAIR>() + static_cast<int>(rank) * GEMM_BM;  // this CTA's rows
  const int n0 = tn * BN;
  const int kpc = a.Cp / BK;  // k-blocks per chunk

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&accf[s], 1); mbar_init(&acce[s], PAIR ? 512 : 256); }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_map(&mapR);
    tma_prefetch_map(&mapK);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 512);
      tmem_relinquish();
    }
    tc_fence_before();
  }
  // A pair meets here before any arrival or byte count crosses to rank 0.
  if constexpr (PAIR)
    cluster_sync_all();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (warp == 0 && lane == 0) {
      int it = 0;
      bool ok = true;
      // Pair: both CTAs count their bytes on rank 0's full barriers.
      const uint32_t full0 = PAIR ? mapa_shared(smem_u32(full), 0) : 0u;
      for (int i = 0; i < a.Nc && ok; ++i) {
        for (int kb = 0; kb < kpc; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait<PAIR>(&empty[s], ((it / STAGES) & 1) ^ 1, st, abort)) { ok = false; break; }
          uint8_t* sa = smem + s * STAGE_BYTES;
          const int ci = a.reverse ? a.Nc - 1 - i : i;
          const int y = (b * a.Nc + ci) * a.Cp + kb * BK;  // first token of the k-block
          if constexpr (PAIR) {
            const uint32_t fb = full0 + 8u * static_cast<uint32_t>(s);
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * STAGE_BYTES);
#pragma unroll
            for (int q = 0; q < GEMM_BM / BK; ++q)
              tma_load_2d_pair(sa + q * BOX_BYTES, &mapR, fb, m0 + q * BK, y);
            const int nb = n0 + static_cast<int>(rank) * B_COLS;
#pragma unroll
            for (int q = 0; q < 2; ++q)
              tma_load_2d_pair(sa + A_BYTES + q * BOX_BYTES, &mapK, fb, nb + q * BK, y);
          } else {
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
      }
      volatile int no_abort = 0;
      if constexpr (PAIR) {
        // Until rank 0's MMAs have consumed the last stages: then no load of
        // this CTA and no commit to its stage barriers is still in flight.
        for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
          mbar_wait<true>(&empty[j % STAGES], (j / STAGES) & 1, st, abort);
      } else {
        for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
          mbar_wait(&full[j % STAGES], (j / STAGES) & 1, st, &no_abort);
      }
    } else if (warp == 1 && rank == 0) {
      // MMA issuer (rank 0 of a pair): the whole warp walks the loop, one
      // elected lane issues.
      constexpr uint32_t HI = sdesc_hi_sw128(1024);
      const uint32_t lo0 = sdesc_lo(smem_u32(smem), MN ? BOX_BYTES : 16);
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait<PAIR>(bar, parity, st, abort));
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
              if constexpr (PAIR)
                mma_bf16_ss_lh_pair(tmem + ab * BN, a_lo + off, HI, b_lo + off, HI, IDESC,
                                    (kb | k) != 0 ? 1u : 0u);
              else
                mma_ss_lh<E>(tmem + ab * BN, a_lo + off, HI, b_lo + off, HI, IDESC,
                             (kb | k) != 0 ? 1u : 0u);
            }
            if constexpr (PAIR)
              mma_commit_pair_mask(&empty[s], 0x3);
            else
              mma_commit(&empty[s]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) {
          if constexpr (PAIR)
            mma_commit_pair_mask(&accf[ab], 0x3);
          else
            mma_commit(&accf[ab]);
        }
        __syncwarp();
      }
      if (elect_one()) {
        if constexpr (PAIR)
          mma_commit_pair_own(drain);
        else
          mma_commit(drain);
      }
      __syncwarp();
      volatile int no_abort = 0;
      mbar_wait(drain, 0, st, &no_abort);
      if constexpr (PAIR) {
        // The epilogues' releases of the last two accumulators (some arrive
        // from the other CTA) land before this CTA may leave.
        for (int i = a.Nc; i < a.Nc + 2; ++i)
          if (i >= 2) mbar_wait<true>(&acce[i & 1], ((i >> 1) & 1) ^ 1, st, abort);
      }
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
    // bf16: the thread's HC columns of W_down stay in registers as packed
    // pairs, so the chunk loop below issues no global loads (they would queue
    // in L2 behind the operand stream and stall the release of the next
    // accumulator), and each W entry is packed into the warp's staging rows
    // and written row-contiguously: a store instruction then covers about
    // three rows' 192-byte segments instead of 16 bytes in each of 32 rows.
    constexpr bool WREG = sizeof(E) == 2;
    uint32_t wd[WREG ? HC / 2 : 1];
    uint8_t* wst = wstage + (warp - 4) * 32 * SCAN_WROW;
    auto emit_w = [&](int j) {
      __syncwarp();  // the previous entry's reads of the staging rows are done
#pragma unroll
      for (int k = 0; k < HC / 8; ++k) {  // 16-byte chunk k: columns 8k .. 8k+7
        uint32_t pk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = 8 * k + 2 * u;
          pk[u] = pack_bf16x2(bf16lo_to_f32(wd[e / 2]) + S[e], bf16hi_to_f32(wd[e / 2]) + S[e + 1]);
        }
        *reinterpret_cast<uint4*>(wst + lane * SCAN_WROW + 16 * k) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      __syncwarp();
      E* dst = a.w_all + w_index(j) * dfs;
      const int r0 = m0 + q * 32;
#pragma unroll 1
      for (int it = 0; it < HC / 8; ++it) {  // the warp's 32 x 12 chunks, 32 at a time
        const int idx = it * 32 + lane;
        const int rr = idx / (HC / 8), kk = idx - rr * (HC / 8);
        const int grow = r0 + rr, gcol = c0 + 8 * kk;
        if (grow < a.d && gcol < a.f)
          *reinterpret_cast<uint4*>(dst + static_cast<long long>(grow) * a.f + gcol) =
              *reinterpret_cast<const uint4*>(wst + rr * SCAN_WROW + 16 * kk);
      }
    };
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
      if constexpr (WREG) {
        const bool have = wrow && row_ok && col < a.f && a.w_all;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint4 w4 = have ? reinterpret_cast<const uint4*>(wrow + col)[u]
                                : make_uint4(0u, 0u, 0u, 0u);
          wd[cc / 2 + 4 * u + 0] = w4.x;
          wd[cc / 2 + 4 * u + 1] = w4.y;
          wd[cc / 2 + 4 * u + 2] = w4.z;
          wd[cc / 2 + 4 * u + 3] = w4.w;
        }
      } else if (row_ok && col < a.f && a.w_all) {
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
    if constexpr (WREG) {
      if (a.w_all) emit_w(0);
    }
    // Pair: the accumulator is released on rank 0's barrier.
    const uint32_t acce0 = PAIR ? mapa_shared(smem_u32(acce), 0) : 0u;
    for (int i = 0; i < a.Nc; ++i) {
      const int ab = i & 1;
      if (!mbar_wait<PAIR>(&accf[ab], (i >> 1) & 1, st, abort)) break;
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
      if constexpr (PAIR)
        mbar_arrive_cluster(acce0 + 8u * static_cast<uint32_t>(ab));
      else
        mbar_arrive(&acce[ab]);
      if constexpr (WREG) {
        if (!last && a.w_all) emit_w(i + 1);
      }
#pragma unroll
      for (int cc = 0; cc < HC; cc += 32) {
        const int col = c0 + cc;
        if (!row_ok || col >= a.f) continue;
        float v[32];
        if (!last) {
          if (WREG || !a.w_all) continue;
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
  if constexpr (PAIR) {
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc_pair(tmem, 512);
    }
  } else {
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  }
}

}  // namespace ttcd
