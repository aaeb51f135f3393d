// Fused dual-window causal sliding-window attention (teacher window w_T and
// student window w_S over the same Q/K/V, GQA) for sm_100a.
//
// Definition: GitHub README "TTCD: Test-Time Training via Context
// Distillation", section "Fused inference kernels" (both windowed outputs in
// one pass over K/V); papernotes.org review "Learning What to Remember", 方法详解
// (long-window teacher and short-window student over a shared backbone);
// podcast cue 19 (each token sees the last w tokens).
//
// One CTA owns a 128-row query tile of one (sequence, query head).  K/V tiles
// of 128 keys are visited from the diagonal outwards ("near to far").  Every
// Q.K^T tile is computed once; its exponentials are shared by both windows:
//   - while the tile touches some row's student window, the student part of P
//     accumulates into O_S (TMEM) and the teacher-only part into O_X;
//   - afterwards only O_X accumulates.
// Each accumulator keeps the running-max reference it was last rescaled to;
// at the end  O_T = (O_S a + O_X) / (l_S a + l_X),  a = 2^(m_S - m_X).
// Rescaling is lazy: the reference only moves when a row maximum grows by more
// than 2^8, which keeps every exponential <= 256 and is exact in real
// arithmetic (the same reference divides out in l).
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2..5 softmax (thread = query row) and epilogue.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O_S [256,256+HD), O_X [384,384+HD).
// P of tile j overwrites S_{j%2}: P_S in columns [0,64), P_X in [64,128) as bf16 pairs.
#pragma once
#include "gemm.cuh"

namespace ttcd {

struct AttnArgs {
  __nv_bfloat16* o_T;  // [B, T, Hq, HD]
  __nv_bfloat16* o_S;
  float* lse_T;  // [B, Hq, T], nullable
  float* lse_S;
  int B, T, Hq, Hkv;
  int w_S, w_T;
  float scale_log2;  // softmax scale * log2(e)
  int n_qt;          // query tiles per sequence
};

constexpr int ATT_BM = 128;
constexpr int ATT_BN = 128;
constexpr int ATT_KS = 3;  // K stages
constexpr int ATT_VS = 2;  // V stages
constexpr int ATT_THREADS = 192;
constexpr float ATT_RESCALE_THRESHOLD = 8.0f;  // log2 units

template <int HD>
struct AttnCfg {
  static constexpr int PANELS = HD > 64 ? 2 : 1;  // 64-column (128-byte) panels per tile
  static constexpr int TILE_BYTES = PANELS * ATT_BM * 128;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE_BYTES;
  static constexpr int V_OFF = K_OFF + ATT_KS * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + ATT_VS * TILE_BYTES;
  // at least 120 KB so that a single CTA (which takes all 512 TMEM columns)
  // is resident per SM
  static constexpr int SMEM = (1024 + BAR_OFF + 512) > 122880 ? (1024 + BAR_OFF + 512) : 122880;
  // bytes each TMA tile load delivers (box is 64 columns even when HD = 32)
  static constexpr uint32_t LOAD_BYTES = PANELS * ATT_BM * 128;
};

// Key-window geometry of a (query tile, key tile) pair.
struct TileGeom {
  int q0, k0;
  __device__ bool has_S(int w_S) const { return k0 + ATT_BN - 1 >= q0 - w_S + 1; }
  __device__ bool has_X(int w_S, int w_T) const {
    return k0 <= q0 + ATT_BM - 1 - w_S && k0 + ATT_BN - 1 >= q0 - w_T + 1;
  }
  // every (row, key) of the tile lies in the window w
  __device__ bool full(int w) const { return k0 + ATT_BN - 1 <= q0 && k0 >= q0 + ATT_BM - w; }
};

__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float (&v)[128]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + 32 * c, r);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[32 * c + i] = __uint_as_float(r[i]);
  }
  tmem_ld_wait();
}

template <int HD>
__device__ __forceinline__ void tmem_scale_rows(uint32_t taddr, float alpha) {
#pragma unroll
  for (int c = 0; c < HD; c += 32) {
    uint32_t r[32];
    tmem_ld32(taddr + c, r);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
    tmem_st32(taddr + c, r);
  }
  tmem_st_wait();
}

template <int HD>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    dual_window_attn_kernel(const __grid_constant__ CUtensorMap mapQ,
                            const __grid_constant__ CUtensorMap mapK,
                            const __grid_constant__ CUtensorMap mapV, const AttnArgs a,
                            const DevStatus st) {
  using Cfg = AttnCfg<HD>;
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(ATT_BM, ATT_BN, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(ATT_BM, HD, false, true);
  constexpr uint32_t COL_O_S = 256, COL_O_X = 384;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + ATT_KS;
  uint64_t* v_full = k_empty + ATT_KS;
  uint64_t* v_empty = v_full + ATT_VS;
  uint64_t* s_full = v_empty + ATT_VS;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_done = pv_done + 1;
  uint64_t* drain = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work item: longest (latest) query tiles first; heads of a GQA group adjacent.
  const int per_tile = a.B * a.Hq;
  const int qt = a.n_qt - 1 - static_cast<int>(blockIdx.x) / per_tile;
  const int bh = static_cast<int>(blockIdx.x) % per_tile;
  const int b = bh / a.Hq;
  const int h = bh % a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const int q0 = qt * ATT_BM;
  const int n_tiles = min(qt, (a.w_T + ATT_BN - 2) / ATT_BN) + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ATT_KS; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < ATT_VS; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&s_full[s], 1); mbar_init(&p_full[s], 128); }
    mbar_init(pv_done, 1);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_map(&mapQ);
    tma_prefetch_map(&mapK);
    tma_prefetch_map(&mapV);
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
      // ------------------------------------------------------------- TMA producer
      const int row_base = b * a.T;
      int issued_k = 0, issued_v = 0;
      mbar_arrive_expect_tx(q_full, Cfg::LOAD_BYTES);
#pragma unroll
      for (int p = 0; p < Cfg::PANELS; ++p)
        tma_load_2d(smem + Cfg::Q_OFF + p * ATT_BM * 128, &mapQ, q_full, h * HD + 64 * p,
                    row_base + q0);
      for (int j = 0; j < n_tiles; ++j) {
        const int row = row_base + q0 - ATT_BN * j;
        const int ks = j % ATT_KS, vs = j % ATT_VS;
        if (!mbar_wait(&k_empty[ks], ((j / ATT_KS) & 1) ^ 1, st, abort)) break;
        mbar_arrive_expect_tx(&k_full[ks], Cfg::LOAD_BYTES);
#pragma unroll
        for (int p = 0; p < Cfg::PANELS; ++p)
          tma_load_2d(smem + Cfg::K_OFF + ks * Cfg::TILE_BYTES + p * ATT_BN * 128, &mapK,
                      &k_full[ks], g * HD + 64 * p, row);
        ++issued_k;
        if (!mbar_wait(&v_empty[vs], ((j / ATT_VS) & 1) ^ 1, st, abort)) break;
        mbar_arrive_expect_tx(&v_full[vs], Cfg::LOAD_BYTES);
#pragma unroll
        for (int p = 0; p < Cfg::PANELS; ++p)
          tma_load_2d(smem + Cfg::V_OFF + vs * Cfg::TILE_BYTES + p * ATT_BN * 128, &mapV,
                      &v_full[vs], g * HD + 64 * p, row);
        ++issued_v;
      }
      volatile int no_abort = 0;
      mbar_wait(q_full, 0, st, &no_abort);
      for (int j = max(0, issued_k - ATT_KS); j < issued_k; ++j)
        mbar_wait(&k_full[j % ATT_KS], (j / ATT_KS) & 1, st, &no_abort);
      for (int j = max(0, issued_v - ATT_VS); j < issued_v; ++j)
        mbar_wait(&v_full[j % ATT_VS], (j / ATT_VS) & 1, st, &no_abort);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------- MMA issuer
      bool ok = mbar_wait(q_full, 0, st, abort);
      const uint32_t sq = smem_u32(smem + Cfg::Q_OFF);
      bool x_started = false;
      auto issue_pv = [&](int jj) -> bool {
        if (!mbar_wait(&p_full[jj & 1], (jj >> 1) & 1, st, abort)) return false;
        if (!mbar_wait(&v_full[jj % ATT_VS], (jj / ATT_VS) & 1, st, abort)) return false;
        tc_fence_after();
        const TileGeom tg{q0, q0 - ATT_BN * jj};
        const uint32_t sv = smem_u32(smem + Cfg::V_OFF + (jj % ATT_VS) * Cfg::TILE_BYTES);
        const uint32_t p_col = tmem + (jj & 1) * 128;
        if (tg.has_S(a.w_S)) {
#pragma unroll
          for (int kk = 0; kk < ATT_BN / 16; ++kk)
            mma_bf16_ts(tmem + COL_O_S, p_col + kk * 8, sdesc_sw128(sv + kk * 2048, ATT_BM * 128, 1024),
                        IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        if (tg.has_X(a.w_S, a.w_T)) {
#pragma unroll
          for (int kk = 0; kk < ATT_BN / 16; ++kk)
            mma_bf16_ts(tmem + COL_O_X, p_col + 64 + kk * 8,
                        sdesc_sw128(sv + kk * 2048, ATT_BM * 128, 1024), IDESC_PV,
                        (x_started || kk > 0) ? 1u : 0u);
          x_started = true;
        }
        mma_commit(&v_empty[jj % ATT_VS]);
        mma_commit(pv_done);
        return true;
      };
      for (int j = 0; j < n_tiles && ok; ++j) {
        const int ks = j % ATT_KS;
        if (!mbar_wait(&k_full[ks], (j / ATT_KS) & 1, st, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sk = smem_u32(smem + Cfg::K_OFF + ks * Cfg::TILE_BYTES);
        const uint32_t s_col = tmem + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (ATT_BM * 128) + (kk & 3) * 32;
          mma_bf16_ss(s_col, sdesc_sw128(sq + off, 16, 1024), sdesc_sw128(sk + off, 16, 1024),
                      IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[j & 1]);
        mma_commit(&k_empty[ks]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && issue_pv(n_tiles - 1)) mma_commit(o_done);
      mma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, st, &no_abort);
    }
  } else {
    // --------------------------------------------------------------- softmax rows
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int t = q0 + r;  // query position inside the sequence
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    float m_ref = 0.f, mS = 0.f, mX = 0.f, lS = 0.f, lX = 0.f;
    bool x_started = false;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const TileGeom tg{q0, q0 - ATT_BN * j};
      const bool hs = tg.has_S(a.w_S);
      const bool hx = tg.has_X(a.w_S, a.w_T);
      if (!mbar_wait(&s_full[j & 1], (j >> 1) & 1, st, abort)) { ok = false; break; }
      tc_fence_after();
      float s[128];
      tmem_ld128(lane_addr + (j & 1) * 128, s);
      // Masks: teacher-valid keys, and which of those are student keys.
      const bool maskT = !tg.full(a.w_T);
      const bool all_student = hs && !hx && tg.full(a.w_S);
      float tile_max = -INFINITY;
      uint32_t in_S_bits[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const int key = tg.k0 + c;
        const bool vT = !maskT || (key <= t && key >= t - a.w_T + 1);
        const bool vS = key <= t && key >= t - a.w_S + 1;
        if (vS) in_S_bits[c >> 5] |= 1u << (c & 31);
        s[c] = vT ? s[c] * a.scale_log2 : -INFINITY;
        tile_max = fmaxf(tile_max, s[c]);
      }
      if (j == 0) {
        m_ref = tile_max;
        mS = m_ref;
      } else {
        const bool grow = tile_max > m_ref + ATT_RESCALE_THRESHOLD;
        if (__any_sync(0xffffffffu, grow)) {
          const float m_new = grow ? tile_max : m_ref;
          // O may only be touched once the previous PV product has landed.
          if (!mbar_wait(pv_done, (j - 1) & 1, st, abort)) { ok = false; break; }
          tc_fence_after();
          if (hs) {
            const float al = ex2_approx(mS - m_new);
            tmem_scale_rows<HD>(lane_addr + COL_O_S, al);
            lS *= al;
            mS = m_new;
          }
          if (hx && x_started) {
            const float al = ex2_approx(mX - m_new);
            tmem_scale_rows<HD>(lane_addr + COL_O_X, al);
            lX *= al;
            mX = m_new;
          }
          m_ref = m_new;
        }
      }
      if (hx && !x_started) { mX = m_ref; x_started = true; }
      // Exponentials once; split into the student and teacher-only parts.
      uint32_t pS[64], pX[64];
      float sumS = 0.f, sumX = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float e0 = ex2_approx(s[c] - m_ref);
        const float e1 = ex2_approx(s[c + 1] - m_ref);
        const bool s0 = all_student || ((in_S_bits[c >> 5] >> (c & 31)) & 1u);
        const bool s1 = all_student || ((in_S_bits[(c + 1) >> 5] >> ((c + 1) & 31)) & 1u);
        const float a0 = s0 ? e0 : 0.f, a1 = s1 ? e1 : 0.f;
        const float b0 = s0 ? 0.f : e0, b1 = s1 ? 0.f : e1;
        sumS += a0 + a1;
        sumX += b0 + b1;
        pS[c >> 1] = pack_bf16x2(a0, a1);
        pX[c >> 1] = pack_bf16x2(b0, b1);
      }
      const uint32_t p_addr = lane_addr + (j & 1) * 128;
      if (hs) {
        lS += sumS;
        tmem_st32(p_addr, *reinterpret_cast<uint32_t(*)[32]>(&pS[0]));
        tmem_st32(p_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&pS[32]));
      }
      if (hx) {
        lX += sumX;
        tmem_st32(p_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&pX[0]));
        tmem_st32(p_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&pX[32]));
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[j & 1]);
    }
    // ------------------------------------------------------------------ epilogue
    if (ok && mbar_wait(o_done, 0, st, abort)) {
      tc_fence_after();
      const bool row_ok = t < a.T;
      const float inv_S = 1.f / lS;
      const float sc = x_started ? ex2_approx(mS - mX) : 0.f;
      const float lT = x_started ? lS * sc + lX : lS;
      const float inv_T = 1.f / lT;
      const long long orow = (static_cast<long long>(b) * a.T + t) * a.Hq + h;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        float os[32], ox[32];
        tmem_ld32f(lane_addr + COL_O_S + c, os);
        if (x_started) {
          tmem_ld32f(lane_addr + COL_O_X + c, ox);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ox[i] = 0.f;
        }
        float vs[32], vt[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          vs[i] = os[i] * inv_S;
          vt[i] = x_started ? (os[i] * sc + ox[i]) * inv_T : vs[i];
        }
        if (row_ok) {
          store_bf16x32(a.o_S + orow * HD + c, vs);
          store_bf16x32(a.o_T + orow * HD + c, vt);
        }
      }
      if (row_ok) {
        const float ln2 = 0.6931471805599453f;
        const long long li = (static_cast<long long>(b) * a.Hq + h) * a.T + t;
        if (a.lse_S) a.lse_S[li] = (mS + __log2f(lS)) * ln2;
        if (a.lse_T) a.lse_T[li] = ((x_started ? mX : mS) + __log2f(lT)) * ln2;
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
