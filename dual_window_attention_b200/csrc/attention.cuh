// Fused dual-window causal sliding-window attention (teacher window w_T and
// student window w_S over the same Q/K/V, GQA) for sm_100a.
//
// Definition: GitHub README "TTCD: Test-Time Training via Context
// Distillation", section "Fused inference kernels" (both windowed outputs in
// one pass over K/V); papernotes.org review "Learning What to Remember", 方法详解
// (long-window teacher and short-window student over a shared backbone);
// podcast cue 19 (each token sees the last w tokens).
//
// Work unit: one CTA owns the same 128-row query block of up to two query
// heads that share one KV head (GQA), so every K/V tile it loads serves both.
// Each head's rows have one TMEM accumulator O and run in two phases over key
// tiles of 128, visited from the diagonal outwards:
//   phase 1 (student): tiles 0..jS, scores masked to the student window
//            [t-w_S+1, t]; when it ends, O/l is the student output o_S;
//   phase 2 (teacher): tiles jX..n-1, scores masked to the teacher-only band
//            [t-w_T+1, t-w_S], accumulated on top of the same O, m, l; at the
//            end O/l is the teacher output o_T.
// So each Q.K^T product and each exponential serves both windows; the one
// tile that straddles the student edge (jX <= jS) is computed in both phases.
//
// Pipeline (one CTA, 384 threads):
//   warp 0      TMA producer: Q of both heads once, then K and V per visit
//   warp 1      TMEM owner and tcgen05.mma issuer (one thread), ping-pong:
//               PV_A(v), QK_A(v+1), PV_B(v), QK_B(v+1), ...
//   warps 4..7  softmax of head A (thread = query row), warps 8..11 head B
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,256+HD), O_B [384,384+HD);
// P (bf16 pairs) overwrites the first 64 columns of its S and is the A operand
// of the PV product straight from TMEM.  Because QK_A(v) is issued after
// PV_A(v-1), "S_A(v) ready" implies O_A holds every earlier tile, so the
// softmax warps may rescale or read O without a further wait.
// Rescaling is lazy: the running-max reference moves only when a row maximum
// grows by more than 2^8 (exponentials stay <= 256; exact in real arithmetic).
#pragma once
#include "gemm.cuh"

namespace ttcd {

template <class OutT>
struct AttnArgs {
  OutT* o_T;  // [B, T, Hq, HD]
  OutT* o_S;
  float* lse_T;  // [B, Hq, T], nullable
  float* lse_S;
  OutT* o_far;     // split form only: far band [t-w_T+1, t-w_S], [B, T, Hq, HD]
  float* lse_far;  // split form only: [B, Hq, T]
  int B, T, Hq, Hkv;
  int w_S, w_T;
  float scale_log2;  // softmax scale * log2(e)
  int n_qt;          // query tiles per sequence
  int pairs;         // head pairs per KV group = ceil(G / 2)
  // First query row that is computed and stored (0 for a whole sequence).  A
  // sequence shard puts the keys and values of the tokens before it in rows
  // [0, q_begin): they are visible to its queries, but no query of theirs is
  // computed.  The grid covers query tiles q_begin/128 .. n_qt-1, and outputs
  // and lse rows are indexed by t - q_begin, T - q_begin rows per sequence.
  int q_begin;
};

// Per-visit clock64 timeline of the CTA with blockIdx.x == 0 (the longest
// query tile of the first head pair), recorded by lane 0 of each head's first
// softmax warp and by the MMA issuer.  Compiled in only with
// -DTTCD_ATTN_TIMELINE=1 (`build --attn-timeline` makes a separate library);
// the library build leaves it out.  Marks per (head, visit):
//   0 S ready (its mbarrier completed)     4 P stored and published
//   1 S in registers                       5 MMA issuer: PV of this visit issued
//   2 row maximum formed                   6 MMA issuer: QK of the next visit issued
//   3 rescale check done
#ifndef TTCD_ATTN_TIMELINE
#define TTCD_ATTN_TIMELINE 0
#endif
constexpr int ATT_TL_VISITS = 128;
constexpr int ATT_TL_MARKS = 8;
#if TTCD_ATTN_TIMELINE
__device__ long long g_attn_timeline[2 * ATT_TL_VISITS * ATT_TL_MARKS];
#endif
__device__ __forceinline__ void attn_mark(bool on, int h, int v, int k) {
#if TTCD_ATTN_TIMELINE
  if (on && v < ATT_TL_VISITS) {
    long long t;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(t)::"memory");
    g_attn_timeline[(h * ATT_TL_VISITS + v) * ATT_TL_MARKS + k] = t;
  }
#else
  (void)on; (void)h; (void)v; (void)k;
#endif
}

constexpr int ATT_BM = 128;
constexpr int ATT_BN = 128;
constexpr int ATT_KS = 2;  // K stages
constexpr int ATT_VS = 2;  // V stages
constexpr int ATT_THREADS = 384;
constexpr float ATT_RESCALE_THRESHOLD = 8.0f;  // log2 units

template <int HD>
struct AttnCfg {
  static constexpr int PANELS = HD > 64 ? 2 : 1;  // 64-column (128-byte) panels per tile
  static constexpr int TILE_BYTES = PANELS * ATT_BM * 128;
  static constexpr int QA_OFF = 0;
  static constexpr int QB_OFF = TILE_BYTES;
  static constexpr int K_OFF = 2 * TILE_BYTES;
  static constexpr int V_OFF = K_OFF + ATT_KS * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + ATT_VS * TILE_BYTES;
  // at least 120 KB so that a single CTA (which takes all 512 TMEM columns)
  // is resident per SM
  static constexpr int SMEM_RAW = 1024 + BAR_OFF + 512;
  static constexpr int SMEM = SMEM_RAW > 122880 ? SMEM_RAW : 122880;
  static constexpr uint32_t LOAD_BYTES = PANELS * ATT_BM * 128;  // box is 64 columns even at HD 32
};

// Visit schedule of one 128-row query tile; identical for every role.
struct Visits {
  int n_tiles;  // key tiles that touch the teacher window
  int jS;       // last student tile
  int jX;       // first teacher-only tile
  int nv;       // visits
  int vX;       // first phase-2 visit (== nv when there is no phase 2)
  __device__ Visits(int qt, int w_S, int w_T) {
    n_tiles = min(qt, (w_T + ATT_BN - 2) / ATT_BN) + 1;
    jS = min(n_tiles - 1, (w_S + ATT_BN - 2) / ATT_BN);
    jX = w_S / ATT_BN;
    const bool phase2 = w_T > w_S && jX <= n_tiles - 1;
    vX = jS + 1;
    nv = vX + (phase2 ? n_tiles - jX : 0);
  }
  __device__ int tile(int v) const { return v < vX ? v : jX + (v - vX); }
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x on the FMA pipe for a pair: round-to-nearest range reduction with the
// 1.5 * 2^23 shifter, then 2^f for f in [-0.5, 0.5] by a cubic whose
// coefficients were fitted to 2^f (relative error weighted least squares on
// Chebyshev nodes, Lawson reweighting; max relative error 1.0e-4), and the
// integer part added to the exponent field.  Inputs are clamped at -126.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
  constexpr float SHIFT = 12582912.0f;  // 1.5 * 2^23
  constexpr float C1 = 0.6932829022407532f, C2 = 0.24221095442771912f,
                  C3 = 0.05500892922282219f;
  float x0, x1;
  f2unpack(x, x0, x1);
  x0 = fmaxf(x0, -126.0f);
  x1 = fmaxf(x1, -126.0f);
  const uint64_t xc = f2pack(x0, x1);
  const uint64_t t = add2(xc, f2pack(SHIFT, SHIFT));
  const uint64_t n = add2(t, f2pack(-SHIFT, -SHIFT));
  const uint64_t fr = fma2(n, f2pack(-1.0f, -1.0f), xc);
  uint64_t p = fma2(fr, f2pack(C3, C3), f2pack(C2, C2));
  p = fma2(p, fr, f2pack(C1, C1));
  p = fma2(p, fr, f2pack(1.0f, 1.0f));
  float p0, p1, t0, t1;
  f2unpack(p, p0, p1);
  f2unpack(t, t0, t1);
  const float r0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  const float r1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
  return f2pack(r0, r1);
}

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[N]) {
#pragma unroll
  for (int c = 0; c < N / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + 32 * c, r);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[32 * c + i] = __uint_as_float(r[i]);
  }
  tmem_ld_wait();
}

template <int HD>
__device__ __forceinline__ void tmem_scale_row(uint32_t taddr, float alpha) {
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

// Normalise this thread's O row by 1/l and store it to dst.
template <int HD, class OutT>
__device__ __forceinline__ void tmem_store_row(uint32_t taddr, float inv_l, OutT* dst, bool ok) {
#pragma unroll
  for (int c = 0; c < HD; c += 32) {
    float v[32];
    tmem_ld32f(taddr + c, v);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= inv_l;
    if (ok) store_x32(dst + c, v);
  }
}

// SPLIT = false: the fused form (o_T, o_S).  SPLIT = true: the LSE-combination
// form of the README's lse_dual_attn: the accumulator restarts at the student
// edge, so phase 2 yields the far band alone (o_far, lse_far) and o_T comes from
// merging it with the student window through the log-sum-exp (lse_merge_kernel).
template <int HD, class OutT, bool SPLIT>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    dual_window_attn_kernel(const __grid_constant__ CUtensorMap mapQ,
                            const __grid_constant__ CUtensorMap mapK,
                            const __grid_constant__ CUtensorMap mapV, const AttnArgs<OutT> a,
                            const DevStatus st) {
  using Cfg = AttnCfg<HD>;
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(ATT_BM, ATT_BN, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(ATT_BM, HD, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BAR_OFF);
  uint64_t* q_full = bars;                  // 1
  uint64_t* k_full = bars + 1;              // KS
  uint64_t* k_empty = k_full + ATT_KS;      // KS
  uint64_t* v_full = k_empty + ATT_KS;      // VS
  uint64_t* v_empty = v_full + ATT_VS;      // VS
  uint64_t* s_full = v_empty + ATT_VS;      // 2 (per head)
  uint64_t* p_full = s_full + 2;            // 2 (per head, 128 arrivals)
  uint64_t* o_done = p_full + 2;            // 2 (per head)
  uint64_t* drain = o_done + 2;             // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work item: longest (latest) query tiles first.
  const int G = a.Hq / a.Hkv;
  const int per_qt = a.B * a.Hkv * a.pairs;
  const int qt = a.n_qt - 1 - static_cast<int>(blockIdx.x) / per_qt;
  int rem = static_cast<int>(blockIdx.x) % per_qt;
  const int pair = rem % a.pairs;
  rem /= a.pairs;
  const int g = rem % a.Hkv;
  const int b = rem / a.Hkv;
  const int hA = g * G + 2 * pair;
  const bool hasB = 2 * pair + 1 < G;
  const int hB = hasB ? hA + 1 : hA;
  const int q0 = qt * ATT_BM;
  const Visits vis(qt, a.w_S, a.w_T);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ATT_KS; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < ATT_VS; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&o_done[s], 1);
    }
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
  // Register split: the launch gives 384 x 168 = 64512 registers; the control
  // warpgroup (warps 0-3) keeps 128 x 56, the two softmax warpgroups take
  // 256 x 224, which adds up to the same 64512.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------- TMA producer
      const int row_base = b * a.T;
      int issued_k = 0, issued_v = 0;
      mbar_arrive_expect_tx(q_full, (hasB ? 2 : 1) * Cfg::LOAD_BYTES);
#pragma unroll
      for (int p = 0; p < Cfg::PANELS; ++p) {
        tma_load_2d(smem + Cfg::QA_OFF + p * ATT_BM * 128, &mapQ, q_full, hA * HD + 64 * p,
                    row_base + q0);
        if (hasB)
          tma_load_2d(smem + Cfg::QB_OFF + p * ATT_BM * 128, &mapQ, q_full, hB * HD + 64 * p,
                      row_base + q0);
      }
      for (int v = 0; v < vis.nv; ++v) {
        const int row = row_base + q0 - ATT_BN * vis.tile(v);
        const int ks = v % ATT_KS, vs = v % ATT_VS;
        if (!mbar_wait(&k_empty[ks], ((v / ATT_KS) & 1) ^ 1, st, abort)) break;
        mbar_arrive_expect_tx(&k_full[ks], Cfg::LOAD_BYTES);
#pragma unroll
        for (int p = 0; p < Cfg::PANELS; ++p)
          tma_load_2d(smem + Cfg::K_OFF + ks * Cfg::TILE_BYTES + p * ATT_BN * 128, &mapK,
                      &k_full[ks], g * HD + 64 * p, row);
        ++issued_k;
        if (!mbar_wait(&v_empty[vs], ((v / ATT_VS) & 1) ^ 1, st, abort)) break;
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
    } else if (warp == 1) {
      // ------------------------------------------------------------- MMA issuer
      // The whole warp walks the loop and one elected lane issues: the MMA
      // queue holds only a few instructions, so the issuer must not spend its
      // time rebuilding operand words between groups.  Descriptor low words
      // (start address, LBO) advance by (offset >> 4); the high words are
      // constants.
      constexpr uint32_t HI = sdesc_hi_sw128(1024);
      const uint32_t q_lo[2] = {sdesc_lo(smem_u32(smem + Cfg::QA_OFF), 16),
                                sdesc_lo(smem_u32(smem + Cfg::QB_OFF), 16)};
      const uint32_t k_lo0 = sdesc_lo(smem_u32(smem + Cfg::K_OFF), 16);
      const uint32_t v_lo0 = sdesc_lo(smem_u32(smem + Cfg::V_OFF), ATT_BM * 128);
      const int nh = hasB ? 2 : 1;
      auto issue_qk = [&](int h, int v) {
        const uint32_t k_lo = k_lo0 + (((v % ATT_KS) * Cfg::TILE_BYTES) >> 4);
        const uint32_t qh = h ? q_lo[1] : q_lo[0];
        const uint32_t d = tmem + h * 128;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * (ATT_BM * 128) + (kk & 3) * 32) >> 4;
            mma_bf16_ss_lh(d, qh + off, HI, k_lo + off, HI, IDESC_QK, kk > 0 ? 1u : 0u);
          }
          mma_commit(&s_full[h]);
        }
        __syncwarp();
      };
      auto issue_pv = [&](int h, int v) {
        const uint32_t v_lo = v_lo0 + (((v % ATT_VS) * Cfg::TILE_BYTES) >> 4);
        const uint32_t d = tmem + 256 + h * 128, pa = tmem + h * 128;
        // the first visit, and in the split form the first far-band visit, start O afresh
        const uint32_t acc0 = (v > 0 && !(SPLIT && v == vis.vX)) ? 1u : 0u;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < ATT_BN / 16; ++kk)
            mma_bf16_ts_lh(d, pa + kk * 8, v_lo + ((kk * 2048) >> 4), HI, IDESC_PV,
                           kk > 0 ? 1u : acc0);
          mma_commit(&o_done[h]);
        }
        __syncwarp();
      };
      // every lane waits; a wait that gave up in any lane ends the loop in all
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, st, abort));
      };
      bool ok = wait(q_full, 0) && wait(&k_full[0], 0);
      if (ok) {
        tc_fence_after();
        for (int h = 0; h < nh; ++h) issue_qk(h, 0);
        if (elect_one()) mma_commit(&k_empty[0]);
        __syncwarp();
      }
      for (int v = 0; v < vis.nv && ok; ++v) {
        const bool more = v + 1 < vis.nv;
        if (!wait(&v_full[v % ATT_VS], (v / ATT_VS) & 1)) { ok = false; break; }
        if (more && !wait(&k_full[(v + 1) % ATT_KS], ((v + 1) / ATT_KS) & 1)) {
          ok = false;
          break;
        }
        const bool tl = TTCD_ATTN_TIMELINE && blockIdx.x == 0 && lane == 0;
        for (int h = 0; h < nh; ++h) {
          if (!wait(&p_full[h], v & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv(h, v);
          attn_mark(tl, h, v, 5);
          if (more) issue_qk(h, v + 1);
          attn_mark(tl, h, v, 6);
        }
        if (!ok) break;
        if (elect_one()) {
          if (more) mma_commit(&k_empty[(v + 1) % ATT_KS]);
          mma_commit(&v_empty[v % ATT_VS]);
        }
        __syncwarp();
      }
      if (elect_one()) mma_commit(drain);
      __syncwarp();
      volatile int no_abort = 0;
      mbar_wait(drain, 0, st, &no_abort);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
    // --------------------------------------------------------------- softmax rows
    const int h_local = (warp - 4) >> 2;  // 0: head A, 1: head B
    const bool active = h_local == 0 || hasB;
    const int head = h_local == 0 ? hA : hB;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int t = q0 + r;  // query position inside the sequence
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + h_local * 128;
    const uint32_t o_addr = tmem + lane_off + 256 + h_local * 128;
    const bool row_ok = t < a.T && t >= a.q_begin;
    const int T_out = a.T - a.q_begin;
    const long long orow = (static_cast<long long>(b) * T_out + (t - a.q_begin)) * a.Hq + head;
    const long long li = (static_cast<long long>(b) * a.Hq + head) * T_out + (t - a.q_begin);
    const float sl2 = a.scale_log2;
    // m_ref = -inf: nothing visible yet (the first tile, or the far band of the
    // split form before its first visible key); O is zero for such a row.
    float m_ref = -INFINITY, l = 0.f;
    bool ok = active;
    const bool tl = TTCD_ATTN_TIMELINE && blockIdx.x == 0 && quarter == 0 && lane == 0;
    for (int v = 0; v < vis.nv && ok; ++v) {
      const int j = vis.tile(v);
      const int k0 = q0 - ATT_BN * j;
      const bool ph2 = v >= vis.vX;
      if (!mbar_wait(&s_full[h_local], v & 1, st, abort)) { ok = false; break; }
      attn_mark(tl, h_local, v, 0);
      tc_fence_after();
      if (v == vis.vX) {
        // end of the student phase: O / l is o_S (PV of every earlier tile has landed)
        tmem_store_row<HD, OutT>(o_addr, 1.f / l, a.o_S + orow * HD, row_ok);
        if (row_ok && a.lse_S) a.lse_S[li] = (m_ref + __log2f(l)) * 0.6931471805599453f;
        if (SPLIT) {
          m_ref = -INFINITY;
          l = 0.f;
        }
      }
      float s[128];
      tmem_ld_cols<128>(s_addr, s);
      attn_mark(tl, h_local, v, 1);
      // visible key columns [lo, hi] of this row in this tile
      const int lo = ph2 ? t - a.w_T + 1 - k0 : t - a.w_S + 1 - k0;
      const int hi = ph2 ? t - a.w_S - k0 : t - k0;
      const bool unmasked = ph2 ? (k0 >= q0 + ATT_BM - a.w_T && k0 + ATT_BN - 1 <= q0 - a.w_S)
                                : (j >= 1 && k0 >= q0 + ATT_BM - a.w_S);
      if (!unmasked) {
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = (c >= lo && c <= hi) ? s[c] : -INFINITY;
      }
      // row maximum as four independent chains (short dependency latency)
      float mx4[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float m = fmax3(s[32 * q], s[32 * q + 1], s[32 * q + 2]);
#pragma unroll
        for (int c = 3; c < 31; c += 2) m = fmax3(m, s[32 * q + c], s[32 * q + c + 1]);
        mx4[q] = fmaxf(m, s[32 * q + 31]);
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      attn_mark(tl, h_local, v, 2);
      const float m_tile = mx * sl2;
      const bool fresh = m_ref == -INFINITY;
      const bool grow = !fresh && m_tile > m_ref + ATT_RESCALE_THRESHOLD;
      if (__any_sync(0xffffffffu, grow)) {
        const float m_new = grow ? m_tile : m_ref;
        const float al = grow ? ex2_approx(m_ref - m_new) : 1.f;
        tmem_scale_row<HD>(o_addr, al);
        l *= al;
        m_ref = m_new;
      }
      if (fresh) m_ref = m_tile;  // may stay -inf: a row with no visible key in this tile
      attn_mark(tl, h_local, v, 3);
      // exponentials, row sum, bf16 pack (a row still at -inf has only masked scores)
      const float nm = m_ref == -INFINITY ? 0.f : -m_ref;
      const uint64_t sc2 = f2pack(sl2, sl2);
      const uint64_t nm2 = f2pack(nm, nm);
      uint64_t acc4[4] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f), f2pack(0.f, 0.f),
                          f2pack(0.f, 0.f)};
      uint32_t P[64];
      if (unmasked) {
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          uint64_t x = fma2(f2pack(s[c], s[c + 1]), sc2, nm2);
          uint64_t e;
          if (((c >> 1) & 3) == 3) {  // one pair in four on the FMA pipe
            e = exp2_poly2(x);
          } else {
            float x0, x1;
            f2unpack(x, x0, x1);
            e = f2pack(ex2_approx(x0), ex2_approx(x1));
          }
          acc4[(c >> 1) & 3] = add2(acc4[(c >> 1) & 3], e);
          float e0, e1;
          f2unpack(e, e0, e1);
          P[c >> 1] = pack_bf16x2(e0, e1);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          uint64_t x = fma2(f2pack(s[c], s[c + 1]), sc2, nm2);
          float x0, x1;
          f2unpack(x, x0, x1);
          const uint64_t e = f2pack(ex2_approx(x0), ex2_approx(x1));
          acc4[(c >> 1) & 3] = add2(acc4[(c >> 1) & 3], e);
          float e0, e1;
          f2unpack(e, e0, e1);
          P[c >> 1] = pack_bf16x2(e0, e1);
        }
      }
      const uint64_t acc = add2(add2(acc4[0], acc4[1]), add2(acc4[2], acc4[3]));
      float a0, a1;
      f2unpack(acc, a0, a1);
      l += a0 + a1;
      tmem_st32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&P[0]));
      tmem_st32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&P[32]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[h_local]);
      attn_mark(tl, h_local, v, 4);
    }
    // ------------------------------------------------------------------ epilogue
    if (ok && mbar_wait(&o_done[h_local], (vis.nv - 1) & 1, st, abort)) {
      tc_fence_after();
      // l = 0 only for an empty far band (split form): o = 0, lse = -inf
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const float lse = l > 0.f ? (m_ref + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      const bool no_band = vis.vX == vis.nv;  // no teacher-only keys in this tile
      if (!SPLIT) {
        tmem_store_row<HD, OutT>(o_addr, inv_l, a.o_T + orow * HD, row_ok);
        if (row_ok && a.lse_T) a.lse_T[li] = lse;
      }
      if (no_band) {  // the accumulator holds the student window: o_T == o_S
        tmem_store_row<HD, OutT>(o_addr, inv_l, a.o_S + orow * HD, row_ok);
        if (row_ok && a.lse_S) a.lse_S[li] = lse;
      }
      if (SPLIT) {
        tmem_store_row<HD, OutT>(o_addr, no_band ? 0.f : inv_l, a.o_far + orow * HD, row_ok);
        if (row_ok) a.lse_far[li] = no_band ? -INFINITY : lse;
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// o_T = (o_S e^{lse_S} + o_far e^{lse_far}) / (e^{lse_S} + e^{lse_far}) and
// lse_T = logaddexp(lse_S, lse_far): the exact merge of two partial softmax
// attentions over disjoint key sets (GitHub README "TTCD", "Fused inference
// kernels", lse_dual_attn).  One thread per 8 output elements of one row
// (b, t, h); lse [B, Hq, T], o [B, T, Hq, HD].
template <int HD, class OutT>
__global__ void lse_merge_kernel(const OutT* __restrict__ o_S, const float* __restrict__ lse_S,
                                 const OutT* __restrict__ o_far,
                                 const float* __restrict__ lse_far, OutT* __restrict__ o_T,
                                 float* __restrict__ lse_T, int T, int Hq, long long rows) {
  constexpr int PER = 8, TPR = HD / PER;  // elements per thread, threads per row
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = idx / TPR;  // (b * T + t) * Hq + h
  if (row >= rows) return;
  const int c = static_cast<int>(idx % TPR) * PER;
  const int h = static_cast<int>(row % Hq);
  const long long bt = row / Hq;
  const int t = static_cast<int>(bt % T);
  const long long li = (bt / T * Hq + h) * T + t;
  const float ls = lse_S[li], lf = lse_far[li];
  const float m = fmaxf(ls, lf);  // lse_S is finite: the diagonal key is in every window
  const float ws = __expf(ls - m), wf = lf == -INFINITY ? 0.f : __expf(lf - m);
  const float inv = 1.f / (ws + wf);
  float x[PER], y[PER];
  ld8f(o_S + row * HD + c, x);
  ld8f(o_far + row * HD + c, y);
#pragma unroll
  for (int i = 0; i < PER; ++i) x[i] = (x[i] * ws + y[i] * wf) * inv;
  st8f(o_T + row * HD + c, x);
  if (c == 0 && lse_T) lse_T[li] = m + __logf(ws + wf);
}

}  // namespace ttcd
