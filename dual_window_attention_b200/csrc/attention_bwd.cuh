// Backward of the fused dual-window causal attention (teacher window w_T and
// student window w_S over the same Q/K/V, GQA) for sm_100a.
//
// papernotes.org review "Learning What to Remember", 方法详解 and 局限与展望
// (training the block costs about 1.1-1.2x a plain transformer, so both
// attention windows are differentiated); definition of each window's softmax
// attention: podcast cue 19 (each token sees the last w tokens).  For one
// window with P = softmax(scale Q K^T) over the visible keys and O = P V:
//   dV = P^T dO,  dP = dO V^T,  dS = P (dP - delta) scale,  delta_t = dO_t . O_t,
//   dK = dS^T Q,  dQ = dS K;
// the two windows add.  P is rebuilt from the forward's log-sum-exp.
//
// Work unit: one CTA owns one 128-key tile of one KV head and walks every
// (query head of the group, query tile, window) visit that can see those keys:
// per head, the teacher passes over query tiles kt .. kt + ceil((w_T-1)/128)
// and then the student passes over kt .. kt + ceil((w_S-1)/128).  Scores are
// formed transposed, S^T = K Q^T, so that keys are TMEM lanes: P^T and dS^T are
// then the A operands of dV += P^T dO and dK += dS^T Q, which accumulate in TMEM
// over all visits and are stored once, without atomics.  dQ = dS K of each
// visit is added to the fp32 dq in global memory by TMA reductions.
//
// Pipeline (one CTA, 384 threads):
//   warp 0      TMA producer: K and V once, then per visit Q with the visit's
//               128 rows of lse (base 2) and delta (two stages; Q is last read
//               by dK), and dO (one stage; last read by dV, early in the visit)
//   warp 1      TMEM owner and tcgen05.mma issuer (one thread), per visit v:
//               dV(v), S(v+1), dK(v) dQ(v), dP(v+1), so that the next visit's
//               scores form while the key-row threads work on dS(v)
//   warps 4..7  thread = key row: P^T (into TMEM, over its S^T row) and dS^T
//               (into shared memory), and at the end the dK and dV rows
//   warps 8..11 thread = query row: the dQ tile of each visit into dq (TMA
//               reduce-add of 32 x 32 boxes staged in shared memory)
// TMEM (512 columns): S^T [0,128), whose first 64 columns take P^T as packed
// bf16 pairs (the A operand of dV, as P is for O in the forward); dP^T
// [128,256), reused for the dQ tile once dS^T is formed; dK [256, 256+HD), dV
// [256+HD, 256+2HD).  The tensor pipe runs one CTA's MMAs in issue order, so
// S(v+1) overwrites P^T(v) only after dV(v) has read it.
// Shared memory operands (128-byte swizzle, 64-column panels of 128 rows):
// K, V, two stages of Q and one of dO as loaded by TMA; dS^T written by the
// key-row threads.  The same tile is read K-major or MN-major by choosing the
// descriptor: Q is the B operand of S^T (K-major) and of dK (MN-major), dS^T is
// the A operand of dK (K-major) and, read as dS, of dQ (MN-major).
#pragma once
#include "attention.cuh"

namespace ttcd {

struct AttnBwdArgs {
  float* dq;  // [B, T, Hq, HD], accumulated (zeroed by the caller)
  float* dk;  // [B, T, Hkv, HD]
  float* dv;
  // per (b, h) rows of Tp = n_kt * 128 floats, padded past T (lse2 +inf, delta 0):
  const float* lse2_T;   // log2(e) lse_T
  const float* lse2_S;
  const float* delta_T;  // rowsum(dO_T o_T)
  const float* delta_S;
  int B, T, Hq, Hkv;
  int w_S, w_T;
  float scale;       // softmax scale
  float scale_log2;  // softmax scale * log2(e)
  int n_kt;          // key tiles per sequence (= query tiles)
};

constexpr int ATTB_THREADS = 384;

template <int HD>
struct AttnBwdCfg {
  static_assert(HD == 64 || HD == 128, "head_dim 64 or 128");
  static constexpr int PANELS = HD / 64;
  static constexpr int TILE = PANELS * 128 * 128;  // K, V, Q, dO tiles
  static constexpr int DS_TILE = 2 * 128 * 128;    // dS^T: 128 x 128 bf16
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + TILE;
  static constexpr int Q_OFF = V_OFF + TILE;       // two stages
  static constexpr int DO_OFF = Q_OFF + 2 * TILE;  // one stage
  static constexpr int DS_OFF = DO_OFF + TILE;
  static constexpr int DQ_OFF = DS_OFF + DS_TILE;   // 4 warps x 32 rows x 128 bytes
  static constexpr int LSE_OFF = DQ_OFF + 4 * 4096;  // 2 stages of 128 floats
  static constexpr int DEL_OFF = LSE_OFF + 1024;    // 2 stages of 128 floats
  static constexpr int BAR_OFF = DEL_OFF + 1024;
  static constexpr int SMEM = 1024 + BAR_OFF + 256;
};

// Visits of one key tile: per query head of the group, nT teacher passes then
// nS student passes; identical in every role.
struct BwdVisits {
  int kt, nT, nS;
  __device__ BwdVisits(int kt_, int n_qt, int w_S, int w_T) : kt(kt_) {
    nT = min(n_qt - 1 - kt, (w_T + ATT_BN - 2) / ATT_BN) + 1;
    nS = min(n_qt - 1 - kt, (w_S + ATT_BN - 2) / ATT_BN) + 1;
  }
  __device__ int per_head() const { return nT + nS; }
  __device__ void get(int v, int& hg, int& qt, bool& student) const {
    hg = v / per_head();
    const int u = v % per_head();
    student = u >= nT;
    qt = kt + (student ? u - nT : u);
  }
};

// One 128-byte row of a P^T / dS^T tile: 64 bf16 (32 packed words) of row r in
// panel `panel`, 16-byte chunks placed by the 128-byte swizzle.
__device__ __forceinline__ void st_tile_row(uint8_t* tile, int panel, int r, const uint32_t* w) {
  uint8_t* row = tile + panel * (128 * 128) + r * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) =
        make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}

template <int HD>
__global__ void __launch_bounds__(ATTB_THREADS, 1)
    dual_window_attn_bwd_kernel(const __grid_constant__ CUtensorMap mapQ,
                                const __grid_constant__ CUtensorMap mapK,
                                const __grid_constant__ CUtensorMap mapV,
                                const __grid_constant__ CUtensorMap mapDOT,
                                const __grid_constant__ CUtensorMap mapDOS,
                                const __grid_constant__ CUtensorMap mapDQ,
                                const AttnBwdArgs a, const DevStatus st) {
  using Cfg = AttnBwdCfg<HD>;
  constexpr uint32_t ID_SS = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
  constexpr uint32_t ID_KB = idesc_bf16_f32(128, HD, false, true);    // dV, dK
  constexpr uint32_t ID_MM = idesc_bf16_f32(128, HD, true, true);     // dQ
  constexpr uint32_t LOAD_BYTES = Cfg::TILE;
  constexpr int PANEL = 128 * 128;  // bytes of one 64-column panel of 128 rows

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BAR_OFF);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;    // 2 stages (Q, lse2, delta)
  uint64_t* q_empty = bars + 3;   // 2 stages
  uint64_t* do_full = bars + 5;
  uint64_t* do_empty = bars + 6;
  uint64_t* s_full = bars + 7;
  uint64_t* dp_full = bars + 8;
  uint64_t* dp_free = bars + 9;   // 128 arrivals
  uint64_t* p_ready = bars + 10;  // 128 arrivals
  uint64_t* ds_ready = bars + 11; // 128 arrivals
  uint64_t* dst_free = bars + 12;
  uint64_t* dq_full = bars + 13;
  uint64_t* kv_done = bars + 14;
  uint64_t* drain = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv;
  const int kt = static_cast<int>(blockIdx.x) % a.n_kt;
  const int hk = (static_cast<int>(blockIdx.x) / a.n_kt) % a.Hkv;
  const int b = static_cast<int>(blockIdx.x) / (a.n_kt * a.Hkv);
  const int k0 = kt * ATT_BN;
  const BwdVisits vis(kt, a.n_kt, a.w_S, a.w_T);
  const int nv = G * vis.per_head();

  if (threadIdx.x == 0) {
    for (int i = 0; i < 16; ++i) {
      const bool many = bars + i == dp_free || bars + i == p_ready || bars + i == ds_ready;
      mbar_init(bars + i, many ? 128 : 1);
    }
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_map(&mapQ);
    tma_prefetch_map(&mapK);
    tma_prefetch_map(&mapV);
    tma_prefetch_map(&mapDOT);
    tma_prefetch_map(&mapDOS);
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
      // ------------------------------------------------------------- TMA producer
      const int row_base = b * a.T;
      mbar_arrive_expect_tx(kv_full, 2 * LOAD_BYTES);
#pragma unroll
      for (int p = 0; p < Cfg::PANELS; ++p) {
        tma_load_2d(smem + Cfg::K_OFF + p * PANEL, &mapK, kv_full, hk * HD + 64 * p, row_base + k0);
        tma_load_2d(smem + Cfg::V_OFF + p * PANEL, &mapV, kv_full, hk * HD + 64 * p, row_base + k0);
      }
      int issued = 0, issued_do = 0;
      for (int v = 0; v < nv; ++v) {
        int hg, qt;
        bool stu;
        vis.get(v, hg, qt, stu);
        const int h = hk * G + hg;
        const int sg = v & 1;
        if (!mbar_wait(&q_empty[sg], ((v >> 1) & 1) ^ 1, st, abort)) break;
        mbar_arrive_expect_tx(&q_full[sg], LOAD_BYTES + 2 * 512);
#pragma unroll
        for (int p = 0; p < Cfg::PANELS; ++p)
          tma_load_2d(smem + Cfg::Q_OFF + sg * Cfg::TILE + p * PANEL, &mapQ, &q_full[sg],
                      h * HD + 64 * p, row_base + qt * ATT_BM);
        const long long li = (static_cast<long long>(b) * a.Hq + h) * (a.n_kt * ATT_BM) + qt * ATT_BM;
        bulk_load(smem + Cfg::LSE_OFF + sg * 512, (stu ? a.lse2_S : a.lse2_T) + li, 512,
                  &q_full[sg]);
        bulk_load(smem + Cfg::DEL_OFF + sg * 512, (stu ? a.delta_S : a.delta_T) + li, 512,
                  &q_full[sg]);
        if (!mbar_wait(do_empty, (v & 1) ^ 1, st, abort)) { ++issued; break; }
        mbar_arrive_expect_tx(do_full, LOAD_BYTES);
        const CUtensorMap* mdo = stu ? &mapDOS : &mapDOT;
#pragma unroll
        for (int p = 0; p < Cfg::PANELS; ++p)
          tma_load_2d(smem + Cfg::DO_OFF + p * PANEL, mdo, do_full, h * HD + 64 * p,
                      row_base + qt * ATT_BM);
        ++issued_do;
        ++issued;
      }
      // every load issued lands before the CTA can exit
      volatile int no_abort = 0;
      mbar_wait(kv_full, 0, st, &no_abort);
      for (int j = max(0, issued - 2); j < issued; ++j)
        mbar_wait(&q_full[j & 1], (j >> 1) & 1, st, &no_abort);
      if (issued_do > 0) mbar_wait(do_full, (issued_do - 1) & 1, st, &no_abort);
    } else if (warp == 1) {
      // ------------------------------------------------------------- MMA issuer
      constexpr uint32_t HI = sdesc_hi_sw128(1024);
      const uint32_t k_lo = sdesc_lo(smem_u32(smem + Cfg::K_OFF), 16);
      const uint32_t v_lo = sdesc_lo(smem_u32(smem + Cfg::V_OFF), 16);
      const uint32_t q_lo = sdesc_lo(smem_u32(smem + Cfg::Q_OFF), 16);
      const uint32_t do_lo = sdesc_lo(smem_u32(smem + Cfg::DO_OFF), 16);
      const uint32_t ds_lo = sdesc_lo(smem_u32(smem + Cfg::DS_OFF), 16);
      // MN-major views: leading byte offset = one 64-column panel
      const uint32_t q_mn = sdesc_lo(smem_u32(smem + Cfg::Q_OFF), PANEL);
      const uint32_t do_mn = sdesc_lo(smem_u32(smem + Cfg::DO_OFF), PANEL);
      const uint32_t k_mn = sdesc_lo(smem_u32(smem + Cfg::K_OFF), PANEL);
      const uint32_t ds_mn = sdesc_lo(smem_u32(smem + Cfg::DS_OFF), PANEL);
      constexpr uint32_t STAGE = Cfg::TILE >> 4;  // descriptor step of one Q / dO stage
      // K-major step kk of 16 elements: panel kk/4, 32 bytes within the row
      auto koff = [](int kk) { return static_cast<uint32_t>(((kk >> 2) * PANEL + (kk & 3) * 32) >> 4); };
      // MN-major step kk of 16 rows: 16 x 128 bytes
      auto moff = [](int kk) { return static_cast<uint32_t>((kk * 2048) >> 4); };
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, st, abort));
      };
      auto issue_s = [&](int v) {  // S^T = K Q^T
        const uint32_t qs = q_lo + (v & 1) * STAGE;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            mma_bf16_ss_lh(tmem, k_lo + koff(kk), HI, qs + koff(kk), HI, ID_SS, kk > 0 ? 1u : 0u);
          mma_commit(s_full);
        }
        __syncwarp();
      };
      auto issue_dp = [&](int v) {  // dP^T = V dO^T
        const uint32_t ds_ = do_lo;
        (void)v;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            mma_bf16_ss_lh(tmem + 128, v_lo + koff(kk), HI, ds_ + koff(kk), HI, ID_SS,
                           kk > 0 ? 1u : 0u);
          mma_commit(dp_full);
        }
        __syncwarp();
      };
      bool ok = wait(kv_full, 0) && wait(&q_full[0], 0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        ok = wait(do_full, 0);
        if (ok) {
          tc_fence_after();
          issue_dp(0);
        }
      }
      for (int v = 0; v < nv && ok; ++v) {
        const uint32_t ph = v & 1;
        const int sg = v & 1;
        const bool more = v + 1 < nv;
        if (!wait(p_ready, ph)) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {  // dV += P^T dO, P^T from TMEM
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts_lh(tmem + 256 + HD, tmem + kk * 8, do_mn + moff(kk), HI, ID_KB,
                           (v > 0 || kk > 0) ? 1u : 0u);
          mma_commit(do_empty);  // dO(v) is read for the last time
        }
        __syncwarp();
        if (more) {  // the next visit's scores, behind dV in the tensor pipe
          if (!wait(&q_full[(v + 1) & 1], ((v + 1) >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_s(v + 1);
        }
        if (!wait(ds_ready, ph)) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // dK += dS^T Q
            mma_bf16_ss_lh(tmem + 256, ds_lo + koff(kk), HI, q_mn + sg * STAGE + moff(kk), HI,
                           ID_KB, (v > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // dQ = dS K, into the dP^T columns
            mma_bf16_ss_lh(tmem + 128, ds_mn + moff(kk), HI, k_mn + moff(kk), HI, ID_MM,
                           kk > 0 ? 1u : 0u);
          mma_commit(dq_full);
          mma_commit(dst_free);
          mma_commit(&q_empty[sg]);
        }
        __syncwarp();
        if (more) {  // the next dP^T once dQ(v) has left its columns
          if (!wait(dp_free, ph) || !wait(do_full, (v + 1) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_dp(v + 1);
        }
      }
      if (elect_one()) {
        mma_commit(kv_done);
        mma_commit(drain);
      }
      __syncwarp();
      volatile int no_abort = 0;
      mbar_wait(drain, 0, st, &no_abort);
    }
  } else if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
    // --------------------------------------------------- key rows: P^T and dS^T
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row of the tile, TMEM lane
    const int j = k0 + r;               // key position
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_off;
    const uint32_t dp_addr = tmem + lane_off + 128;
    uint8_t* ds_tile = smem + Cfg::DS_OFF;
    bool ok = true;
    for (int v = 0; v < nv; ++v) {
      const uint32_t ph = v & 1;
      int hg, qt;
      bool stu;
      vis.get(v, hg, qt, stu);
      const int q0 = qt * ATT_BM;
      const int w = stu ? a.w_S : a.w_T;
      // this visit's lse (base 2) and delta per query column, copied with Q and dO
      if (!mbar_wait(&q_full[v & 1], (v >> 1) & 1, st, abort)) { ok = false; break; }
      const float* lse2 = reinterpret_cast<const float*>(smem + Cfg::LSE_OFF + (v & 1) * 512);
      const float* dlt = reinterpret_cast<const float*>(smem + Cfg::DEL_OFF + (v & 1) * 512);
      // visible query columns of key j: c - lo in [0, w - 1], lo = j - q0
      const int lo = j - q0;
      if (!mbar_wait(s_full, ph, st, abort)) { ok = false; break; }
      tc_fence_after();
      uint32_t P[64];
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        float s[32];
        tmem_ld32f(s_addr + cc, s);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int c = cc + i;
          const float p0 = (c - lo >= 0 && c - lo < w) ? ex2_approx(s[i] * a.scale_log2 - lse2[c]) : 0.f;
          const float p1 = (c + 1 - lo >= 0 && c + 1 - lo < w)
                               ? ex2_approx(s[i + 1] * a.scale_log2 - lse2[c + 1]) : 0.f;
          P[c >> 1] = pack_bf16x2(p0, p1);
        }
      }
      // P^T over the first 64 columns of this row's S^T (the A operand of dV)
      tmem_st32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&P[0]));
      tmem_st32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&P[32]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_ready);
      // dS^T = P^T (dP^T - delta) scale
      if (!mbar_wait(dp_full, ph, st, abort)) { ok = false; break; }
      tc_fence_after();
      uint32_t D[64];
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        float dp[32];
        tmem_ld32f(dp_addr + cc, dp);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int c = cc + i;
          const uint32_t pw = P[c >> 1];
          const float d0 = bf16lo_to_f32(pw) * (dp[i] - dlt[c]) * a.scale;
          const float d1 = bf16hi_to_f32(pw) * (dp[i + 1] - dlt[c + 1]) * a.scale;
          D[c >> 1] = pack_bf16x2(d0, d1);
        }
      }
      tc_fence_before();
      if (!mbar_wait(dst_free, ph ^ 1, st, abort)) { ok = false; break; }
      st_tile_row(ds_tile, 0, r, &D[0]);
      st_tile_row(ds_tile, 1, r, &D[32]);
      fence_async_smem();
      mbar_arrive(ds_ready);
    }
    // -------------------------------------------------------- dK and dV rows
    if (ok && mbar_wait(kv_done, 0, st, abort)) {
      tc_fence_after();
      const bool row_ok = j < a.T;
      const long long orow = (static_cast<long long>(b) * a.T + j) * a.Hkv + hk;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        float x[32];
        tmem_ld32f(tmem + lane_off + 256 + c, x);
        if (row_ok) store_f32x32(a.dk + orow * HD + c, x);
        tmem_ld32f(tmem + lane_off + 256 + HD + c, x);
        if (row_ok) store_f32x32(a.dv + orow * HD + c, x);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
    // ----------------------------------------------------- query rows: dQ tiles
    // Each visit's dQ tile is added to dq by TMA reductions (fp32 add in L2),
    // 32 rows x 32 columns at a time through this warp's 4 KB staging box
    // (128-byte swizzle).  Rows past a sequence's end carry exact zeros (P = 0
    // there), so a box reaching into the next sequence adds nothing to it.
    const int quarter = warp & 3;
    const uint32_t dq_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 128;
    uint8_t* box = smem + Cfg::DQ_OFF + quarter * 4096;
    for (int v = 0; v < nv; ++v) {
      int hg, qt;
      bool stu;
      vis.get(v, hg, qt, stu);
      const int h = hk * G + hg;
      if (!mbar_wait(dq_full, v & 1, st, abort)) break;
      tc_fence_after();
      // the whole row into registers first: the columns are free for the next
      // dP^T as soon as they have been read
      float x[HD];
#pragma unroll
      for (int c = 0; c < HD; c += 32) tmem_ld32f(dq_addr + c, *reinterpret_cast<float(*)[32]>(&x[c]));
      tc_fence_before();
      mbar_arrive(dp_free);
      const int y = b * a.T + qt * ATT_BM + quarter * 32;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        if (lane == 0) bulk_wait_read<0>();  // the previous box has been read out
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(box + lane * 128 + ((j ^ (lane & 7)) << 4)) =
              make_float4(x[c + 4 * j], x[c + 4 * j + 1], x[c + 4 * j + 2], x[c + 4 * j + 3]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(&mapDQ, box, h * HD + c, y);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait<0>();  // every reduction has completed
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Per (b, h) row of Tp floats, both windows: delta[t] = sum_d dO[b, t, h, d]
// O[b, t, h, d] and lse2[t] = log2(e) lse[b, h, t] for t < T; past T, delta 0 and
// lse2 +inf (so that the rebuilt P is 0 there).  One thread per (window, b, h, t).
template <int HD>
__global__ void attn_bwd_rows_kernel(const __nv_bfloat16* __restrict__ o_T,
                                     const __nv_bfloat16* __restrict__ o_S,
                                     const __nv_bfloat16* __restrict__ do_T,
                                     const __nv_bfloat16* __restrict__ do_S,
                                     const float* __restrict__ lse_T,
                                     const float* __restrict__ lse_S, float* __restrict__ delta_T,
                                     float* __restrict__ delta_S, float* __restrict__ lse2_T,
                                     float* __restrict__ lse2_S, int T, int Tp, int Hq,
                                     long long rows) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= 2 * rows * Tp) return;
  const bool stu = idx >= rows * Tp;
  const long long e = stu ? idx - rows * Tp : idx;
  const int t = static_cast<int>(e % Tp);
  const long long bh = e / Tp;  // b * Hq + h
  float* delta = stu ? delta_S : delta_T;
  float* lse2 = stu ? lse2_S : lse2_T;
  if (t >= T) {
    delta[e] = 0.f;
    lse2[e] = INFINITY;
    return;
  }
  const long long b = bh / Hq;
  const int h = static_cast<int>(bh % Hq);
  const long long row = (b * T + t) * Hq + h;  // (b, t, h) row of o and dO
  const __nv_bfloat16* o = (stu ? o_S : o_T) + row * HD;
  const __nv_bfloat16* g = (stu ? do_S : do_T) + row * HD;
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < HD; c += 8) {
    float x[8], y[8];
    ld8f(o + c, x);
    ld8f(g + c, y);
#pragma unroll
    for (int i = 0; i < 8; ++i) s = fmaf(x[i], y[i], s);
  }
  delta[e] = s;
  lse2[e] = (stu ? lse_S : lse_T)[bh * T + t] * 1.4426950408889634f;
}

}  // namespace ttcd
