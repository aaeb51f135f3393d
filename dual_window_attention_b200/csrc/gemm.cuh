// Persistent warp-specialised tcgen05 GEMM for sm_100a:  C = A * B^T.
//
//   A [rows, K] bf16 K-major, B [N, K] bf16 K-major, fp32 accumulators in TMEM.
//   warp 0      : TMA producer (one elected lane), STAGES-deep smem ring
//   warp 1      : TMEM allocation + tcgen05.mma issue (one elected lane)
//   warps 2..5  : epilogue, each owns one 32-lane quarter of the accumulator
//   Two TMEM accumulators (2*BN columns) let the epilogue of tile j overlap the
//   main loop of tile j+1.
//
// The A rows may be cut into groups (fast-weight chunks): sequence b, chunk i
// covers rows [b*T + i*C, b*T + min((i+1)*C, T)) and reads B rows starting at
// (b*Nc + i) * b_group_rows.  A plain GEMM is one sequence with one chunk.
#pragma once
#include <type_traits>

#include "ptx.cuh"

namespace ttcd {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;  // bf16 elements per 128-byte swizzled row

struct TileCtx {
  int row0;        // first A row (== output row) of the tile
  int valid_rows;  // rows of this tile inside its group (<= 128)
  int tn;          // column-tile index
  int group;       // b * Nc + i (paired tiles: the sequence b)
  int b_row0;      // first B row of this group
  int tok0;        // paired tiles: token of accumulator row 0 (and of row 64)
};

struct GemmGeom {
  static constexpr bool kPaired = false;
  int n_seq, T, C, Nc;  // row groups
  int K;                // reduction length (multiple of 64 not required: TMA zero-fills)
  int tiles_m;          // ceil(C / 128)
  int tiles_n;          // column tiles
  int b_group_rows;     // B row offset per group (0 = shared B)
  int row_off = 0;      // first A (and output) row of the geometry
  __host__ __device__ int total() const { return n_seq * Nc * tiles_m * tiles_n; }
  // CTA pairs: pair tile t covers row tiles 2p and 2p + 1 of one group; `rank`
  // picks this CTA's.  True while the pair's first tile has rows; the second
  // may have none (valid_rows 0), and its CTA still takes part in the MMAs.
  __host__ __device__ int tiles_m2() const { return (tiles_m + 1) / 2; }
  __host__ __device__ int total_pairs() const { return n_seq * Nc * tiles_m2() * tiles_n; }
  __device__ bool tile_pair(int t, int rank, TileCtx& c) const {
    const int tn = t % tiles_n;
    const int r = t / tiles_n;
    const int pm = r % tiles_m2();
    const int g = r / tiles_m2();
    const int b = g / Nc, i = g % Nc;
    const int len = min(C, T - i * C);
    const int m0 = (2 * pm + rank) * GEMM_BM;
    c.valid_rows = max(0, min(GEMM_BM, len - m0));
    c.row0 = row_off + b * T + i * C + m0;
    c.tn = tn;
    c.group = g;
    c.b_row0 = g * b_group_rows;
    return len - 2 * pm * GEMM_BM > 0;
  }
  __device__ bool tile(int t, TileCtx& c) const {
    const int tn = t % tiles_n;
    const int r = t / tiles_n;
    const int tm = r % tiles_m;
    const int g = r / tiles_m;
    const int b = g / Nc, i = g % Nc;
    const int len = min(C, T - i * C);
    const int m0 = tm * GEMM_BM;
    c.valid_rows = min(GEMM_BM, len - m0);
    c.row0 = row_off + b * T + i * C + m0;
    c.tn = tn;
    c.group = g;
    c.b_row0 = g * b_group_rows;
    return c.valid_rows > 0;
  }
};

// Paired tiles: accumulator rows 0-63 are the teacher rows of tokens
// [tok0, tok0 + 64) of sequence b and rows 64-127 the student rows of the same
// tokens (A = [u_T; u_S], the student half `half_rows` rows further down).
// Consecutive tiles of a sequence overlap by H = conv_k - 1 tokens, so the
// epilogue holds the H rows before its first output token and the causal conv
// needs nothing from other tiles: tile tm outputs tokens [tm (64-H), tm (64-H) +
// 64-H) and starts at tok0 = tm (64-H) - H (rows before token 0 of sequence 0
// are zero-filled by the TMA load, and zeroed by the epilogue for every b).
struct PairGeom {
  static constexpr bool kPaired = true;
  int n_seq, T, H, K;
  int tiles_m;  // ceil(T / (64 - H))
  int tiles_n;
  long long half_rows;  // B*T: row offset of the student half of A
  __host__ __device__ int total() const { return n_seq * tiles_m * tiles_n; }
  __device__ bool tile(int t, TileCtx& c) const {
    const int tn = t % tiles_n;
    const int r = t / tiles_n;
    const int tm = r % tiles_m;
    const int b = r / tiles_m;
    c.tn = tn;
    c.group = b;
    c.b_row0 = 0;
    c.tok0 = tm * (64 - H) - H;
    c.row0 = b * T + c.tok0;
    c.valid_rows = GEMM_BM;
    return true;
  }
};

// Barrier and AND-vote over the NT epilogue threads (named barrier 1).
// Collective epilogues call them the same number of times in every warp; the
// vote on each tile's accumulator wait makes an abort uniform, so no warp
// leaves the tile loop while another waits at a barrier.
template <int NT = 128>
__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}
template <int NT = 128>
__device__ __forceinline__ bool epi_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(NT)
      : "memory");
  return r != 0;
}

// Epilogue warps of a GEMM: Epi::kWarps when the epilogue declares it (8: two
// warps per TMEM lane quarter), else 4.  With 4 the kernel runs warps 0-5 (0 TMA,
// 1 MMA, 2-5 epilogue); with 8 it runs warps 0-11, the epilogue on warps 4-11
// (two whole warpgroups, 2-3 idle), and setmaxnreg moves registers from the
// control warpgroup (56) to the epilogue warpgroups (224).
template <class Epi, class = void>
struct EpiWarps {
  static constexpr int value = 4;
};
template <class Epi>
struct EpiWarps<Epi, std::void_t<decltype(Epi::kWarps)>> {
  static constexpr int value = Epi::kWarps;
};
template <class Epi>
constexpr int gemm_epi_warp0() {
  return EpiWarps<Epi>::value == 8 ? 4 : 2;
}
template <class Epi>
constexpr int gemm_threads() {
  return 32 * gemm_epi_warp0<Epi>() + 32 * EpiWarps<Epi>::value;
}
// Shared memory the epilogue keeps after the operand stages: Epi::kStagingBytes
// when declared, else 4 warps x 8 KB of TMA-store staging for staged epilogues.
template <class Epi, class = void>
struct EpiStagingBytes {
  static constexpr int value = Epi::kStaged ? 4 * 8192 : 0;
};
template <class Epi>
struct EpiStagingBytes<Epi, std::void_t<decltype(Epi::kStagingBytes)>> {
  static constexpr int value = Epi::kStagingBytes;
};
// Extra mbarriers for the epilogue's own use (Epi::kExtraBars, each initialised
// with Epi::kExtraBarCount arrivals), and whether the epilogue releases the
// TMEM accumulator itself (Epi::kSelfRelease: it arrives on stg.release).
template <class Epi, class = void>
struct EpiExtraBars {
  static constexpr int value = 0;
  static constexpr int count = 1;
};
template <class Epi>
struct EpiExtraBars<Epi, std::void_t<decltype(Epi::kExtraBars)>> {
  static constexpr int value = Epi::kExtraBars;
  static constexpr int count = Epi::kExtraBarCount;
};
template <class Epi, class = void>
struct EpiSelfRelease {
  static constexpr bool value = false;
};
template <class Epi>
struct EpiSelfRelease<Epi, std::void_t<decltype(Epi::kSelfRelease)>> {
  static constexpr bool value = Epi::kSelfRelease;
};

__device__ __forceinline__ void tmem_ld16f(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  tmem_ld16(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld32f(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = w;
  }
}
__device__ __forceinline__ void store_f32x32(float* dst, const float (&v)[32]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}
__device__ __forceinline__ void store_x32(__nv_bfloat16* dst, const float (&v)[32]) { store_bf16x32(dst, v); }
__device__ __forceinline__ void store_x32(float* dst, const float (&v)[32]) { store_f32x32(dst, v); }

__device__ __forceinline__ void load_x32(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w = s[q];
    v[8 * q + 0] = bf16lo_to_f32(w.x); v[8 * q + 1] = bf16hi_to_f32(w.x);
    v[8 * q + 2] = bf16lo_to_f32(w.y); v[8 * q + 3] = bf16hi_to_f32(w.y);
    v[8 * q + 4] = bf16lo_to_f32(w.z); v[8 * q + 5] = bf16hi_to_f32(w.z);
    v[8 * q + 6] = bf16lo_to_f32(w.w); v[8 * q + 7] = bf16hi_to_f32(w.w);
  }
}
__device__ __forceinline__ void load_x32(const float* src, float (&v)[32]) {
  const float4* s = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float4 w = s[q];
    v[4 * q] = w.x; v[4 * q + 1] = w.y; v[4 * q + 2] = w.z; v[4 * q + 3] = w.w;
  }
}

// Per-warp staging of epilogue output for TMA stores: two 4 KB buffers, each
// 32 rows x 128 bytes in the 128-byte swizzle (16-byte chunk j of row r sits
// at slot j ^ (r & 7)), so a warp writing one chunk per row touches every bank
// once per 8 rows.  One lane issues the store of the whole 32-row box.
struct EpiStage {
  uint8_t* buf;             // 2 x 4096 bytes, 1024-aligned; nullptr: direct stores
  const CUtensorMap* map;   // first output tensor map (box: 128 bytes x 32 rows)
  const CUtensorMap* map2;  // second output tensor map (same box), when an epilogue has two
  int toggle;
  uint64_t* xbars = nullptr;    // the epilogue's extra mbarriers
  uint64_t* release = nullptr;  // the tile's accumulator-empty barrier (self-releasing epilogues)
  int tiles = 0;                // tiles this thread has run (self-releasing epilogues count them)
  __device__ bool on() const { return buf != nullptr; }
  // Before writing into the current buffer: its previous store has read it.
  __device__ void acquire() {
    if ((threadIdx.x & 31) == 0) bulk_wait_read<1>();
    __syncwarp();
  }
  __device__ void write_f32(int r, const float (&v)[32]) {
    uint8_t* b = buf + toggle * 4096 + r * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(b + ((j ^ (r & 7)) << 4)) =
          make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  }
  __device__ void write_bf16(int r, const float (&lo)[32], const float (&hi)[32]) {
    uint8_t* b = buf + toggle * 4096 + r * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float* v = j < 4 ? &lo[8 * j] : &hi[8 * (j - 4)];
      uint4 w;
      w.x = pack_bf16x2(v[0], v[1]);
      w.y = pack_bf16x2(v[2], v[3]);
      w.z = pack_bf16x2(v[4], v[5]);
      w.w = pack_bf16x2(v[6], v[7]);
      *reinterpret_cast<uint4*>(b + ((j ^ (r & 7)) << 4)) = w;
    }
  }
  __device__ void flush(const CUtensorMap* m, int x, int y) {
    fence_async_smem();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
      tma_store_2d(m, buf + toggle * 4096, x, y);
      bulk_commit();
    }
    toggle ^= 1;
  }
  __device__ void flush(int x, int y) { flush(map, x, y); }
  __device__ void drain() {
    if (buf && (threadIdx.x & 31) == 0) bulk_wait<0>();
  }
};

// B_MN = true (bf16 only): B is given as B^T, a row-major [K, N] matrix (N
// contiguous), and is read as an MN-major tcgen05 operand: TMA boxes of 64
// N-elements x 64 K-rows, leading-byte offset = one box, 16 K-rows (2048 bytes)
// per MMA step.  With row groups (b_group_rows > 0) group g's B^T starts at row
// g * b_group_rows, so K must then be a multiple of 64.
//
// PAIR = true (bf16, one K-major B, plain row tiles): clusters of two CTAs run
// 256-row tiles as M = 256 MMAs (tcgen05 .cta_group::2).  Each CTA loads its
// own 128 rows of A and half of the tile's B rows (B is given with BN/2-row
// boxes), so a k-block moves a third less into each SM.  Rank 0 counts both
// CTAs' bytes on its full barriers, issues the MMAs and commits them to both
// CTAs' barriers; each CTA's epilogue handles its own 128 rows and releases
// the accumulator on rank 0's barrier.
template <class E, int BN, int STAGES, bool DUAL_B, class Epi, class Geom = GemmGeom,
          bool B_MN = false, bool PAIR = false>
__global__ void __launch_bounds__(gemm_threads<Epi>(), 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA,
                   const __grid_constant__ CUtensorMap mapB0,
                   const __grid_constant__ CUtensorMap mapB1,
                   const __grid_constant__ CUtensorMap mapOut,
                   const __grid_constant__ CUtensorMap mapOut2, const Geom geo,
                   const Epi epi, const DevStatus st) {
  constexpr bool STAGED = Epi::kStaged;
  constexpr int A_BYTES = GEMM_BM * 128;
  constexpr int B_BYTES = (PAIR ? BN / 2 : BN) * 128;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of 2");
  static_assert(!B_MN || (sizeof(E) == 2 && !DUAL_B), "MN-major B: bf16, single B operand");
  static_assert(!PAIR || (sizeof(E) == 2 && !DUAL_B && !Geom::kPaired &&
                          !EpiSelfRelease<Epi>::value),
                "CTA pairs: bf16, one B operand, plain row tiles, kernel-released accumulator");
  constexpr uint32_t IDESC =
      idesc_f32acc(PAIR ? 2 * GEMM_BM : GEMM_BM, BN, ElemTraits<E>::FMT, false, B_MN);
  constexpr int MN_BOX_BYTES = 64 * 64 * 2;  // 64 N-elements x 64 K-rows, bf16
  constexpr int BK = ElemTraits<E>::BK;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  constexpr int NX = EpiExtraBars<Epi>::value;
  uint8_t* staging = smem + STAGES * STAGE_BYTES;  // the epilogue's shared memory
  uint64_t* xbars = reinterpret_cast<uint64_t*>(staging + EpiStagingBytes<Epi>::value);
  uint64_t* full = xbars + NX;
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    if (STAGED) {
      tma_prefetch_map(&mapOut);
      tma_prefetch_map(&mapOut2);
    }
    for (int i = 0; i < NX; ++i) mbar_init(&xbars[i], EpiExtraBars<Epi>::count);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], (PAIR ? 2 : 1) * 32 * EpiWarps<Epi>::value);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_map(&mapA);
    tma_prefetch_map(&mapB0);
    if (DUAL_B) tma_prefetch_map(&mapB1);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
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
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  // Tiles of this CTA: pair tiles (one per cluster) or row tiles.
  const int total = [&]() {
    if constexpr (PAIR)
      return geo.total_pairs();
    else
      return geo.total();
  }();
  const int t_first = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int t_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  auto get_tile = [&](int t, TileCtx& c) -> bool {
    if constexpr (PAIR)
      return geo.tile_pair(t, static_cast<int>(rank), c);
    else
      return geo.tile(t, c);
  };
  const int nk = (geo.K + BK - 1) / BK;
  constexpr int EPI0 = gemm_epi_warp0<Epi>();
  // 8 epilogue warps: the launch's 384 x 168 registers are split 128 x 56 (warps
  // 0-3) + 256 x 224 (warps 4-11), each warp setting its limit in its own branch
  constexpr bool SPLIT_REGS = EpiWarps<Epi>::value == 8;

  if (warp == 0) {
    if constexpr (SPLIT_REGS) asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      int it = 0;
      bool ok = true;
      const uint32_t full0 = PAIR ? mapa_shared(smem_u32(full), 0) : 0u;
      for (int t = t_first; t < total && ok; t += t_step) {
        TileCtx c;
        if (!get_tile(t, c)) continue;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait<PAIR>(&empty[s], ph ^ 1, st, abort)) { ok = false; break; }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          if constexpr (PAIR) {
            // both CTAs' bytes land on rank 0's full barrier
            const uint32_t fb = full0 + 8u * static_cast<uint32_t>(s);
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * STAGE_BYTES);
            tma_load_2d_pair(sa, &mapA, fb, kb * BK, c.row0);
            if constexpr (B_MN) {  // this CTA's BN/2 columns as 64-column boxes
#pragma unroll
              for (int q = 0; q < BN / 128; ++q)
                tma_load_2d_pair(sb + q * MN_BOX_BYTES, &mapB0, fb,
                                 c.tn * BN + static_cast<int>(rank) * (BN / 2) + 64 * q,
                                 c.b_row0 + kb * BK);
            } else {
              tma_load_2d_pair(sb, &mapB0, fb, kb * BK,
                               c.b_row0 + c.tn * BN + static_cast<int>(rank) * (BN / 2));
            }
            continue;
          }
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          if constexpr (Geom::kPaired) {  // two 64-row boxes: teacher rows, student rows
            tma_load_2d(sa, &mapA, &full[s], kb * BK, c.row0);
            tma_load_2d(sa + (GEMM_BM / 2) * 128, &mapA, &full[s], kb * BK,
                        static_cast<int>(c.row0 + geo.half_rows));
          } else {
            tma_load_2d(sa, &mapA, &full[s], kb * BK, c.row0);
          }
          if (DUAL_B) {
            tma_load_2d(sb, &mapB0, &full[s], kb * BK, c.b_row0 + c.tn * (BN / 2));
            tma_load_2d(sb + (BN / 2) * 128, &mapB1, &full[s], kb * BK,
                        c.b_row0 + c.tn * (BN / 2));
          } else if constexpr (B_MN) {
#pragma unroll
            for (int q = 0; q < BN / 64; ++q)
              tma_load_2d(sb + q * MN_BOX_BYTES, &mapB0, &full[s], c.tn * BN + 64 * q,
                          c.b_row0 + kb * BK);
          } else {
            tma_load_2d(sb, &mapB0, &full[s], kb * BK, c.b_row0 + c.tn * BN);
          }
        }
      }
      // Let every load this thread issued land before the CTA can exit (a
      // pair: until rank 0's MMAs have consumed them, so no commit to this
      // CTA's stage barriers is still in flight either).
      volatile int no_abort = 0;
      for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j) {
        if constexpr (PAIR)
          mbar_wait<true>(&empty[j % STAGES], (j / STAGES) & 1, st, abort);
        else
          mbar_wait(&full[j % STAGES], (j / STAGES) & 1, st, &no_abort);
      }
    }
  } else if (warp == 1) {
    if constexpr (SPLIT_REGS) asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop (operand words stay warp-uniform) and one
    // elected lane issues; descriptor low words advance by (byte offset >> 4).
    constexpr uint32_t HI = sdesc_hi_sw128(1024);
    const uint32_t lo0 = sdesc_lo(smem_u32(smem), 16);
    // MN-major B: its leading-byte offset is one box (the low word differs by it)
    constexpr uint32_t B_LBO_FIX = B_MN ? ((MN_BOX_BYTES >> 4) - 1) << 16 : 0;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait<PAIR>(bar, parity, st, abort));
    };
    int it = 0, j = 0;
    bool ok = rank == 0;  // a pair's MMAs are issued by rank 0 alone
    for (int t = t_first; t < total && ok; t += t_step) {
      TileCtx c;
      if (!get_tile(t, c)) continue;
      const int ab = j & 1;
      if (!wait(&acce[ab], ((j >> 1) & 1) ^ 1)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + ab * BN;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % STAGES;
        if (!wait(&full[s], (it / STAGES) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_lo = lo0 + ((s * STAGE_BYTES) >> 4);
        const uint32_t b_lo = a_lo + (A_BYTES >> 4) + B_LBO_FIX;
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 4 MMAs of 32 bytes of K per 128-byte row
            if constexpr (PAIR)
              mma_bf16_ss_lh_pair(d_tmem, a_lo + 2 * k, HI, b_lo + (B_MN ? k * (2048 >> 4) : 2 * k),
                                  HI, IDESC, (kb | k) != 0 ? 1u : 0u);
            else
              mma_ss_lh<E>(d_tmem, a_lo + 2 * k, HI, b_lo + (B_MN ? k * (2048 >> 4) : 2 * k), HI,
                           IDESC, (kb | k) != 0 ? 1u : 0u);
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
      ++j;
    }
    if (!PAIR || rank == 0) {
      // Drain: all MMAs issued by the elected lane complete before TMEM is freed.
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
        // the epilogues' releases of the last two accumulators (half of them
        // arrive from the other CTA) land before this CTA may leave
        for (int jj = j; jj < j + 2; ++jj)
          if (jj >= 2) mbar_wait<true>(&acce[jj & 1], ((jj >> 1) & 1) ^ 1, st, abort);
      }
    }
  } else if (warp < EPI0) {
    if constexpr (SPLIT_REGS) asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
  } else {
    if constexpr (SPLIT_REGS) asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    // staging slots of 8 KB per lane quarter (8-warp epilogues share them by quarter)
    EpiStage stg{STAGED ? staging + ((warp - EPI0) & 3) * 8192 : nullptr, &mapOut, &mapOut2, 0};
    stg.xbars = xbars;
    int j = 0;
    const uint32_t acce0 = PAIR ? mapa_shared(smem_u32(acce), 0) : 0u;
    for (int t = t_first; t < total; t += t_step) {
      TileCtx c;
      if (!get_tile(t, c)) continue;
      const int ab = j & 1;
      // per-row inputs of the epilogue are fetched while the tile is still computing
      const float pre = epi.pre(c, r);
      bool ok = mbar_wait<PAIR>(&accf[ab], (j >> 1) & 1, st, abort);
      if constexpr (Epi::kCollective) ok = epi_bar_and<32 * EpiWarps<Epi>::value>(ok);
      if (!ok) break;
      tc_fence_after();
      stg.release = &acce[ab];
      epi.template run<BN>(c, tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * BN, r,
                           stg, pre);
      if constexpr (!EpiSelfRelease<Epi>::value) {
        tc_fence_before();
        if constexpr (PAIR)
          mbar_arrive_cluster(acce0 + 8u * static_cast<uint32_t>(ab));
        else
          mbar_arrive(&acce[ab]);
      }
      ++j;
    }
    stg.drain();
  }
  if constexpr (PAIR) {
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
  } else {
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem_base, TMEM_COLS);
    }
  }
}

template <int BN, int STAGES, bool STAGED = false>
constexpr int gemm_smem_bytes() {
  return 1024 + STAGES * (GEMM_BM * 128 + BN * 128) + (STAGED ? 4 * 8192 : 0) + 256;
}
template <class Epi, int BN, int STAGES, bool PAIR = false>
constexpr int gemm_smem_bytes_for() {
  return 1024 + STAGES * (GEMM_BM * 128 + (PAIR ? BN / 2 : BN) * 128) +
         EpiStagingBytes<Epi>::value + 8 * EpiExtraBars<Epi>::value + 256;
}

// ------------------------------------------------------------------ epilogues

// Writes one row's 32 (fp32) or 64 (bf16) output columns starting at `col`:
// through the warp's staging buffer and a TMA store when all 32 rows of the
// warp lie inside the tile, else with direct stores for the valid rows.
template <class OutT>
struct OutChunk {
  static constexpr int COLS = sizeof(OutT) == 4 ? 32 : 64;
};
__device__ __forceinline__ void emit(EpiStage& stg, const CUtensorMap* m, bool staged, bool ok,
                                     float* out_row, int col, int y, const float (&v)[32],
                                     const float (&)[32]) {
  if (staged) {
    stg.acquire();
    stg.write_f32(threadIdx.x & 31, v);
    stg.flush(m, col, y);
  } else if (ok) {
    store_f32x32(out_row + col, v);
  }
}
__device__ __forceinline__ void emit(EpiStage& stg, const CUtensorMap* m, bool staged, bool ok,
                                     __nv_bfloat16* out_row, int col, int y,
                                     const float (&lo)[32], const float (&hi)[32]) {
  if (staged) {
    stg.acquire();
    stg.write_bf16(threadIdx.x & 31, lo, hi);
    stg.flush(m, col, y);
  } else if (ok) {
    store_bf16x32(out_row + col, lo);
    store_bf16x32(out_row + col + 32, hi);
  }
}
template <class OutT>
__device__ __forceinline__ void emit(EpiStage& stg, bool staged, bool ok, OutT* out_row, int col,
                                     int y, const float (&lo)[32], const float (&hi)[32]) {
  emit(stg, stg.map, staged, ok, out_row, col, y, lo, hi);
}

// C[row, col] = OutT(acc * row_scale[row]) (row_scale nullable), columns < N.
// N must be a multiple of 64 for bf16 output.
template <class OutT>
struct EpiStore {
  static constexpr bool kStaged = true;
  static constexpr bool kCollective = false;
  OutT* out;
  long long ldo;
  int N;
  const float* row_scale;
  __device__ float pre(const TileCtx& c, int r) const {
    return (row_scale && r < c.valid_rows) ? __ldg(row_scale + c.row0 + r) : 1.f;
  }
  template <int BN>
  __device__ void run(const TileCtx& c, uint32_t taddr, int r, EpiStage& stg, float sc) const {
    const bool ok = r < c.valid_rows;
    const long long row = c.row0 + r;
    const int wrow = r & ~31;
    const bool staged = stg.on() && wrow + 32 <= c.valid_rows;
    constexpr int CW = OutChunk<OutT>::COLS;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += CW) {
      const int col = c.tn * BN + cc;
      if (col >= N) break;
      float lo[32], hi[32];
      tmem_ld32f(taddr + cc, lo);
#pragma unroll
      for (int i = 0; i < 32; ++i) lo[i] *= sc;
      if (CW == 64) {
        tmem_ld32f(taddr + cc + 32, hi);
#pragma unroll
        for (int i = 0; i < 32; ++i) hi[i] *= sc;
      }
      emit(stg, staged, ok, out + row * ldo, col, c.row0 + wrow, lo, hi);
    }
  }
};
using EpiStoreBF16 = EpiStore<__nv_bfloat16>;

// out[row, col] = resid[row % resid_rows, col] + acc;  columns < N.
template <class OutT, class ResT>
struct EpiResidual {
  static constexpr bool kStaged = true;
  static constexpr bool kCollective = false;
  OutT* out;
  long long ldo;
  const ResT* resid;  // nullable
  long long ld_res;
  long long resid_rows;
  int N;
  __device__ float pre(const TileCtx&, int) const { return 1.f; }
  template <int BN>
  __device__ void run(const TileCtx& c, uint32_t taddr, int r, EpiStage& stg, float) const {
    const bool ok = r < c.valid_rows;
    const long long row = c.row0 + r;
    const int wrow = r & ~31;
    const bool staged = stg.on() && wrow + 32 <= c.valid_rows;
    const ResT* res_row = resid ? resid + (row % resid_rows) * ld_res : nullptr;
    constexpr int CW = OutChunk<OutT>::COLS;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += CW) {
      const int col = c.tn * BN + cc;
      if (col >= N) break;
      float lo[32], hi[32];
      tmem_ld32f(taddr + cc, lo);
      if (CW == 64) tmem_ld32f(taddr + cc + 32, hi);
      if (ok && res_row) {
        float x[32];
        load_x32(res_row + col, x);
#pragma unroll
        for (int i = 0; i < 32; ++i) lo[i] += x[i];
        if (CW == 64) {
          load_x32(res_row + col + 32, x);
#pragma unroll
          for (int i = 0; i < 32; ++i) hi[i] += x[i];
        }
      }
      emit(stg, staged, ok, out + row * ldo, col, c.row0 + wrow, lo, hi);
    }
  }
};

// o_proj of both paths with the residual, feeding the MLP RMSNorm:
//   h = x[row % BT] + acc                (rows [0, BT) teacher, [BT, 2BT) student)
//   hg[row]       = h * g_mlp            (gate/up operand; stored through mapOut)
//   h_S[row - BT] = h  for student rows  (fp32 residual of the output; mapOut2)
//   ssq[tn][row]  = sum over this tile's columns of h^2  (fixed order)
template <class E, class ResT>
struct EpiOprojNorm {
  static constexpr bool kStaged = true;
  static constexpr bool kCollective = false;
  E* hg;
  float* hS;
  float* ssq;
  const ResT* x;
  const E* g;
  long long BT;
  int d;
  __device__ float pre(const TileCtx&, int) const { return 1.f; }
  template <int BN>
  __device__ void run(const TileCtx& c, uint32_t taddr, int r, EpiStage& stg, float) const {
    const bool ok = r < c.valid_rows;
    const long long row = c.row0 + r;
    const long long wrow0 = c.row0 + (r & ~31);  // first row of this warp
    const bool wvalid = stg.on() && (r & ~31) + 32 <= c.valid_rows;
    const bool w_student = wrow0 >= BT;            // whole warp in the student half
    const bool w_teacher = wrow0 + 32 <= BT;       // whole warp in the teacher half
    const bool is_student = row >= BT;
    const ResT* xrow = x + (row % BT) * d;
    float* hs_row = is_student ? hS + (row - BT) * d : hS;
    float ss = 0.f;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 64) {
      const int col = c.tn * BN + cc;
      if (col >= d) break;
      float lo[32], hi[32], glo[32], ghi[32];
      tmem_ld32f(taddr + cc, lo);
      tmem_ld32f(taddr + cc + 32, hi);
      if (ok) {
        float t[32];
        load_x32(xrow + col, t);
#pragma unroll
        for (int i = 0; i < 32; ++i) lo[i] += t[i];
        load_x32(xrow + col + 32, t);
#pragma unroll
        for (int i = 0; i < 32; ++i) hi[i] += t[i];
      }
      load_x32(g + col, glo);
      load_x32(g + col + 32, ghi);
#pragma unroll
      for (int i = 0; i < 32; ++i) ss += lo[i] * lo[i] + hi[i] * hi[i];
      // fp32 student residual
      if (wvalid && w_student) {
        emit(stg, stg.map2, true, ok, hs_row, col, static_cast<int>(wrow0 - BT), lo, lo);
        emit(stg, stg.map2, true, ok, hs_row, col + 32, static_cast<int>(wrow0 - BT), hi, hi);
      } else if (!(wvalid && w_teacher) && ok && is_student) {
        store_f32x32(hs_row + col, lo);
        store_f32x32(hs_row + col + 32, hi);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        glo[i] *= lo[i];
        ghi[i] *= hi[i];
      }
      E* hg_row = hg + row * d;
      if constexpr (sizeof(E) == 2) {
        emit(stg, stg.map, wvalid, ok, hg_row, col, static_cast<int>(wrow0), glo, ghi);
      } else {
        emit(stg, stg.map, wvalid, ok, hg_row, col, static_cast<int>(wrow0), glo, glo);
        emit(stg, stg.map, wvalid, ok, hg_row, col + 32, static_cast<int>(wrow0), ghi, ghi);
      }
    }
    if (ok) ssq[static_cast<long long>(c.tn) * (2 * BT) + row] = ss;
  }
};

// Gate/up tile: accumulator columns [0, BN/2) are gate, [BN/2, BN) are up for
// output columns tn*BN/2 + [0, BN/2).  Z = silu(gate) * up, fp32.
// When `rstd` is set, the A operand was h * g and RMSNorm is finished here as
// the row scale rstd[row] on gate and up alike (u W^T = rstd * ((h * g) W^T));
// otherwise A already holds u.
//
// OutT = bf16 writes 64 columns per step (N a multiple of 64).  Output row of
// accumulator row `row` is row - out_row0 (the output may start at a later row
// than A, e.g. the student half of [u_T; u_S]).
template <class OutT = float>
struct EpiSwiGLU {
  static constexpr bool kStaged = true;
  static constexpr bool kCollective = false;
  OutT* out;
  long long ldo;
  int N;  // d_ff
  const float* rstd;  // [rows], nullable
  long long out_row0 = 0;
  __device__ float pre(const TileCtx& c, int r) const {
    return (rstd && r < c.valid_rows) ? __ldg(rstd + c.row0 + r) : 1.f;
  }
  __device__ static void swiglu32(uint32_t taddr, int cc, int half, float rs, float (&z)[32]) {
    float u[32];
    tmem_ld32f(taddr + cc, z);
    tmem_ld32f(taddr + half + cc, u);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float gg = z[i] * rs;
      z[i] = __fdividef(gg, 1.0f + __expf(-gg)) * (u[i] * rs);
    }
  }
  template <int BN>
  __device__ void run(const TileCtx& c, uint32_t taddr, int r, EpiStage& stg, float rs) const {
    constexpr int STEP = sizeof(OutT) == 2 ? 64 : 32;
    const bool ok = r < c.valid_rows;
    const long long row = c.row0 + r - out_row0;
    const int wrow = r & ~31;
    const bool staged = stg.on() && wrow + 32 <= c.valid_rows;
    const int y = static_cast<int>(c.row0 - out_row0) + wrow;
#pragma unroll 1
    for (int cc = 0; cc < BN / 2; cc += STEP) {
      const int col = c.tn * (BN / 2) + cc;
      if (col >= N) break;
      float lo[32], hi[32];
      swiglu32(taddr, cc, BN / 2, rs, lo);
      if constexpr (STEP == 64) swiglu32(taddr, cc + 32, BN / 2, rs, hi);
      emit(stg, staged, ok, out + row * ldo, col, y, lo, hi);
    }
  }
};

// Gate/up with SwiGLU, the two short convs, the value-residual difference and
// the student keys in one epilogue (papernotes.org review "Learning What to
// Remember", 关键设计 3: Zbar_P = conv_P(Z_P), D = Zbar_T - Zbar_S, K =
// l2-norm(Zbar_S); the fast weight reads the raw Z_S, 关键设计 2), on paired
// tiles (PairGeom): accumulator rows 0-63 hold the teacher rows of 64 tokens and
// rows 64-127 the student rows of the same tokens; columns [0, 128) are gate and
// [128, 256) up for output columns tn*128 + [0, 128).
//
// Eight epilogue warps in two groups that pass the tile's four 32-column
// slices through four shared z tiles (16 KB each: [path][row][column] fp32,
// 16-byte slots swizzled by row, so both the row-wise writes and the column
// reads are conflict-free), with one full and one free mbarrier per slice:
//   producers (warps 4-7, thread = accumulator row) form z = silu(rstd g)
//      (rstd u) for each slice and write it to the slice's tile once the
//      consumers have freed it; after the last TMEM read they release the
//      accumulator, so the next-but-one tile's MMAs need not wait for the convs;
//   consumers (warps 8-11, thread = rows R and R + 32 of column group cg of 8
//      columns) form the causal depthwise convs of both paths from the k rows
//      R - k + 1 .. R of the tile (16-byte shared loads; the taps of the 8
//      columns come from a bf16 table [path][f/8][KMAX][8] made once per call,
//      loaded before the slice is waited for), and write 8 columns of
//      D = Zbar_T - Zbar_S and Kp = Zbar_S (padded chunk layout) and of the
//      bf16 Z_S (output-GEMM operand) with one 16-byte store each.  Kp^2
//      accumulates per row; four lanes share a row and reduce once per tile
//      (the key norm becomes a row scale of R).
// The producers run up to one tile ahead of the consumers.  Every wait is a
// bounded mbarrier wait; no named barrier is used, so the tile loop needs no
// collective vote.
// The tile's first k-1 rows only feed the conv (their outputs belong to the
// previous tile); fp32 Z never reaches memory.
//   z_halo [2, B, k-1, f] fp32: Z rows before token 0 (nullable: zeros)
//   z_tail [2, B, k-1, f] fp32: written with the last k-1 rows of Z (nullable)
template <int KMAX>  // conv width k <= KMAX
struct EpiSwiGLUConv {
  static constexpr bool kStaged = true;
  static constexpr bool kCollective = false;
  static constexpr int kWarps = 8;
  static constexpr int kStagingBytes = 4 * 16384;  // the four slice tiles
  static constexpr int kExtraBars = 8;             // slice full [0, 4), slice free [4, 8)
  static constexpr int kExtraBarCount = 128;
  static constexpr bool kSelfRelease = true;
  __nv_bfloat16* D;
  __nv_bfloat16* Kp;
  __nv_bfloat16* Zs;
  float* ssq;          // [ceil(f/128), P]
  const float* rstd;   // [2BT] MLP RMSNorm row scales, nullable (u already normalised)
  const __nv_bfloat16* taps;  // [2][f/8][KMAX][8]: conv_T then conv_S, tap m of column 8c + i
  const float* z_halo;
  float* z_tail;
  int B, T, f, k, C, Cp, Nc;
  long long BT, P;
  DevStatus st;        // where a wait that gives up is recorded

  __device__ float pre(const TileCtx& c, int r) const {
    const int t = c.tok0 + (r & 63);
    if (!rstd || t < 0 || t >= T) return 1.f;
    return __ldg(rstd + (r < 64 ? 0 : BT) + static_cast<long long>(c.group) * T + t);
  }
  // padded index of token t of sequence b in the chunk layout of D, Kp, R
  __device__ long long pidx(int b, int t) const {
    return (static_cast<long long>(b) * Nc + t / C) * Cp + t % C;
  }

  template <int BN>
  __device__ void run(const TileCtx& c, uint32_t taddr, int r, EpiStage& stg, float rs) const {
    static_assert(BN == 256, "gate/up tiles are 128 gate + 128 up columns");
    const int et = static_cast<int>(threadIdx.x) - 128;  // epilogue thread 0..255 (warps 4-11)
    const uint32_t par = stg.tiles & 1;                  // each slice barrier completes once per tile
    ++stg.tiles;
    uint64_t* full = stg.xbars;
    uint64_t* freed = stg.xbars + 4;
    uint8_t* tiles = stg.buf - ((et >> 5) & 3) * 8192;  // the 64 KB slice-tile area
    const int b = c.group;
    const int H = k - 1;
    const int nslice = min(4, (f - c.tn * 128) / 32);  // f is a multiple of 64
    volatile int no_abort = 0;
    if (et < 128) {
      // ------------------------------------------------------------ producers
      const int rin = r & 63;
      const int path = r >= 64 ? 1 : 0;
      const int ta = c.tok0 + rin;
      const int R = path * 64 + rin;
#pragma unroll 1
      for (int s = 0; s < 4; ++s) {
        float z[32];
        const int col0 = c.tn * 128 + 32 * s;
        if (s < nslice) {
          float gt[32], up[32];
          tmem_ld32f(taddr + 32 * s, gt);
          tmem_ld32f(taddr + 128 + 32 * s, up);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float gg = gt[i] * rs;
            z[i] = __fdividef(gg, 1.0f + __expf(-gg)) * (up[i] * rs);
          }
          if (ta < 0 || ta >= T) {
            if (ta < 0 && z_halo) {
              load_x32(z_halo + ((static_cast<long long>(path) * B + b) * H + (ta + H)) * f + col0, z);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) z[i] = 0.f;
            }
          }
          if (z_tail && rin >= H && ta >= T - H && ta < T && ta >= 0)
            store_f32x32(z_tail + ((static_cast<long long>(path) * B + b) * H + (ta - (T - H))) * f + col0, z);
        }
        if (s == nslice - 1) {  // the accumulator has been read: release it
          tc_fence_before();
          mbar_arrive(stg.release);
        }
        mbar_wait(&freed[s], par ^ 1, st, &no_abort);
        if (s < nslice) {
          uint8_t* tile = tiles + s * 16384;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(tile + R * 128 + ((j ^ (R & 7)) << 4)) =
                make_float4(z[4 * j], z[4 * j + 1], z[4 * j + 2], z[4 * j + 3]);
        }
        mbar_arrive(&full[s]);
      }
      return;
    }
    // -------------------------------------------------------------- consumers
    mbar_arrive(stg.release);  // consumers never touch the accumulator
    const int ec = et - 128;
    const int cg = ec & 3;
    int brow[2];
    bool bval[2];
    long long bp[2], bz[2];
    float ssq_acc[2] = {0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      brow[u] = (ec >> 2) + 32 * u;
      const int t = c.tok0 + brow[u];
      bval[u] = brow[u] >= H && t >= 0 && t < T;
      const int tt = bval[u] ? t : 0;
      bp[u] = pidx(b, tt) * f;
      bz[u] = (static_cast<long long>(b) * T + tt) * f;
    }
#pragma unroll 1
    for (int s = 0; s < 4; ++s) {
      const int col = c.tn * 128 + 32 * s + 8 * cg;
      uint4 tw[2][KMAX];
      if (s < nslice) {
        const uint4* src = reinterpret_cast<const uint4*>(taps) + static_cast<long long>(col >> 3) * KMAX;
#pragma unroll
        for (int m = 0; m < KMAX; ++m) {
          tw[0][m] = m < k ? __ldg(src + m) : make_uint4(0u, 0u, 0u, 0u);
          tw[1][m] = m < k ? __ldg(src + static_cast<long long>(f / 8) * KMAX + m)
                           : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      mbar_wait(&full[s], par, st, &no_abort);
      if (s < nslice) {
        const uint8_t* tile = tiles + s * 16384;
        float aT[2][8], aS[2][8], z0[2][8];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int i = 0; i < 8; ++i) { aT[u][i] = 0.f; aS[u][i] = 0.f; z0[u][i] = 0.f; }
#pragma unroll
        for (int m = 0; m < KMAX; ++m) {  // tap m multiplies position t - m
          if (m >= k) break;
          float wT[8], wS[8];
          {
            const uint32_t uT[4] = {tw[0][m].x, tw[0][m].y, tw[0][m].z, tw[0][m].w};
            const uint32_t uS[4] = {tw[1][m].x, tw[1][m].y, tw[1][m].z, tw[1][m].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              wT[2 * i] = bf16lo_to_f32(uT[i]);
              wT[2 * i + 1] = bf16hi_to_f32(uT[i]);
              wS[2 * i] = bf16lo_to_f32(uS[i]);
              wS[2 * i + 1] = bf16hi_to_f32(uS[i]);
            }
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int RT = brow[u] - m, RS = 64 + brow[u] - m;
            if (RT < 0) continue;
            float zt[8], zs[8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int j = 2 * cg + h;
              const float4 x = *reinterpret_cast<const float4*>(tile + RT * 128 + ((j ^ (RT & 7)) << 4));
              const float4 y = *reinterpret_cast<const float4*>(tile + RS * 128 + ((j ^ (RS & 7)) << 4));
              zt[4 * h] = x.x; zt[4 * h + 1] = x.y; zt[4 * h + 2] = x.z; zt[4 * h + 3] = x.w;
              zs[4 * h] = y.x; zs[4 * h + 1] = y.y; zs[4 * h + 2] = y.z; zs[4 * h + 3] = y.w;
            }
            if (m == 0) {
#pragma unroll
              for (int i = 0; i < 8; ++i) z0[u][i] = zs[i];
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              aT[u][i] = fmaf(wT[i], zt[i], aT[u][i]);
              aS[u][i] = fmaf(wS[i], zs[i], aS[u][i]);
            }
          }
        }
        // the slice's reads are done: the producers may refill it
        mbar_arrive(&freed[s]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (!bval[u]) continue;
          float dd[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            dd[i] = aT[u][i] - aS[u][i];
            ssq_acc[u] = fmaf(aS[u][i], aS[u][i], ssq_acc[u]);
          }
          st8f(D + bp[u] + col, dd);
          st8f(Kp + bp[u] + col, aS[u]);
          st8f(Zs + bz[u] + col, z0[u]);
        }
      } else {
        mbar_arrive(&freed[s]);
      }
    }
    // per-token sums of Kp^2 over the tile's columns: the four lanes of a row
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float v = ssq_acc[u];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      if (cg == 0 && bval[u]) ssq[static_cast<long long>(c.tn) * P + pidx(b, c.tok0 + brow[u])] = v;
    }
  }
};

// taps[path][c / 8][m][c % 8] = conv_path[c, m] (bf16, zero for m >= k): the
// table the gate/up conv epilogue reads, 8 columns of one tap per 16 bytes.
template <int KMAX>
__global__ void conv_tap_table_kernel(const __nv_bfloat16* __restrict__ conv_T,
                                      const __nv_bfloat16* __restrict__ conv_S,
                                      __nv_bfloat16* __restrict__ taps, int f, int k) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= 2 * f * KMAX) return;
  const int path = idx / (f * KMAX);
  const int e = idx % (f * KMAX);
  const int c8 = e / (KMAX * 8), m = (e / 8) % KMAX, ci = e % 8;
  const int col = c8 * 8 + ci;
  const __nv_bfloat16* w = path ? conv_S : conv_T;
  taps[idx] = m < k ? w[static_cast<long long>(col) * k + m] : __float2bfloat16_rn(0.f);
}

// QKV projection with rotary embedding on the query and key heads, written to
// one token-major tensor qkv [rows, (Hq + 2 Hkv) HD]: q heads, then k heads,
// then v heads (column n of the accumulator is column n of qkv).  Each head's
// HD columns are rotated in registers (pairs i, i + HD/2) and leave through the
// staged TMA store in 64-column pieces.
template <int HD>
struct EpiQKVRope {
  static constexpr bool kStaged = true;
  static constexpr bool kCollective = false;
  static constexpr int NF = HD / 2;  // rotation frequencies
  __nv_bfloat16* qkv;
  int ld;         // (Hq + 2 Hkv) * HD
  int n_rope;     // (Hq + Hkv) * HD: columns that get the rotation
  int T;
  const __half2* rope_cs;  // [HD/2][T] (cos, sin), frequency-major
  const float* rstd;       // [rows] input RMSNorm row scale (the gain is in the weight), nullable
  // Rows reserved before each sequence's rows in qkv (a sequence shard's K/V
  // halo): output row = row + (b + 1) * row_shift for sequence b = tile group
  // (tiles must not straddle sequences when it is nonzero).
  int row_shift;
  __device__ float pre(const TileCtx& c, int r) const {
    return (rstd && r < c.valid_rows) ? __ldg(rstd + c.row0 + r) : 1.f;
  }

  // (x_i, x_{i+NF}) -> (x_i c - x_{i+NF} s, x_{i+NF} c + x_i s) for NF frequencies
  // starting at f0, in place.
  template <int N>
  __device__ static void rotate(float* a, float* b, const uint32_t* tab, int f0, int T) {
    uint32_t cs[N];
#pragma unroll
    for (int i = 0; i < N; ++i) cs[i] = __ldg(tab + static_cast<long long>(f0 + i) * T);
#pragma unroll
    for (int i = 0; i < N; ++i) {
      __half2 h;
      memcpy(&h, &cs[i], 4);
      const float2 e = __half22float2(h);
      const float x = a[i], y = b[i];
      a[i] = x * e.x - y * e.y;
      b[i] = y * e.x + x * e.y;
    }
  }

  template <int BN>
  __device__ void run(const TileCtx& c, uint32_t taddr, int r, EpiStage& stg, float rs) const {
    static_assert(BN % 64 == 0 && BN % HD == 0, "column tile must hold whole heads");
    const bool ok = r < c.valid_rows;
    const long long row = c.row0 + r;
    const int shift = (c.group + 1) * row_shift;
    const int wrow = r & ~31;
    const bool staged = stg.on() && wrow + 32 <= c.valid_rows;
    const int t = static_cast<int>(row % T);
    const int tcol = c.tn * BN;
    const uint32_t* tab = reinterpret_cast<const uint32_t*>(rope_cs) + t;
    // Rotate the q/k heads of the tile in place in TMEM, 32-column slices at a
    // time (few live registers), then emit the tile as plain rows.
    if (tcol < n_rope) {
#pragma unroll 1
      for (int h0 = 0; h0 < BN; h0 += HD) {
        if (tcol + h0 >= n_rope) break;
        const uint32_t th = taddr + h0;
        if constexpr (HD == 32) {
          uint32_t raw[32];
          tmem_ld32(th, raw);
          tmem_ld_wait();
          float* x = reinterpret_cast<float*>(raw);
          rotate<16>(x, x + 16, tab, 0, T);
          tmem_st32(th, raw);
        } else {
#pragma unroll 1
          for (int q = 0; q < NF; q += 32) {
            uint32_t ra[32], rb[32];
            tmem_ld32(th + q, ra);
            tmem_ld32(th + NF + q, rb);
            tmem_ld_wait();
            rotate<32>(reinterpret_cast<float*>(ra), reinterpret_cast<float*>(rb), tab, q, T);
            tmem_st32(th + q, ra);
            tmem_st32(th + NF + q, rb);
          }
        }
      }
      tmem_st_wait();
    }
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 64) {
      if (tcol + cc >= ld) break;
      float lo[32], hi[32];
      tmem_ld32f(taddr + cc, lo);
      tmem_ld32f(taddr + cc + 32, hi);
#pragma unroll
      for (int i = 0; i < 32; ++i) {  // the rotation is linear: the row scale commutes with it
        lo[i] *= rs;
        hi[i] *= rs;
      }
      emit(stg, staged, ok, qkv + (row + shift) * ld, tcol + cc, c.row0 + wrow + shift, lo, hi);
    }
  }
};

}  // namespace ttcd
