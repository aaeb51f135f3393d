// libttcd: host side of the C ABI declared in include/ttcd.h.
//
// Argument validation, workspace carving, TMA tensor-map construction and the
// launch sequence of the IP-TTCD block forward.  Every step of the path runs in
// the kernels included below; the host only marshals pointers and sizes.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/ttcd.h"
#include "attention.cuh"
#include "elementwise.cuh"
#include "gemm.cuh"
#include "ptx.cuh"
#include "scan.cuh"
#include "decode.cuh"
#include "backward.cuh"
#include "attention_bwd.cuh"

using namespace ttcd;

// ------------------------------------------------------------------ device state
// Status word of the entry points that take no workspace (the two attention
// calls, the MLP without caller scratch, the bounded-wait self-test without a
// status region): one per device, shared by every caller of those entry points.
// Entry points with a workspace or a decode state keep their status word in its
// first bytes instead (kStatusBytes), so concurrent callers never see each
// other's timeouts.
__device__ uint32_t g_ttcd_err;

namespace {

constexpr size_t kStatusBytes = TTCD_STATUS_BYTES;

constexpr int kMaxDevices = 64;
uint64_t g_timeout_ns = 2000000000ull;
std::mutex g_mu;
uint32_t* g_err_ptr[kMaxDevices] = {nullptr};
int g_num_sms[kMaxDevices] = {0};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool init_device(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ttcd_err) != cudaSuccess) return false;
    g_err_ptr[dev] = static_cast<uint32_t*>(p);
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    g_num_sms[dev] = n;
  }
  return true;
}

constexpr int kMaxStageEvents = 16;

// Everything one call needs to launch: device, stream, where its kernels record
// a timeout, and (profiled calls only) the caller's stage-boundary events.
struct Ctx {
  int dev;
  cudaStream_t s;
  DevStatus st;
  int sms;
  cudaEvent_t const* events;
  int n_events;
};

// `status` is the call's status word (the first word of its workspace or decode
// state), or null for the per-device word of the entry points without one.
ttcd_status make_ctx(void* stream, Ctx& c, void* status = nullptr) {
  if (cudaGetDevice(&c.dev) != cudaSuccess) return TTCD_ERR_CUDA;
  if (!init_device(c.dev)) return TTCD_ERR_CUDA;
  c.s = static_cast<cudaStream_t>(stream);
  c.st.err = status ? static_cast<uint32_t*>(status) : g_err_ptr[c.dev];
  c.st.timeout_ns = g_timeout_ns;
  c.sms = g_num_sms[c.dev];
  c.events = nullptr;
  c.n_events = 0;
  return TTCD_OK;
}

// Records the caller's stage-boundary event `k` on the call's stream (profiled
// calls only).  A failed record is not a launch error: it is cleared and skipped.
void stage_mark(const Ctx& c, int k) {
  if (k < c.n_events && cudaEventRecord(c.events[k], c.s) != cudaSuccess) cudaGetLastError();
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 2-D tensor map of element type E (bf16 or fp32): `outer` rows of `inner`
// elements, row pitch in bytes, box of box_inner x box_outer elements,
// 128-byte swizzle.
template <class E>
bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      sizeof(E) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
// Row-major [rows, cols] operand; the box spans one 128-byte swizzle row of K.
template <class E>
bool map_rows(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return make_map<E>(m, ptr, cols, rows, cols * sizeof(E), ElemTraits<E>::BK, box_rows);
}

// Kernels that move registers between warp groups with setmaxnreg: a group's
// setmaxnreg.inc waits until the registers it asks for are free in the block's
// launch allocation, so the split must fit in (launch registers x threads) or
// the block never proceeds.  The split of each such kernel, in registers per
// block, is checked against the compiled launch count before every launch.
struct RegSplit {
  int threads_low, regs_low;    // warps that give registers back (setmaxnreg.dec)
  int threads_high, regs_high;  // warps that take them (setmaxnreg.inc)
};
constexpr RegSplit kAttnRegSplit{128, 56, 256, 224};  // dual_window_attn_kernel
constexpr RegSplit kScanRegSplit{128, 56, 256, 224};  // fastweight_scan_kernel
constexpr RegSplit kGemm8RegSplit{128, 56, 256, 224};  // gemm_tc_kernel with 8 epilogue warps
ttcd_status check_reg_split(const void* kern, int threads, const RegSplit& s) {
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return TTCD_ERR_CUDA;
  const long long pool = static_cast<long long>(attr.numRegs) * threads;
  const long long need = static_cast<long long>(s.threads_low) * s.regs_low +
                         static_cast<long long>(s.threads_high) * s.regs_high;
  return need <= pool ? TTCD_OK : TTCD_ERR_UNSUPPORTED;
}

// Process-wide diagnostic counter of kernel launches (atomic; not call state).
std::atomic<unsigned long long> g_launches{0};

#define TTCD_CHECK_LAUNCH()                                      \
  do {                                                           \
    if (cudaGetLastError() != cudaSuccess) return TTCD_ERR_CUDA; \
    g_launches.fetch_add(1, std::memory_order_relaxed);          \
  } while (0)

// Output tensor map for the staged epilogue: boxes of 128 bytes x 32 rows.
template <class OutT>
bool make_out_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols,
                  uint64_t ld_elems) {
  return make_map<OutT>(m, ptr, cols, rows, ld_elems * sizeof(OutT), 128 / sizeof(OutT), 32);
}

// PAIR: CTA pairs on 256-row tiles (plain row tiles, one K-major B whose map
// has BN/2-row boxes), launched as clusters of two.
template <class E, int BN, int STAGES, bool DUAL, class Epi, class Geom = GemmGeom,
          bool B_MN = false, bool PAIR = false>
ttcd_status launch_gemm(const Ctx& c, const CUtensorMap& A, const CUtensorMap& B0,
                        const CUtensorMap& B1, const CUtensorMap* out_map, const Geom& geo,
                        const Epi& epi, const CUtensorMap* out_map2 = nullptr) {
  int total;
  if constexpr (PAIR)
    total = geo.total_pairs();
  else
    total = geo.total();
  if (total <= 0) return TTCD_OK;
  if (Epi::kStaged && !out_map) return TTCD_ERR_INVALID_ARG;
  auto kern = gemm_tc_kernel<E, BN, STAGES, DUAL, Epi, Geom, B_MN, PAIR>;
  constexpr int smem = gemm_smem_bytes_for<Epi, BN, STAGES, PAIR>();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TTCD_ERR_CUDA;
  if constexpr (EpiWarps<Epi>::value == 8) {
    const ttcd_status rs = check_reg_split(reinterpret_cast<const void*>(kern), gemm_threads<Epi>(),
                                           kGemm8RegSplit);
    if (rs != TTCD_OK) return rs;
  }
  const CUtensorMap& o1 = out_map ? *out_map : A;
  const CUtensorMap& o2 = out_map2 ? *out_map2 : A;
  if constexpr (PAIR) {
    const int pairs = total < c.sms / 2 ? total : c.sms / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2u * static_cast<unsigned>(pairs));
    cfg.blockDim = dim3(gemm_threads<Epi>());
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, A, B0, B1, o1, o2, geo, epi, c.st) != cudaSuccess) {
      cudaGetLastError();
      return TTCD_ERR_CUDA;
    }
  } else {
    const int grid = total < c.sms ? total : c.sms;
    kern<<<grid, gemm_threads<Epi>(), smem, c.s>>>(A, B0, B1, o1, o2, geo, epi, c.st);
  }
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

// bf16 GEMMs over plain row tiles with one K-major B run on CTA pairs (256-row
// tiles, 6 stages); their B operand is then mapped in 128-row boxes.
template <class E>
constexpr bool kPairGemm = sizeof(E) == 2;
template <class E>
constexpr uint32_t gemm_b_box() {
  return kPairGemm<E> ? 128u : 256u;
}
template <class E, class Epi>
ttcd_status launch_rows_gemm(const Ctx& c, const CUtensorMap& A, const CUtensorMap& B,
                             const CUtensorMap* out_map, const GemmGeom& geo, const Epi& epi,
                             const CUtensorMap* out_map2 = nullptr) {
  if constexpr (kPairGemm<E>)
    return launch_gemm<E, 256, 6, false, Epi, GemmGeom, false, true>(c, A, B, B, out_map, geo, epi,
                                                                     out_map2);
  else
    return launch_gemm<E, 256, 4, false>(c, A, B, B, out_map, geo, epi, out_map2);
}

// The same with B given transposed (MN-major, bf16): pairs need no change of map.
template <class Epi>
ttcd_status launch_rows_gemm_bmn(const Ctx& c, const CUtensorMap& A, const CUtensorMap& B,
                                 const CUtensorMap* out_map, const GemmGeom& geo, const Epi& epi) {
  return launch_gemm<__nv_bfloat16, 256, 6, false, Epi, GemmGeom, true, true>(c, A, B, B, out_map,
                                                                               geo, epi);
}

GemmGeom plain_geom(long long rows, int N_tiles, int K) {
  GemmGeom g;
  g.n_seq = 1;
  g.T = static_cast<int>(rows);
  g.C = static_cast<int>(rows);
  g.Nc = 1;
  g.K = K;
  g.tiles_m = static_cast<int>((rows + GEMM_BM - 1) / GEMM_BM);
  g.tiles_n = N_tiles;
  g.b_group_rows = 0;
  return g;
}

int cdiv(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

// ------------------------------------------------------------------ validation
ttcd_status check_params(const ttcd_block_params* p) {
  if (!p) return TTCD_ERR_INVALID_ARG;
  if (p->B < 1 || p->T < 1 || p->d_model < 1 || p->n_q_heads < 1 || p->n_kv_heads < 1 ||
      p->d_ff < 1 || p->chunk < 1 || p->w_S < 1 || p->w_T < p->w_S)
    return TTCD_ERR_INVALID_ARG;
  if (p->n_q_heads % p->n_kv_heads != 0) return TTCD_ERR_INVALID_ARG;
  if (p->conv_k < 1 || p->conv_k > 8) return TTCD_ERR_INVALID_ARG;
  if (p->dtype != TTCD_F32 && p->dtype != TTCD_BF16) return TTCD_ERR_INVALID_ARG;
  if (!(p->rms_eps >= 0.f) || !(p->l2_eps >= 0.f) || !(p->rope_theta > 0.f) ||
      !(p->softmax_scale >= 0.f))
    return TTCD_ERR_INVALID_ARG;
  if (p->head_dim != 32 && p->head_dim != 64 && p->head_dim != 128) return TTCD_ERR_UNSUPPORTED;
  if (p->d_model % 64 != 0 || p->d_ff % 64 != 0) return TTCD_ERR_UNSUPPORTED;
  if ((p->n_q_heads + 2 * p->n_kv_heads) * p->head_dim % 64 != 0) return TTCD_ERR_UNSUPPORTED;
  const long long BT = static_cast<long long>(p->B) * p->T;
  if (2 * BT >= (1ll << 31) || static_cast<long long>(p->d_ff) * p->d_model >= (1ll << 31))
    return TTCD_ERR_UNSUPPORTED;
  return TTCD_OK;
}

// ------------------------------------------------------------------ workspace layout
struct Layout {
  size_t off[32];
  size_t total;
};
enum Buf {
  B_STATUS, B_WQKVG, B_RSTDIN, B_QKV, B_O, B_H, B_ROPE, B_U, B_Z, B_ZS16, B_D, B_KP, B_SSQ,
  B_KSCALE, B_R, B_WALL, B_M, B_WPROJT, B_RT, B_KT, B_HSSQ, B_RSTD, B_X32, B_OUT32, B_HS32,
  B_W32, B_QKVX, B_ZH, B_UH, B_TAPS, B_COUNT
};
static_assert(B_COUNT <= 32, "workspace layout table too small");
const char* kBufNames[B_COUNT] = {"status", "wqkv_g", "rstd_in", "qkv", "o", "h", "rope", "u",
                                  "Z", "Zs16", "D", "Kp", "ssq", "kscale", "R", "Wall", "M",
                                  "WprojT", "Rt", "Kt", "hssq", "rstd", "x32", "out32", "hS32",
                                  "w32", "qkv_ext", "z_halo", "u_halo", "taps"};

// bf16 problems shorter than one chunk run with fp32 operands (kind::tf32 MMAs):
// their fast-weight state is the sum of fewer than C rank-1 writes, so the bf16
// rounding of the MLP input and of D, M, R, K' does not average out over the
// chunk.  Inputs and weights are widened exactly into the workspace, the output
// is rounded back to bf16 once.
bool wide_mode(const ttcd_block_params* p) { return p->dtype == TTCD_BF16 && p->T < p->chunk; }

// fp32 copies of the weights for the wide route, in ttcd_block_weights order.
struct W32Layout {
  size_t off[10];
  size_t total;
};
W32Layout w32_layout(const ttcd_block_params* p) {
  const size_t d = p->d_model, f = p->d_ff, hd = p->head_dim;
  const size_t dqkv = (p->n_q_heads + 2 * p->n_kv_heads) * hd, dq = p->n_q_heads * hd;
  const size_t n[10] = {dqkv * d, d * dq, d, d, f * d, f * d, d * f, f * f,
                        f * p->conv_k, f * p->conv_k};
  W32Layout L;
  size_t o = 0;
  for (int i = 0; i < 10; ++i) {
    L.off[i] = o;
    o += (n[i] * 4 + 255) / 256 * 256;
  }
  L.total = o;
  return L;
}

struct Dims {
  long long BT, P;
  int Nc, Cp, d, f, Hq, Hkv, hd, dqkv;
};
Dims dims_of(const ttcd_block_params* p) {
  Dims m;
  m.BT = static_cast<long long>(p->B) * p->T;
  m.Nc = (p->T + p->chunk - 1) / p->chunk;
  m.Cp = (p->chunk + 63) / 64 * 64;
  m.P = static_cast<long long>(p->B) * m.Nc * m.Cp;
  m.d = p->d_model;
  m.f = p->d_ff;
  m.Hq = p->n_q_heads;
  m.Hkv = p->n_kv_heads;
  m.hd = p->head_dim;
  m.dqkv = (m.Hq + 2 * m.Hkv) * m.hd;
  return m;
}

// Operand buffers hold bf16 for TTCD_BF16 and fp32 (tf32 tensor-core operands)
// for TTCD_F32 and the wide route; q, k, v stay bf16 (the attention kernel takes
// bf16).  The status word comes first in every workspace.
Layout make_layout(const ttcd_block_params* p, bool block, bool shard = false,
                   bool allow_wide = true) {
  const Dims m = dims_of(p);
  size_t sz[B_COUNT] = {0};
  const bool wide = allow_wide && !shard && wide_mode(p);
  const size_t e = (p->dtype == TTCD_F32 || wide) ? 4 : 2;
  sz[B_STATUS] = kStatusBytes;
  if (block) {
    sz[B_WQKVG] = static_cast<size_t>(m.dqkv) * m.d * e;  // W_qkv diag(g_attn)
    sz[B_RSTDIN] = m.BT * 4;                              // input RMSNorm row scales
    sz[B_QKV] = m.BT * m.dqkv * 2;
    sz[B_O] = 2 * m.BT * m.Hq * m.hd * e;
    sz[B_H] = m.BT * m.d * 4;                        // student residual stream, fp32
    sz[B_HSSQ] = static_cast<size_t>(cdiv(m.d, 256)) * 2 * m.BT * 4;  // RMSNorm partial sums
    sz[B_RSTD] = 2 * m.BT * 4;                                           // RMSNorm row scales
    sz[B_ROPE] = static_cast<size_t>(p->T) * (m.hd / 2) * 4;
  }
  sz[B_U] = 2 * m.BT * m.d * e;
  sz[B_Z] = e == 4 ? 2 * m.BT * m.f * 4 : 0;  // bf16: Z stays on chip (fused gate/up + conv)
  sz[B_ZS16] = e == 2 ? m.BT * m.f * 2 : 0;  // fp32 mode reads Z_S directly
  sz[B_TAPS] = e == 2 ? 2 * static_cast<size_t>(m.f) * 8 * 2 : 0;  // bf16 conv tap table
  sz[B_D] = m.P * m.f * e;
  sz[B_KP] = m.P * m.f * e;
  sz[B_SSQ] = m.P * 4 * (m.f / 64);
  sz[B_KSCALE] = m.P * 4;
  sz[B_R] = m.P * m.d * e;
  sz[B_WALL] = static_cast<size_t>(p->B) * m.Nc * m.d * m.f * e;
  sz[B_M] = static_cast<size_t>(m.d) * m.f * e;
  sz[B_WPROJT] = e == 4 ? static_cast<size_t>(m.f) * m.f * e : 0;  // bf16 reads W_proj MN-major
  if (e == 4) {  // tf32 operands stay K-major: transposed copies for the chunk scan
    sz[B_RT] = m.P * m.d * e;
    sz[B_KT] = m.P * m.f * e;
  }
  if (shard) {  // sequence shard: qkv with room for the K/V halo, conv history
    const size_t H = static_cast<size_t>(p->conv_k - 1);
    sz[B_QKV] = 0;
    sz[B_QKVX] = static_cast<size_t>(p->B) * (p->w_T - 1 + p->T) * m.dqkv * 2;
    sz[B_ZH] = 2 * static_cast<size_t>(p->B) * H * m.f * 4;
    sz[B_UH] = 2 * static_cast<size_t>(p->B) * H * m.d * e;
  }
  if (wide) {  // fp32 copies of the bf16 interface tensors
    if (block) sz[B_X32] = m.BT * m.d * 4;
    else sz[B_HS32] = m.BT * m.d * 4;
    sz[B_OUT32] = m.BT * m.d * 4;
    sz[B_W32] = w32_layout(p).total;
  }
  Layout L;
  size_t o = 0;
  for (int i = 0; i < B_COUNT; ++i) {
    L.off[i] = o;
    o += (sz[i] + 1023) / 1024 * 1024;
  }
  L.total = o;
  return L;
}

template <class T>
T* at(void* ws, const Layout& L, Buf b) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + L.off[b]);
}

#define TTCD_TRY(x)                    \
  do {                                 \
    ttcd_status _s = (x);              \
    if (_s != TTCD_OK) return _s;      \
  } while (0)

// ------------------------------------------------------------------ attention
// q rows have `ld_q` elements between tokens, k and v rows `ld_kv` (equal to
// Hq*HD / Hkv*HD for separate tensors, or the qkv width for one packed tensor).
template <int HD, class OutT, bool SPLIT = false>
ttcd_status launch_attn(const Ctx& c, const void* q, const void* k, const void* v, OutT* o_T,
                        OutT* o_S, float* lse_T, float* lse_S, int B, int T, int Hq, int Hkv,
                        int w_S, int w_T, float scale, long long ld_q, long long ld_kv,
                        OutT* o_far = nullptr, float* lse_far = nullptr, int q_begin = 0) {
  CUtensorMap mq, mk, mv;
  const long long BT = static_cast<long long>(B) * T;
  using bf = __nv_bfloat16;
  if (!make_map<bf>(&mq, q, static_cast<uint64_t>(Hq) * HD, BT, ld_q * 2, 64, 128) ||
      !make_map<bf>(&mk, k, static_cast<uint64_t>(Hkv) * HD, BT, ld_kv * 2, 64, 128) ||
      !make_map<bf>(&mv, v, static_cast<uint64_t>(Hkv) * HD, BT, ld_kv * 2, 64, 128))
    return TTCD_ERR_CUDA;
  AttnArgs<OutT> a;
  a.o_T = o_T;
  a.o_S = o_S;
  a.lse_T = lse_T;
  a.lse_S = lse_S;
  a.o_far = o_far;
  a.lse_far = lse_far;
  a.B = B;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.w_S = w_S;
  a.w_T = w_T;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.n_qt = (T + ATT_BM - 1) / ATT_BM;
  a.pairs = (Hq / Hkv + 1) / 2;
  a.q_begin = q_begin;
  if (q_begin < 0 || q_begin >= T) return TTCD_ERR_INVALID_ARG;
  auto kern = dual_window_attn_kernel<HD, OutT, SPLIT>;
  constexpr int smem = AttnCfg<HD>::SMEM;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TTCD_ERR_CUDA;
  const long long grid =
      static_cast<long long>(a.n_qt - q_begin / ATT_BM) * B * Hkv * a.pairs;
  if (grid >= (1ll << 31)) return TTCD_ERR_UNSUPPORTED;
  TTCD_TRY(check_reg_split(reinterpret_cast<const void*>(kern), ATT_THREADS, kAttnRegSplit));
  kern<<<static_cast<unsigned>(grid), ATT_THREADS, smem, c.s>>>(mq, mk, mv, a, c.st);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

template <class OutT>
ttcd_status run_attn(const Ctx& c, const void* q, const void* k, const void* v, OutT* o_T,
                     OutT* o_S, float* lse_T, float* lse_S, int B, int T, int Hq, int Hkv, int hd,
                     int w_S, int w_T, float scale, long long ld_q, long long ld_kv,
                     int q_begin = 0) {
  switch (hd) {
    case 32: return launch_attn<32>(c, q, k, v, o_T, o_S, lse_T, lse_S, B, T, Hq, Hkv, w_S, w_T, scale, ld_q, ld_kv, static_cast<OutT*>(nullptr), nullptr, q_begin);
    case 64: return launch_attn<64>(c, q, k, v, o_T, o_S, lse_T, lse_S, B, T, Hq, Hkv, w_S, w_T, scale, ld_q, ld_kv, static_cast<OutT*>(nullptr), nullptr, q_begin);
    case 128: return launch_attn<128>(c, q, k, v, o_T, o_S, lse_T, lse_S, B, T, Hq, Hkv, w_S, w_T, scale, ld_q, ld_kv, static_cast<OutT*>(nullptr), nullptr, q_begin);
    default: return TTCD_ERR_UNSUPPORTED;
  }
}

// The LSE-combination form: the split kernel gives o_S, lse_S and the far band
// (o_far, lse_far); the merge kernel combines them into o_T (and lse_T).
template <int HD>
ttcd_status launch_attn_lse(const Ctx& c, const void* q, const void* k, const void* v,
                            __nv_bfloat16* o_T, __nv_bfloat16* o_S, __nv_bfloat16* o_far,
                            float* lse_T, float* lse_S, float* lse_far, int B, int T, int Hq,
                            int Hkv, int w_S, int w_T, float scale) {
  TTCD_TRY((launch_attn<HD, __nv_bfloat16, true>(c, q, k, v, nullptr, o_S, nullptr, lse_S, B, T,
                                                 Hq, Hkv, w_S, w_T, scale,
                                                 static_cast<long long>(Hq) * HD,
                                                 static_cast<long long>(Hkv) * HD, o_far, lse_far)));
  const long long rows = static_cast<long long>(B) * T * Hq;
  const long long threads = rows * (HD / 8);
  lse_merge_kernel<HD, __nv_bfloat16><<<static_cast<unsigned>(cdiv(threads, 256)), 256, 0, c.s>>>(
      o_S, lse_S, o_far, lse_far, o_T, lse_T, T, Hq, rows);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

// ------------------------------------------------------------------ fast-weight MLP body
// u (operand type E, [2BT, d], teacher rows first) is already in the workspace.
// With `hssq` set, u holds h * g_mlp and RMSNorm is finished as a row scale in
// the gate/up epilogue, from the partial sums of squares hssq [n_part, 2BT]
// reduced to one 1/rms per row first.
// Front half of the fast-weight MLP: from u (operand type E, [2BT, d], teacher
// rows first, already in the workspace) to D, the keys and R.  When `rstd` is
// set, u holds h * g_mlp and the MLP RMSNorm is finished as the row scale rstd
// in the gate/up epilogue.  `z_halo` (bf16 operands only, nullable): Z_T, Z_S of
// the conv_k - 1 tokens before token 0 ([2, B, conv_k-1, f] fp32; a sequence
// shard's conv history), zeros when null.
template <class E>
ttcd_status mlp_front(const Ctx& c, const ttcd_block_params* p, const Layout& L, void* ws,
                      const E* w_gate, const E* w_up, const E* w_down, const E* w_proj,
                      const E* conv_T, const E* conv_S, const float* beta, int mark,
                      const float* rstd, const float* z_halo) {
  const Dims m = dims_of(p);
  E* u = at<E>(ws, L, B_U);
  float* Z = at<float>(ws, L, B_Z);
  E* Zs = sizeof(E) == 2 ? at<E>(ws, L, B_ZS16) : nullptr;
  E* D = at<E>(ws, L, B_D);
  E* Kp = at<E>(ws, L, B_KP);
  float* ssq = at<float>(ws, L, B_SSQ);
  float* kscale = at<float>(ws, L, B_KSCALE);
  E* R = at<E>(ws, L, B_R);
  E* M = at<E>(ws, L, B_M);
  E* WprojT = at<E>(ws, L, B_WPROJT);
  stage_mark(c, mark);

  if constexpr (sizeof(E) == 2) {
    // Z_P = silu(u_P W_gate^T) * (u_P W_up^T) for both paths of the same tokens
    // in one tile, with the convs, D, the unnormalised keys, their sums of
    // squares and the bf16 Z_S in the epilogue (slow weights, off-policy).
    const int H = p->conv_k - 1;
    CUtensorMap mA, mB0, mB1;
    if (!map_rows<E>(&mA, u, 2 * m.BT, m.d, 64) || !map_rows<E>(&mB0, w_gate, m.f, m.d, 128) ||
        !map_rows<E>(&mB1, w_up, m.f, m.d, 128))
      return TTCD_ERR_CUDA;
    PairGeom g;
    g.n_seq = p->B;
    g.T = p->T;
    g.H = H;
    g.K = m.d;
    g.tiles_m = cdiv(p->T, 64 - H);
    g.tiles_n = cdiv(m.f, 128);
    g.half_rows = m.BT;
    __nv_bfloat16* taps = at<__nv_bfloat16>(ws, L, B_TAPS);
    if (p->conv_k <= 4) {
      conv_tap_table_kernel<4><<<cdiv(2 * m.f * 4, 256), 256, 0, c.s>>>(conv_T, conv_S, taps, m.f,
                                                                        p->conv_k);
      TTCD_CHECK_LAUNCH();
      EpiSwiGLUConv<4> e{D, Kp, Zs, ssq, rstd, taps, z_halo, nullptr,
                         p->B, p->T, m.f, p->conv_k, p->chunk, m.Cp, m.Nc, m.BT, m.P, c.st};
      TTCD_TRY((launch_gemm<E, 256, 3, true, EpiSwiGLUConv<4>, PairGeom>(c, mA, mB0, mB1, &mA, g, e)));
    } else {
      conv_tap_table_kernel<8><<<cdiv(2 * m.f * 8, 256), 256, 0, c.s>>>(conv_T, conv_S, taps, m.f,
                                                                        p->conv_k);
      TTCD_CHECK_LAUNCH();
      EpiSwiGLUConv<8> e{D, Kp, Zs, ssq, rstd, taps, z_halo, nullptr,
                         p->B, p->T, m.f, p->conv_k, p->chunk, m.Cp, m.Nc, m.BT, m.P, c.st};
      TTCD_TRY((launch_gemm<E, 256, 3, true, EpiSwiGLUConv<8>, PairGeom>(c, mA, mB0, mB1, &mA, g, e)));
    }
    stage_mark(c, mark + 1);
    if (m.Cp != p->chunk || p->T % p->chunk != 0) {
      const long long n = m.P * (m.f / 8);
      pad_rows_zero_kernel<E><<<static_cast<unsigned>(cdiv(n, 256)), 256, 0, c.s>>>(
          D, Kp, m.f, p->T, p->chunk, m.Cp, m.Nc, m.P);
      TTCD_CHECK_LAUNCH();
    }
    key_scale_kernel<<<cdiv(m.P, 256), 256, 0, c.s>>>(ssq, cdiv(m.f, 128), beta, kscale, p->T,
                                                      p->chunk, m.Cp, m.Nc, m.P, p->l2_eps);
    TTCD_CHECK_LAUNCH();
  } else {
    // fp32 operands (tf32): Z_P = silu(u_P W_gate^T) * (u_P W_up^T) for the stacked
    // paths into fp32 Z, then the conv/residual/key kernel.
    {
      CUtensorMap mA, mB0, mB1;
      if (!map_rows<E>(&mA, u, 2 * m.BT, m.d, 128) || !map_rows<E>(&mB0, w_gate, m.f, m.d, 128) ||
          !map_rows<E>(&mB1, w_up, m.f, m.d, 128))
        return TTCD_ERR_CUDA;
      CUtensorMap mo;
      if (!make_out_map<float>(&mo, Z, 2 * m.BT, m.f, m.f)) return TTCD_ERR_CUDA;
      EpiSwiGLU<float> e{Z, m.f, m.f, rstd};
      TTCD_TRY((launch_gemm<E, 256, 4, true>(c, mA, mB0, mB1, &mo, plain_geom(2 * m.BT, cdiv(m.f, 128), m.d), e)));
    }
    stage_mark(c, mark + 1);
    // Short convs, residual difference, student keys (unnormalised) and their squares.
    {
      dim3 grid(m.f / CONV_TC, static_cast<unsigned>(m.P / CONV_TP));
      if (p->conv_k <= 4)
        conv_residual_key_kernel<E, E, 4><<<grid, 256, 0, c.s>>>(Z, conv_T, conv_S, D, Kp, Zs, ssq,
                                                                 p->T, m.f, p->conv_k, p->chunk,
                                                                 m.Cp, m.Nc, m.BT, m.P);
      else
        conv_residual_key_kernel<E, E, 8><<<grid, 256, 0, c.s>>>(Z, conv_T, conv_S, D, Kp, Zs, ssq,
                                                                 p->T, m.f, p->conv_k, p->chunk,
                                                                 m.Cp, m.Nc, m.BT, m.P);
      TTCD_CHECK_LAUNCH();
      key_scale_kernel<<<cdiv(m.P, 256), 256, 0, c.s>>>(ssq, m.f / CONV_TC, beta, kscale, p->T,
                                                        p->chunk, m.Cp, m.Nc, m.P, p->l2_eps);
      TTCD_CHECK_LAUNCH();
    }
  }
  stage_mark(c, mark + 2);
  // M = W_down W_proj (associativity of W_down (W_proj d_t)).  bf16: W_proj
  // [K = f, N = f] row-major is read as an MN-major operand; fp32 (tf32
  // operands stay K-major): through a transposed copy.
  {
    CUtensorMap mA, mB;
    if (!map_rows<E>(&mA, w_down, m.d, m.f, 128)) return TTCD_ERR_CUDA;
    CUtensorMap mo;
    if (!make_out_map<E>(&mo, M, m.d, m.f, m.f)) return TTCD_ERR_CUDA;
    EpiStore<E> e{M, m.f, m.f, nullptr};
    const GemmGeom g = plain_geom(m.d, cdiv(m.f, 256), m.f);
    if constexpr (sizeof(E) == 2) {
      if (!make_map<E>(&mB, w_proj, m.f, m.f, m.f * sizeof(E), 64, 64)) return TTCD_ERR_CUDA;
      TTCD_TRY((launch_gemm<E, 256, 4, false, EpiStore<E>, GemmGeom, true>(c, mA, mB, mB, &mo, g, e)));
    } else {
      dim3 tb(32, 8), tg(cdiv(m.f, 32), cdiv(m.f, 32));
      transpose_kernel<E, E><<<tg, tb, 0, c.s>>>(w_proj, WprojT, m.f, m.f);
      TTCD_CHECK_LAUNCH();
      if (!map_rows<E>(&mB, WprojT, m.f, m.f, 256)) return TTCD_ERR_CUDA;
      TTCD_TRY((launch_gemm<E, 256, 4, false>(c, mA, mB, mB, &mo, g, e)));
    }
  }
  stage_mark(c, mark + 3);
  // R = D M^T (token-major), each row scaled by beta_t / ||Zbar_S[t]||.
  {
    CUtensorMap mA, mB;
    if (!map_rows<E>(&mA, D, m.P, m.f, 128) || !map_rows<E>(&mB, M, m.d, m.f, gemm_b_box<E>()))
      return TTCD_ERR_CUDA;
    CUtensorMap mo;
    if (!make_out_map<E>(&mo, R, m.P, m.d, m.d)) return TTCD_ERR_CUDA;
    EpiStore<E> e{R, m.d, m.d, kscale};
    TTCD_TRY(launch_rows_gemm<E>(c, mA, mB, &mo, plain_geom(m.P, cdiv(m.d, 256), m.f), e));
  }
  stage_mark(c, mark + 4);
  return TTCD_OK;
}

// The bf16 chunk scan on CTA pairs: `tiles` pair tiles, two CTAs each, launched
// as clusters of two.
ttcd_status launch_scan_pair(const Ctx& c, const CUtensorMap& mR, const CUtensorMap& mK,
                             const ScanArgs<__nv_bfloat16>& a, int tiles) {
  constexpr int STAGES = 5;
  constexpr int smem = scan_smem_bytes<__nv_bfloat16, STAGES, true>();
  auto kern = fastweight_scan_kernel<__nv_bfloat16, STAGES, true, true>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TTCD_ERR_CUDA;
  TTCD_TRY(check_reg_split(reinterpret_cast<const void*>(kern), SCAN_THREADS, kScanRegSplit));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2u * static_cast<unsigned>(tiles));
  cfg.blockDim = dim3(SCAN_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mR, mK, a, c.st) != cudaSuccess) {
    cudaGetLastError();
    return TTCD_ERR_CUDA;
  }
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

// The chunk scan over R and the keys: Delta W_i = R_i^T K'_i, the fp32 exclusive
// prefix S_i from state_in, and (w_all set) W_i = W_down + S_i per chunk.  With
// `whole` set, the padded tokens of each sequence form one chunk: state_out is
// state_in + the sum of all chunk increments (a sequence shard's total).
template <class E>
ttcd_status launch_scan(const Ctx& c, const ttcd_block_params* p, const Layout& L, void* ws,
                        const E* w_down, const float* state_in, float* state_out, E* w_all,
                        bool whole) {
  const Dims m = dims_of(p);
  E* R = at<E>(ws, L, B_R);
  E* Kp = at<E>(ws, L, B_KP);
  {
    CUtensorMap mR, mK;
    constexpr uint32_t BK = ElemTraits<E>::BK;
    constexpr bool MN = sizeof(E) == 2;
    // bf16 with more than one 128-row tile of d: CTA pairs on 256 x 192 tiles.
    const bool pair = MN && m.d > GEMM_BM;
    if (MN) {
      if (!make_map<E>(&mR, R, m.d, m.P, m.d * sizeof(E), BK, BK) ||
          !make_map<E>(&mK, Kp, m.f, m.P, m.f * sizeof(E), BK, BK))
        return TTCD_ERR_CUDA;
    } else {
      E* Rt = at<E>(ws, L, B_RT);
      E* Kt = at<E>(ws, L, B_KT);
      dim3 tb(32, 8);
      transpose_kernel<E, E><<<dim3(cdiv(m.d, 32), cdiv(m.P, 32)), tb, 0, c.s>>>(R, Rt, static_cast<int>(m.P), m.d);
      TTCD_CHECK_LAUNCH();
      transpose_kernel<E, E><<<dim3(cdiv(m.f, 32), cdiv(m.P, 32)), tb, 0, c.s>>>(Kp, Kt, static_cast<int>(m.P), m.f);
      TTCD_CHECK_LAUNCH();
      if (!make_map<E>(&mR, Rt, m.P, m.d, m.P * sizeof(E), BK, 128) ||
          !make_map<E>(&mK, Kt, m.P, m.f, m.P * sizeof(E), BK, SCAN_BN))
        return TTCD_ERR_CUDA;
    }
    ScanArgs<E> a{};
    a.d = m.d;
    a.f = m.f;
    a.Nc = whole ? 1 : m.Nc;
    a.Cp = whole ? m.Nc * m.Cp : m.Cp;
    a.w_down = w_down;
    a.state_in = state_in;
    a.state_out = state_out;
    a.w_all = w_all;
    a.tiles_m = cdiv(m.d, pair ? 2 * GEMM_BM : GEMM_BM);
    a.tiles_n = cdiv(m.f, SCAN_BN);
    a.commit_pos = nullptr;
    a.commit_C = 1;
    if constexpr (MN) {
      if (pair) return launch_scan_pair(c, mR, mK, a, p->B * a.tiles_m * a.tiles_n);
    }
    constexpr int STAGES = 4;
    constexpr int smem = scan_smem_bytes<E, STAGES, false>();
    auto kern = fastweight_scan_kernel<E, STAGES, MN>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return TTCD_ERR_CUDA;
    TTCD_TRY(check_reg_split(reinterpret_cast<const void*>(kern), SCAN_THREADS, kScanRegSplit));
    kern<<<p->B * a.tiles_m * a.tiles_n, SCAN_THREADS, smem, c.s>>>(mR, mK, a, c.st);
    TTCD_CHECK_LAUNCH();
  }
  return TTCD_OK;
}

// Back half of the fast-weight MLP: the chunk scan from state_in, then
// y = h_S + (W_down + S_i) Z_S, one GEMM per chunk with its own weight.
template <class E, class OutT, class ResT>
ttcd_status mlp_back(const Ctx& c, const ttcd_block_params* p, const Layout& L, void* ws,
                     const E* w_down, const float* state_in, float* state_out, const ResT* h_S,
                     OutT* y, int mark) {
  const Dims m = dims_of(p);
  float* Z = at<float>(ws, L, B_Z);
  E* Zs = sizeof(E) == 2 ? at<E>(ws, L, B_ZS16) : nullptr;
  E* Wall = at<E>(ws, L, B_WALL);
  TTCD_TRY(launch_scan<E>(c, p, L, ws, w_down, state_in, state_out, Wall, false));
  stage_mark(c, mark + 5);
  // y = h_S + (W_down + S_i) Z_S, one GEMM per chunk with its own weight.
  {
    CUtensorMap mA, mB;
    const void* zs = Zs ? static_cast<const void*>(Zs) : static_cast<const void*>(Z + m.BT * m.f);
    if (!map_rows<E>(&mA, zs, m.BT, m.f, 128) ||
        !map_rows<E>(&mB, Wall, static_cast<long long>(p->B) * m.Nc * m.d, m.f, gemm_b_box<E>()))
      return TTCD_ERR_CUDA;
    GemmGeom g;
    g.n_seq = p->B;
    g.T = p->T;
    g.C = p->chunk;
    g.Nc = m.Nc;
    g.K = m.f;
    g.tiles_m = cdiv(p->chunk, 128);
    g.tiles_n = cdiv(m.d, 256);
    g.b_group_rows = m.d;
    CUtensorMap mo;
    if (!make_out_map<OutT>(&mo, y, m.BT, m.d, m.d)) return TTCD_ERR_CUDA;
    EpiResidual<OutT, ResT> e{y, m.d, h_S, m.d, m.BT, m.d};
    TTCD_TRY(launch_rows_gemm<E>(c, mA, mB, &mo, g, e));
  }
  stage_mark(c, mark + 6);
  return TTCD_OK;
}

template <class E, class OutT, class ResT>
ttcd_status run_mlp_core(const Ctx& c, const ttcd_block_params* p, const Layout& L, void* ws,
                         const E* w_gate, const E* w_up, const E* w_down, const E* w_proj,
                         const E* conv_T, const E* conv_S, const float* beta,
                         const float* state_in, float* state_out, const ResT* h_S, OutT* y,
                         int mark, const float* rstd) {
  TTCD_TRY(mlp_front<E>(c, p, L, ws, w_gate, w_up, w_down, w_proj, conv_T, conv_S, beta, mark,
                        rstd, nullptr));
  return mlp_back<E, OutT, ResT>(c, p, L, ws, w_down, state_in, state_out, h_S, y, mark);
}

bool weights_ok(const ttcd_block_weights* w, bool block) {
  if (!w) return false;
  const void* need[] = {w->g_mlp, w->w_gate, w->w_up, w->w_down, w->w_proj, w->conv_T, w->conv_S};
  for (const void* q : need)
    if (!aligned16(q)) return false;
  if (block && (!aligned16(w->w_qkv) || !aligned16(w->w_o) || !aligned16(w->g_attn))) return false;
  return true;
}

// Casts n elements (grid-stride) on the call's stream.
template <class InT, class OutT>
ttcd_status launch_cast(const Ctx& c, const void* in, void* out, long long n) {
  if (n <= 0) return TTCD_OK;
  const long long blocks = std::min<long long>(cdiv(n, 256), 8ll * c.sms);
  cast_kernel<InT, OutT><<<static_cast<unsigned>(blocks), 256, 0, c.s>>>(
      static_cast<const InT*>(in), static_cast<OutT*>(out), n);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

// The wide route: exact fp32 copies of the bf16 weights in the workspace, and a
// weight table that points at them.  Weights the call does not use may be null.
ttcd_status widen_weights(const Ctx& c, const ttcd_block_params* p, const ttcd_block_weights* w,
                          void* ws, const Layout& L, ttcd_block_weights* w32) {
  const W32Layout WL = w32_layout(p);
  uint8_t* base = at<uint8_t>(ws, L, B_W32);
  const size_t d = p->d_model, f = p->d_ff, hd = p->head_dim;
  const size_t dqkv = (p->n_q_heads + 2 * p->n_kv_heads) * hd, dq = p->n_q_heads * hd;
  const long long n[10] = {static_cast<long long>(dqkv * d), static_cast<long long>(d * dq),
                           static_cast<long long>(d), static_cast<long long>(d),
                           static_cast<long long>(f * d), static_cast<long long>(f * d),
                           static_cast<long long>(d * f), static_cast<long long>(f * f),
                           static_cast<long long>(f * p->conv_k),
                           static_cast<long long>(f * p->conv_k)};
  const void* src[10] = {w->w_qkv, w->w_o,    w->g_attn, w->g_mlp,  w->w_gate,
                         w->w_up,  w->w_down, w->w_proj, w->conv_T, w->conv_S};
  const void** dst[10] = {&w32->w_qkv, &w32->w_o,    &w32->g_attn, &w32->g_mlp,  &w32->w_gate,
                          &w32->w_up,  &w32->w_down, &w32->w_proj, &w32->conv_T, &w32->conv_S};
  for (int i = 0; i < 10; ++i) {
    *dst[i] = nullptr;
    if (!src[i]) continue;
    *dst[i] = base + WL.off[i];
    TTCD_TRY((launch_cast<__nv_bfloat16, float>(c, src[i], base + WL.off[i], n[i])));
  }
  return TTCD_OK;
}

// Reads the status word at `word` after all work queued on s, and clears it.
ttcd_status read_clear_status(uint32_t* word, cudaStream_t s, uint32_t* flags) {
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return TTCD_ERR_CUDA;
  if (v && cudaMemsetAsync(word, 0, sizeof(v), s) != cudaSuccess) return TTCD_ERR_CUDA;
  if (flags) *flags = v;
  if (v & DEV_ERR_TIMEOUT) return TTCD_ERR_TIMEOUT;
  return v ? TTCD_ERR_CUDA : TTCD_OK;
}

// ttcd_fastweight_mlp with its status word at `status` (null: the per-device word).
ttcd_status mlp_entry(const void* u_T, const void* u_S, const void* h_S, const float* beta,
                      const ttcd_block_weights* w, const ttcd_block_params* p,
                      const float* state_in, float* state_out, void* y, void* workspace,
                      size_t ws_bytes, void* stream, void* status) {
  TTCD_TRY(check_params(p));
  if (!aligned16(u_T) || !aligned16(u_S) || !aligned16(beta) || !aligned16(y) ||
      !weights_ok(w, false) || !aligned16(workspace))
    return TTCD_ERR_INVALID_ARG;
  if ((h_S && !aligned16(h_S)) || (state_in && !aligned16(state_in)) ||
      (state_out && !aligned16(state_out)))
    return TTCD_ERR_INVALID_ARG;
  const Layout L = make_layout(p, false);
  if (ws_bytes < L.total) return TTCD_ERR_WORKSPACE;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, status));
  const Dims m = dims_of(p);
  const long long n_u = m.BT * m.d;
  using bf = __nv_bfloat16;
  if (wide_mode(p)) {
    ttcd_block_weights w32;
    TTCD_TRY(widen_weights(c, p, w, workspace, L, &w32));
    float* u = at<float>(workspace, L, B_U);
    TTCD_TRY((launch_cast<bf, float>(c, u_T, u, n_u)));
    TTCD_TRY((launch_cast<bf, float>(c, u_S, u + n_u, n_u)));
    float* hs = nullptr;
    if (h_S) {
      hs = at<float>(workspace, L, B_HS32);
      TTCD_TRY((launch_cast<bf, float>(c, h_S, hs, n_u)));
    }
    float* y32 = at<float>(workspace, L, B_OUT32);
    TTCD_TRY((run_mlp_core<float, float, float>(
        c, p, L, workspace, static_cast<const float*>(w32.w_gate),
        static_cast<const float*>(w32.w_up), static_cast<const float*>(w32.w_down),
        static_cast<const float*>(w32.w_proj), static_cast<const float*>(w32.conv_T),
        static_cast<const float*>(w32.conv_S), beta, state_in, state_out, hs, y32, 0, nullptr)));
    return launch_cast<float, bf>(c, y32, y, n_u);
  }
  const size_t e = p->dtype == TTCD_F32 ? 4 : 2;
  uint8_t* u = at<uint8_t>(workspace, L, B_U);
  if (cudaMemcpyAsync(u, u_T, n_u * e, cudaMemcpyDeviceToDevice, c.s) != cudaSuccess ||
      cudaMemcpyAsync(u + n_u * e, u_S, n_u * e, cudaMemcpyDeviceToDevice, c.s) != cudaSuccess)
    return TTCD_ERR_CUDA;
  if (p->dtype == TTCD_BF16) {
    return run_mlp_core<bf, bf, bf>(
        c, p, L, workspace, static_cast<const bf*>(w->w_gate), static_cast<const bf*>(w->w_up),
        static_cast<const bf*>(w->w_down), static_cast<const bf*>(w->w_proj),
        static_cast<const bf*>(w->conv_T), static_cast<const bf*>(w->conv_S), beta, state_in,
        state_out, static_cast<const bf*>(h_S), static_cast<bf*>(y), 0, nullptr);
  }
  return run_mlp_core<float, float, float>(
      c, p, L, workspace, static_cast<const float*>(w->w_gate),
      static_cast<const float*>(w->w_up), static_cast<const float*>(w->w_down),
      static_cast<const float*>(w->w_proj), static_cast<const float*>(w->conv_T),
      static_cast<const float*>(w->conv_S), beta, state_in, state_out,
      static_cast<const float*>(h_S), static_cast<float*>(y), 0, nullptr);
}

// S0: rotary table at positions pos0 .., the input RMSNorm as row scales with
// its gain folded into a copy of W_qkv, and the QKV GEMM with RoPE into qkv.
// With n_halo > 0 (a sequence shard), each sequence's rows are preceded by
// n_halo rows reserved for the K/V of the tokens before it, and the GEMM tiles
// keep to one sequence.
template <class E>
ttcd_status block_qkv(const Ctx& c, const E* xin, const ttcd_block_weights* w,
                      const ttcd_block_params* p, void* ws, const Layout& L,
                      __nv_bfloat16* qkv, int n_halo, long long pos0) {
  const Dims m = dims_of(p);
  E* wg = at<E>(ws, L, B_WQKVG);
  float* rstd_in = at<float>(ws, L, B_RSTDIN);
  __half2* rope = at<__half2>(ws, L, B_ROPE);
  stage_mark(c, 0);
  rope_table_kernel<<<cdiv(static_cast<long long>(p->T) * (m.hd / 2), 256), 256, 0, c.s>>>(
      rope, p->T, m.hd, std::log2(static_cast<double>(p->rope_theta)), pos0);
  TTCD_CHECK_LAUNCH();
  rms_rowscale_kernel<E><<<cdiv(m.BT, 8), 256, 0, c.s>>>(xin, rstd_in, m.BT, m.d, p->rms_eps);
  TTCD_CHECK_LAUNCH();
  {
    const long long n8 = static_cast<long long>(m.dqkv) * m.d / 8;
    scale_cols_kernel<E><<<cdiv(n8, 256), 256, 0, c.s>>>(
        static_cast<const E*>(w->w_qkv), static_cast<const E*>(w->g_attn), wg, n8, m.d);
    TTCD_CHECK_LAUNCH();
  }
  stage_mark(c, 1);
  CUtensorMap mA, mB;
  if (!map_rows<E>(&mA, xin, m.BT, m.d, 128) || !map_rows<E>(&mB, wg, m.dqkv, m.d, gemm_b_box<E>()))
    return TTCD_ERR_CUDA;
  GemmGeom g = plain_geom(m.BT, cdiv(m.dqkv, 256), m.d);
  if (n_halo > 0) {  // one row group per sequence
    g.n_seq = p->B;
    g.T = p->T;
    g.C = p->T;
    g.tiles_m = cdiv(p->T, GEMM_BM);
  }
  CUtensorMap mo;
  const long long rows_out = m.BT + static_cast<long long>(p->B) * n_halo;
  if (!make_out_map<__nv_bfloat16>(&mo, qkv, rows_out, m.dqkv, m.dqkv)) return TTCD_ERR_CUDA;
  const int n_rope = (m.Hq + m.Hkv) * m.hd;
  switch (m.hd) {
    case 32: TTCD_TRY(launch_rows_gemm<E>(c, mA, mB, &mo, g, EpiQKVRope<32>{qkv, m.dqkv, n_rope, p->T, rope, rstd_in, n_halo})); break;
    case 64: TTCD_TRY(launch_rows_gemm<E>(c, mA, mB, &mo, g, EpiQKVRope<64>{qkv, m.dqkv, n_rope, p->T, rope, rstd_in, n_halo})); break;
    default: TTCD_TRY(launch_rows_gemm<E>(c, mA, mB, &mo, g, EpiQKVRope<128>{qkv, m.dqkv, n_rope, p->T, rope, rstd_in, n_halo})); break;
  }
  stage_mark(c, 2);
  return TTCD_OK;
}

// S1-S2b: dual-window attention of each sequence's T rows over keys that start
// n_halo rows earlier (qkv as block_qkv left it), o_proj of both paths with the
// residual, and the MLP RMSNorm row scales.
template <class E>
ttcd_status block_attend(const Ctx& c, const E* xin, const ttcd_block_weights* w,
                         const ttcd_block_params* p, void* ws, const Layout& L,
                         const __nv_bfloat16* qkv, int n_halo) {
  const Dims m = dims_of(p);
  E* o = at<E>(ws, L, B_O);
  float* h = at<float>(ws, L, B_H);
  E* u = at<E>(ws, L, B_U);
  float* hssq = at<float>(ws, L, B_HSSQ);
  // Dual-window attention: o_T rows then o_S rows.
  const float sc = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(m.hd));
  TTCD_TRY(run_attn<E>(c, qkv, qkv + static_cast<long long>(m.Hq) * m.hd,
                       qkv + static_cast<long long>(m.Hq + m.Hkv) * m.hd, o,
                       o + m.BT * m.Hq * m.hd, nullptr, nullptr, p->B, p->T + n_halo, m.Hq,
                       m.Hkv, m.hd, p->w_S, p->w_T, sc, m.dqkv, m.dqkv, n_halo));
  stage_mark(c, 3);
  // h_P = x + o_P W_o^T (fp32), both paths in one GEMM.
  {
    CUtensorMap mA, mB;
    if (!map_rows<E>(&mA, o, 2 * m.BT, static_cast<long long>(m.Hq) * m.hd, 128) ||
        !map_rows<E>(&mB, w->w_o, m.d, static_cast<long long>(m.Hq) * m.hd, gemm_b_box<E>()))
      return TTCD_ERR_CUDA;
    const GemmGeom g = plain_geom(2 * m.BT, cdiv(m.d, 256), m.Hq * m.hd);
    // h_P = x + o_P W_o^T; stores h * g_mlp (gate/up operand), the student
    // h in fp32, and per-tile sums of h^2 for the MLP RMSNorm.
    CUtensorMap mo, mo2;
    if (!make_out_map<E>(&mo, u, 2 * m.BT, m.d, m.d) ||
        !make_out_map<float>(&mo2, h, m.BT, m.d, m.d))
      return TTCD_ERR_CUDA;
    EpiOprojNorm<E, E> e{u, h, hssq, xin, static_cast<const E*>(w->g_mlp), m.BT, m.d};
    TTCD_TRY(launch_rows_gemm<E>(c, mA, mB, &mo, g, e, &mo2));
  }
  // The MLP RMSNorm's 1/rms per row, from the o_proj epilogue's partial sums.
  rms_rstd_kernel<<<cdiv(2 * m.BT, 256), 256, 0, c.s>>>(hssq, cdiv(m.d, 256), 2 * m.BT,
                                                        1.0f / m.d, p->rms_eps,
                                                        at<float>(ws, L, B_RSTD));
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

// The block for operand type E (bf16: kind::f16 tensor cores; fp32: kind::tf32).
// x, the weights and out are E; the wide route calls it with fp32 copies.
template <class E>
ttcd_status run_block(const Ctx& c, const void* x, const float* beta,
                      const ttcd_block_weights* w, const ttcd_block_params* p,
                      const float* state_in, float* state_out, void* out, void* ws,
                      const Layout& L) {
  const E* xin = static_cast<const E*>(x);
  __nv_bfloat16* qkv = at<__nv_bfloat16>(ws, L, B_QKV);
  TTCD_TRY(block_qkv<E>(c, xin, w, p, ws, L, qkv, 0, 0));
  TTCD_TRY(block_attend<E>(c, xin, w, p, ws, L, qkv, 0));
  return run_mlp_core<E, E, float>(c, p, L, ws, static_cast<const E*>(w->w_gate),
                                   static_cast<const E*>(w->w_up),
                                   static_cast<const E*>(w->w_down),
                                   static_cast<const E*>(w->w_proj),
                                   static_cast<const E*>(w->conv_T),
                                   static_cast<const E*>(w->conv_S), beta, state_in, state_out,
                                   at<float>(ws, L, B_H), static_cast<E*>(out), 4,
                                   at<float>(ws, L, B_RSTD));
}

// ttcd_block_forward with optional stage-boundary events (profiled calls).
ttcd_status block_entry(const void* x, const float* beta, const ttcd_block_weights* w,
                        const ttcd_block_params* p, const float* state_in, float* state_out,
                        void* out, void* workspace, size_t ws_bytes, void* stream,
                        const cudaEvent_t* events, int n_events) {
  TTCD_TRY(check_params(p));
  if (!aligned16(x) || !aligned16(beta) || !aligned16(out) || !weights_ok(w, true) ||
      !aligned16(workspace) || (state_out && !aligned16(state_out)) ||
      (state_in && !aligned16(state_in)))
    return TTCD_ERR_INVALID_ARG;
  const Layout L = make_layout(p, true);
  if (ws_bytes < L.total) return TTCD_ERR_WORKSPACE;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, at<void>(workspace, L, B_STATUS)));
  c.events = events;
  c.n_events = n_events;
  if (p->dtype == TTCD_F32)
    return run_block<float>(c, x, beta, w, p, state_in, state_out, out, workspace, L);
  if (wide_mode(p)) {
    using bf = __nv_bfloat16;
    const long long n_x = static_cast<long long>(p->B) * p->T * p->d_model;
    ttcd_block_weights w32;
    TTCD_TRY(widen_weights(c, p, w, workspace, L, &w32));
    float* x32 = at<float>(workspace, L, B_X32);
    float* out32 = at<float>(workspace, L, B_OUT32);
    TTCD_TRY((launch_cast<bf, float>(c, x, x32, n_x)));
    TTCD_TRY(run_block<float>(c, x32, beta, &w32, p, state_in, state_out, out32, workspace, L));
    return launch_cast<float, bf>(c, out32, out, n_x);
  }
  return run_block<__nv_bfloat16>(c, x, beta, w, p, state_in, state_out, out, workspace, L);
}

// A plain sliding-window block (a layer outside ttt_layers): QKV with RoPE,
// one attention window w_T (the fused kernel with w_S = w_T writes the same
// output twice: o_T into the teacher half of o, o_S into the student half),
// o_proj + residual + RMS statistics over the student half only, SwiGLU with
// the static weights over the same rows, and out = h + W_down Z.
template <class E>
ttcd_status run_swa_block(const Ctx& c, const void* x, const ttcd_block_weights* w,
                          const ttcd_block_params* p, void* out, void* ws, const Layout& L) {
  const Dims m = dims_of(p);
  const E* xin = static_cast<const E*>(x);
  __nv_bfloat16* qkv = at<__nv_bfloat16>(ws, L, B_QKV);
  TTCD_TRY(block_qkv<E>(c, xin, w, p, ws, L, qkv, 0, 0));
  E* o = at<E>(ws, L, B_O);
  float* h = at<float>(ws, L, B_H);
  E* u = at<E>(ws, L, B_U);
  float* hssq = at<float>(ws, L, B_HSSQ);
  float* rstd = at<float>(ws, L, B_RSTD);
  const float sc = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(m.hd));
  TTCD_TRY(run_attn<E>(c, qkv, qkv + static_cast<long long>(m.Hq) * m.hd,
                       qkv + static_cast<long long>(m.Hq + m.Hkv) * m.hd, o,
                       o + m.BT * m.Hq * m.hd, nullptr, nullptr, p->B, p->T, m.Hq, m.Hkv, m.hd,
                       p->w_T, p->w_T, sc, m.dqkv, m.dqkv, 0));
  stage_mark(c, 3);
  {  // h = x + o W_o^T over the student rows [BT, 2BT) of o
    CUtensorMap mA, mB, mo, mo2;
    if (!map_rows<E>(&mA, o, 2 * m.BT, static_cast<long long>(m.Hq) * m.hd, 128) ||
        !map_rows<E>(&mB, w->w_o, m.d, static_cast<long long>(m.Hq) * m.hd, gemm_b_box<E>()) ||
        !make_out_map<E>(&mo, u, 2 * m.BT, m.d, m.d) ||
        !make_out_map<float>(&mo2, h, m.BT, m.d, m.d))
      return TTCD_ERR_CUDA;
    GemmGeom g = plain_geom(m.BT, cdiv(m.d, 256), m.Hq * m.hd);
    g.row_off = static_cast<int>(m.BT);
    EpiOprojNorm<E, E> e{u, h, hssq, xin, static_cast<const E*>(w->g_mlp), m.BT, m.d};
    TTCD_TRY(launch_rows_gemm<E>(c, mA, mB, &mo, g, e, &mo2));
  }
  rms_rstd_kernel<<<cdiv(m.BT, 256), 256, 0, c.s>>>(hssq, cdiv(m.d, 256), 2 * m.BT, 1.0f / m.d,
                                                    p->rms_eps, rstd, m.BT);
  TTCD_CHECK_LAUNCH();
  stage_mark(c, 4);
  // Z = silu(u W_gate^T) * (u W_up^T) over the same rows: bf16 Z_S, or fp32 into
  // the student half of Z
  E* zs = sizeof(E) == 2 ? at<E>(ws, L, B_ZS16) : reinterpret_cast<E*>(at<float>(ws, L, B_Z) + m.BT * m.f);
  {
    CUtensorMap mA, mB0, mB1, mo;
    if (!map_rows<E>(&mA, u, 2 * m.BT, m.d, 128) ||
        !map_rows<E>(&mB0, w->w_gate, m.f, m.d, 128) || !map_rows<E>(&mB1, w->w_up, m.f, m.d, 128) ||
        !make_out_map<E>(&mo, zs, m.BT, m.f, m.f))
      return TTCD_ERR_CUDA;
    GemmGeom g = plain_geom(m.BT, cdiv(m.f, 128), m.d);
    g.row_off = static_cast<int>(m.BT);
    EpiSwiGLU<E> e{zs, m.f, m.f, rstd, m.BT};
    TTCD_TRY((launch_gemm<E, 256, 4, true>(c, mA, mB0, mB1, &mo, g, e)));
  }
  stage_mark(c, 5);
  {  // out = h + W_down Z
    CUtensorMap mA, mB, mo;
    if (!map_rows<E>(&mA, zs, m.BT, m.f, 128) ||
        !map_rows<E>(&mB, w->w_down, m.d, m.f, gemm_b_box<E>()) ||
        !make_out_map<E>(&mo, out, m.BT, m.d, m.d))
      return TTCD_ERR_CUDA;
    EpiResidual<E, float> e{static_cast<E*>(out), m.d, h, m.d, m.BT, m.d};
    TTCD_TRY(launch_rows_gemm<E>(c, mA, mB, &mo, plain_geom(m.BT, cdiv(m.d, 256), m.f), e));
  }
  stage_mark(c, 6);
  return TTCD_OK;
}

ttcd_status swa_block_entry(const void* x, const ttcd_block_weights* w,
                            const ttcd_block_params* p, void* out, void* workspace,
                            size_t ws_bytes, void* stream) {
  TTCD_TRY(check_params(p));
  if (!aligned16(x) || !aligned16(out) || !aligned16(workspace) || !w || !aligned16(w->w_qkv) ||
      !aligned16(w->w_o) || !aligned16(w->g_attn) || !aligned16(w->g_mlp) ||
      !aligned16(w->w_gate) || !aligned16(w->w_up) || !aligned16(w->w_down))
    return TTCD_ERR_INVALID_ARG;
  const Layout L = make_layout(p, true, false, false);
  if (ws_bytes < L.total) return TTCD_ERR_WORKSPACE;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, at<void>(workspace, L, B_STATUS)));
  if (p->dtype == TTCD_F32) return run_swa_block<float>(c, x, w, p, out, workspace, L);
  return run_swa_block<__nv_bfloat16>(c, x, w, p, out, workspace, L);
}

}  // namespace

// ===================================================================== C ABI
extern "C" {

size_t ttcd_swa_block_forward_workspace_size(const ttcd_block_params* p) {
  if (check_params(p) != TTCD_OK) return 0;
  return make_layout(p, true, false, false).total;
}

ttcd_status ttcd_swa_block_forward(const void* x, const ttcd_block_weights* w,
                                   const ttcd_block_params* p, void* out, void* workspace,
                                   size_t ws_bytes, void* stream) {
  return swa_block_entry(x, w, p, out, workspace, ws_bytes, stream);
}

const char* ttcd_status_string(ttcd_status s) {
  switch (s) {
    case TTCD_OK: return "ok";
    case TTCD_ERR_INVALID_ARG: return "invalid argument";
    case TTCD_ERR_UNSUPPORTED: return "unsupported configuration";
    case TTCD_ERR_CUDA: return "CUDA error";
    case TTCD_ERR_TIMEOUT: return "device wait timed out";
    case TTCD_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

const char* ttcd_version(void) { return "ttcd 0.2 sm_100a"; }

unsigned long long ttcd_kernel_launch_count(void) { return g_launches.load(); }

void ttcd_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns = ns ? ns : 1; }

size_t ttcd_fastweight_mlp_workspace_size(const ttcd_block_params* p) {
  if (check_params(p) != TTCD_OK) return 0;
  return make_layout(p, false).total;
}

size_t ttcd_block_forward_workspace_size(const ttcd_block_params* p) {
  if (check_params(p) != TTCD_OK) return 0;
  return make_layout(p, true).total;
}

ttcd_status ttcd_block_workspace_offset(const ttcd_block_params* p, const char* name,
                                        size_t* offset) {
  if (check_params(p) != TTCD_OK || !name || !offset) return TTCD_ERR_INVALID_ARG;
  const Layout L = make_layout(p, true);
  for (int i = 0; i < B_COUNT; ++i) {
    if (std::strcmp(name, kBufNames[i]) == 0) {
      *offset = L.off[i];
      return TTCD_OK;
    }
  }
  return TTCD_ERR_INVALID_ARG;
}

ttcd_status ttcd_check_device_status(void* workspace, void* stream) {
  if (!aligned16(workspace)) return TTCD_ERR_INVALID_ARG;
  return read_clear_status(static_cast<uint32_t*>(workspace), static_cast<cudaStream_t>(stream),
                           nullptr);
}

ttcd_status ttcd_get_device_error(uint32_t* flags, void* stream) {
  Ctx c;
  TTCD_TRY(make_ctx(stream, c));
  return read_clear_status(c.st.err, c.s, flags);
}

ttcd_status ttcd_dual_window_attn(const void* q, const void* k, const void* v, void* o_T,
                                  void* o_S, float* lse_T, float* lse_S, int B, int T, int Hq,
                                  int Hkv, int hd, int w_S, int w_T, float scale,
                                  ttcd_dtype dtype, void* stream) {
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || w_S < 1 || w_T < w_S ||
      !(scale >= 0.f))
    return TTCD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_T) || !aligned16(o_S))
    return TTCD_ERR_INVALID_ARG;
  if ((lse_T && !aligned16(lse_T)) || (lse_S && !aligned16(lse_S))) return TTCD_ERR_INVALID_ARG;
  if (dtype != TTCD_BF16) return dtype == TTCD_F32 ? TTCD_ERR_UNSUPPORTED : TTCD_ERR_INVALID_ARG;
  if (hd != 32 && hd != 64 && hd != 128) return TTCD_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * T >= (1ll << 31)) return TTCD_ERR_UNSUPPORTED;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c));
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(hd));
  return run_attn<__nv_bfloat16>(c, q, k, v, static_cast<__nv_bfloat16*>(o_T),
                                 static_cast<__nv_bfloat16*>(o_S), lse_T, lse_S, B, T, Hq, Hkv,
                                 hd, w_S, w_T, sc, static_cast<long long>(Hq) * hd,
                                 static_cast<long long>(Hkv) * hd);
}

ttcd_status ttcd_dual_window_attn_lse(const void* q, const void* k, const void* v, void* o_T,
                                      void* o_S, void* o_far, float* lse_T, float* lse_S,
                                      float* lse_far, int B, int T, int Hq, int Hkv, int hd,
                                      int w_S, int w_T, float scale, ttcd_dtype dtype,
                                      void* stream) {
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || w_S < 1 || w_T < w_S ||
      !(scale >= 0.f))
    return TTCD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_T) || !aligned16(o_S) ||
      !aligned16(o_far) || !aligned16(lse_S) || !aligned16(lse_far))
    return TTCD_ERR_INVALID_ARG;
  if (lse_T && !aligned16(lse_T)) return TTCD_ERR_INVALID_ARG;
  if (dtype != TTCD_BF16) return dtype == TTCD_F32 ? TTCD_ERR_UNSUPPORTED : TTCD_ERR_INVALID_ARG;
  if (hd != 32 && hd != 64 && hd != 128) return TTCD_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * T * Hq * (hd / 8) >= (1ll << 31) * 256ll)
    return TTCD_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * T >= (1ll << 31)) return TTCD_ERR_UNSUPPORTED;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c));
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(hd));
  using bf = __nv_bfloat16;
  bf *oT = static_cast<bf*>(o_T), *oS = static_cast<bf*>(o_S), *oF = static_cast<bf*>(o_far);
  switch (hd) {
    case 32: return launch_attn_lse<32>(c, q, k, v, oT, oS, oF, lse_T, lse_S, lse_far, B, T, Hq, Hkv, w_S, w_T, sc);
    case 64: return launch_attn_lse<64>(c, q, k, v, oT, oS, oF, lse_T, lse_S, lse_far, B, T, Hq, Hkv, w_S, w_T, sc);
    default: return launch_attn_lse<128>(c, q, k, v, oT, oS, oF, lse_T, lse_S, lse_far, B, T, Hq, Hkv, w_S, w_T, sc);
  }
}

ttcd_status ttcd_fastweight_mlp(const void* u_T, const void* u_S, const void* h_S,
                                const float* beta, const ttcd_block_weights* w,
                                const ttcd_block_params* p, const float* state_in,
                                float* state_out, void* y, void* workspace, size_t ws_bytes,
                                void* stream) {
  return mlp_entry(u_T, u_S, h_S, beta, w, p, state_in, state_out, y, workspace, ws_bytes,
                   stream, workspace);
}

ttcd_status ttcd_block_forward(const void* x, const float* beta, const ttcd_block_weights* w,
                               const ttcd_block_params* p, float* state_out, void* out,
                               void* workspace, size_t ws_bytes, void* stream) {
  return block_entry(x, beta, w, p, nullptr, state_out, out, workspace, ws_bytes, stream,
                     nullptr, 0);
}

ttcd_status ttcd_block_forward_profiled(const void* x, const float* beta,
                                        const ttcd_block_weights* w, const ttcd_block_params* p,
                                        float* state_out, void* out, void* workspace,
                                        size_t ws_bytes, void* stream, void* const* events,
                                        int n_events) {
  if (n_events < 0 || n_events > kMaxStageEvents || (n_events > 0 && !events))
    return TTCD_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return TTCD_ERR_INVALID_ARG;
  return block_entry(x, beta, w, p, nullptr, state_out, out, workspace, ws_bytes, stream,
                     reinterpret_cast<const cudaEvent_t*>(events), n_events);
}

// ---------------------------------------------------------------- sequence shards
size_t ttcd_shard_workspace_size(const ttcd_block_params* p) {
  if (check_params(p) != TTCD_OK || p->dtype != TTCD_BF16) return 0;
  return make_layout(p, true, true).total;
}

}  // extern "C"

namespace {
// Common checks of the shard phases; on success fills the layout and the
// context (status word in the workspace) and the K/V halo length.
ttcd_status shard_begin(const ttcd_block_params* p, long long pos0, void* workspace,
                        size_t ws_bytes, void* stream, Layout& L, Ctx& c, int& n_halo) {
  TTCD_TRY(check_params(p));
  if (p->dtype != TTCD_BF16) return TTCD_ERR_UNSUPPORTED;
  if (pos0 < 0 || pos0 % p->chunk != 0 || !aligned16(workspace)) return TTCD_ERR_INVALID_ARG;
  if (pos0 + p->T >= (1ll << 31)) return TTCD_ERR_UNSUPPORTED;
  L = make_layout(p, true, true);
  if (ws_bytes < L.total) return TTCD_ERR_WORKSPACE;
  TTCD_TRY(make_ctx(stream, c, at<void>(workspace, L, B_STATUS)));
  n_halo = static_cast<int>(std::min<long long>(p->w_T - 1, pos0));
  return TTCD_OK;
}

// Strided copy of `rows` rows of `width` bytes per sequence, as B 2-D copies.
ttcd_status copy_rows(const Ctx& c, int B, void* dst, size_t dpitch, size_t dseq,
                      const void* src, size_t spitch, size_t sseq, size_t width, size_t rows) {
  if (rows == 0) return TTCD_OK;
  for (int b = 0; b < B; ++b) {
    if (cudaMemcpy2DAsync(static_cast<uint8_t*>(dst) + b * dseq, dpitch,
                          static_cast<const uint8_t*>(src) + b * sseq, spitch, width, rows,
                          cudaMemcpyDeviceToDevice, c.s) != cudaSuccess)
      return TTCD_ERR_CUDA;
  }
  return TTCD_OK;
}
}  // namespace

extern "C" {

ttcd_status ttcd_shard_qkv(const void* x, const ttcd_block_weights* w, const ttcd_block_params* p,
                           long long pos0, void* kv_tail, void* workspace, size_t ws_bytes,
                           void* stream) {
  if (!aligned16(x) || !weights_ok(w, true) || (kv_tail && !aligned16(kv_tail)))
    return TTCD_ERR_INVALID_ARG;
  Layout L;
  Ctx c;
  int n_halo = 0;
  TTCD_TRY(shard_begin(p, pos0, workspace, ws_bytes, stream, L, c, n_halo));
  using bf = __nv_bfloat16;
  const Dims m = dims_of(p);
  bf* qkvx = at<bf>(workspace, L, B_QKVX);
  TTCD_TRY(block_qkv<bf>(c, static_cast<const bf*>(x), w, p, workspace, L, qkvx, n_halo, pos0));
  if (kv_tail) {  // K, V of this shard's last min(T, w_T - 1) tokens
    const size_t kvw = 2 * static_cast<size_t>(m.Hkv) * m.hd * 2, rowb = m.dqkv * 2;
    const size_t nt = std::min(p->T, p->w_T - 1);
    TTCD_TRY(copy_rows(c, p->B, kv_tail, kvw, nt * kvw,
                       reinterpret_cast<uint8_t*>(qkvx) + (n_halo + p->T - nt) * rowb +
                           static_cast<size_t>(m.Hq) * m.hd * 2,
                       rowb, (n_halo + p->T) * rowb, kvw, nt));
  }
  return TTCD_OK;
}

ttcd_status ttcd_shard_attend(const void* x, const void* kv_halo, const ttcd_block_weights* w,
                              const ttcd_block_params* p, long long pos0, void* u_tail,
                              void* workspace, size_t ws_bytes, void* stream) {
  if (!aligned16(x) || !weights_ok(w, true) || (u_tail && !aligned16(u_tail)) ||
      (kv_halo && !aligned16(kv_halo)))
    return TTCD_ERR_INVALID_ARG;
  Layout L;
  Ctx c;
  int n_halo = 0;
  TTCD_TRY(shard_begin(p, pos0, workspace, ws_bytes, stream, L, c, n_halo));
  if (n_halo > 0 && !kv_halo) return TTCD_ERR_INVALID_ARG;
  using bf = __nv_bfloat16;
  const Dims m = dims_of(p);
  bf* qkvx = at<bf>(workspace, L, B_QKVX);
  const size_t kvw = 2 * static_cast<size_t>(m.Hkv) * m.hd * 2, rowb = m.dqkv * 2;
  const size_t qw = static_cast<size_t>(m.Hq) * m.hd * 2, seqb = (n_halo + p->T) * rowb;
  // the halo's K and V in front of each sequence's rows; its query columns zeroed
  TTCD_TRY(copy_rows(c, p->B, reinterpret_cast<uint8_t*>(qkvx) + qw, rowb, seqb, kv_halo, kvw,
                     n_halo * kvw, kvw, n_halo));
  for (int b = 0; n_halo > 0 && b < p->B; ++b)
    if (cudaMemset2DAsync(reinterpret_cast<uint8_t*>(qkvx) + b * seqb, rowb, 0, qw, n_halo,
                          c.s) != cudaSuccess)
      return TTCD_ERR_CUDA;
  TTCD_TRY(block_attend<bf>(c, static_cast<const bf*>(x), w, p, workspace, L, qkvx, n_halo));
  if (u_tail && p->conv_k > 1) {  // normalised MLP inputs of the last min(T, k-1) tokens
    const int n = std::min(p->T, p->conv_k - 1);
    const long long threads = 2ll * p->B * n * (m.d / 8);
    u_tail_kernel<bf><<<static_cast<unsigned>(cdiv(threads, 256)), 256, 0, c.s>>>(
        at<bf>(workspace, L, B_U), at<float>(workspace, L, B_RSTD), static_cast<bf*>(u_tail),
        p->B, p->T, m.d, n, m.BT);
    TTCD_CHECK_LAUNCH();
  }
  return TTCD_OK;
}

ttcd_status ttcd_shard_mix(const float* beta, const void* u_halo, const ttcd_block_weights* w,
                           const ttcd_block_params* p, long long pos0, float* total,
                           void* workspace, size_t ws_bytes, void* stream) {
  if (!aligned16(beta) || !weights_ok(w, false) || !aligned16(total) ||
      (u_halo && !aligned16(u_halo)))
    return TTCD_ERR_INVALID_ARG;
  Layout L;
  Ctx c;
  int n_halo = 0;
  TTCD_TRY(shard_begin(p, pos0, workspace, ws_bytes, stream, L, c, n_halo));
  using bf = __nv_bfloat16;
  const Dims m = dims_of(p);
  const int H = p->conv_k - 1;
  const int nh = static_cast<int>(std::min<long long>(H, pos0));
  if (nh > 0 && !u_halo) return TTCD_ERR_INVALID_ARG;
  float* zh = nullptr;
  if (H > 0) {
    // Z_T, Z_S of the H tokens before the shard from the previous shard's u rows
    // (zero rows, hence zero Z, before the sequence start).
    bf* uh = at<bf>(workspace, L, B_UH);
    zh = at<float>(workspace, L, B_ZH);
    const size_t rowb = static_cast<size_t>(m.d) * 2;
    if (cudaMemsetAsync(uh, 0, 2 * static_cast<size_t>(p->B) * H * rowb, c.s) != cudaSuccess)
      return TTCD_ERR_CUDA;
    for (int pb = 0; nh > 0 && pb < 2 * p->B; ++pb)
      if (cudaMemcpyAsync(reinterpret_cast<uint8_t*>(uh) + (static_cast<size_t>(pb) * H + (H - nh)) * rowb,
                          static_cast<const uint8_t*>(u_halo) + static_cast<size_t>(pb) * nh * rowb,
                          nh * rowb, cudaMemcpyDeviceToDevice, c.s) != cudaSuccess)
        return TTCD_ERR_CUDA;
    CUtensorMap mA, mB0, mB1, mo;
    const long long rows = 2ll * p->B * H;
    if (!map_rows<bf>(&mA, uh, rows, m.d, 128) || !map_rows<bf>(&mB0, w->w_gate, m.f, m.d, 128) ||
        !map_rows<bf>(&mB1, w->w_up, m.f, m.d, 128) ||
        !make_out_map<float>(&mo, zh, rows, m.f, m.f))
      return TTCD_ERR_CUDA;
    EpiSwiGLU<float> e{zh, m.f, m.f, nullptr};
    TTCD_TRY((launch_gemm<bf, 256, 4, true>(c, mA, mB0, mB1, &mo, plain_geom(rows, cdiv(m.f, 128), m.d), e)));
  }
  TTCD_TRY(mlp_front<bf>(c, p, L, workspace, static_cast<const bf*>(w->w_gate),
                         static_cast<const bf*>(w->w_up), static_cast<const bf*>(w->w_down),
                         static_cast<const bf*>(w->w_proj), static_cast<const bf*>(w->conv_T),
                         static_cast<const bf*>(w->conv_S), beta, 4,
                         at<float>(workspace, L, B_RSTD), zh));
  // this shard's total: all its padded tokens as one chunk, from a zero state
  return launch_scan<bf>(c, p, L, workspace, static_cast<const bf*>(w->w_down), nullptr, total,
                         nullptr, true);
}

ttcd_status ttcd_shard_finish(const ttcd_block_weights* w, const ttcd_block_params* p,
                              long long pos0, const float* state_in, float* state_out, void* out,
                              void* workspace, size_t ws_bytes, void* stream) {
  if (!weights_ok(w, false) || !aligned16(out) || (state_in && !aligned16(state_in)) ||
      (state_out && !aligned16(state_out)))
    return TTCD_ERR_INVALID_ARG;
  Layout L;
  Ctx c;
  int n_halo = 0;
  TTCD_TRY(shard_begin(p, pos0, workspace, ws_bytes, stream, L, c, n_halo));
  using bf = __nv_bfloat16;
  return mlp_back<bf, bf, float>(c, p, L, workspace, static_cast<const bf*>(w->w_down), state_in,
                                 state_out, at<float>(workspace, L, B_H), static_cast<bf*>(out),
                                 4);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Fast-weight MLP without caller-provided scratch.
//
// Some callers cannot hand this library a workspace: a host framework may own
// every byte of device memory through its own pool and expose no way to borrow
// from it, and a latency-critical loop may not be allowed to call cudaMalloc
// (which can synchronise the device).  For them the scratch of one
// ttcd_fastweight_mlp call lives in this fixed array instead.  It is part of
// the library image, so every GPU that loads the library holds these 32 MiB
// until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_ttcd_noalloc_scratch[kNoAllocScratchBytes];
namespace {
// Device address of the array, looked up once per device (host-side state of
// this file only: not exported).
void* g_noalloc_scratch_addr[kMaxDevices] = {nullptr};
}  // namespace

extern "C" {

ttcd_status ttcd_fastweight_mlp_noalloc(const void* u_T, const void* u_S, const void* h_S,
                                        const float* beta, const ttcd_block_weights* w,
                                        const ttcd_block_params* p, const float* state_in,
                                        float* state_out, void* y, void* stream) {
  TTCD_TRY(check_params(p));
  const size_t need = make_layout(p, false).total;
  if (need > kNoAllocScratchBytes) return TTCD_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TTCD_ERR_CUDA;
  {
    // One-time set-up per device, made with that device current: the array's
    // name is only a host-side stand-in, the kernels need its device address.
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_noalloc_scratch_addr[dev]) {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_ttcd_noalloc_scratch) != cudaSuccess || !addr)
        return TTCD_ERR_CUDA;
      g_noalloc_scratch_addr[dev] = addr;
    }
  }
  // Every byte of scratch that a call reads is written earlier in the same
  // call, so nothing has to be cleared between calls.  Timeouts go to the
  // per-device status word (ttcd_get_device_error): the caller holds no
  // workspace to keep one in.
  return mlp_entry(u_T, u_S, h_S, beta, w, p, state_in, state_out, y,
                   g_noalloc_scratch_addr[dev], kNoAllocScratchBytes, stream, nullptr);
}

size_t ttcd_fastweight_mlp_noalloc_capacity(void) { return kNoAllocScratchBytes; }

__global__ void bounded_wait_test_kernel(DevStatus st) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, st, &abort_flag);  // nothing ever arrives
  __syncthreads();
}

// Copies the attention kernel's clock64 timeline (instrumented build only).
ttcd_status ttcd_attn_timeline_read(long long* out, size_t n) {
#if TTCD_ATTN_TIMELINE
  const size_t total = 2 * ATT_TL_VISITS * ATT_TL_MARKS;
  if (!out || n < total) return TTCD_ERR_INVALID_ARG;
  if (cudaMemcpyFromSymbol(out, g_attn_timeline, total * sizeof(long long)) != cudaSuccess)
    return TTCD_ERR_CUDA;
  void* dev = nullptr;  // cleared for the next launch
  if (cudaGetSymbolAddress(&dev, g_attn_timeline) != cudaSuccess ||
      cudaMemset(dev, 0, total * sizeof(long long)) != cudaSuccess)
    return TTCD_ERR_CUDA;
  return TTCD_OK;
#else
  (void)out;
  (void)n;
  return TTCD_ERR_UNSUPPORTED;
#endif
}

// Evaluates the attention kernel's FMA-pipe 2^x (exp2_poly2) at x[0..n-1].
__global__ void exp2_poly_test_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const long long i = 2ll * (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x1 = i + 1 < n ? x[i + 1] : x[i];
  float y0, y1;
  f2unpack(exp2_poly2(f2pack(x[i], x1)), y0, y1);
  y[i] = y0;
  if (i + 1 < n) y[i + 1] = y1;
}

ttcd_status ttcd_test_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y)) || (reinterpret_cast<uintptr_t>(x) & 3u) ||
      (reinterpret_cast<uintptr_t>(y) & 3u))
    return TTCD_ERR_INVALID_ARG;
  if (n == 0) return TTCD_OK;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c));
  const int threads = (n + 1) / 2;
  exp2_poly_test_kernel<<<cdiv(threads, 256), 256, 0, c.s>>>(x, y, n);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

ttcd_status ttcd_test_bounded_wait(uint64_t timeout_ns, void* status, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return TTCD_ERR_INVALID_ARG;
  if (status && !aligned16(status)) return TTCD_ERR_INVALID_ARG;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, status));
  DevStatus st = c.st;
  st.timeout_ns = timeout_ns;
  bounded_wait_test_kernel<<<1, 32, 0, c.s>>>(st);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

}  // extern "C"

// ===================================================================== decode
namespace {

// Decode state (per sequence unless noted), 1 KiB-aligned pieces; the status
// word of every decode call comes first.
struct DecState {
  size_t status, kc, vc, hist, rc, kx, S, weff, M, wprojT, total;
};
DecState dec_state_layout(const ttcd_block_params* p) {
  const long long B = p->B, d = p->d_model, f = p->d_ff, hd = p->head_dim;
  const long long W = p->w_T, H = p->conv_k > 1 ? p->conv_k - 1 : 1;
  const long long Cp = (p->chunk + 63) / 64 * 64;
  size_t sz[10] = {kStatusBytes,                                          // status word
                   static_cast<size_t>(B * W * p->n_kv_heads * hd * 2),   // K cache ring
                   static_cast<size_t>(B * W * p->n_kv_heads * hd * 2),   // V cache ring
                   static_cast<size_t>(2 * B * H * f * 4),                // conv history
                   static_cast<size_t>(B * Cp * d * 2),                   // r rows of the chunk
                   static_cast<size_t>(B * Cp * f * 2),                   // k' rows of the chunk
                   static_cast<size_t>(B * d * f * 4),                    // S
                   static_cast<size_t>(B * d * f * 2),                    // W_down + S
                   static_cast<size_t>(d * f * 2),                        // M (shared)
                   static_cast<size_t>(f * f * 2)};                       // W_proj^T (shared)
  DecState L;
  size_t* fields[10] = {&L.status, &L.kc, &L.vc, &L.hist, &L.rc, &L.kx, &L.S, &L.weff, &L.M,
                        &L.wprojT};
  size_t off = 0;
  for (int i = 0; i < 10; ++i) {
    *fields[i] = off;
    off += (sz[i] + 1023) / 1024 * 1024;
  }
  L.total = off;
  return L;
}

// Per-step scratch.
struct DecWs {
  size_t xn, qkv, qrot, o, hp, hS, u, Z, Zs, D, ks, r, pm, pl, po, ssq, total;
  int nsplit;
};
DecWs dec_ws_layout(const ttcd_block_params* p) {
  const long long B = p->B, d = p->d_model, f = p->d_ff, hd = p->head_dim;
  const long long Hq = p->n_q_heads, dqkv = (p->n_q_heads + 2 * p->n_kv_heads) * hd;
  DecWs L;
  L.nsplit = static_cast<int>(cdiv(p->w_T, DEC_KC));
  const long long np = B * Hq * 2 * L.nsplit;
  const size_t sz[16] = {static_cast<size_t>(B * d * 2), static_cast<size_t>(B * dqkv * 4),
                         static_cast<size_t>(B * Hq * hd * 2), static_cast<size_t>(2 * B * Hq * hd * 2),
                         static_cast<size_t>(2 * B * d * 4), static_cast<size_t>(B * d * 4),
                         static_cast<size_t>(2 * B * d * 2), static_cast<size_t>(2 * B * f * 4),
                         static_cast<size_t>(B * f * 2), static_cast<size_t>(B * f * 2),
                         static_cast<size_t>(B * 4), static_cast<size_t>(B * d * 2),
                         static_cast<size_t>(np * 4), static_cast<size_t>(np * 4),
                         static_cast<size_t>(np * hd * 4),
                         static_cast<size_t>(B * cdiv(f, 256) * 4)};
  size_t* fields[16] = {&L.xn, &L.qkv, &L.qrot, &L.o, &L.hp, &L.hS, &L.u, &L.Z, &L.Zs, &L.D,
                        &L.ks, &L.r, &L.pm, &L.pl, &L.po, &L.ssq};
  size_t off = 0;
  for (int i = 0; i < 16; ++i) {
    *fields[i] = off;
    off += (sz[i] + 1023) / 1024 * 1024;
  }
  L.total = off;
  return L;
}

ttcd_status check_decode_params(const ttcd_block_params* p) {
  TTCD_TRY(check_params(p));
  if (p->dtype != TTCD_BF16) return TTCD_ERR_UNSUPPORTED;
  if (p->n_q_heads / p->n_kv_heads > DEC_MAXG) return TTCD_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->B) * p->d_model * p->d_ff >= (1ll << 40)) return TTCD_ERR_UNSUPPORTED;
  return TTCD_OK;
}

template <class T>
T* dat(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

// S (in place) += the chunk buffers' R^T K' over their first Cp rows (rows past
// the chunk's tokens are zero), by the chunk-scan kernel with one chunk.
ttcd_status dec_commit(const Ctx& c, const ttcd_block_params* p, void* state, const DecState& L,
                       const __nv_bfloat16* w_down, const float* S_in, float* S_out,
                       const long long* commit_pos = nullptr) {
  using bf = __nv_bfloat16;
  const int d = p->d_model, f = p->d_ff, Cp = (p->chunk + 63) / 64 * 64;
  CUtensorMap mR, mK;
  constexpr uint32_t BK = ElemTraits<bf>::BK;
  if (!make_map<bf>(&mR, dat<bf>(state, L.rc), d, static_cast<uint64_t>(p->B) * Cp, d * 2, BK, BK) ||
      !make_map<bf>(&mK, dat<bf>(state, L.kx), f, static_cast<uint64_t>(p->B) * Cp, f * 2, BK, BK))
    return TTCD_ERR_CUDA;
  ScanArgs<bf> a{};
  a.d = d;
  a.f = f;
  a.Nc = 1;
  a.Cp = Cp;
  a.w_down = w_down;
  a.state_in = S_in;
  a.state_out = S_out;
  a.w_all = nullptr;
  a.tiles_m = cdiv(d, 128);
  a.tiles_n = cdiv(f, SCAN_BN);
  a.commit_pos = commit_pos;
  a.commit_C = p->chunk;
  constexpr int STAGES = 4;
  constexpr int smem = scan_smem_bytes<bf, STAGES, false>();
  auto kern = fastweight_scan_kernel<bf, STAGES, true>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TTCD_ERR_CUDA;
  TTCD_TRY(check_reg_split(reinterpret_cast<const void*>(kern), SCAN_THREADS, kScanRegSplit));
  kern<<<p->B * a.tiles_m * a.tiles_n, SCAN_THREADS, smem, c.s>>>(mR, mK, a, c.st);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

ttcd_status dec_weff(const Ctx& c, const ttcd_block_params* p, void* state, const DecState& L,
                     const __nv_bfloat16* w_down, const long long* commit_pos = nullptr) {
  const long long df = static_cast<long long>(p->d_model) * p->d_ff;
  const long long n4 = p->B * df / 4;
  const long long blocks = std::min<long long>(cdiv(n4, 256), 2LL * c.sms);
  decode_weff_kernel<<<static_cast<unsigned>(blocks), 256, 0, c.s>>>(
      w_down, dat<float>(state, L.S), dat<__nv_bfloat16>(state, L.weff), df, n4, commit_pos,
      p->chunk);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

template <int HD>
ttcd_status dec_attention(const Ctx& c, const ttcd_block_params* p, void* state,
                          const DecState& S, void* ws, const DecWs& L, int t, float scale,
                          const long long* pos) {
  using bf = __nv_bfloat16;
  const int B = p->B, Hq = p->n_q_heads, Hkv = p->n_kv_heads;
  const int G = Hq / Hkv;
  const int smem = dec_attn_smem_bytes<HD>(G);
  auto kern = G <= 2 ? decode_attn_partial_kernel<HD, 2>
                     : (G <= 4 ? decode_attn_partial_kernel<HD, 4> : decode_attn_partial_kernel<HD, 8>);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TTCD_ERR_CUDA;
  kern<<<dim3(B * Hkv, L.nsplit), DEC_THREADS, smem, c.s>>>(
      dat<bf>(ws, L.qrot), dat<bf>(state, S.kc), dat<bf>(state, S.vc), dat<float>(ws, L.pm),
      dat<float>(ws, L.pl), dat<float>(ws, L.po), Hq, Hkv, p->w_T, t, p->w_S, p->w_T,
      scale * 1.4426950408889634f, L.nsplit, pos);
  TTCD_CHECK_LAUNCH();
  decode_attn_combine_kernel<HD><<<B * Hq * 2, HD, 0, c.s>>>(
      dat<float>(ws, L.pm), dat<float>(ws, L.pl), dat<float>(ws, L.po), dat<bf>(ws, L.o), B, Hq,
      L.nsplit);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

// One token.  pos null: the token's position is t (host).  pos set: every
// kernel reads the position from *pos, the chunk commit runs every step and
// acts only at a chunk's last token, and the last launch advances *pos.
ttcd_status run_decode(const Ctx& c, const __nv_bfloat16* x, const float* beta, int t,
                       const ttcd_block_weights* w, const ttcd_block_params* p, void* state,
                       const DecState& S, __nv_bfloat16* y, void* ws, const DecWs& L,
                       long long* pos = nullptr, bool commit = true) {
  using bf = __nv_bfloat16;
  const int B = p->B, d = p->d_model, f = p->d_ff, hd = p->head_dim;
  const int Hq = p->n_q_heads, Hkv = p->n_kv_heads, dqkv = (Hq + 2 * Hkv) * hd;
  const int C = p->chunk, Cp = (C + 63) / 64 * 64;
  // input RMSNorm and Q/K/V (fp32, rotated once)
  rmsnorm_kernel<bf, bf, bf><<<cdiv(B, 8), 256, 0, c.s>>>(
      x, static_cast<const bf*>(w->g_attn), dat<bf>(ws, L.xn), B, d, p->rms_eps);
  TTCD_CHECK_LAUNCH();
  // few rows: warp-per-row GEMV; otherwise the tcgen05 GEMM
  const bool gemv_B = B <= DEC_GEMV_SWITCH_B;      // QKV and r: B rows
  const bool gemv = 2 * B <= DEC_GEMV_SWITCH;       // o_proj and gate/up: both paths, 2B rows
  if (gemv_B) {
    decode_gemv_kernel<0><<<cdiv(dqkv, 8), 256, 0, c.s>>>(
        static_cast<const bf*>(w->w_qkv), nullptr, dat<bf>(ws, L.xn), dat<float>(ws, L.qkv), B,
        dqkv, d, dqkv);
    TTCD_CHECK_LAUNCH();
  } else {
    CUtensorMap mA, mB, mo;
    if (!map_rows<bf>(&mA, dat<bf>(ws, L.xn), B, d, 128) ||
        !map_rows<bf>(&mB, w->w_qkv, dqkv, d, 256) ||
        !make_out_map<float>(&mo, dat<float>(ws, L.qkv), B, dqkv, dqkv))
      return TTCD_ERR_CUDA;
    EpiStore<float> e{dat<float>(ws, L.qkv), dqkv, dqkv, nullptr};
    TTCD_TRY((launch_gemm<bf, 256, 4, false>(c, mA, mB, mB, &mo, plain_geom(B, cdiv(dqkv, 256), d), e)));
  }
  decode_rope_cache_kernel<<<dim3(B, Hq + 2 * Hkv), hd / 2, 0, c.s>>>(
      dat<float>(ws, L.qkv), dat<bf>(ws, L.qrot), dat<bf>(state, S.kc), dat<bf>(state, S.vc), Hq,
      Hkv, hd, t, p->w_T, static_cast<double>(p->rope_theta), pos);
  TTCD_CHECK_LAUNCH();
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(hd));
  switch (hd) {
    case 32: TTCD_TRY(dec_attention<32>(c, p, state, S, ws, L, t, scale, pos)); break;
    case 64: TTCD_TRY(dec_attention<64>(c, p, state, S, ws, L, t, scale, pos)); break;
    default: TTCD_TRY(dec_attention<128>(c, p, state, S, ws, L, t, scale, pos)); break;
  }
  // o_proj for both paths, residual, MLP RMSNorm
  if (gemv) {
    decode_gemv_kernel<0><<<cdiv(d, 8), 256, 0, c.s>>>(
        static_cast<const bf*>(w->w_o), nullptr, dat<bf>(ws, L.o), dat<float>(ws, L.hp), 2 * B, d,
        Hq * hd, d);
    TTCD_CHECK_LAUNCH();
  } else {
    CUtensorMap mA, mB, mo;
    if (!map_rows<bf>(&mA, dat<bf>(ws, L.o), 2 * B, Hq * hd, 128) ||
        !map_rows<bf>(&mB, w->w_o, d, Hq * hd, 256) ||
        !make_out_map<float>(&mo, dat<float>(ws, L.hp), 2 * B, d, d))
      return TTCD_ERR_CUDA;
    EpiStore<float> e{dat<float>(ws, L.hp), d, d, nullptr};
    TTCD_TRY((launch_gemm<bf, 256, 4, false>(c, mA, mB, mB, &mo, plain_geom(2 * B, cdiv(d, 256), Hq * hd), e)));
  }
  decode_residual_norm_kernel<<<2 * B, 256, 0, c.s>>>(x, dat<float>(ws, L.hp),
                                                      static_cast<const bf*>(w->g_mlp),
                                                      dat<bf>(ws, L.u), dat<float>(ws, L.hS), B,
                                                      d, p->rms_eps);
  TTCD_CHECK_LAUNCH();
  // SwiGLU with the slow weights, both paths
  if (gemv) {
    decode_gemv_kernel<1><<<cdiv(f, 8), 256, 0, c.s>>>(
        static_cast<const bf*>(w->w_gate), static_cast<const bf*>(w->w_up), dat<bf>(ws, L.u),
        dat<float>(ws, L.Z), 2 * B, f, d, f);
    TTCD_CHECK_LAUNCH();
  } else {
    CUtensorMap mA, mB0, mB1, mo;
    if (!map_rows<bf>(&mA, dat<bf>(ws, L.u), 2 * B, d, 128) ||
        !map_rows<bf>(&mB0, w->w_gate, f, d, 128) || !map_rows<bf>(&mB1, w->w_up, f, d, 128) ||
        !make_out_map<float>(&mo, dat<float>(ws, L.Z), 2 * B, f, f))
      return TTCD_ERR_CUDA;
    EpiSwiGLU<float> e{dat<float>(ws, L.Z), f, f, nullptr};
    TTCD_TRY((launch_gemm<bf, 256, 4, true>(c, mA, mB0, mB1, &mo, plain_geom(2 * B, cdiv(f, 128), d), e)));
  }
  // convs, residual, key (into the chunk buffer), key scale
  const int n_part = cdiv(f, 256);
  decode_conv_kernel<<<dim3(n_part, B), 256, 0, c.s>>>(
      dat<float>(ws, L.Z), static_cast<const bf*>(w->conv_T), static_cast<const bf*>(w->conv_S),
      dat<float>(state, S.hist), dat<bf>(ws, L.D), dat<bf>(state, S.kx), dat<bf>(ws, L.Zs),
      dat<float>(ws, L.ssq), B, f, p->conv_k, t, C, Cp, pos);
  TTCD_CHECK_LAUNCH();
  // r = (D M^T) beta / ||zbar_S||, into the chunk buffer: the GEMV forms the
  // key scale and writes the chunk slot itself
  if (gemv_B) {
    DecKeyRowEpi kr{dat<float>(ws, L.ssq), n_part, beta, p->l2_eps, pos, t, C, Cp};
    decode_gemv_kernel<2><<<cdiv(d, 8), 256, 0, c.s>>>(
        dat<bf>(state, S.M), nullptr, dat<bf>(ws, L.D), dat<bf>(state, S.rc), B, d, f, d, kr);
    TTCD_CHECK_LAUNCH();
  } else {
    decode_kscale_kernel<<<B, 32, 0, c.s>>>(dat<float>(ws, L.ssq), n_part, beta,
                                            dat<float>(ws, L.ks), p->l2_eps);
    TTCD_CHECK_LAUNCH();
    CUtensorMap mA, mB, mo;
    if (!map_rows<bf>(&mA, dat<bf>(ws, L.D), B, f, 128) ||
        !map_rows<bf>(&mB, dat<bf>(state, S.M), d, f, 256) ||
        !make_out_map<bf>(&mo, dat<bf>(ws, L.r), B, d, d))
      return TTCD_ERR_CUDA;
    EpiStore<bf> e{dat<bf>(ws, L.r), d, d, dat<float>(ws, L.ks)};
    TTCD_TRY((launch_gemm<bf, 256, 4, false>(c, mA, mB, mB, &mo, plain_geom(B, cdiv(d, 256), f), e)));
    decode_row_copy_kernel<<<static_cast<unsigned>(cdiv(static_cast<long long>(B) * d, 256)), 256, 0, c.s>>>(
        dat<bf>(ws, L.r), dat<bf>(state, S.rc), B, d, Cp, t % C, pos, C);
    TTCD_CHECK_LAUNCH();
  }
  // output with the current chunk's weight W_down + S
  decode_out_kernel<<<dim3(cdiv(d, 8), B), 256, 0, c.s>>>(dat<bf>(state, S.weff), dat<bf>(ws, L.Zs),
                                                         dat<float>(ws, L.hS), y, d, f);
  TTCD_CHECK_LAUNCH();
  // last token of a chunk: S += this chunk's Delta W, then W_down + S
  float* Sp = dat<float>(state, S.S);
  if (pos) {  // launched unless the caller omits them; they act only at a chunk's last token
    if (commit) {
      TTCD_TRY(dec_commit(c, p, state, S, static_cast<const bf*>(w->w_down), Sp, Sp, pos));
      TTCD_TRY(dec_weff(c, p, state, S, static_cast<const bf*>(w->w_down), pos));
    }
    decode_advance_kernel<<<1, 1, 0, c.s>>>(pos);
    TTCD_CHECK_LAUNCH();
  } else if (t % C == C - 1) {
    TTCD_TRY(dec_commit(c, p, state, S, static_cast<const bf*>(w->w_down), Sp, Sp));
    TTCD_TRY(dec_weff(c, p, state, S, static_cast<const bf*>(w->w_down)));
  }
  return TTCD_OK;
}

}  // namespace

extern "C" {

size_t ttcd_decode_state_size(const ttcd_block_params* p) {
  if (check_decode_params(p) != TTCD_OK) return 0;
  return dec_state_layout(p).total;
}

size_t ttcd_decode_workspace_size(const ttcd_block_params* p) {
  if (check_decode_params(p) != TTCD_OK) return 0;
  return dec_ws_layout(p).total;
}

ttcd_status ttcd_decode_state_init(const ttcd_block_weights* w, const ttcd_block_params* p,
                                   const float* state_in, void* state, size_t state_bytes,
                                   void* workspace, size_t ws_bytes, void* stream) {
  TTCD_TRY(check_decode_params(p));
  if (!weights_ok(w, true) || !aligned16(state) || (state_in && !aligned16(state_in)))
    return TTCD_ERR_INVALID_ARG;
  const DecState S = dec_state_layout(p);
  if (state_bytes < S.total) return TTCD_ERR_WORKSPACE;
  (void)workspace;
  (void)ws_bytes;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, dat<void>(state, S.status)));
  using bf = __nv_bfloat16;
  const int d = p->d_model, f = p->d_ff;
  if (cudaMemsetAsync(state, 0, S.total, c.s) != cudaSuccess) return TTCD_ERR_CUDA;
  if (state_in && cudaMemcpyAsync(dat<float>(state, S.S), state_in,
                                  static_cast<size_t>(p->B) * d * f * 4,
                                  cudaMemcpyDeviceToDevice, c.s) != cudaSuccess)
    return TTCD_ERR_CUDA;
  TTCD_TRY(dec_weff(c, p, state, S, static_cast<const bf*>(w->w_down)));
  // M = W_down W_proj
  dim3 tb(32, 8), tg(cdiv(f, 32), cdiv(f, 32));
  transpose_kernel<bf, bf><<<tg, tb, 0, c.s>>>(static_cast<const bf*>(w->w_proj),
                                               dat<bf>(state, S.wprojT), f, f);
  TTCD_CHECK_LAUNCH();
  CUtensorMap mA, mB, mo;
  if (!map_rows<bf>(&mA, w->w_down, d, f, 128) ||
      !map_rows<bf>(&mB, dat<bf>(state, S.wprojT), f, f, 256) ||
      !make_out_map<bf>(&mo, dat<bf>(state, S.M), d, f, f))
    return TTCD_ERR_CUDA;
  EpiStore<bf> e{dat<bf>(state, S.M), f, f, nullptr};
  return launch_gemm<bf, 256, 4, false>(c, mA, mB, mB, &mo, plain_geom(d, cdiv(f, 256), f), e);
}

ttcd_status ttcd_block_decode(const void* x_t, const float* beta_t, int t,
                              const ttcd_block_weights* w, const ttcd_block_params* p,
                              void* state, size_t state_bytes, void* y, void* workspace,
                              size_t ws_bytes, void* stream) {
  TTCD_TRY(check_decode_params(p));
  if (t < 0 || !aligned16(x_t) || !beta_t || (reinterpret_cast<uintptr_t>(beta_t) & 3u) ||
      !aligned16(y) || !weights_ok(w, true) || !aligned16(state) || !aligned16(workspace))
    return TTCD_ERR_INVALID_ARG;
  const DecState S = dec_state_layout(p);
  const DecWs L = dec_ws_layout(p);
  if (state_bytes < S.total || ws_bytes < L.total) return TTCD_ERR_WORKSPACE;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, dat<void>(state, S.status)));
  return run_decode(c, static_cast<const __nv_bfloat16*>(x_t), beta_t, t, w, p, state, S,
                    static_cast<__nv_bfloat16*>(y), workspace, L);
}

ttcd_status ttcd_block_decode_next(const void* x_t, const float* beta_t,
                                   const ttcd_block_weights* w, const ttcd_block_params* p,
                                   void* state, size_t state_bytes, void* y, void* workspace,
                                   size_t ws_bytes, void* stream) {
  return ttcd_block_decode_next_ex(x_t, beta_t, w, p, state, state_bytes, y, workspace, ws_bytes,
                                   1, stream);
}

ttcd_status ttcd_block_decode_next_ex(const void* x_t, const float* beta_t,
                                      const ttcd_block_weights* w, const ttcd_block_params* p,
                                      void* state, size_t state_bytes, void* y, void* workspace,
                                      size_t ws_bytes, int commit, void* stream) {
  TTCD_TRY(check_decode_params(p));
  if (!aligned16(x_t) || !beta_t || (reinterpret_cast<uintptr_t>(beta_t) & 3u) ||
      !aligned16(y) || !weights_ok(w, true) || !aligned16(state) || !aligned16(workspace))
    return TTCD_ERR_INVALID_ARG;
  const DecState S = dec_state_layout(p);
  const DecWs L = dec_ws_layout(p);
  if (state_bytes < S.total || ws_bytes < L.total) return TTCD_ERR_WORKSPACE;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, dat<void>(state, S.status)));
  // the position counter sits after the status word in the state's status region
  long long* pos = dat<long long>(state, S.status + 8);
  return run_decode(c, static_cast<const __nv_bfloat16*>(x_t), beta_t, 0, w, p, state, S,
                    static_cast<__nv_bfloat16*>(y), workspace, L, pos, commit != 0);
}

ttcd_status ttcd_decode_state_read(const ttcd_block_params* p, int t_next, void* state,
                                   size_t state_bytes, float* state_out, void* stream) {
  TTCD_TRY(check_decode_params(p));
  if (t_next < 0 || !aligned16(state) || !aligned16(state_out)) return TTCD_ERR_INVALID_ARG;
  const DecState S = dec_state_layout(p);
  if (state_bytes < S.total) return TTCD_ERR_WORKSPACE;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, dat<void>(state, S.status)));
  const int d = p->d_model, f = p->d_ff, C = p->chunk, Cp = (C + 63) / 64 * 64;
  const int n = t_next % C;  // tokens of the current, partial chunk
  if (n == 0) {
    return cudaMemcpyAsync(state_out, dat<float>(state, S.S), static_cast<size_t>(p->B) * d * f * 4,
                           cudaMemcpyDeviceToDevice, c.s) == cudaSuccess
               ? TTCD_OK
               : TTCD_ERR_CUDA;
  }
  // rows n.. of the chunk buffers still hold the previous chunk: clear them (the
  // coming tokens of this chunk overwrite them anyway), then S + R^T K'
  using bf = __nv_bfloat16;
  for (int b = 0; b < p->B; ++b) {
    if (cudaMemsetAsync(dat<bf>(state, S.rc) + (static_cast<size_t>(b) * Cp + n) * d, 0,
                        static_cast<size_t>(Cp - n) * d * 2, c.s) != cudaSuccess ||
        cudaMemsetAsync(dat<bf>(state, S.kx) + (static_cast<size_t>(b) * Cp + n) * f, 0,
                        static_cast<size_t>(Cp - n) * f * 2, c.s) != cudaSuccess)
      return TTCD_ERR_CUDA;
  }
  return dec_commit(c, p, state, S, nullptr, dat<float>(state, S.S), state_out);
}

}  // extern "C"

// ================================================================== MLP backward
// The chain rule of the fast-weight MLP (backward.cuh has the formulas), bf16
// operands and fp32 accumulation: the forward's front half and chunk scan are
// recomputed into the forward workspace, then
//   dZ_S (read)  = dy (W_down + S_i)                  chunk-grouped GEMM
//   G_i, dS_in   = reverse prefix of dy_C^T Z_S,C    chunk scan walked backwards
//   dRt, s dRt   = Zbar_S G_i^T                       chunk-grouped GEMM
//   E, dD, ds    = dRt M                              GEMM (M read MN-major)
//   dbeta, coef  = from ds and the key norms
//   dZbar_S      = (s r) G_i + coef Zbar_S - dD       chunk-grouped GEMM
//   dM           = sum_t s dRt_t D_t^T;  dW_down, dW_proj from dM
//   dZ_P         = conv_P^T dZbar_P (+ dZ_S read);  tap gradients
//   da, db, Z    = gate/up recomputed with dZ          GEMM
//   du_P         = [da | db] [W_gate; W_up]            GEMM (MN-major)
//   dW_gate, dW_up = sum_rows da^T u, db^T u           token contractions
namespace {

struct BwdLayout {
  Layout F;  // the forward MLP's workspace (bf16 operands), first
  size_t dyp, zsp, dzsy, drt, dr, dd, epart, coef, dzbs, dm, dm16, dwd, dz, dab, zall, wgu,
      tpart, dsi, total;
};

BwdLayout bwd_layout(const ttcd_block_params* p) {
  const Dims m = dims_of(p);
  BwdLayout L;
  L.F = make_layout(p, false, false, false);
  const size_t n_epart = static_cast<size_t>(cdiv(m.f, 256));
  const size_t sz[18] = {
      static_cast<size_t>(m.P) * m.d * 2,                                    // dy, chunk-padded
      static_cast<size_t>(m.P) * m.f * 2,                                    // Z_S, chunk-padded
      static_cast<size_t>(m.BT) * m.f * 4,                                   // dZ_S of the read
      static_cast<size_t>(m.P) * m.d * 2,                                    // dRt
      static_cast<size_t>(m.P) * m.d * 2,                                    // s dRt
      static_cast<size_t>(m.P) * m.f * 4,                                    // dD
      n_epart * m.P * 4,                                                     // ds partials
      static_cast<size_t>(m.P) * 4,                                          // coef
      static_cast<size_t>(m.P) * m.f * 4,                                    // dZbar_S
      static_cast<size_t>(m.d) * m.f * 4,                                    // dM
      static_cast<size_t>(m.d) * m.f * 2,                                    // dM bf16
      static_cast<size_t>(m.d) * m.f * 4,                                    // dM W_proj^T
      2 * static_cast<size_t>(m.BT) * m.f * 4,                               // dZ
      2 * static_cast<size_t>(m.BT) * 2 * m.f * 2,                           // [da | db]
      2 * static_cast<size_t>(m.BT) * m.f * 2,                               // Z (recomputed)
      2 * static_cast<size_t>(m.f) * m.d * 2,                                // [W_gate; W_up]
      static_cast<size_t>(TAP_SPLITS) * 2 * m.f * p->conv_k * 4,             // tap partials
      static_cast<size_t>(p->B) * m.d * m.f * 4};                            // dL/dstate_in
  size_t* f[18] = {&L.dyp, &L.zsp, &L.dzsy, &L.drt, &L.dr, &L.dd, &L.epart, &L.coef, &L.dzbs,
                   &L.dm, &L.dm16, &L.dwd, &L.dz, &L.dab, &L.zall, &L.wgu, &L.tpart, &L.dsi};
  size_t off = L.F.total;
  for (int i = 0; i < 18; ++i) {
    *f[i] = off;
    off += (sz[i] + 1023) / 1024 * 1024;
  }
  L.total = off;
  return L;
}

ttcd_status check_bwd_params(const ttcd_block_params* p) {
  TTCD_TRY(check_params(p));
  if (p->dtype != TTCD_BF16) return TTCD_ERR_UNSUPPORTED;
  const Dims m = dims_of(p);
  if (2 * m.BT * 2 * m.f >= (1ll << 40) || m.P * static_cast<long long>(m.f) >= (1ll << 40))
    return TTCD_ERR_UNSUPPORTED;
  return TTCD_OK;
}

// Token contraction out[i, j] = sum_r A[r, i] B[r, j] (A [rows, m_dim] and B
// [rows, n_dim] token-major bf16, row pitches lda / ldb elements), fp32 out
// [m_dim, n_dim]: the chunk-scan kernel with one chunk of all rows.
ttcd_status launch_tsum(const Ctx& c, const __nv_bfloat16* A, long long lda, int m_dim,
                        const __nv_bfloat16* Bm, long long ldb, int n_dim, long long rows,
                        float* out) {
  using bf = __nv_bfloat16;
  CUtensorMap mA, mB;
  if (!make_map<bf>(&mA, A, m_dim, rows, lda * 2, 64, 64) ||
      !make_map<bf>(&mB, Bm, n_dim, rows, ldb * 2, 64, 64))
    return TTCD_ERR_CUDA;
  ScanArgs<bf> a{};
  a.d = m_dim;
  a.f = n_dim;
  a.Nc = 1;
  a.Cp = static_cast<int>((rows + 63) / 64 * 64);
  a.state_out = out;
  a.tiles_m = cdiv(m_dim, 128);
  a.tiles_n = cdiv(n_dim, SCAN_BN);
  a.commit_C = 1;
  constexpr int STAGES = 4;
  constexpr int smem = scan_smem_bytes<bf, STAGES, false>();
  auto kern = fastweight_scan_kernel<bf, STAGES, true>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TTCD_ERR_CUDA;
  TTCD_TRY(check_reg_split(reinterpret_cast<const void*>(kern), SCAN_THREADS, kScanRegSplit));
  kern<<<a.tiles_m * a.tiles_n, SCAN_THREADS, smem, c.s>>>(mA, mB, a, c.st);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

// Chunk-grouped geometry over the chunk-padded rows (every chunk Cp rows).
GemmGeom padded_chunk_geom(const ttcd_block_params* p, const Dims& m, int K, int tiles_n) {
  GemmGeom g;
  g.n_seq = p->B;
  g.T = m.Nc * m.Cp;
  g.C = m.Cp;
  g.Nc = m.Nc;
  g.K = K;
  g.tiles_m = cdiv(m.Cp, 128);
  g.tiles_n = tiles_n;
  g.b_group_rows = m.d;
  return g;
}

ttcd_status mlp_backward_bf16(const Ctx& c, const __nv_bfloat16* u_T, const __nv_bfloat16* u_S,
                              const float* beta, const ttcd_block_weights* w,
                              const ttcd_block_params* p, const float* state_in,
                              const __nv_bfloat16* d_y, const float* d_state_out, float* du_T,
                              float* du_S, float* d_beta, float* d_state_in,
                              const ttcd_mlp_grads* g, void* ws, const BwdLayout& L) {
  using bf = __nv_bfloat16;
  const Dims m = dims_of(p);
  const Layout& F = L.F;
  const bf* w_gate = static_cast<const bf*>(w->w_gate);
  const bf* w_up = static_cast<const bf*>(w->w_up);
  const bf* w_down = static_cast<const bf*>(w->w_down);
  const bf* w_proj = static_cast<const bf*>(w->w_proj);
  bf* U = at<bf>(ws, F, B_U);
  bf* Zs = at<bf>(ws, F, B_ZS16);
  bf* D = at<bf>(ws, F, B_D);
  bf* Kp = at<bf>(ws, F, B_KP);
  float* ssq = at<float>(ws, F, B_SSQ);
  float* kscale = at<float>(ws, F, B_KSCALE);
  bf* R = at<bf>(ws, F, B_R);
  bf* Wall = at<bf>(ws, F, B_WALL);  // W_down + S_i, then G_i
  bf* M = at<bf>(ws, F, B_M);
  bf* dyp = dat<bf>(ws, L.dyp);
  bf* zsp = dat<bf>(ws, L.zsp);
  float* dzsy = dat<float>(ws, L.dzsy);
  bf* drt = dat<bf>(ws, L.drt);
  bf* dr = dat<bf>(ws, L.dr);
  float* dD = dat<float>(ws, L.dd);
  float* epart = dat<float>(ws, L.epart);
  float* coef = dat<float>(ws, L.coef);
  float* dzbs = dat<float>(ws, L.dzbs);
  float* dM = dat<float>(ws, L.dm);
  bf* dM16 = dat<bf>(ws, L.dm16);
  float* dwd = dat<float>(ws, L.dwd);
  float* dZ = dat<float>(ws, L.dz);
  bf* dab = dat<bf>(ws, L.dab);
  bf* zall = dat<bf>(ws, L.zall);
  bf* wgu = dat<bf>(ws, L.wgu);
  float* tpart = dat<float>(ws, L.tpart);
  float* dsi = d_state_in ? d_state_in : dat<float>(ws, L.dsi);
  const long long n_u = m.BT * m.d;

  // forward front half and chunk scan, recomputed
  if (cudaMemcpyAsync(U, u_T, n_u * 2, cudaMemcpyDeviceToDevice, c.s) != cudaSuccess ||
      cudaMemcpyAsync(U + n_u, u_S, n_u * 2, cudaMemcpyDeviceToDevice, c.s) != cudaSuccess)
    return TTCD_ERR_CUDA;
  TTCD_TRY(mlp_front<bf>(c, p, F, ws, w_gate, w_up, w_down, w_proj,
                         static_cast<const bf*>(w->conv_T), static_cast<const bf*>(w->conv_S),
                         beta, 0, nullptr, nullptr));
  TTCD_TRY(launch_scan<bf>(c, p, F, ws, w_down, state_in, nullptr, Wall, false));

  // dZ_S of the read: dy (W_down + S_i), W_i [d, f] read MN-major per chunk
  {
    CUtensorMap mA, mB, mo;
    if (!map_rows<bf>(&mA, d_y, m.BT, m.d, 128) ||
        !make_map<bf>(&mB, Wall, m.f, static_cast<uint64_t>(p->B) * m.Nc * m.d, m.f * 2, 64, 64) ||
        !make_out_map<float>(&mo, dzsy, m.BT, m.f, m.f))
      return TTCD_ERR_CUDA;
    GemmGeom gg;
    gg.n_seq = p->B;
    gg.T = p->T;
    gg.C = p->chunk;
    gg.Nc = m.Nc;
    gg.K = m.d;
    gg.tiles_m = cdiv(p->chunk, 128);
    gg.tiles_n = cdiv(m.f, 256);
    gg.b_group_rows = m.d;
    EpiStore<float> e{dzsy, m.f, m.f, nullptr};
    TTCD_TRY((launch_rows_gemm_bmn<EpiStore<float>>(c, mA, mB, &mo, gg, e)));
  }
  // G_i and dL/dstate_in: the scan walked backwards over dy_C^T Z_S,C
  {
    const long long nd = m.P * (m.d / 8), nf = m.P * (m.f / 8);
    chunk_pad_rows_kernel<bf><<<static_cast<unsigned>(cdiv(nd, 256)), 256, 0, c.s>>>(
        d_y, dyp, m.d, p->T, p->chunk, m.Cp, m.Nc, m.P);
    TTCD_CHECK_LAUNCH();
    chunk_pad_rows_kernel<bf><<<static_cast<unsigned>(cdiv(nf, 256)), 256, 0, c.s>>>(
        Zs, zsp, m.f, p->T, p->chunk, m.Cp, m.Nc, m.P);
    TTCD_CHECK_LAUNCH();
    CUtensorMap mA, mB;
    if (!make_map<bf>(&mA, dyp, m.d, m.P, m.d * 2, 64, 64) ||
        !make_map<bf>(&mB, zsp, m.f, m.P, m.f * 2, 64, 64))
      return TTCD_ERR_CUDA;
    ScanArgs<bf> a{};
    a.d = m.d;
    a.f = m.f;
    a.Nc = m.Nc;
    a.Cp = m.Cp;
    a.w_down = nullptr;
    a.state_in = d_state_out;
    a.state_out = dsi;
    a.w_all = Wall;
    a.tiles_m = cdiv(m.d, 128);
    a.tiles_n = cdiv(m.f, SCAN_BN);
    a.commit_C = 1;
    a.reverse = true;
    constexpr int STAGES = 4;
    constexpr int smem = scan_smem_bytes<bf, STAGES, false>();
    auto kern = fastweight_scan_kernel<bf, STAGES, true>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return TTCD_ERR_CUDA;
    TTCD_TRY(check_reg_split(reinterpret_cast<const void*>(kern), SCAN_THREADS, kScanRegSplit));
    kern<<<p->B * a.tiles_m * a.tiles_n, SCAN_THREADS, smem, c.s>>>(mA, mB, a, c.st);
    TTCD_CHECK_LAUNCH();
  }
  // dRt = Zbar_S G_i^T and s dRt
  {
    CUtensorMap mA, mB;
    if (!map_rows<bf>(&mA, Kp, m.P, m.f, 128) ||
        !map_rows<bf>(&mB, Wall, static_cast<long long>(p->B) * m.Nc * m.d, m.f, gemm_b_box<bf>()))
      return TTCD_ERR_CUDA;
    EpiStoreScaledPair e{drt, dr, m.d, m.d, kscale};
    TTCD_TRY(launch_rows_gemm<bf>(c, mA, mB, nullptr, padded_chunk_geom(p, m, m.f, cdiv(m.d, 256)), e));
  }
  // E = dRt M: dD = s E and the partial dots D . E
  {
    CUtensorMap mA, mB;
    if (!map_rows<bf>(&mA, drt, m.P, m.d, 128) ||
        !make_map<bf>(&mB, M, m.f, m.d, m.f * 2, 64, 64))
      return TTCD_ERR_CUDA;
    EpiBwdE e{dD, D, epart, m.P, m.f, kscale};
    TTCD_TRY((launch_rows_gemm_bmn<EpiBwdE>(c, mA, mB, nullptr, plain_geom(m.P, cdiv(m.f, 256), m.d), e)));
  }
  key_backward_kernel<<<cdiv(m.P, 256), 256, 0, c.s>>>(epart, cdiv(m.f, 256), ssq,
                                                       cdiv(m.f, 128), beta, d_beta, coef, p->T,
                                                       p->chunk, m.Cp, m.Nc, m.P, p->l2_eps);
  TTCD_CHECK_LAUNCH();
  // dZbar_S = (s r) G_i + coef Zbar_S - dD
  {
    CUtensorMap mA, mB;
    if (!map_rows<bf>(&mA, R, m.P, m.d, 128) ||
        !make_map<bf>(&mB, Wall, m.f, static_cast<uint64_t>(p->B) * m.Nc * m.d, m.f * 2, 64, 64))
      return TTCD_ERR_CUDA;
    EpiBwdZbS e{dzbs, Kp, dD, m.f, coef};
    TTCD_TRY((launch_rows_gemm_bmn<EpiBwdZbS>(c, mA, mB, nullptr, padded_chunk_geom(p, m, m.d, cdiv(m.f, 256)), e)));
  }
  // dM = sum_t (s dRt)_t D_t^T;  dW_proj = W_down^T dM;  dW_down = dM W_proj^T + the read's
  TTCD_TRY(launch_tsum(c, dr, m.d, m.d, D, m.f, m.f, m.P, dM));
  TTCD_TRY((launch_cast<float, bf>(c, dM, dM16, static_cast<long long>(m.d) * m.f)));
  TTCD_TRY(launch_tsum(c, w_down, m.f, m.f, dM16, m.f, m.f, m.d, g->w_proj));
  {
    CUtensorMap mA, mB, mo;
    if (!map_rows<bf>(&mA, dM16, m.d, m.f, 128) || !map_rows<bf>(&mB, w_proj, m.f, m.f, 256) ||
        !make_out_map<float>(&mo, dwd, m.d, m.f, m.f))
      return TTCD_ERR_CUDA;
    EpiStore<float> e{dwd, m.f, m.f, nullptr};
    TTCD_TRY((launch_gemm<bf, 256, 4, false>(c, mA, mB, mB, &mo, plain_geom(m.d, cdiv(m.f, 256), m.f), e)));
  }
  {
    const long long n = static_cast<long long>(m.d) * m.f;
    dw_down_combine_kernel<<<static_cast<unsigned>(cdiv(n, 256)), 256, 0, c.s>>>(
        dwd, dsi, d_state_out, g->w_down, p->B, n);
    TTCD_CHECK_LAUNCH();
  }
  // dZ_P through the convs (teacher: dZbar_T = dD), plus the read's dZ_S
  {
    const bf* taps = at<bf>(ws, F, B_TAPS);  // the forward's table, [path][f/8][KMAX][8]
    const long long n = 2ll * p->B * cdiv(p->T, CONV_BWD_ROWS) * (m.f / 4);
    if (p->conv_k <= 4)
      conv_backward_kernel<4><<<static_cast<unsigned>(cdiv(n, 256)), 256, 0, c.s>>>(
          dD, dzbs, dzsy, taps, dZ, p->B, p->T, m.f, p->conv_k, p->chunk, m.Cp, m.Nc);
    else
      conv_backward_kernel<8><<<static_cast<unsigned>(cdiv(n, 256)), 256, 0, c.s>>>(
          dD, dzbs, dzsy, taps, dZ, p->B, p->T, m.f, p->conv_k, p->chunk, m.Cp, m.Nc);
    TTCD_CHECK_LAUNCH();
  }
  // gate/up recomputed: [da | db] and Z
  {
    CUtensorMap mA, mB0, mB1;
    if (!map_rows<bf>(&mA, U, 2 * m.BT, m.d, 128) || !map_rows<bf>(&mB0, w_gate, m.f, m.d, 128) ||
        !map_rows<bf>(&mB1, w_up, m.f, m.d, 128))
      return TTCD_ERR_CUDA;
    EpiSwiGLUBwd e{dZ, dab, zall, m.f};
    TTCD_TRY((launch_gemm<bf, 256, 4, true>(c, mA, mB0, mB1, nullptr,
                                            plain_geom(2 * m.BT, cdiv(m.f, 128), m.d), e)));
  }
  // tap gradients
  {
    // one wave: as many token splits as resident threads allow, at most TAP_SPLITS
    auto tap_kernel = p->conv_k <= 4 ? conv_tap_grad_kernel<4> : conv_tap_grad_kernel<8>;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tap_kernel, TAP_THREADS, 0) !=
        cudaSuccess)
      return TTCD_ERR_CUDA;
    const long long resident = static_cast<long long>(std::max(per_sm, 1)) * c.sms * TAP_THREADS;
    const int nsplit = static_cast<int>(
        std::min<long long>(TAP_SPLITS, std::max<long long>(1, resident / (2 * (m.f / 4)))));
    const int nt = 2 * (m.f / 4) * nsplit;
    tap_kernel<<<cdiv(nt, TAP_THREADS), TAP_THREADS, 0, c.s>>>(
        dD, dzbs, zall, tpart, p->B, p->T, m.f, p->conv_k, p->chunk, m.Cp, m.Nc, nsplit);
    TTCD_CHECK_LAUNCH();
    conv_tap_reduce_kernel<<<cdiv(2 * m.f * p->conv_k, 256), 256, 0, c.s>>>(
        tpart, g->conv_T, g->conv_S, m.f, p->conv_k, nsplit);
    TTCD_CHECK_LAUNCH();
  }
  // du_P = [da | db] [W_gate; W_up]
  {
    const size_t wbytes = static_cast<size_t>(m.f) * m.d * 2;
    if (cudaMemcpyAsync(wgu, w_gate, wbytes, cudaMemcpyDeviceToDevice, c.s) != cudaSuccess ||
        cudaMemcpyAsync(wgu + static_cast<size_t>(m.f) * m.d, w_up, wbytes,
                        cudaMemcpyDeviceToDevice, c.s) != cudaSuccess)
      return TTCD_ERR_CUDA;
    CUtensorMap mB;
    if (!make_map<bf>(&mB, wgu, m.d, 2 * m.f, m.d * 2, 64, 64)) return TTCD_ERR_CUDA;
    float* du[2] = {du_T, du_S};
    for (int path = 0; path < 2; ++path) {
      CUtensorMap mA, mo;
      if (!map_rows<bf>(&mA, dab + path * m.BT * 2 * m.f, m.BT, 2 * m.f, 128) ||
          !make_out_map<float>(&mo, du[path], m.BT, m.d, m.d))
        return TTCD_ERR_CUDA;
      EpiStore<float> e{du[path], m.d, m.d, nullptr};
      TTCD_TRY((launch_rows_gemm_bmn<EpiStore<float>>(c, mA, mB, &mo, plain_geom(m.BT, cdiv(m.d, 256), 2 * m.f), e)));
    }
  }
  // dW_gate = sum_rows da^T u, dW_up = sum_rows db^T u (both paths)
  TTCD_TRY(launch_tsum(c, dab, 2 * m.f, m.f, U, m.d, m.d, 2 * m.BT, g->w_gate));
  TTCD_TRY(launch_tsum(c, dab + m.f, 2 * m.f, m.f, U, m.d, m.d, 2 * m.BT, g->w_up));
  return TTCD_OK;
}

}  // namespace

extern "C" {

size_t ttcd_fastweight_mlp_backward_workspace_size(const ttcd_block_params* p) {
  if (check_bwd_params(p) != TTCD_OK) return 0;
  return bwd_layout(p).total;
}

ttcd_status ttcd_fastweight_mlp_backward(const void* u_T, const void* u_S, const float* beta,
                                         const ttcd_block_weights* w, const ttcd_block_params* p,
                                         const float* state_in, const void* d_y,
                                         const float* d_state_out, float* du_T, float* du_S,
                                         float* d_beta, float* d_state_in,
                                         const ttcd_mlp_grads* grads, void* workspace,
                                         size_t ws_bytes, void* stream) {
  TTCD_TRY(check_bwd_params(p));
  if (!aligned16(u_T) || !aligned16(u_S) || !aligned16(beta) || !aligned16(d_y) ||
      !aligned16(du_T) || !aligned16(du_S) || !aligned16(d_beta) || !weights_ok(w, false) ||
      !aligned16(workspace) || !grads)
    return TTCD_ERR_INVALID_ARG;
  if ((state_in && !aligned16(state_in)) || (d_state_out && !aligned16(d_state_out)) ||
      (d_state_in && !aligned16(d_state_in)))
    return TTCD_ERR_INVALID_ARG;
  const float* gp[6] = {grads->w_gate, grads->w_up,   grads->w_down,
                        grads->w_proj, grads->conv_T, grads->conv_S};
  for (const float* q : gp)
    if (!aligned16(q)) return TTCD_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(p);
  if (ws_bytes < L.total) return TTCD_ERR_WORKSPACE;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, workspace));
  using bf = __nv_bfloat16;
  return mlp_backward_bf16(c, static_cast<const bf*>(u_T), static_cast<const bf*>(u_S), beta, w,
                           p, state_in, static_cast<const bf*>(d_y), d_state_out, du_T, du_S,
                           d_beta, d_state_in, grads, workspace, L);
}

}  // extern "C"

// ================================================================== attention backward
namespace {

// status word, then delta_T, delta_S, lse2_T, lse2_S: [B Hq][Tp] fp32 each,
// Tp = T rounded up to the 128-query tile.
size_t attn_bwd_rows_bytes(int B, int T, int Hq) {
  const size_t Tp = static_cast<size_t>(T + ATT_BM - 1) / ATT_BM * ATT_BM;
  return (static_cast<size_t>(B) * Hq * Tp * 4 + 1023) / 1024 * 1024;
}
size_t attn_bwd_ws_bytes(int B, int T, int Hq) {
  return kStatusBytes + 4 * attn_bwd_rows_bytes(B, T, Hq);
}

// q rows have ld_q elements between tokens, k and v rows ld_kv (as launch_attn);
// o, dO, dq, dk, dv are dense.
template <int HD>
ttcd_status launch_attn_bwd(const Ctx& c, const void* q, const void* k, const void* v,
                            const void* o_T, const void* o_S, const float* lse_T,
                            const float* lse_S, const void* do_T, const void* do_S, float* dq,
                            float* dk, float* dv, int B, int T, int Hq, int Hkv, int w_S,
                            int w_T, float scale, void* ws, long long ld_q, long long ld_kv) {
  using bf = __nv_bfloat16;
  const long long BT = static_cast<long long>(B) * T;
  const size_t rows_bytes = attn_bwd_rows_bytes(B, T, Hq);
  float* delta_T = dat<float>(ws, kStatusBytes);
  float* delta_S = dat<float>(ws, kStatusBytes + rows_bytes);
  float* lse2_T = dat<float>(ws, kStatusBytes + 2 * rows_bytes);
  float* lse2_S = dat<float>(ws, kStatusBytes + 3 * rows_bytes);
  // dq is accumulated over the key tiles
  if (cudaMemsetAsync(dq, 0, static_cast<size_t>(BT) * Hq * HD * 4, c.s) != cudaSuccess)
    return TTCD_ERR_CUDA;
  const int n_kt = cdiv(T, ATT_BN);
  const int Tp = n_kt * ATT_BN;
  const long long rows = static_cast<long long>(B) * Hq;
  attn_bwd_rows_kernel<HD><<<static_cast<unsigned>(cdiv(2 * rows * Tp, 256)), 256, 0, c.s>>>(
      static_cast<const bf*>(o_T), static_cast<const bf*>(o_S), static_cast<const bf*>(do_T),
      static_cast<const bf*>(do_S), lse_T, lse_S, delta_T, delta_S, lse2_T, lse2_S, T, Tp, Hq,
      rows);
  TTCD_CHECK_LAUNCH();
  CUtensorMap mq, mk, mv, mdt, mds;
  const uint64_t wq = static_cast<uint64_t>(Hq) * HD, wkv = static_cast<uint64_t>(Hkv) * HD;
  if (!make_map<bf>(&mq, q, wq, BT, ld_q * 2, 64, 128) ||
      !make_map<bf>(&mk, k, wkv, BT, ld_kv * 2, 64, 128) ||
      !make_map<bf>(&mv, v, wkv, BT, ld_kv * 2, 64, 128) ||
      !make_map<bf>(&mdt, do_T, wq, BT, wq * 2, 64, 128) ||
      !make_map<bf>(&mds, do_S, wq, BT, wq * 2, 64, 128))
    return TTCD_ERR_CUDA;
  CUtensorMap mdq;  // dq as [BT, Hq * HD] fp32, boxes of 32 columns x 32 rows
  if (!make_map<float>(&mdq, dq, wq, BT, wq * 4, 32, 32)) return TTCD_ERR_CUDA;
  AttnBwdArgs a;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.lse2_T = lse2_T;
  a.lse2_S = lse2_S;
  a.delta_T = delta_T;
  a.delta_S = delta_S;
  a.B = B;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.w_S = w_S;
  a.w_T = w_T;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.n_kt = n_kt;
  auto kern = dual_window_attn_bwd_kernel<HD>;
  constexpr int smem = AttnBwdCfg<HD>::SMEM;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TTCD_ERR_CUDA;
  const long long grid = static_cast<long long>(a.n_kt) * B * Hkv;
  if (grid >= (1ll << 31)) return TTCD_ERR_UNSUPPORTED;
  TTCD_TRY(check_reg_split(reinterpret_cast<const void*>(kern), ATTB_THREADS, kAttnRegSplit));
  kern<<<static_cast<unsigned>(grid), ATTB_THREADS, smem, c.s>>>(mq, mk, mv, mdt, mds, mdq, a, c.st);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

}  // namespace

extern "C" {

size_t ttcd_dual_window_attn_backward_workspace_size(int B, int T, int Hq) {
  if (B < 1 || T < 1 || Hq < 1) return 0;
  return attn_bwd_ws_bytes(B, T, Hq);
}

ttcd_status ttcd_dual_window_attn_backward(const void* q, const void* k, const void* v,
                                           const void* o_T, const void* o_S, const float* lse_T,
                                           const float* lse_S, const void* do_T,
                                           const void* do_S, float* dq, float* dk, float* dv,
                                           int B, int T, int Hq, int Hkv, int hd, int w_S,
                                           int w_T, float scale, void* workspace,
                                           size_t ws_bytes, void* stream) {
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || w_S < 1 || w_T < w_S ||
      !(scale >= 0.f))
    return TTCD_ERR_INVALID_ARG;
  const void* need[] = {q, k, v, o_T, o_S, lse_T, lse_S, do_T, do_S, dq, dk, dv, workspace};
  for (const void* x : need)
    if (!aligned16(x)) return TTCD_ERR_INVALID_ARG;
  if (hd != 64 && hd != 128) return TTCD_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * T * Hq >= (1ll << 31)) return TTCD_ERR_UNSUPPORTED;
  if (ws_bytes < attn_bwd_ws_bytes(B, T, Hq)) return TTCD_ERR_WORKSPACE;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, workspace));
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(hd));
  const long long lq = static_cast<long long>(Hq) * hd, lkv = static_cast<long long>(Hkv) * hd;
  if (hd == 64)
    return launch_attn_bwd<64>(c, q, k, v, o_T, o_S, lse_T, lse_S, do_T, do_S, dq, dk, dv, B, T,
                               Hq, Hkv, w_S, w_T, sc, workspace, lq, lkv);
  return launch_attn_bwd<128>(c, q, k, v, o_T, o_S, lse_T, lse_S, do_T, do_S, dq, dk, dv, B, T,
                              Hq, Hkv, w_S, w_T, sc, workspace, lq, lkv);
}

}  // extern "C"

// ================================================================== block backward
// The chain rule of the block forward (run_block) in reverse, bf16 operands:
// the forward up to the MLP inputs is recomputed (q, k, v with RoPE, both
// attention outputs with their log-sum-exps, h_P = x + o_P W_o^T in fp32, u_P),
// then the MLP backward, the MLP RMSNorm backward with the output residual,
// o_proj's two GEMMs, the attention backward, RoPE's transpose, the QKV GEMMs
// and the input RMSNorm backward.
namespace {

constexpr int NORM_BLOCKS = 296;  // blocks of the RMSNorm backward kernels (2 per SM)

struct BlockBwdLayout {
  Layout F;    // the forward block workspace: qkv, o, the RoPE table, row scales
  BwdLayout M; // the MLP backward's workspace, at offset `mlp`
  size_t mlp, lse_T, lse_S, h, u, du, dh, dO, dq, dk, dv, dqkv, xn, dxn, gpart, attn, total;
};

BlockBwdLayout block_bwd_layout(const ttcd_block_params* p) {
  const Dims m = dims_of(p);
  BlockBwdLayout L;
  L.F = make_layout(p, true, false, false);
  L.M = bwd_layout(p);
  const size_t BT = static_cast<size_t>(m.BT), d = m.d, dq = static_cast<size_t>(m.Hq) * m.hd,
               dkv = static_cast<size_t>(m.Hkv) * m.hd;
  const size_t sz[16] = {L.M.total,
                         static_cast<size_t>(p->B) * m.Hq * p->T * 4,  // lse_T
                         static_cast<size_t>(p->B) * m.Hq * p->T * 4,  // lse_S
                         2 * BT * d * 4,                               // h_T, h_S
                         2 * BT * d * 2,                               // u_T, u_S
                         2 * BT * d * 4,                               // du_T, du_S
                         2 * BT * d * 2,                               // dh (bf16)
                         2 * BT * dq * 2,                              // do_T, do_S
                         BT * dq * 4,                                  // dq
                         BT * dkv * 4,                                 // dk
                         BT * dkv * 4,                                 // dv
                         BT * static_cast<size_t>(m.dqkv) * 2,         // dqkv (bf16)
                         BT * d * 2,                                   // xn (bf16)
                         BT * d * 4,                                   // dxn
                         2 * static_cast<size_t>(NORM_BLOCKS) * d * 4, // RMSNorm gain partials
                         attn_bwd_ws_bytes(p->B, p->T, m.Hq)};
  size_t* f[16] = {&L.mlp, &L.lse_T, &L.lse_S, &L.h, &L.u, &L.du, &L.dh, &L.dO, &L.dq, &L.dk,
                   &L.dv, &L.dqkv, &L.xn, &L.dxn, &L.gpart, &L.attn};
  size_t off = L.F.total;
  for (int i = 0; i < 16; ++i) {
    *f[i] = off;
    off += (sz[i] + 1023) / 1024 * 1024;
  }
  L.total = off;
  return L;
}

ttcd_status block_backward_bf16(const Ctx& c, const __nv_bfloat16* x, const float* beta,
                                const ttcd_block_weights* w, const ttcd_block_params* p,
                                const float* state_in, const __nv_bfloat16* d_out,
                                const float* d_state_out, float* dx, float* d_beta,
                                float* d_state_in, const ttcd_block_grads* g, void* ws,
                                const BlockBwdLayout& L) {
  using bf = __nv_bfloat16;
  const Dims m = dims_of(p);
  const Layout& F = L.F;
  const long long BT = m.BT, dq = static_cast<long long>(m.Hq) * m.hd;
  bf* qkv = at<bf>(ws, F, B_QKV);
  bf* o = at<bf>(ws, F, B_O);
  float* lse_T = dat<float>(ws, L.lse_T);
  float* lse_S = dat<float>(ws, L.lse_S);
  float* h = dat<float>(ws, L.h);
  bf* u = dat<bf>(ws, L.u);
  float* du = dat<float>(ws, L.du);
  bf* dh = dat<bf>(ws, L.dh);
  bf* dO = dat<bf>(ws, L.dO);
  float* gq = dat<float>(ws, L.dq);
  float* gk = dat<float>(ws, L.dk);
  float* gv = dat<float>(ws, L.dv);
  bf* dqkv = dat<bf>(ws, L.dqkv);
  bf* xn = dat<bf>(ws, L.xn);
  float* dxn = dat<float>(ws, L.dxn);
  float* gpart = dat<float>(ws, L.gpart);
  const float sc = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(m.hd));

  // ---- forward up to the MLP inputs
  TTCD_TRY(block_qkv<bf>(c, x, w, p, ws, F, qkv, 0, 0));
  TTCD_TRY(run_attn<bf>(c, qkv, qkv + dq, qkv + dq + static_cast<long long>(m.Hkv) * m.hd, o,
                        o + BT * dq, lse_T, lse_S, p->B, p->T, m.Hq, m.Hkv, m.hd, p->w_S, p->w_T,
                        sc, m.dqkv, m.dqkv));
  {  // h_P = x + o_P W_o^T, fp32, both paths
    CUtensorMap mA, mB, mo;
    if (!map_rows<bf>(&mA, o, 2 * BT, dq, 128) || !map_rows<bf>(&mB, w->w_o, m.d, dq, gemm_b_box<bf>()) ||
        !make_out_map<float>(&mo, h, 2 * BT, m.d, m.d))
      return TTCD_ERR_CUDA;
    EpiResidual<float, bf> e{h, m.d, x, m.d, BT, m.d};
    TTCD_TRY(launch_rows_gemm<bf>(c, mA, mB, &mo, plain_geom(2 * BT, cdiv(m.d, 256), static_cast<int>(dq)), e));
  }
  rmsnorm_kernel<float, bf, bf><<<cdiv(2 * BT, 8), 256, 0, c.s>>>(
      h, static_cast<const bf*>(w->g_mlp), u, 2 * BT, m.d, p->rms_eps);
  TTCD_CHECK_LAUNCH();

  // ---- the fast-weight MLP
  const ttcd_mlp_grads mg{g->w_gate, g->w_up, g->w_down, g->w_proj, g->conv_T, g->conv_S};
  TTCD_TRY(mlp_backward_bf16(c, u, u + BT * m.d, beta, w, p, state_in, d_out, d_state_out, du,
                             du + BT * m.d, d_beta, d_state_in, &mg, dat<void>(ws, L.mlp), L.M));

  // ---- MLP RMSNorm of both paths and the output residual: dh (bf16), dx = dh_T + dh_S
  const size_t norm_smem = static_cast<size_t>(m.d) * 4;
  mlp_norm_backward_kernel<<<NORM_BLOCKS, 256, norm_smem, c.s>>>(
      h, du, static_cast<const bf*>(w->g_mlp), d_out, dh, dx, gpart, BT, m.d, p->rms_eps);
  TTCD_CHECK_LAUNCH();
  column_sum_kernel<<<cdiv(m.d, 256), 256, 0, c.s>>>(gpart, g->g_mlp, NORM_BLOCKS, m.d);
  TTCD_CHECK_LAUNCH();

  // ---- o_proj: dO = dh W_o (W_o [d, Hq hd] read MN-major), dW_o = dh^T o
  {
    CUtensorMap mA, mB, mo;
    if (!map_rows<bf>(&mA, dh, 2 * BT, m.d, 128) ||
        !make_map<bf>(&mB, w->w_o, dq, m.d, dq * 2, 64, 64) ||
        !make_out_map<bf>(&mo, dO, 2 * BT, dq, dq))
      return TTCD_ERR_CUDA;
    EpiStore<bf> e{dO, dq, static_cast<int>(dq), nullptr};
    TTCD_TRY((launch_rows_gemm_bmn<EpiStore<bf>>(c, mA, mB, &mo, plain_geom(2 * BT, cdiv(dq, 256), m.d), e)));
  }
  TTCD_TRY(launch_tsum(c, dh, m.d, m.d, o, dq, static_cast<int>(dq), 2 * BT, g->w_o));

  // ---- attention (q, k, v are strided views of qkv)
  {
    void* aws = dat<void>(ws, L.attn);
    const bf* qp = qkv;
    const bf* kp = qkv + dq;
    const bf* vp = qkv + dq + static_cast<long long>(m.Hkv) * m.hd;
    if (m.hd == 64)
      TTCD_TRY(launch_attn_bwd<64>(c, qp, kp, vp, o, o + BT * dq, lse_T, lse_S, dO, dO + BT * dq,
                                   gq, gk, gv, p->B, p->T, m.Hq, m.Hkv, p->w_S, p->w_T, sc, aws,
                                   m.dqkv, m.dqkv));
    else
      TTCD_TRY(launch_attn_bwd<128>(c, qp, kp, vp, o, o + BT * dq, lse_T, lse_S, dO, dO + BT * dq,
                                    gq, gk, gv, p->B, p->T, m.Hq, m.Hkv, p->w_S, p->w_T, sc, aws,
                                    m.dqkv, m.dqkv));
  }
  {  // RoPE's transpose, packed with dv into one bf16 row per token
    const long long n = BT * (m.Hq + 2 * m.Hkv) * (m.hd / 2);
    rope_backward_pack_kernel<<<static_cast<unsigned>(cdiv(n, 256)), 256, 0, c.s>>>(
        gq, gk, gv, at<__half2>(ws, F, B_ROPE), dqkv, BT, p->T, m.Hq, m.Hkv, m.hd);
    TTCD_CHECK_LAUNCH();
  }

  // ---- QKV: dxn = dqkv W_qkv (W_qkv [dqkv, d] read MN-major), dW_qkv = dqkv^T xn
  {
    CUtensorMap mA, mB, mo;
    if (!map_rows<bf>(&mA, dqkv, BT, m.dqkv, 128) ||
        !make_map<bf>(&mB, w->w_qkv, m.d, m.dqkv, static_cast<uint64_t>(m.d) * 2, 64, 64) ||
        !make_out_map<float>(&mo, dxn, BT, m.d, m.d))
      return TTCD_ERR_CUDA;
    EpiStore<float> e{dxn, m.d, m.d, nullptr};
    TTCD_TRY((launch_rows_gemm_bmn<EpiStore<float>>(c, mA, mB, &mo, plain_geom(BT, cdiv(m.d, 256), m.dqkv), e)));
  }
  rmsnorm_kernel<bf, bf, bf><<<cdiv(BT, 8), 256, 0, c.s>>>(
      x, static_cast<const bf*>(w->g_attn), xn, BT, m.d, p->rms_eps);
  TTCD_CHECK_LAUNCH();
  TTCD_TRY(launch_tsum(c, dqkv, m.dqkv, m.dqkv, xn, m.d, m.d, BT, g->w_qkv));

  // ---- input RMSNorm
  input_norm_backward_kernel<<<NORM_BLOCKS, 256, norm_smem, c.s>>>(
      x, dxn, static_cast<const bf*>(w->g_attn), dx, gpart + static_cast<long long>(NORM_BLOCKS) * m.d,
      BT, m.d, p->rms_eps);
  TTCD_CHECK_LAUNCH();
  column_sum_kernel<<<cdiv(m.d, 256), 256, 0, c.s>>>(
      gpart + static_cast<long long>(NORM_BLOCKS) * m.d, g->g_attn, NORM_BLOCKS, m.d);
  TTCD_CHECK_LAUNCH();
  return TTCD_OK;
}

}  // namespace

extern "C" {

size_t ttcd_block_backward_workspace_size(const ttcd_block_params* p) {
  if (check_bwd_params(p) != TTCD_OK) return 0;
  if (p->head_dim != 64 && p->head_dim != 128) return 0;
  return block_bwd_layout(p).total;
}

ttcd_status ttcd_block_backward(const void* x, const float* beta, const ttcd_block_weights* w,
                                const ttcd_block_params* p, const float* state_in,
                                const void* d_out, const float* d_state_out, float* dx,
                                float* d_beta, float* d_state_in, const ttcd_block_grads* grads,
                                void* workspace, size_t ws_bytes, void* stream) {
  TTCD_TRY(check_bwd_params(p));
  if (p->head_dim != 64 && p->head_dim != 128) return TTCD_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(beta) || !aligned16(d_out) || !aligned16(dx) ||
      !aligned16(d_beta) || !weights_ok(w, true) || !aligned16(workspace) || !grads)
    return TTCD_ERR_INVALID_ARG;
  if ((state_in && !aligned16(state_in)) || (d_state_out && !aligned16(d_state_out)) ||
      (d_state_in && !aligned16(d_state_in)))
    return TTCD_ERR_INVALID_ARG;
  const float* gp[10] = {grads->w_qkv, grads->w_o,    grads->g_attn, grads->g_mlp,
                         grads->w_gate, grads->w_up,  grads->w_down, grads->w_proj,
                         grads->conv_T, grads->conv_S};
  for (const float* q : gp)
    if (!aligned16(q)) return TTCD_ERR_INVALID_ARG;
  if (static_cast<size_t>(p->d_model) * 4 > 48 * 1024) return TTCD_ERR_UNSUPPORTED;
  const BlockBwdLayout L = block_bwd_layout(p);
  if (ws_bytes < L.total) return TTCD_ERR_WORKSPACE;
  Ctx c;
  TTCD_TRY(make_ctx(stream, c, workspace));
  using bf = __nv_bfloat16;
  return block_backward_bf16(c, static_cast<const bf*>(x), beta, w, p, state_in,
                             static_cast<const bf*>(d_out), d_state_out, dx, d_beta, d_state_in,
                             grads, workspace, L);
}

}  // extern "C"
