// Host-side helpers shared by the library's translation units: error reporting,
// tensor-map construction, per-phase timing, the GEMM / row-kernel launchers, split and
// tile choices, and the status-word hand-off of every entry point.  Globals are C++17
// inline variables (one definition across the library).
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <vector>

#include "lora_mlp.h"
#include "gemm_sm100.cuh"
#include "rowops.cuh"
#include "rope.cuh"
#include "lowrank_dual.cuh"

namespace lm {
namespace host {

inline thread_local char g_err[512] = "no error";

inline int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

#define CUDA_TRY(expr)                                                                   \
  do {                                                                                   \
    cudaError_t e_ = (expr);                                                             \
    if (e_ != cudaSuccess)                                                               \
      return fail(LORA_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_));        \
  } while (0)

#define TRY(expr)            \
  do {                       \
    int rc_ = (expr);        \
    if (rc_ != LORA_OK) return rc_; \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

inline bool debug_mode() {
  static int v = [] {
    const char* e = getenv("LORA_MLP_DEBUG");
    return (e && e[0] && e[0] != '0') ? 1 : 0;
  }();
  return v != 0;
}

// Which rank-r products run in the single-pass streaming kernel (lowrank_dual.cuh) rather
// than as split-K / split-T GEMMs; both forms compute the same quantities.  LORA_MLP_DUAL:
//   1 (default): the fused backward passes (Q with dB from one read of dY, of dG / dU) and
//                the reductions over T (dAg / dAu, dAd), where it measured faster;
//   2: every rank-r product (also the forward projections P, Pd, which measured a few us
//      slower than the split-K GEMM);
//   0: none (two passes over each activation gradient).
// Read once per process.
inline int dual_mode() {
  static int v = [] {
    const char* e = getenv("LORA_MLP_DUAL");
    if (!e || !e[0]) return 1;
    return e[0] == '0' ? 0 : (e[0] == '2' ? 2 : 1);
  }();
  return v;
}

inline unsigned long long wait_limit_ns() {
  const char* e = getenv("LORA_MLP_WAIT_LIMIT_MS");
  long long ms = e ? atoll(e) : 5000;
  if (ms < 1) ms = 1;
  return static_cast<unsigned long long>(ms) * 1000000ull;
}

// ------------------------------------------------------------------ driver API
inline PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

inline int get_encoder() {
  if (g_encode) return LORA_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
    return fail(LORA_ERR_CUDA, "cannot resolve cuTensorMapEncodeTiled");
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return LORA_OK;
}

// 2-D bf16 tensor map, 128-byte swizzle (or `swz`): `inner` contiguous elements per row,
// `outer` rows `ld` elements apart, box of box_inner x box_outer elements.
inline int make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
             uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  TRY(get_encoder());
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                        box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(LORA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): inner=%llu outer=%llu ld=%llu box=%ux%u",
                static_cast<int>(r), (unsigned long long)inner, (unsigned long long)outer,
                (unsigned long long)ld, box_inner, box_outer);
  return LORA_OK;
}
// Untyped 2-D map without swizzle (4-bit codes as bytes, block absmax as fp32).
inline int make_map_raw(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, uint32_t esize, uint64_t inner,
                 uint64_t outer, uint64_t ld, uint32_t box_inner, uint32_t box_outer) {
  TRY(get_encoder());
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * esize};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(LORA_ERR_CUDA, "cuTensorMapEncodeTiled (raw) failed (%d): inner=%llu outer=%llu box=%ux%u",
                static_cast<int>(r), (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
  return LORA_OK;
}
// 4-bit weight W [rows x cols] (codes: rows x cols/2 bytes; absmax: rows x cols/64 fp32)
// read with K = cols contiguous (forward use): boxes {32 B, n_rows} and {4 floats, n_rows}.
inline int map_q4_k(CUtensorMap* mq, CUtensorMap* ma, const uint8_t* q, const float* am, uint64_t rows, uint64_t cols,
             uint32_t n_rows) {
  TRY(make_map_raw(mq, q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cols / 2, rows, cols / 2, 32, n_rows));
  return make_map_raw(ma, am, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, cols / 64, rows, cols / 64, 4, n_rows);
}
// The same weight read with N = cols contiguous and K = rows (backward use): boxes
// {n_cols / 2 B, 64 K rows} and {4 floats, 64 K rows}.
inline int map_q4_mn(CUtensorMap* mq, CUtensorMap* ma, const uint8_t* q, const float* am, uint64_t rows, uint64_t cols,
              uint32_t n_cols) {
  TRY(make_map_raw(mq, q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cols / 2, rows, cols / 2, n_cols / 2, 64));
  return make_map_raw(ma, am, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, cols / 64, rows, cols / 64, 4, 64);
}

// Operand with K contiguous: [rows x K], box 64 (K) x box_rows.
inline int map_k(CUtensorMap* m, const void* p, uint64_t rows, uint64_t K, uint64_t ld, uint32_t box_rows) {
  return make_map(m, p, K, rows, ld, 64, box_rows);
}
// Operand with M/N contiguous: [K x MN], box 64 (MN) x 64 (K).
inline int map_mn(CUtensorMap* m, const void* p, uint64_t K, uint64_t MN, uint64_t ld) {
  return make_map(m, p, MN, K, ld, 64, 64);
}
// The same operand as a 3-D view {64 elements, K rows, MN/64 chunks} (MN % 64 == 0),
// box {64, 64, chunks}: one load fills `chunks` chunk-major 8 KB sub-tiles.
inline int map_mn3(CUtensorMap* m, const void* p, uint64_t K, uint64_t MN, uint64_t ld, uint32_t chunks) {
  TRY(get_encoder());
  cuuint64_t dims[3] = {64, K, MN / 64};
  cuuint64_t strides[2] = {ld * 2, 128};
  cuuint32_t box[3] = {64, 64, chunks};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(LORA_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d): K=%llu MN=%llu ld=%llu chunks=%u",
                static_cast<int>(r), (unsigned long long)K, (unsigned long long)MN, (unsigned long long)ld, chunks);
  return LORA_OK;
}

// --------------------------------------------------------------------- timing
inline const char* kPhaseNames[LORA_NUM_PHASES] = {
    "rmsnorm_fwd", "proj_P_gate_up", "gemm_gate_up_swiglu", "proj_P_down", "gemm_down",
    "lowrank_bwd_down", "gemm_dact_swiglu_bwd", "lowrank_bwd_gate_up", "gemm_dH", "rmsnorm_bwd",
    "zero_grads", "reduce_dA_gate_up", "reduce_dB_gate_up", "reduce_dB_down", "reduce_dA_down",
    "norm_weight_grad", "other", "qkv_gemm", "qkv_gemm_dH", "qkv_lowrank", "o_gemm", "o_gemm_dX", "o_lowrank",
    "rope", "ce_gemm_lse", "ce_finalize", "ce_gemm_dlogits", "ce_gemm_dH"};
enum Phase {
  PH_RMS_FWD = 0, PH_P_GU, PH_GATEUP, PH_P_D, PH_DOWN, PH_Q_D, PH_DACT, PH_Q_GU, PH_DH,
  PH_RMS_BWD, PH_ZERO, PH_RED_DA_GU, PH_RED_DB_GU, PH_RED_DB_D, PH_RED_DA_D, PH_DW, PH_OTHER,
  PH_QKV_GEMM, PH_QKV_DH, PH_QKV_LOWRANK, PH_O_GEMM, PH_O_DX, PH_O_LOWRANK, PH_ROPE, PH_CE_LSE, PH_CE_FIN,
  PH_CE_DZ, PH_CE_DH
};

struct Timing {
  std::mutex mu;
  bool on = false;
  struct Rec { cudaEvent_t a, b; int phase; };
  std::vector<Rec> pending;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
inline Timing g_timing;

struct PhaseScope {
  cudaStream_t st;
  int phase;
  cudaEvent_t a = nullptr, b = nullptr;
  PhaseScope(cudaStream_t s, int ph) : st(s), phase(ph) {
    std::lock_guard<std::mutex> lk(g_timing.mu);
    if (!g_timing.on) return;
    a = g_timing.get();
    b = g_timing.get();
    cudaEventRecord(a, st);
  }
  ~PhaseScope() {
    if (!a) return;
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> lk(g_timing.mu);
    g_timing.pending.push_back({a, b, phase});
  }
};

// ------------------------------------------------------------------ launches
inline int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

constexpr int kSmemLimit = 232448;  // 227 KB per CTA on sm_100

// Launch one GEMM.  PAIR = 2 runs clusters of two CTAs sharing 256-row tiles
// (tcgen05 cta_group::2); the caller sets tiles_m = ceil(M / (128 * PAIR)).
// MT = 2 runs units of two M tiles (2 x 128 x PAIR rows) that share every B stage; the
// caller sets tiles_m = ceil(M / (128 * PAIR * MT)).
template <int A_MN, int B_MN, int NACC, int EPI, int PAIR = 1, int FUSE = 0, int Q4 = 0, int MT = 1>
int launch_gemm(GemmArgs& a, cudaStream_t st, int phase) {
  static_assert(PAIR == 1 || (PAIR == 2 && !A_MN), "CTA pairs take a K-major A operand");
  static_assert(MT == 1 || (MT == 2 && !A_MN), "two M tiles per unit take a K-major A operand");
  if (a.bn < 16 || a.bn > 256 || a.bn % 16 || (B_MN && a.bn % (64 * PAIR)) || (!B_MN && (a.bn / PAIR) % 8))
    return fail(LORA_ERR_UNSUPPORTED, "internal: bad N tile %d", a.bn);
  a.stage_bytes = MT * BM * BK * 2 + NACC * (a.bn / PAIR) * BK * 2;
  a.cr_bytes = 0;
  if (Q4) {  // 4-bit B: expanded B slots per stage; codes + absmax in a ring of their own
    const Q4Layout QL = q4_layout(a.bn, PAIR, FUSE, B_MN, NACC);
    a.stage_bytes = MT * BM * BK * 2 + QL.slots * QL.b_unit;
    a.cr_bytes = (QL.slots * (QL.q_unit + QL.m_unit) + 1023) & ~1023u;
  }
  a.stage_bytes = (a.stage_bytes + 1023) & ~1023u;
  const int extra = Q4 ? 2560 : 256;  // barriers (+ the 4-bit code table)
  const int ring = Q4 ? code_ring(MT) * static_cast<int>(a.cr_bytes) : 0;
  const int stg = a.epi_tma ? kEpiWarps * kEpiStageBytes : 0;  // epilogue staging for TMA stores
  const int avail = kSmemLimit - 1024 - extra - ring - stg;
  a.stages = std::min(kMaxStages, avail / static_cast<int>(a.stage_bytes));
  static const int stage_cap = [] {
    const char* e = getenv("LORA_MLP_MAX_STAGES");  // tuning knob: cap the TMA ring depth
    return e ? atoi(e) : 0;
  }();
  if (stage_cap >= 2) a.stages = std::min(a.stages, stage_cap);
  if (a.stages < 2) return fail(LORA_ERR_UNSUPPORTED, "internal: stage does not fit");
  // accumulator sets: two when they fit in TMEM's 512 columns, else one
  const int set_cols = MT * NACC * a.bn;
  a.nbuf = 2 * set_cols <= 512 ? 2 : 1;
  const int cols = a.nbuf * set_cols;
  uint32_t tc = 32;
  while (tc < static_cast<uint32_t>(cols)) tc <<= 1;
  if (tc > 512) return fail(LORA_ERR_UNSUPPORTED, "internal: TMEM columns %d > 512", cols);
  a.tmem_cols = tc;
  int smem = 1024 + a.stages * static_cast<int>(a.stage_bytes) + ring + stg + extra;
  // more than half of TMEM per CTA: keep one CTA per SM so allocation never waits
  if (tc > 256) smem = std::max(smem, kSmemLimit / 2 + 4096);
  a.limit_ns = wait_limit_ns();
  const long long tiles = static_cast<long long>(a.tiles_m) * a.tiles_n * a.splits;
  if (tiles <= 0) return LORA_OK;
  if (tiles > 0x7fffffffLL) return fail(LORA_ERR_UNSUPPORTED, "too many tiles");
  const int units = static_cast<int>(std::min<long long>(tiles, sm_count() / PAIR));
  auto kern = gemm_kernel<A_MN, B_MN, NACC, EPI, PAIR, FUSE, Q4, MT>;
  CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  PhaseScope ps(st, phase);
  if (PAIR == 1) {
    kern<<<units, gemm_threads(Q4), smem, st>>>(a);
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units * PAIR, 1, 1);
    cfg.blockDim = dim3(gemm_threads(Q4), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = PAIR;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, a));
  }
  CUDA_TRY(cudaGetLastError());
  return LORA_OK;
}

inline int launch_rms_fwd(cudaStream_t st, const void* X, const void* w, void* H, float* rstd, long long T, int d,
                   float eps) {
  const int nvec = d / 8;
  int threads = kRowThreads, vpt = (nvec + threads - 1) / threads;
  if (vpt > 8) {
    vpt = 8;
    threads = round_up((nvec + 7) / 8, 32);
  }
  if (threads > 1024) return fail(LORA_ERR_UNSUPPORTED, "d = %d too large for the row kernel", d);
  int v = vpt <= 1 ? 1 : vpt <= 2 ? 2 : vpt <= 4 ? 4 : 8;
  auto X16 = static_cast<const uint16_t*>(X);
  auto w16 = static_cast<const uint16_t*>(w);
  auto H16 = static_cast<uint16_t*>(H);
  PhaseScope ps(st, PH_RMS_FWD);
  for (long long r0 = 0; r0 < T; r0 += 0x7fffffffLL) {
    unsigned int rows = static_cast<unsigned int>(std::min<long long>(T - r0, 0x7fffffffLL));
    const uint16_t* x = X16 + r0 * d;
    uint16_t* h = H16 + r0 * d;
    if (threads <= kRowThreads) {
      switch (v) {
        case 1: rmsnorm_fwd_kernel<1, kRowThreads><<<rows, threads, 0, st>>>(x, w16, h, rstd + r0, d, eps); break;
        case 2: rmsnorm_fwd_kernel<2, kRowThreads><<<rows, threads, 0, st>>>(x, w16, h, rstd + r0, d, eps); break;
        case 4: rmsnorm_fwd_kernel<4, kRowThreads><<<rows, threads, 0, st>>>(x, w16, h, rstd + r0, d, eps); break;
        default: rmsnorm_fwd_kernel<8, kRowThreads><<<rows, threads, 0, st>>>(x, w16, h, rstd + r0, d, eps); break;
      }
    } else {
      rmsnorm_fwd_kernel<8, 1024><<<rows, threads, 0, st>>>(x, w16, h, rstd + r0, d, eps);
    }
  }
  CUDA_TRY(cudaGetLastError());
  return LORA_OK;
}

inline int launch_rms_bwd(cudaStream_t st, const float* dH, const void* X, const void* w, const float* rstd, void* dX,
                   long long T, int d, const void* dY = nullptr) {
  const int nvec = d / 8;
  int threads = kRowThreads, vpt = (nvec + threads - 1) / threads;
  if (vpt > 4) {
    vpt = 4;
    threads = round_up((nvec + 3) / 4, 32);
  }
  if (threads > 1024) return fail(LORA_ERR_UNSUPPORTED, "d = %d too large for the row kernel", d);
  int v = vpt <= 1 ? 1 : vpt <= 2 ? 2 : 4;
  auto X16 = static_cast<const uint16_t*>(X);
  auto w16 = static_cast<const uint16_t*>(w);
  auto dX16 = static_cast<uint16_t*>(dX);
  auto dY16 = static_cast<const uint16_t*>(dY);
  PhaseScope ps(st, PH_RMS_BWD);
  for (long long r0 = 0; r0 < T; r0 += 0x7fffffffLL) {
    unsigned int rows = static_cast<unsigned int>(std::min<long long>(T - r0, 0x7fffffffLL));
    const float* g = dH + r0 * d;
    const uint16_t* x = X16 + r0 * d;
    const uint16_t* y = dY16 ? dY16 + r0 * d : nullptr;
    uint16_t* o = dX16 + r0 * d;
    if (threads <= kRowThreads) {
      switch (v) {
        case 1: rmsnorm_bwd_kernel<1, kRowThreads><<<rows, threads, 0, st>>>(g, x, w16, rstd + r0, y, o, d); break;
        case 2: rmsnorm_bwd_kernel<2, kRowThreads><<<rows, threads, 0, st>>>(g, x, w16, rstd + r0, y, o, d); break;
        default: rmsnorm_bwd_kernel<4, kRowThreads><<<rows, threads, 0, st>>>(g, x, w16, rstd + r0, y, o, d); break;
      }
    } else {
      rmsnorm_bwd_kernel<4, 1024><<<rows, threads, 0, st>>>(g, x, w16, rstd + r0, y, o, d);
    }
  }
  CUDA_TRY(cudaGetLastError());
  return LORA_OK;
}

// Upper bound of the K-split count of a rank-r projection (fixed, so workspace sizes
// do not depend on the device).
constexpr int kProjMaxSplits = 16;
// Number of K splits for `tiles` output tiles over nkb k-blocks: the split that
// fills whole waves of a 148-SM part best (at most max_splits), preferring fewer
// splits among those within 3 % of the best.  Depends only on the sizes, so
// workspace sizes do not depend on the device.
inline int balanced_splits(long long tiles, long long nkb, int max_splits) {
  const double sms = 148.0;
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= max_splits && s <= nkb; ++s) {
    const long long per = (nkb + s - 1) / s;
    const long long ss = (nkb + per - 1) / per;        // splits actually formed
    const double w = static_cast<double>(tiles * ss) / sms;
    double eff = w / std::ceil(w);
    if (tiles * ss < sms) eff = w;                      // a partial single wave
    if (eff > best_eff + 0.03) { best_eff = eff; best = static_cast<int>(ss); }
  }
  return best;
}
inline int proj_splits(long long T, long long K) {
  const long long tiles = (T + 127) / 128;
  const long long nkb = (K + 63) / 64;
  return balanced_splits(tiles, nkb, kProjMaxSplits);
}

template <class P>
inline P* at(void* base, size_t off) { return reinterpret_cast<P*>(static_cast<char*>(base) + off); }
template <class P>
inline const P* at(const void* base, size_t off) { return reinterpret_cast<const P*>(static_cast<const char*>(base) + off); }

inline int check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return fail(LORA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (!aligned16(p)) return fail(LORA_ERR_ALIGNMENT, "pointer %p is not 16-byte aligned", p);
  }
  return LORA_OK;
}

// Every call clears its status word first (in every mode), so the word reports the
// bounded waits of the most recent call that used it (lora_mlp_status reads it).
inline int begin_call(int* status, cudaStream_t st) {
  if (status) CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), st));
  return LORA_OK;
}

inline int end_call(int* status, cudaStream_t st) {
  if (!debug_mode()) return LORA_OK;
  CUDA_TRY(cudaStreamSynchronize(st));
  if (status) {
    int v = 0;
    CUDA_TRY(cudaMemcpy(&v, status, sizeof(int), cudaMemcpyDeviceToHost));
    if ((v & 0xF00) == kDevBadIndex)
      return fail(LORA_ERR_INVALID_ARG, "a device-side index input was out of range (code 0x%x)", v);
    if (v) return fail(LORA_ERR_TIMEOUT, "device-side bounded wait gave up (code 0x%x)", v);
  }
  return LORA_OK;
}

inline GemmArgs new_args(int* status) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.splits = 1;
  a.alpha = 1.0f;
  a.status = status;
  for (int s = 0; s < kMaxSegs; ++s) a.seg[s].b_map[0] = a.seg[s].b_map[1] = -1;
  return a;
}

// Banded tile order for a dense GEMM: `group_m` row tiles per band (the band's A
// panels are re-read from L2 by every N tile).  LORA_MLP_RASTER=0 selects the plain
// M-fastest order instead, LORA_MLP_BAND=g sets every band to g row tiles (tuning
// comparisons).
inline void set_band(GemmArgs& a, int group_m) {
  static const int off = [] {
    const char* e = getenv("LORA_MLP_RASTER");
    return e && e[0] == '0' ? 1 : 0;
  }();
  static const int forced = [] {
    const char* e = getenv("LORA_MLP_BAND");
    return e ? atoi(e) : 0;
  }();
  if (forced >= 1) group_m = forced;
  if (off || group_m >= a.tiles_m) return;
  a.raster = 2;
  a.group_m = group_m;
}

// Epilogue outputs ([rows x cols] bf16 or fp32, row stride ld) written by TMA stores from
// shared-memory staging, for GEMMs run with MT = 2 (one accumulator set: the epilogue no longer
// hides behind the next unit's main loop): maps at a.maps[first ...].  LORA_MLP_EPI_TMA=0 keeps
// the per-thread stores (tuning comparison).
inline bool epilogue_tma_enabled() {
  static const int on = [] {
    const char* e = getenv("LORA_MLP_EPI_TMA");
    return e && e[0] == '0' ? 0 : 1;
  }();
  return on != 0;
}
// MT = 2 gain for a short-K bf16 GEMM whose epilogue only stores (gate/up, the Q/K/V and
// o_proj GEMMs): worth it when the stores leave by TMA (see kMtGainBf16Swiglu), not otherwise.
inline double mt_gain_bf16_stores() { return epilogue_tma_enabled() ? 0.8 : 1.02; }
inline int set_epilogue_tma(GemmArgs& a, int first, std::initializer_list<const void*> outs, long long rows,
                            long long cols, long long ld, bool fp32 = false) {
  if (!epilogue_tma_enabled()) return LORA_OK;
  if (first < 0 || first + static_cast<int>(outs.size()) > kMaxMaps)
    return fail(LORA_ERR_UNSUPPORTED, "internal: bad epilogue maps");
  int i = first;
  for (const void* p : outs)
    TRY(make_map_raw(&a.maps[i++], p, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     fp32 ? 4 : 2, cols, rows, ld, 16, 32));
  static const int drain_mode = [] {
    // tuning knob: 0 = convert straight from TMEM, 1 = hold the second M tile, 2 = hold both
    const char* e = getenv("LORA_MLP_EPI_DRAIN");
    const int v = e ? atoi(e) : 2;
    return v >= 0 && v <= 2 ? v : 2;
  }();
  // empty TMEM into registers first: one bf16 output with N tile 256, or the SwiGLU forward's
  // three outputs with N tile 128 (the kernel takes it only with two M tiles per unit)
  const bool drainable = !fp32 && (outs.size() == 3 ? a.bn == 128 : outs.size() == 1 && a.bn == 256);
  a.epi_drain = drainable ? drain_mode : 0;
  a.epi_tma = 1;
  a.out_map0 = first;
  return LORA_OK;
}

inline void set_hints(GemmArgs& a, int a_hint, int b_hint) {
  for (int s = 0; s < a.nseg; ++s) {
    a.seg[s].a_hint = a_hint;
    a.seg[s].b_hint = b_hint;
  }
}

inline void set_seg(GemmArgs& a, int s, int amap, int ak0, int b0, int bk0, int b1, int bk1, int klen) {
  a.seg[s].a_map = amap;
  a.seg[s].a_k0 = ak0;
  a.seg[s].b_map[0] = b0;
  a.seg[s].b_k0[0] = bk0;
  a.seg[s].b_map[1] = b1;
  a.seg[s].b_k0[1] = bk1;
  a.seg[s].k_len = klen;
  a.nseg = std::max(a.nseg, s + 1);
}

// Tile shape of a dense GEMM (M = T rows, N columns): CTA pair (256-row tiles) or
// single CTA, N tile 256 or 128 — the option that fills whole waves of the 148 SMs
// best (ties within 2 % go to the larger tile, then to the pair).
struct TileChoice { int pair, bn; };
inline TileChoice pick_tiles(long long T, int N, bool mn_major) {
  TileChoice best{T > 128 ? 2 : 1, N >= 256 ? 256 : (mn_major ? round_up(N, 64) : round_up(N, 16))};
  if (N < 256 || T <= 128) return best;
  // Cost = whole waves x time of one tile.  A tile of N = 128 takes about 0.8 of an
  // N = 256 tile's time (measured: the per-k-block issue and barrier work of the MMA
  // thread does not shrink with N), so N = 128 only pays where it saves many waves.
  double best_cost = 1e30;
  const int bns[2] = {256, 128};
  for (int pair = 2; pair >= 1; --pair) {
    for (int bn : bns) {
      const long long units = ((T + 128LL * pair - 1) / (128LL * pair)) * ((N + bn - 1) / bn);
      const double waves = std::ceil(units / (148.0 / pair));
      const double cost = waves * (bn == 256 ? 1.0 : 0.8);
      if (cost < best_cost - 1e-9) {
        best_cost = cost;
        best = TileChoice{pair, bn};
      }
    }
  }
  return best;
}

// M tiles per unit for a K-major-A GEMM with M = T rows and N columns in tiles of bn.
// Two M tiles per unit share every B stage (a quarter fewer operand bytes per FLOP, and
// for 4-bit weights half the expansion work per FLOP) but leave one accumulator set in
// TMEM, so the epilogue no longer overlaps the next unit's main loop.  `gain` is the
// measured per-FLOP time of MT = 2 relative to MT = 1 for the kind of GEMM (8B shape:
// 4-bit gate/up 0.79, cross-entropy logits 0.81-0.87, bf16 gate/up with its three-output
// epilogue 1.02); MT = 2 is taken when its waves of a 148-SM part cost less.
// LORA_MLP_MT=1 or 2 forces the choice (tuning comparison, tests).
inline int pick_mt(long long T, int pair, int bn, long long N, double gain) {
  static const int force = [] {
    const char* e = getenv("LORA_MLP_MT");
    return e ? atoi(e) : 0;
  }();
  if (force == 1 || force == 2) return force;
  const double per_wave = 148.0 / pair;
  const long long nt = (N + bn - 1) / bn;
  const long long u1 = ((T + 128LL * pair - 1) / (128LL * pair)) * nt;
  const long long u2 = ((T + 256LL * pair - 1) / (256LL * pair)) * nt;
  const double w1 = std::ceil(u1 / per_wave), w2 = std::ceil(u2 / per_wave);
  return (u2 >= per_wave && 2.0 * gain * w2 < w1) ? 2 : 1;
}

// Expected MT = 2 gains by GEMM kind (see pick_mt).
constexpr double kMtGain4bit = 0.8, kMtGainCe = 0.85, kMtGainBf16 = 1.02;
// bf16 gate/up with its SwiGLU outputs leaving by TMA stores: MT = 2 measured 1.74 -> 1.45 ms at
// the 8B shape (with per-thread stores the exposed epilogue cancelled the gain: 1.73 ms)
constexpr double kMtGainBf16Swiglu = 0.8;
// bf16 dAct (SwiGLU' epilogue): MT = 2 measured slower (0.91 -> 1.08 ms) even with dG, dU leaving by
// TMA stores, since its per-thread loads of G, U stay exposed; it keeps MT = 1 unless forced
constexpr double kMtGainBf16Dact = 1.02;
// bf16 GEMMs with a long K (down: K = f, dH: K = 2f, the cross-entropy's dH: K = the
// vocabulary chunk): the epilogue is a small part of a unit, fetching B once per two M tiles
// pays (8B shape: down 0.80 -> 0.71 ms, dH 1.59 -> 1.40 ms; the dAct GEMM, K = d with the
// SwiGLU' epilogue, measured 13 % slower and keeps kMtGainBf16)
constexpr double kMtGainBf16LongK = 0.8;

// Rank-r projection out[T x cols] (bf16) = scale * sum of K-split fp32 partials.
// The GEMM args must already hold maps/segments/M/N/bn/tiles and NACC columns.
template <int B_MN, int NACC>
int launch_proj(GemmArgs& a, long long T, long long K, int cols, float* part, void* out, float scale,
                cudaStream_t st, int phase) {
  const int s = proj_splits(T, K);
  const long long nkb = (K + BK - 1) / BK;
  const long long per = (nkb + s - 1) / s;
  a.splits = s;
  a.k_chunk = static_cast<int>(per * BK);
  a.out[0] = part;
  a.ld_out = cols;
  a.split_stride = T * cols;
  a.alpha = 1.0f;
  TRY((launch_gemm<0, B_MN, NACC, EPI_F32>(a, st, phase)));
  const long long n = T * cols;
  const long long blocks = (n / 4 + 255) / 256;
  PhaseScope ps(st, phase);
  splitk_finalize_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(part, s, T * cols, n, scale,
                                                                        static_cast<uint16_t*>(out));
  CUDA_TRY(cudaGetLastError());
  return LORA_OK;
}

// Split the T reduction of an adapter-gradient GEMM so that the tiles fill whole
// waves (at most 12 splits: every split adds one set of fp32 atomics per output).
inline void choose_splits(GemmArgs& a, long long K) {
  const long long tiles = static_cast<long long>(a.tiles_m) * a.tiles_n;
  const long long nkb = (K + BK - 1) / BK;
  const int s = balanced_splits(tiles, nkb, 12);
  const long long per = (nkb + s - 1) / s;
  a.k_chunk = static_cast<int>(per * BK);
  a.splits = static_cast<int>((nkb + per - 1) / per);
}


// Rank-r projection written into a column block of a wider bf16 matrix:
// out[:, 0:rp] (row stride ld_out) = scale * sum of K-split fp32 partials.
template <int B_MN>
int launch_proj_into(GemmArgs& a, long long T, long long K, int rp, float* part, void* out, long long ld_out,
                     float scale, cudaStream_t st, int phase) {
  const int s = proj_splits(T, K);
  const long long nkb = (K + BK - 1) / BK;
  const long long per = (nkb + s - 1) / s;
  a.splits = s;
  a.k_chunk = static_cast<int>(per * BK);
  a.out[0] = part;
  a.ld_out = rp;
  a.split_stride = T * rp;
  a.alpha = 1.0f;
  TRY((launch_gemm<0, B_MN, 1, EPI_F32>(a, st, phase)));
  const long long n = T * rp;
  const long long blocks = (n / 4 + 255) / 256;
  PhaseScope ps(st, phase);
  splitk_finalize_strided_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      part, s, T * rp, T, rp, ld_out, scale, static_cast<uint16_t*>(out));
  CUDA_TRY(cudaGetLastError());
  return LORA_OK;
}


// ------------------------------------------ rank-r streaming products (lowrank_dual.cuh)
// One problem: X [T x K] (row stride ldx); the row product's skinny operand S (MN-major
// [K x r] with row stride r in S[0], or K-major [r x K] rows, row stride K, in S[0] and
// S[1]); the column product's operand P [T x p_cols] (row stride ldp); its outputs.
struct DualProblem {
  const void* X;
  long long ldx;
  const void* S[2];
  const void* P;
  long long ldp;
  int p_cols;
  float* out[3];
};
// Which products a launch computes and how their operands and outputs are laid out.
struct DualSpec {
  int do_row, do_col;
  int row_kmajor, nbk;  // K-major row operand from nbk [r x K] matrices (else MN-major [K x r])
  int col_trans;        // column product written as [r x K] matrices (else [K x r] per problem)
  int n;                // MMA N: 16 or 32, or a multiple of 64 (MN-major tiles); K-major rows: nbk * rp
  int qw;               // row-product columns written per problem
};
// Q = s [X_m B_m] and dB_m += X_m^T P_m together (the backward of an up-projection)
inline DualSpec dual_spec_both(int r) {
  const int rp = round_up(r, 16);
  const int n = rp <= 32 ? rp : round_up(rp, 64);
  return DualSpec{1, 1, 0, 1, 0, n, rp};
}
// P = s X [A_0; A_1]^T (the forward rank-r projection of nbk adapters sharing X)
inline DualSpec dual_spec_proj(int r, int nbk) {
  const int rp = round_up(r, 16);
  return DualSpec{1, 0, 1, nbk, 0, nbk * rp, nbk * rp};
}
// dA_i += (Q[:, i rp : i rp + r])^T X for the nq (<= 3) column blocks of Q (the reductions over T)
inline DualSpec dual_spec_reduce(int r, int nq) {
  const int rp = round_up(r, 16);
  const int w = nq * rp;
  const int n = w <= 32 ? w : round_up(w, 64);
  return DualSpec{0, 1, 0, 1, 1, n, 0};
}
struct DualShape {
  int R, nrb, nc, nreg, grid, slots;
  long long units;
};
// MN-major skinny tile geometry for MMA N = n: row bytes (= the swizzle width), atoms of 64
// columns, swizzle
inline void dual_tile_geometry(int n, int* prow, int* patoms, CUtensorMapSwizzle* map_swz, uint32_t* smem_swz) {
  *prow = n >= 64 ? 128 : n * 2;
  *patoms = n >= 64 ? n / 64 : 1;
  *map_swz = *prow == 32 ? CU_TENSOR_MAP_SWIZZLE_32B : (*prow == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
  *smem_swz = *prow == 32 ? kSwz32 : (*prow == 64 ? kSwz64 : kSwz128);
}
// Row blocks per region: 2 while a row product keeps R accumulators in TMEM; 8 for a
// column product alone (each region adds one fp32 atomic per output element; at the 8B
// shape R = 8 measured faster than 4 and 16 for both reductions over T).
inline int dual_rows(const DualSpec& sp, long long T, int K, int nx) {
  static const int r_knob = [] {
    const char* e = getenv("LORA_MLP_DUAL_R");  // tuning knob: row blocks per region
    return e ? atoi(e) : 0;
  }();
  (void)T;
  (void)K;
  (void)nx;
  int R = sp.do_row ? 2 : 8;
  if (r_knob >= 1) R = std::max(1, std::min(r_knob, sp.do_row ? 512 / sp.n - 2 : 64));
  return R;
}
// Shape of the unit grid on `max_grid` CTAs; slots = the most CTAs that share one
// (row region, problem), i.e. the partial slots the row product needs.
inline DualShape dual_shape(const DualSpec& sp, long long T, int K, int nx, int max_grid) {
  DualShape s{};
  s.R = dual_rows(sp, T, K, nx);
  s.nrb = static_cast<int>((T + 127) / 128);
  s.nc = (K + 127) / 128;
  s.nreg = (s.nrb + s.R - 1) / s.R;
  s.units = static_cast<long long>(s.nreg) * nx * s.nc;
  s.grid = static_cast<int>(std::min<long long>(s.units, max_grid));
  s.slots = 1;
  if (sp.do_row) {
    for (long long k = 0; k < static_cast<long long>(s.nreg) * nx; ++k) {
      const long long a = dual_owner(k * s.nc, s.units, s.grid);
      const long long b = dual_owner(k * s.nc + s.nc - 1, s.units, s.grid);
      s.slots = std::max(s.slots, static_cast<int>(b - a + 1));
    }
  }
  return s;
}
// Partial slots to reserve whatever the device's SM count: ranges hold at least
// floor(U / G) units, so a run of nc units meets at most 1 + ceil((nc - 1) / floor(U / G))
// of them, largest at the largest grid.
inline int dual_slots_bound(const DualSpec& sp, long long T, int K, int nx) {
  if (!sp.do_row) return 0;
  const DualShape s = dual_shape(sp, T, K, nx, kDualMaxGrid);
  const long long L = std::max<long long>(1, s.units / s.grid);
  return static_cast<int>(1 + (s.nc - 1 + L - 1) / L);
}
// Arrival counters a launch uses (zero on entry, left zero).
inline long long dual_counters(const DualSpec& sp, long long T, int K, int nx) {
  return sp.do_row ? static_cast<long long>(dual_shape(sp, T, K, nx, kDualMaxGrid).nreg) * nx : 0;
}

// Runs the products of `sp` over the nx problems.  The row product goes to Q (bf16, row
// stride ldq; problem m writes columns [m qw, (m + 1) qw), scaled by `scale`); `part` holds
// dual_slots_bound(...) * T * ldq floats and `cnt` dual_counters(...) zeroed ints.  The
// column product is added (fp32 atomics) into outputs the caller has zeroed.
inline int launch_dual(const DualSpec& sp, const DualProblem* pr, int nx, long long T, int K, int r, float scale,
                       void* Q, int ldq, float* part, int* cnt, int* status, cudaStream_t st, int phase) {
  const int rp = round_up(r, 16);
  if (nx < 1 || nx > 2 || K < 8 || K % 8 || r < 8 || r % 8 || r > 128 || sp.n < 16 || sp.n > 256 || sp.n % 16 ||
      (sp.n > 32 && sp.n % 64 && (sp.do_col || !sp.row_kmajor)) || (sp.row_kmajor && sp.n != sp.nbk * rp) ||
      (sp.col_trans && nx != 1) || (sp.do_row && (sp.qw % 16 || sp.qw > sp.n || nx * sp.qw > ldq)))
    return fail(LORA_ERR_UNSUPPORTED, "internal: bad rank-r pass (nx %d, K %d, r %d, n %d)", nx, K, r, sp.n);
  DualArgs a;
  memset(&a, 0, sizeof(a));
  const DualShape s = dual_shape(sp, T, K, nx, std::min(sm_count(), kDualMaxGrid));
  if (s.units <= 0) return LORA_OK;
  if (sp.do_row && s.slots > dual_slots_bound(sp, T, K, nx))
    return fail(LORA_ERR_UNSUPPORTED, "internal: rank-r pass needs %d partial slots", s.slots);
  int prow = 0, patoms = 0;
  CUtensorMapSwizzle map_swz;
  uint32_t smem_swz = 0;
  dual_tile_geometry(sp.n, &prow, &patoms, &map_swz, &smem_swz);
  for (int m = 0; m < nx; ++m) {
    TRY(map_k(&a.x[m], pr[m].X, T, K, pr[m].ldx, 128));
    if (sp.do_row) {
      if (sp.row_kmajor) {
        for (int i = 0; i < sp.nbk; ++i) TRY(map_k(&a.b[m][i], pr[m].S[i], r, K, K, static_cast<uint32_t>(rp)));
      } else {
        TRY(make_map(&a.b[m][0], pr[m].S[0], r, K, r, prow / 2, 128, map_swz));
      }
    }
    if (sp.do_col) TRY(make_map(&a.p[m], pr[m].P, pr[m].p_cols, T, pr[m].ldp, prow / 2, 128, map_swz));
    a.out[m] = pr[m].out[0];
  }
  if (sp.col_trans)
    for (int i = 0; i < 3; ++i) a.out[i] = pr[0].out[i];
  a.nx = nx;
  a.T = T;
  a.K = K;
  a.r = r;
  a.rp = rp;
  a.n = sp.n;
  a.do_row = sp.do_row;
  a.do_col = sp.do_col;
  a.row_kmajor = sp.row_kmajor;
  a.nbk = sp.nbk;
  a.qw = sp.qw;
  a.col_trans = sp.col_trans;
  a.prow = prow;
  a.patoms = patoms;
  a.swz = smem_swz;
  // TMEM's 512 columns: two row sets (so a run's flush overlaps the next run) and two
  // accumulators per product (independent MMA chains) where they fit, in that order
  int sets = 0;
  a.nsplit = 0;
  for (int cfg = 0; cfg < 4 && !a.nsplit; ++cfg) {
    const int rsets = cfg < 2 ? 2 : 1, nsplit = (cfg & 1) ? 1 : 2;
    sets = (sp.do_row ? rsets * s.R : 0) + (sp.do_col ? 2 : 0);
    if (nsplit * sets * sp.n <= 512) {
      a.nsplit = nsplit;
      a.rsets = rsets;
    }
  }
  if (!a.nsplit) return fail(LORA_ERR_UNSUPPORTED, "internal: rank-r accumulators exceed TMEM");
  uint32_t tc = 32;
  while (tc < static_cast<uint32_t>(a.nsplit * sets * sp.n)) tc <<= 1;
  a.tmem_cols = tc;
  a.R = s.R;
  a.nrb = s.nrb;
  a.nc = s.nc;
  a.nreg = s.nreg;
  a.units = s.units;
  a.scale = scale;
  a.Q = static_cast<uint16_t*>(Q);
  a.ldq = ldq;
  a.part = part;
  a.part_slot = T * ldq;
  a.cnt = cnt;
  a.status = status;
  a.limit_ns = wait_limit_ns();
  const uint32_t tile = 256u * static_cast<uint32_t>(sp.n);  // one skinny tile: 128 K rows (or 2 x 64 K) x n
  a.col_off = kDualXBytes;
  a.row_off = kDualXBytes + (sp.do_col ? tile : 0u);
  a.stage_bytes = a.row_off + (sp.do_row ? tile : 0u);  // the bytes of one stage's copies
  // 4 KB of slack past the barriers: no operand read of the ring's last stage can leave the allocation
  a.stages = std::min(kDualMaxStages, (kSmemLimit - 1024 - 256 - 4096) / static_cast<int>(a.stage_bytes));
  static const int stage_cap = [] {
    const char* e = getenv("LORA_MLP_DUAL_STAGES");  // tuning knob: cap the ring depth
    return e ? atoi(e) : 0;
  }();
  if (stage_cap >= 2) a.stages = std::min(a.stages, stage_cap);
  if (a.stages < 2) return fail(LORA_ERR_UNSUPPORTED, "internal: rank-r stage does not fit");
  const int smem = 1024 + a.stages * static_cast<int>(a.stage_bytes) + 256 + 4096;
  CUDA_TRY(cudaFuncSetAttribute(lowrank_dual_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  PhaseScope ps(st, phase);
  lowrank_dual_kernel<<<s.grid, kDualThreads, smem, st>>>(a);
  CUDA_TRY(cudaGetLastError());
  return LORA_OK;
}

// Device addresses of the library's own device memory in the current CUDA context
// (defined in lora_mlp.cu): the no-alloc projection's scratch and the status word of
// the calls that take no workspace.
struct LibSyms {
  unsigned long long ctx_id;
  float* scratch;
  int* status;
};
int lib_syms(LibSyms* out);

}  // namespace host
}  // namespace lm
