// Host side of liblora_mlp.so for the MLP sub-block and the library-wide calls:
// argument validation, the launch sequence of the LoRA-MLP forward/backward, the
// library-owned device memory, per-phase timing and status, and those extern "C"
// entry points of include/lora_mlp.h.  (Q/K/V, o_proj and RoPE: lora_attn.cu;
// the LM-head cross-entropy: lora_ce.cu.)
#include "host.cuh"

using namespace lm;
using namespace lm::host;

namespace {

// --------------------------------------------------------------- layouts
struct WsLayout {
  size_t status, Q, Qd, dG, dU, dH, part, am, cnt, total;
  long long ncnt;  // arrival counters of the rank-r streaming launches (DualLaunch order)
};

int check_dims(const lora_mlp_dims* D) {
  if (!D) return fail(LORA_ERR_INVALID_ARG, "dims is NULL");
  if (D->T < 1 || D->T >= (1LL << 31)) return fail(LORA_ERR_INVALID_ARG, "T = %lld out of range", (long long)D->T);
  if (D->d < 8 || D->f < 8 || D->r < 1) return fail(LORA_ERR_INVALID_ARG, "d, f, r must be positive (d, f >= 8)");
  if (D->d % 8 || D->f % 8 || D->r % 8)
    return fail(LORA_ERR_ALIGNMENT, "d, f, r must be multiples of 8 (16-byte rows); got %d %d %d", D->d, D->f, D->r);
  if (D->d > 65536) return fail(LORA_ERR_UNSUPPORTED, "d = %d > 65536", D->d);
  if (D->r > 128) return fail(LORA_ERR_UNSUPPORTED, "r = %d > 128", D->r);
  if (D->wfmt != LORA_WFMT_BF16 && D->wfmt != LORA_WFMT_4BIT && D->wfmt != LORA_WFMT_4BIT_DQ)
    return fail(LORA_ERR_INVALID_ARG, "bad wfmt");
  if (D->residual != 0 && D->residual != 1) return fail(LORA_ERR_INVALID_ARG, "residual must be 0 or 1");
  if (D->wfmt != LORA_WFMT_BF16) {
    if (D->qblock != 64) return fail(LORA_ERR_UNSUPPORTED, "qblock must be 64");
    if (D->d % 256 || D->f % 256) return fail(LORA_ERR_UNSUPPORTED, "4-bit weights need d, f multiples of 256");
  }
  return LORA_OK;
}

int rp_of(const lora_mlp_dims* D) { return round_up(D->r, 16); }

lora_mlp_ctx_layout ctx_layout(const lora_mlp_dims* D) {
  const size_t T = D->T, d = D->d, f = D->f, rp = rp_of(D);
  lora_mlp_ctx_layout L{};
  size_t o = 0;
  L.rstd = o; o = up256(o + T * 4);
  L.H = o;    o = up256(o + T * d * 2);
  L.G = o;    o = up256(o + T * f * 2);
  L.U = o;    o = up256(o + T * f * 2);
  L.Act = o;  o = up256(o + T * f * 2);
  L.P = o;    o = up256(o + T * 2 * rp * 2);
  L.Pd = o;   o = up256(o + T * rp * 2);
  L.total = o;
  L.rp = static_cast<int32_t>(rp);
  return L;
}

// The rank-r streaming launches of one forward + backward (lowrank_dual.cuh), in the
// order of their arrival counters in the workspace.
enum DualLaunch { DL_P_GU = 0, DL_P_D, DL_BWD_D, DL_BWD_GU, DL_RED_GU, DL_RED_D, DL_COUNT };
struct DualPlan {
  DualSpec sp;
  int K, nx, ldq;
};
DualPlan dual_plan(const lora_mlp_dims* D, int which) {
  const int r = D->r, rp = rp_of(D);
  switch (which) {
    case DL_P_GU: return DualPlan{dual_spec_proj(r, 2), D->d, 1, 2 * rp};    // P  = s H [Ag; Au]^T
    case DL_P_D: return DualPlan{dual_spec_proj(r, 1), D->f, 1, rp};         // Pd = s Act Ad^T
    case DL_BWD_D: return DualPlan{dual_spec_both(r), D->d, 1, rp};          // Qd = s dY Bd, dBd
    case DL_BWD_GU: return DualPlan{dual_spec_both(r), D->f, 2, 2 * rp};     // Q = s [dG Bg | dU Bu], dBg, dBu
    case DL_RED_GU: return DualPlan{dual_spec_reduce(r, 2), D->d, 1, 0};     // dAg, dAu
    default: return DualPlan{dual_spec_reduce(r, 1), D->f, 1, 0};            // dAd
  }
}
long long dual_cnt_offset(const lora_mlp_dims* D, int which) {
  long long o = 0;
  for (int i = 0; i < which; ++i) {
    const DualPlan pl = dual_plan(D, i);
    o += dual_counters(pl.sp, D->T, pl.K, pl.nx);
  }
  return o;
}

WsLayout ws_layout(const lora_mlp_dims* D) {
  const size_t T = D->T, d = D->d, f = D->f, rp = rp_of(D);
  WsLayout L{};
  size_t o = 0;
  L.status = o; o = 256;
  L.Q = o;  o = up256(o + T * 2 * rp * 2);
  L.Qd = o; o = up256(o + T * rp * 2);
  L.dG = o; o = up256(o + T * f * 2);
  L.dU = o; o = up256(o + T * f * 2);
  L.dH = o; o = up256(o + T * d * 4);
  size_t part = 0;
  part = std::max(part, size_t(proj_splits(T, d)) * T * 2 * rp);   // P  = s H [Ag|Au]^T
  part = std::max(part, size_t(proj_splits(T, f)) * T * rp);       // Pd = s Act Ad^T
  part = std::max(part, size_t(proj_splits(T, d)) * T * rp);       // Qd = s dY Bd
  part = std::max(part, size_t(proj_splits(T, f)) * T * 2 * rp);   // Q  = s [dG Bg | dU Bu]
  for (int i = 0; i < DL_COUNT; ++i) {  // the single-pass kernels' partial slots
    const DualPlan pl = dual_plan(D, i);
    part = std::max(part, size_t(dual_slots_bound(pl.sp, D->T, pl.K, pl.nx)) * T * pl.ldq);
  }
  L.part = o; o = up256(o + part * 4);
  // double-quantised constants: the fp32 absmax of Wg, Wu and Wd, decoded at each call
  L.am = o;
  if (D->wfmt == LORA_WFMT_4BIT_DQ) o = up256(o + 3 * (f * d / 64) * 4);
  L.ncnt = dual_cnt_offset(D, DL_COUNT);
  L.cnt = o; o = up256(o + static_cast<size_t>(L.ncnt) * 4);
  L.total = o;
  return L;
}

// Weight constants of a 4-bit call: the caller's fp32 absmax, or for double-quantised
// constants their fp32 expansion in the workspace (one decode launch per call).
struct Absmax3 {
  const float *g, *u, *d;
};
int absmax_for_call(const lora_mlp_dims* D, const lora_mlp_weights* W, void* workspace, const WsLayout& WL,
                    cudaStream_t st, Absmax3* out) {
  if (D->wfmt != LORA_WFMT_4BIT_DQ) {
    *out = Absmax3{W->absmax_g, W->absmax_u, W->absmax_d};
    return LORA_OK;
  }
  const long long n = static_cast<long long>(D->f) * D->d / 64;
  float* base = at<float>(workspace, WL.am);
  Absmax8List L{};
  const uint8_t* codes[3] = {W->absmax8_g, W->absmax8_u, W->absmax8_d};
  const float* sc[3] = {W->scale2_g, W->scale2_u, W->scale2_d};
  for (int m = 0; m < 3; ++m) {
    L.codes[m] = codes[m];
    L.scale2[m] = sc[m];
    L.out[m] = base + m * n;
    L.n[m] = n;
  }
  PhaseScope ps(st, PH_OTHER);
  absmax8_decode_kernel<<<296, 256, 0, st>>>(L);
  CUDA_TRY(cudaGetLastError());
  *out = Absmax3{base, base + n, base + 2 * n};
  return LORA_OK;
}

int check_weights(const lora_mlp_dims* D, const lora_mlp_weights* W) {
  if (D->wfmt == LORA_WFMT_BF16) return check_ptrs({W->Wg, W->Wu, W->Wd});
  TRY(check_ptrs({W->Qg, W->Qu, W->Qd, W->codebook}));
  if (D->wfmt == LORA_WFMT_4BIT) return check_ptrs({W->absmax_g, W->absmax_u, W->absmax_d});
  return check_ptrs({W->absmax8_g, W->absmax8_u, W->absmax8_d, W->scale2_g, W->scale2_u, W->scale2_d});
}


}  // namespace

// ------------------------------------------------- library-owned device memory
// Scratch for lora_lowrank_proj_noalloc: the K-split fp32 partial sums live in a
// file-scope device array instead of caller memory.  Every GPU that loads this
// library holds it until the process exits.
constexpr size_t kNoAllocScratchFloats = size_t(4) << 20;  // 16 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];
// Bounded-wait status word of the calls that take no workspace (lora_gemm_bf16,
// lora_lowrank_proj_noalloc); the calls with a workspace keep theirs at its offset 0.
static __device__ __align__(256) int g_lib_status;

// In host code the names above denote host-side stand-ins, not device addresses.
// Their device addresses belong to one CUDA context (the module is loaded per
// context), so they are looked up with cudaGetSymbolAddress, with the caller's context
// current, and cached under that context's unique id (cuCtxGetId: unlike the CUcontext
// handle, an id is never reused within the process, so a context destroyed by
// cudaDeviceReset and its successor get different entries).
namespace {
std::mutex g_syms_mu;
std::vector<LibSyms> g_syms;
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;

int resolve_ctx_fns() {
  if (g_ctx_current && g_ctx_id) return LORA_OK;
  void* f1 = nullptr;
  void* f2 = nullptr;
  cudaDriverEntryPointQueryResult q1, q2;
  cudaError_t e1 = cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1);
  cudaError_t e2 = cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2);
  if (e1 != cudaSuccess || e2 != cudaSuccess || q1 != cudaDriverEntryPointSuccess ||
      q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
    return fail(LORA_ERR_CUDA, "cannot resolve cuCtxGetCurrent / cuCtxGetId");
  g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
  g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
  return LORA_OK;
}

}  // namespace

int lm::host::lib_syms(LibSyms* out) {
  std::lock_guard<std::mutex> lk(g_syms_mu);
  TRY(resolve_ctx_fns());
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return fail(LORA_ERR_CUDA, "cuCtxGetCurrent failed");
  if (!ctx) {
    // no context current yet: the runtime makes the device's primary context current
    // on its first use, which this lookup is
    void* p = nullptr;
    CUDA_TRY(cudaGetSymbolAddress(&p, g_lib_status));
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return fail(LORA_ERR_CUDA, "no current CUDA context");
  }
  unsigned long long id = 0;
  if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return fail(LORA_ERR_CUDA, "cuCtxGetId failed");
  for (const LibSyms& e : g_syms)
    if (e.ctx_id == id) {
      *out = e;
      return LORA_OK;
    }
  LibSyms e{id, nullptr, nullptr};
  void* p = nullptr;
  cudaError_t err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (err != cudaSuccess || !p)
    return fail(LORA_ERR_CUDA, "cudaGetSymbolAddress(no-alloc scratch) failed: %s", cudaGetErrorString(err));
  e.scratch = static_cast<float*>(p);
  err = cudaGetSymbolAddress(&p, g_lib_status);
  if (err != cudaSuccess || !p)
    return fail(LORA_ERR_CUDA, "cudaGetSymbolAddress(status word) failed: %s", cudaGetErrorString(err));
  e.status = static_cast<int*>(p);
  if (g_syms.size() >= 64) g_syms.erase(g_syms.begin());  // contexts long gone
  g_syms.push_back(e);
  *out = e;
  return LORA_OK;
}

// ======================================================================= ABI
extern "C" {

const char* lora_mlp_last_error(void) { return g_err; }

const char* lora_mlp_phase_name(int32_t phase) {
  if (phase < 0 || phase >= LORA_NUM_PHASES) return "invalid";
  return kPhaseNames[phase];
}

int lora_mlp_timing_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_timing.mu);
  g_timing.on = on != 0;
  return LORA_OK;
}

int lora_mlp_timing_collect(double* ms, int64_t* launches) {
  std::vector<Timing::Rec> recs;
  {
    std::lock_guard<std::mutex> lk(g_timing.mu);
    recs.swap(g_timing.pending);
  }
  if (ms)
    for (int i = 0; i < LORA_NUM_PHASES; ++i) ms[i] = 0.0;
  if (launches)
    for (int i = 0; i < LORA_NUM_PHASES; ++i) launches[i] = 0;
  int rc = LORA_OK;
  for (auto& r : recs) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess) rc = fail(LORA_ERR_CUDA, "timing event: %s", cudaGetErrorString(e));
    if (ms) ms[r.phase] += t;
    if (launches) launches[r.phase] += 1;
  }
  std::lock_guard<std::mutex> lk(g_timing.mu);
  for (auto& r : recs) {
    g_timing.pool.push_back(r.a);
    g_timing.pool.push_back(r.b);
  }
  return rc;
}

int lora_mlp_ctx_layout_get(const lora_mlp_dims* dims, lora_mlp_ctx_layout* out) {
  TRY(check_dims(dims));
  if (!out) return fail(LORA_ERR_INVALID_ARG, "out is NULL");
  *out = ctx_layout(dims);
  return LORA_OK;
}

int lora_mlp_workspace_bytes(const lora_mlp_dims* dims, size_t* bytes) {
  TRY(check_dims(dims));
  if (!bytes) return fail(LORA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = ws_layout(dims).total;
  return LORA_OK;
}

int lora_rmsnorm_fwd(int64_t T, int32_t d, float eps, const void* X, const void* w, void* H, float* rstd,
                     void* stream) {
  if (T < 1 || d < 8 || d % 8 || d > 65536) return fail(LORA_ERR_INVALID_ARG, "bad T/d (%lld, %d)", (long long)T, d);
  TRY(check_ptrs({X, w, H, rstd}));
  return launch_rms_fwd(static_cast<cudaStream_t>(stream), X, w, H, rstd, T, d, eps);
}

int lora_rmsnorm_bwd(int64_t T, int32_t d, const float* dH, const void* X, const void* w, const float* rstd,
                     void* dX, void* stream) {
  if (T < 1 || d < 8 || d % 8 || d > 65536) return fail(LORA_ERR_INVALID_ARG, "bad T/d (%lld, %d)", (long long)T, d);
  TRY(check_ptrs({dH, X, w, rstd, dX}));
  return launch_rms_bwd(static_cast<cudaStream_t>(stream), dH, X, w, rstd, dX, T, d);
}

int lora_merge_weights(int64_t rows, int64_t cols, int32_t r, float scale, const void* W, const void* A,
                       const void* B, void* Wm, void* stream) {
  if (rows < 1 || cols < 8 || cols % 8) return fail(LORA_ERR_INVALID_ARG, "bad rows/cols (%lld, %lld)", (long long)rows, (long long)cols);
  if (r < 1 || r > 256) return fail(LORA_ERR_UNSUPPORTED, "r = %d outside 1..256", r);
  if (!std::isfinite(scale)) return fail(LORA_ERR_INVALID_ARG, "scale is not finite");
  TRY(check_ptrs({W, A, Wm}));
  if (!B) return fail(LORA_ERR_INVALID_ARG, "B is NULL");
  if (reinterpret_cast<uintptr_t>(B) % 2) return fail(LORA_ERR_ALIGNMENT, "B is not 2-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(static_cast<unsigned>((cols / 8 + 127) / 128),
                  static_cast<unsigned>(std::min<long long>((rows + 3) / 4, 65535)));
  PhaseScope ps(st, PH_OTHER);
  merge_weights_kernel<<<grid, 128, 0, st>>>(static_cast<const uint16_t*>(W), static_cast<const uint16_t*>(A),
                                             static_cast<const uint16_t*>(B), static_cast<uint16_t*>(Wm), rows,
                                             cols, r, scale);
  CUDA_TRY(cudaGetLastError());
  return LORA_OK;
}

int lora_quantize_4bit(const void* W, int64_t numel, int32_t block, const float* codebook16, uint8_t* codes,
                       float* absmax, void* stream) {
  if (block != 64) return fail(LORA_ERR_UNSUPPORTED, "block must be 64");
  if (numel < 64 || numel % 64) return fail(LORA_ERR_INVALID_ARG, "numel must be a positive multiple of 64");
  TRY(check_ptrs({W, codebook16, codes, absmax}));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long nb = numel / 64;
  const int threads = 256;
  const long long blocks = std::min<long long>((nb + 7) / 8, 148LL * 16);
  PhaseScope ps(st, PH_OTHER);
  quantize4_kernel<<<static_cast<unsigned>(blocks), threads, 0, st>>>(static_cast<const uint16_t*>(W), nb,
                                                                       codebook16, codes, absmax);
  CUDA_TRY(cudaGetLastError());
  return LORA_OK;
}

int lora_quantize_absmax8(const float* absmax, int64_t n, int32_t block2, uint8_t* codes8, float* scale2,
                          void* stream) {
  if (block2 != kAbsmax8Block) return fail(LORA_ERR_UNSUPPORTED, "block2 must be %d", kAbsmax8Block);
  if (n < 1) return fail(LORA_ERR_INVALID_ARG, "n must be positive");
  TRY(check_ptrs({absmax, codes8, scale2}));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long nblk = (n + kAbsmax8Block - 1) / kAbsmax8Block;
  const long long blocks = std::min<long long>((nblk + 7) / 8, 148LL * 16);
  PhaseScope ps(st, PH_OTHER);
  absmax8_quantize_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(absmax, n, codes8, scale2);
  CUDA_TRY(cudaGetLastError());
  return LORA_OK;
}

int lora_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, int32_t a_mn, const void* B, int32_t b_mn,
                   float* C, int32_t flags, void* stream) {
  if (M < 1 || N < 1 || K < 1 || M >= (1LL << 31) || N >= (1LL << 31) || K >= (1LL << 31))
    return fail(LORA_ERR_INVALID_ARG, "bad M/N/K");
  if (M % 8 || N % 8 || K % 8) return fail(LORA_ERR_ALIGNMENT, "M, N, K must be multiples of 8");
  TRY(check_ptrs({A, B, C}));
  if (flags & ~(LORA_GEMM_CTA_PAIR | LORA_GEMM_TEST_NO_LOADS)) return fail(LORA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if ((flags & LORA_GEMM_TEST_NO_LOADS) && (flags & LORA_GEMM_CTA_PAIR))
    return fail(LORA_ERR_INVALID_ARG, "LORA_GEMM_TEST_NO_LOADS is for single-CTA tiles only");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LibSyms ls;
  TRY(lib_syms(&ls));
  GemmArgs a = new_args(ls.status);
  a.test_no_loads = (flags & LORA_GEMM_TEST_NO_LOADS) ? 1 : 0;
  const int pair = (flags & LORA_GEMM_CTA_PAIR) && !a_mn ? 2 : 1;
  int bn = b_mn ? (N >= 256 ? 256 : round_up(static_cast<int>(N), 64))
                : (N >= 256 ? 256 : round_up(static_cast<int>(N), 16));
  if (pair == 2) bn = b_mn ? std::min(256, round_up(static_cast<int>(N), 128)) : std::max(bn, 32);
  // MN-major operands whose contiguous extent is a multiple of 64 load one 3-D box per tile
  a.mn3d_a = a_mn && M % 64 == 0;
  a.mn3d_b = b_mn && N % 64 == 0;
  if (a.mn3d_a) TRY(map_mn3(&a.maps[0], A, K, M, M, 2));
  else if (a_mn) TRY(map_mn(&a.maps[0], A, K, M, M));
  else TRY(map_k(&a.maps[0], A, M, K, K, 128));
  if (a.mn3d_b) TRY(map_mn3(&a.maps[1], B, K, N, N, bn / pair / 64));
  else if (b_mn) TRY(map_mn(&a.maps[1], B, K, N, N));
  else TRY(map_k(&a.maps[1], B, N, K, K, bn / pair));
  set_seg(a, 0, 0, 0, 1, 0, -1, 0, static_cast<int>(K));
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.bn = bn;
  a.tiles_m = static_cast<int>((M + BM * pair - 1) / (BM * pair));
  a.tiles_n = static_cast<int>((N + bn - 1) / bn);
  a.out[0] = C;
  a.ld_out = N;
  TRY(begin_call(a.status, st));
  if (pair == 2) {
    if (b_mn) TRY((launch_gemm<0, 1, 1, EPI_F32, 2>(a, st, PH_OTHER)));
    else TRY((launch_gemm<0, 0, 1, EPI_F32, 2>(a, st, PH_OTHER)));
  } else if (!a_mn && !b_mn) {
    TRY((launch_gemm<0, 0, 1, EPI_F32>(a, st, PH_OTHER)));
  } else if (!a_mn && b_mn) {
    TRY((launch_gemm<0, 1, 1, EPI_F32>(a, st, PH_OTHER)));
  } else if (a_mn && !b_mn) {
    TRY((launch_gemm<1, 0, 1, EPI_F32>(a, st, PH_OTHER)));
  } else {
    TRY((launch_gemm<1, 1, 1, EPI_F32>(a, st, PH_OTHER)));
  }
  return end_call(a.status, st);
}

int lora_mlp_status(const void* workspace, int32_t* code, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int* word = static_cast<const int*>(workspace);
  if (!word) {
    LibSyms ls;
    TRY(lib_syms(&ls));
    word = ls.status;
  } else if (!aligned16(workspace)) {
    return fail(LORA_ERR_ALIGNMENT, "workspace %p is not 16-byte aligned", workspace);
  }
  CUDA_TRY(cudaStreamSynchronize(st));
  int v = 0;
  CUDA_TRY(cudaMemcpy(&v, word, sizeof(int), cudaMemcpyDeviceToHost));
  if (code) *code = v;
  if ((v & 0xF00) == kDevBadIndex)
    return fail(LORA_ERR_INVALID_ARG, "a device-side index input was out of range (code 0x%x)", v);
  if (v) return fail(LORA_ERR_TIMEOUT, "device-side bounded wait gave up (code 0x%x)", v);
  return LORA_OK;
}

int lora_mlp_fwd(const lora_mlp_dims* D, const void* X, const void* rms_w, const lora_mlp_weights* W,
                 const lora_mlp_adapters* A, void* Y, void* ctx, void* workspace, void* stream) {
  TRY(check_dims(D));
  if (!W || !A) return fail(LORA_ERR_INVALID_ARG, "weights/adapters is NULL");
  const bool q4 = D->wfmt != LORA_WFMT_BF16;
  TRY(check_ptrs({X, rms_w, Y, ctx, workspace, A->Ag, A->Bg, A->Au, A->Bu, A->Ad, A->Bd}));
  TRY(check_weights(D, W));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long T = D->T;
  const int d = D->d, f = D->f, r = D->r, rp = rp_of(D);
  const float s = D->scale;
  const lora_mlp_ctx_layout L = ctx_layout(D);
  const WsLayout WL = ws_layout(D);
  int* status = at<int>(workspace, WL.status);
  void* H = at<char>(ctx, L.H);
  float* rstd = at<float>(ctx, L.rstd);
  void* G = at<char>(ctx, L.G);
  void* U = at<char>(ctx, L.U);
  void* Act = at<char>(ctx, L.Act);
  void* P = at<char>(ctx, L.P);
  void* Pd = at<char>(ctx, L.Pd);
  TRY(begin_call(status, st));
  Absmax3 am{};
  if (q4) TRY(absmax_for_call(D, W, workspace, WL, st, &am));

  // S1: RMSNorm (cached rstd)
  TRY(launch_rms_fwd(st, X, rms_w, H, rstd, T, d, D->eps));

  // S2: P = s * [H Ag^T | H Au^T]  (rank-r projections, padded to rp columns each)
  float* part = at<float>(workspace, WL.part);
  int* cnt = at<int>(workspace, WL.cnt);
  const int dmode = dual_mode();
  if (dmode == 2) {
    CUDA_TRY(cudaMemsetAsync(cnt, 0, static_cast<size_t>(WL.ncnt) * sizeof(int), st));
    const DualPlan pl = dual_plan(D, DL_P_GU);
    DualProblem pr{};
    pr.X = H; pr.ldx = d; pr.S[0] = A->Ag; pr.S[1] = A->Au;
    TRY(launch_dual(pl.sp, &pr, 1, T, d, r, s, P, 2 * rp, part, cnt + dual_cnt_offset(D, DL_P_GU), status, st,
                    PH_P_GU));
  } else {
    GemmArgs a = new_args(status);
    TRY(map_k(&a.maps[0], H, T, d, d, 128));
    TRY(map_k(&a.maps[1], A->Ag, r, d, d, rp));
    TRY(map_k(&a.maps[2], A->Au, r, d, d, rp));
    set_seg(a, 0, 0, 0, 1, 0, 2, 0, d);
    a.M = static_cast<int>(T); a.N = rp; a.bn = rp;
    a.tiles_m = static_cast<int>((T + BM - 1) / BM); a.tiles_n = 1; a.out_acc_col = rp;
    TRY((launch_proj<0, 2>(a, T, d, 2 * rp, part, P, s, st, PH_P_GU)));
  }
  // S3: G = H Wg^T + P_g Bg^T, U = H Wu^T + P_u Bu^T, Act = silu(G) * U.
  // One N = 256 MMA per k-step covers 128 gate and 128 up columns; the LoRA term is
  // one K = 2rp extension [P_g | P_u] x [[Bg | 0]; [0 | Bu]]^T, the zero blocks
  // coming from TMA out-of-range fill (Bu is read from column -rp).
  if (q4) {
    // 4-bit frozen weights: the codes are expanded to bf16 B tiles in shared memory
    // by dequant warps inside the GEMM (each CTA of a pair expands its own branch)
    GemmArgs a = new_args(status);
    const int pair = T > 128 ? 2 : 1;
    TRY(map_k(&a.maps[0], H, T, d, d, 128));
    TRY(map_q4_k(&a.maps[1], &a.maps[6], W->Qg, am.g, f, d, 128));
    TRY(map_q4_k(&a.maps[2], &a.maps[7], W->Qu, am.u, f, d, 128));
    TRY(map_k(&a.maps[3], P, T, 2 * rp, 2 * rp, 128));
    TRY(map_k(&a.maps[4], A->Bg, f, r, r, 128));
    TRY(map_k(&a.maps[5], A->Bu, f, r, r, 128));
    set_seg(a, 0, 0, 0, 1, 0, 2, 0, d);
    a.seg[0].q4 = 1; a.seg[0].b_am[0] = 6; a.seg[0].b_am[1] = 7;
    set_seg(a, 1, 3, 0, 4, 0, 5, -rp, 2 * rp);
    a.codebook = W->codebook;
    const int mt = pair == 2 ? pick_mt(T, pair, 128, f, kMtGain4bit) : 1;
    a.M = static_cast<int>(T); a.N = f; a.bn = 128;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (f + 127) / 128;
    a.out[0] = G; a.out[1] = U; a.out[2] = Act; a.ld_out = f;
    set_hints(a, HINT_EVICT_LAST, HINT_NONE);
    set_band(a, 16 / mt);
    a.stream_out = 1;
    if (mt == 2) TRY((launch_gemm<0, 0, 2, EPI_SWIGLU_FWD, 2, 1, 1, 2>(a, st, PH_GATEUP)));
    else if (pair == 2) TRY((launch_gemm<0, 0, 2, EPI_SWIGLU_FWD, 2, 1, 1>(a, st, PH_GATEUP)));
    else TRY((launch_gemm<0, 0, 2, EPI_SWIGLU_FWD, 1, 1, 1>(a, st, PH_GATEUP)));
  } else {
    GemmArgs a = new_args(status);
    const int pair = T > 128 ? 2 : 1;
    TRY(map_k(&a.maps[0], H, T, d, d, 128));
    TRY(map_k(&a.maps[1], W->Wg, f, d, d, 128));
    TRY(map_k(&a.maps[2], W->Wu, f, d, d, 128));
    TRY(map_k(&a.maps[3], P, T, 2 * rp, 2 * rp, 128));
    TRY(map_k(&a.maps[4], A->Bg, f, r, r, 128));
    TRY(map_k(&a.maps[5], A->Bu, f, r, r, 128));
    set_seg(a, 0, 0, 0, 1, 0, 2, 0, d);
    set_seg(a, 1, 3, 0, 4, 0, 5, -rp, 2 * rp);
    // MT = 2 leaves one accumulator set, so the epilogue no longer hides behind the next
    // unit's main loop: it then writes G, U, Act by TMA stores from shared-memory staging
    const int mt = pair == 2 ? pick_mt(T, pair, 128, f, mt_gain_bf16_stores()) : 1;
    a.M = static_cast<int>(T); a.N = f; a.bn = 128;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (f + 127) / 128;
    a.out[0] = G; a.out[1] = U; a.out[2] = Act; a.ld_out = f;
    if (mt == 2) TRY(set_epilogue_tma(a, 6, {G, U, Act}, T, f, f));
    set_hints(a, HINT_EVICT_LAST, HINT_NONE);  // H is re-read by every N tile: keep it in L2
    set_band(a, 8 / mt);
    a.stream_out = 1;
    if (mt == 2) TRY((launch_gemm<0, 0, 2, EPI_SWIGLU_FWD, 2, 1, 0, 2>(a, st, PH_GATEUP)));
    else if (pair == 2) TRY((launch_gemm<0, 0, 2, EPI_SWIGLU_FWD, 2, 1>(a, st, PH_GATEUP)));
    else TRY((launch_gemm<0, 0, 2, EPI_SWIGLU_FWD, 1, 1>(a, st, PH_GATEUP)));
  }
  // S4a: Pd = s * Act Ad^T
  if (dmode == 2) {
    const DualPlan pl = dual_plan(D, DL_P_D);
    DualProblem pr{};
    pr.X = Act; pr.ldx = f; pr.S[0] = A->Ad;
    TRY(launch_dual(pl.sp, &pr, 1, T, f, r, s, Pd, rp, part, cnt + dual_cnt_offset(D, DL_P_D), status, st, PH_P_D));
  } else {
    GemmArgs a = new_args(status);
    TRY(map_k(&a.maps[0], Act, T, f, f, 128));
    TRY(map_k(&a.maps[1], A->Ad, r, f, f, rp));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, f);
    a.M = static_cast<int>(T); a.N = rp; a.bn = rp;
    a.tiles_m = static_cast<int>((T + BM - 1) / BM); a.tiles_n = 1;
    TRY((launch_proj<0, 1>(a, T, f, rp, part, Pd, s, st, PH_P_D)));
  }
  // S4b: Y = Act Wd^T + Pd Bd^T
  if (q4) {
    GemmArgs a = new_args(status);
    const int bn = 256;  // d is a multiple of 256 for 4-bit weights
    const int pair = T > 128 ? 2 : 1;
    TRY(map_k(&a.maps[0], Act, T, f, f, 128));
    TRY(map_q4_k(&a.maps[1], &a.maps[4], W->Qd, am.d, d, f, bn / pair));
    TRY(map_k(&a.maps[2], Pd, T, rp, rp, 128));
    TRY(map_k(&a.maps[3], A->Bd, d, r, r, bn / pair));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, f);
    a.seg[0].q4 = 1; a.seg[0].b_am[0] = 4;
    set_seg(a, 1, 2, 0, 3, 0, -1, 0, rp);
    a.codebook = W->codebook;
    const int mt = pair == 2 ? pick_mt(T, pair, bn, d, kMtGain4bit) : 1;
    a.M = static_cast<int>(T); a.N = d; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (d + bn - 1) / bn;
    a.out[0] = Y; a.ld_out = d;
    if (D->residual) { a.in[0] = X; a.ld_in = d; }  // Y = X + ...
    a.stream_out = 1;
    set_band(a, 8 / mt);
    if (mt == 2) TRY((launch_gemm<0, 0, 1, EPI_BF16, 2, 0, 1, 2>(a, st, PH_DOWN)));
    else if (pair == 2) TRY((launch_gemm<0, 0, 1, EPI_BF16, 2, 0, 1>(a, st, PH_DOWN)));
    else TRY((launch_gemm<0, 0, 1, EPI_BF16, 1, 0, 1>(a, st, PH_DOWN)));
  } else {
    GemmArgs a = new_args(status);
    const TileChoice tcx = pick_tiles(T, d, false);
    const int bn = tcx.bn;
    const int pair = (tcx.pair == 2 && bn >= 32) ? 2 : 1;
    TRY(map_k(&a.maps[0], Act, T, f, f, 128));
    TRY(map_k(&a.maps[1], W->Wd, d, f, f, bn / pair));
    TRY(map_k(&a.maps[2], Pd, T, rp, rp, 128));
    TRY(map_k(&a.maps[3], A->Bd, d, r, r, bn / pair));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, f);
    set_seg(a, 1, 2, 0, 3, 0, -1, 0, rp);
    const int mt = pair == 2 ? pick_mt(T, pair, bn, d, kMtGainBf16LongK) : 1;
    a.M = static_cast<int>(T); a.N = d; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (d + bn - 1) / bn;
    a.out[0] = Y; a.ld_out = d;
    if (D->residual) { a.in[0] = X; a.ld_in = d; }  // Y = X + ...
    if (mt == 2) TRY(set_epilogue_tma(a, 4, {Y}, T, d, d));
    a.stream_out = 1;
    set_band(a, 8 / mt);
    if (mt == 2) TRY((launch_gemm<0, 0, 1, EPI_BF16, 2, 0, 0, 2>(a, st, PH_DOWN)));
    else if (pair == 2) TRY((launch_gemm<0, 0, 1, EPI_BF16, 2>(a, st, PH_DOWN)));
    else TRY((launch_gemm<0, 0, 1, EPI_BF16>(a, st, PH_DOWN)));
  }
  return end_call(status, st);
}

int lora_mlp_bwd(const lora_mlp_dims* D, const void* dY, const void* X, const void* rms_w, const lora_mlp_weights* W,
                 const lora_mlp_adapters* A, const void* ctx, void* dX, const lora_mlp_grads* gr, void* workspace,
                 void* stream) {
  TRY(check_dims(D));
  if (!W || !A || !gr) return fail(LORA_ERR_INVALID_ARG, "weights/adapters/grads is NULL");
  const bool q4 = D->wfmt != LORA_WFMT_BF16;
  TRY(check_ptrs({dY, X, rms_w, ctx, dX, workspace, A->Ag, A->Bg, A->Au, A->Bu, A->Ad, A->Bd,
                  gr->dAg, gr->dBg, gr->dAu, gr->dBu, gr->dAd, gr->dBd}));
  if (gr->dw) TRY(check_ptrs({gr->dw}));
  TRY(check_weights(D, W));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long T = D->T;
  const int d = D->d, f = D->f, r = D->r, rp = rp_of(D);
  const float s = D->scale;
  const lora_mlp_ctx_layout L = ctx_layout(D);
  const WsLayout WL = ws_layout(D);
  int* status = at<int>(workspace, WL.status);
  const void* H = at<char>(ctx, L.H);
  const float* rstd = at<float>(ctx, L.rstd);
  const void* G = at<char>(ctx, L.G);
  const void* U = at<char>(ctx, L.U);
  const void* Act = at<char>(ctx, L.Act);
  const void* P = at<char>(ctx, L.P);
  const void* Pd = at<char>(ctx, L.Pd);
  void* Q = at<char>(workspace, WL.Q);
  void* Qd = at<char>(workspace, WL.Qd);
  void* dG = at<char>(workspace, WL.dG);
  void* dU = at<char>(workspace, WL.dU);
  float* dH = at<float>(workspace, WL.dH);
  const int tm = static_cast<int>((T + BM - 1) / BM);
  const int qbn = rp <= 64 ? 64 : 128;
  TRY(begin_call(status, st));
  Absmax3 am{};
  if (q4) TRY(absmax_for_call(D, W, workspace, WL, st, &am));

  float* part = at<float>(workspace, WL.part);
  int* cnt = at<int>(workspace, WL.cnt);
  const int dmode = dual_mode();
  const bool dual = dmode >= 1;
  // adapter gradients: overwrite semantics -> zero them (and the arrival counters of the
  // rank-r passes), then accumulate with atomics
  {
    ZeroList z;
    z.p[0] = gr->dAg; z.n[0] = static_cast<long long>(r) * d;
    z.p[1] = gr->dAu; z.n[1] = static_cast<long long>(r) * d;
    z.p[2] = gr->dBg; z.n[2] = static_cast<long long>(f) * r;
    z.p[3] = gr->dBu; z.n[3] = static_cast<long long>(f) * r;
    z.p[4] = gr->dAd; z.n[4] = static_cast<long long>(r) * f;
    z.p[5] = gr->dBd; z.n[5] = static_cast<long long>(d) * r;
    z.p[6] = gr->dw;  z.n[6] = gr->dw ? d : 0;
    z.p[7] = reinterpret_cast<float*>(cnt); z.n[7] = WL.ncnt;  // int zero = float +0 bits
    PhaseScope ps(st, PH_ZERO);
    zero_grads_kernel<<<296, 256, 0, st>>>(z);
    CUDA_TRY(cudaGetLastError());
  }
  if (dual) {
    // S5a + S5c in one read of dY: Qd = s dY Bd, dBd = dY^T Pd
    DualProblem pr{};
    pr.X = dY; pr.ldx = d; pr.S[0] = A->Bd; pr.P = Pd; pr.ldp = rp; pr.p_cols = r; pr.out[0] = gr->dBd;
    TRY(launch_dual(dual_plan(D, DL_BWD_D).sp, &pr, 1, T, d, r, s, Qd, rp, part, cnt + dual_cnt_offset(D, DL_BWD_D),
                    status, st, PH_Q_D));
  } else {
    // S5a: Qd = s * dY Bd
    GemmArgs a = new_args(status);
    TRY(map_k(&a.maps[0], dY, T, d, d, 128));
    TRY(map_mn(&a.maps[1], A->Bd, d, r, r));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, d);
    a.M = static_cast<int>(T); a.N = rp; a.bn = qbn; a.tiles_m = tm; a.tiles_n = 1;
    TRY((launch_proj<1, 1>(a, T, d, rp, part, Qd, s, st, PH_Q_D)));
  }
  // S5b + S6: dAct = dY Wd + Qd Ad  ->  dG = dAct U silu'(G), dU = dAct silu(G)
  if (q4) {
    GemmArgs a = new_args(status);
    const int bn = 256;
    const int pair = T > 128 ? 2 : 1;
    TRY(map_k(&a.maps[0], dY, T, d, d, 128));
    TRY(map_q4_mn(&a.maps[1], &a.maps[4], W->Qd, am.d, d, f, bn / pair));
    TRY(map_k(&a.maps[2], Qd, T, rp, rp, 128));
    a.mn3d_b = 1;
    TRY(map_mn3(&a.maps[3], A->Ad, r, f, f, bn / pair / 64));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, d);
    a.seg[0].q4 = 1; a.seg[0].b_am[0] = 4;
    set_seg(a, 1, 2, 0, 3, 0, -1, 0, rp);
    a.codebook = W->codebook;
    const int mt = pair == 2 ? pick_mt(T, pair, bn, f, kMtGain4bit) : 1;
    a.M = static_cast<int>(T); a.N = f; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (f + bn - 1) / bn;
    a.in[0] = G; a.in[1] = U; a.ld_in = f;
    a.out[0] = dG; a.out[1] = dU; a.ld_out = f;
    a.stream_out = 1;
    set_band(a, 16 / mt);
    if (mt == 2) TRY((launch_gemm<0, 1, 1, EPI_SWIGLU_BWD, 2, 0, 1, 2>(a, st, PH_DACT)));
    else if (pair == 2) TRY((launch_gemm<0, 1, 1, EPI_SWIGLU_BWD, 2, 0, 1>(a, st, PH_DACT)));
    else TRY((launch_gemm<0, 1, 1, EPI_SWIGLU_BWD, 1, 0, 1>(a, st, PH_DACT)));
  } else {
    GemmArgs a = new_args(status);
    const TileChoice tcx = pick_tiles(T, f, true);
    const int bn = tcx.bn;
    const int pair = (tcx.pair == 2 && bn % 128 == 0) ? 2 : 1;
    TRY(map_k(&a.maps[0], dY, T, d, d, 128));
    TRY(map_k(&a.maps[2], Qd, T, rp, rp, 128));
    a.mn3d_b = f % 64 == 0;
    if (a.mn3d_b) {
      TRY(map_mn3(&a.maps[1], W->Wd, d, f, f, bn / pair / 64));
      TRY(map_mn3(&a.maps[3], A->Ad, r, f, f, bn / pair / 64));
    } else {
      TRY(map_mn(&a.maps[1], W->Wd, d, f, f));
      TRY(map_mn(&a.maps[3], A->Ad, r, f, f));
    }
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, d);
    set_seg(a, 1, 2, 0, 3, 0, -1, 0, rp);
    const int mt = pair == 2 ? pick_mt(T, pair, bn, f, kMtGainBf16Dact) : 1;
    a.M = static_cast<int>(T); a.N = f; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (f + bn - 1) / bn;
    a.in[0] = G; a.in[1] = U; a.ld_in = f;
    a.out[0] = dG; a.out[1] = dU; a.ld_out = f;
    if (mt == 2) TRY(set_epilogue_tma(a, 4, {dG, dU}, T, f, f));
    a.stream_out = 1;
    set_band(a, 8 / mt);
    if (mt == 2) TRY((launch_gemm<0, 1, 1, EPI_SWIGLU_BWD, 2, 0, 0, 2>(a, st, PH_DACT)));
    else if (pair == 2) TRY((launch_gemm<0, 1, 1, EPI_SWIGLU_BWD, 2>(a, st, PH_DACT)));
    else TRY((launch_gemm<0, 1, 1, EPI_SWIGLU_BWD>(a, st, PH_DACT)));
  }
  if (dual) {
    // S7a + S7b in one read of dG and dU: Q = s [dG Bg | dU Bu], dBg = dG^T P_g, dBu = dU^T P_u
    DualProblem pg[2] = {};
    pg[0].X = dG; pg[0].ldx = f; pg[0].S[0] = A->Bg; pg[0].P = P; pg[0].ldp = 2 * rp; pg[0].p_cols = r;
    pg[0].out[0] = gr->dBg;
    pg[1].X = dU; pg[1].ldx = f; pg[1].S[0] = A->Bu; pg[1].P = static_cast<const char*>(P) + rp * 2;
    pg[1].ldp = 2 * rp; pg[1].p_cols = r; pg[1].out[0] = gr->dBu;
    TRY(launch_dual(dual_plan(D, DL_BWD_GU).sp, pg, 2, T, f, r, s, Q, 2 * rp, part,
                    cnt + dual_cnt_offset(D, DL_BWD_GU), status, st, PH_Q_GU));
  } else {
    // S7a: Q = s * [dG Bg | dU Bu]
    GemmArgs a = new_args(status);
    TRY(map_k(&a.maps[0], dG, T, f, f, 128));
    TRY(map_k(&a.maps[1], dU, T, f, f, 128));
    TRY(map_mn(&a.maps[2], A->Bg, f, r, r));
    TRY(map_mn(&a.maps[3], A->Bu, f, r, r));
    set_seg(a, 0, 0, 0, 2, 0, -1, 0, f);
    set_seg(a, 1, 1, 0, -1, 0, 3, 0, f);
    a.M = static_cast<int>(T); a.N = rp; a.bn = qbn; a.tiles_m = tm; a.tiles_n = 1; a.out_acc_col = rp;
    TRY((launch_proj<1, 2>(a, T, f, 2 * rp, part, Q, s, st, PH_Q_GU)));
  }
  // S8: dH = dG Wg + dU Wu + Q_g Ag + Q_u Au   (fp32)
  if (q4) {
    GemmArgs a = new_args(status);
    const int bn = 256;
    const int pair = T > 128 ? 2 : 1;
    TRY(map_k(&a.maps[0], dG, T, f, f, 128));
    TRY(map_q4_mn(&a.maps[1], &a.maps[7], W->Qg, am.g, f, d, bn / pair));
    TRY(map_k(&a.maps[2], dU, T, f, f, 128));
    TRY(map_q4_mn(&a.maps[3], &a.maps[8], W->Qu, am.u, f, d, bn / pair));
    TRY(map_k(&a.maps[4], Q, T, 2 * rp, 2 * rp, 128));
    a.mn3d_b = 1;
    TRY(map_mn3(&a.maps[5], A->Ag, r, d, d, bn / pair / 64));
    TRY(map_mn3(&a.maps[6], A->Au, r, d, d, bn / pair / 64));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, f);
    a.seg[0].q4 = 1; a.seg[0].b_am[0] = 7;
    set_seg(a, 1, 2, 0, 3, 0, -1, 0, f);
    a.seg[1].q4 = 1; a.seg[1].b_am[0] = 8;
    set_seg(a, 2, 4, 0, 5, 0, -1, 0, rp);
    set_seg(a, 3, 4, rp, 6, 0, -1, 0, rp);
    a.codebook = W->codebook;
    const int mt = pair == 2 ? pick_mt(T, pair, bn, d, kMtGain4bit) : 1;
    a.M = static_cast<int>(T); a.N = d; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (d + bn - 1) / bn;
    a.out[0] = dH; a.ld_out = d;
    a.stream_out = 1;
    set_band(a, mt == 2 ? 2 : 4);
    if (mt == 2) TRY((launch_gemm<0, 1, 1, EPI_F32, 2, 0, 1, 2>(a, st, PH_DH)));
    else if (pair == 2) TRY((launch_gemm<0, 1, 1, EPI_F32, 2, 0, 1>(a, st, PH_DH)));
    else TRY((launch_gemm<0, 1, 1, EPI_F32, 1, 0, 1>(a, st, PH_DH)));
  } else {
    GemmArgs a = new_args(status);
    const TileChoice tcx = pick_tiles(T, d, true);
    const int bn = tcx.bn;
    const int pair = (tcx.pair == 2 && bn % 128 == 0) ? 2 : 1;
    TRY(map_k(&a.maps[0], dG, T, f, f, 128));
    TRY(map_k(&a.maps[2], dU, T, f, f, 128));
    TRY(map_k(&a.maps[4], Q, T, 2 * rp, 2 * rp, 128));
    a.mn3d_b = d % 64 == 0;
    if (a.mn3d_b) {
      TRY(map_mn3(&a.maps[1], W->Wg, f, d, d, bn / pair / 64));
      TRY(map_mn3(&a.maps[3], W->Wu, f, d, d, bn / pair / 64));
      TRY(map_mn3(&a.maps[5], A->Ag, r, d, d, bn / pair / 64));
      TRY(map_mn3(&a.maps[6], A->Au, r, d, d, bn / pair / 64));
    } else {
      TRY(map_mn(&a.maps[1], W->Wg, f, d, d));
      TRY(map_mn(&a.maps[3], W->Wu, f, d, d));
      TRY(map_mn(&a.maps[5], A->Ag, r, d, d));
      TRY(map_mn(&a.maps[6], A->Au, r, d, d));
    }
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, f);
    set_seg(a, 1, 2, 0, 3, 0, -1, 0, f);
    set_seg(a, 2, 4, 0, 5, 0, -1, 0, rp);
    set_seg(a, 3, 4, rp, 6, 0, -1, 0, rp);
    const int mt = pair == 2 ? pick_mt(T, pair, bn, d, kMtGainBf16LongK) : 1;
    a.M = static_cast<int>(T); a.N = d; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (d + bn - 1) / bn;
    a.out[0] = dH; a.ld_out = d;
    if (mt == 2) TRY(set_epilogue_tma(a, 7, {dH}, T, d, d, true));
    a.stream_out = 1;
    set_band(a, 8 / mt);
    if (mt == 2) TRY((launch_gemm<0, 1, 1, EPI_F32, 2, 0, 0, 2>(a, st, PH_DH)));
    else if (pair == 2) TRY((launch_gemm<0, 1, 1, EPI_F32, 2>(a, st, PH_DH)));
    else TRY((launch_gemm<0, 1, 1, EPI_F32>(a, st, PH_DH)));
  }
  // S10: dX = RMSNorm backward (cached rstd)
  TRY(launch_rms_bwd(st, dH, X, rms_w, rstd, dX, T, d, D->residual ? dY : nullptr));

  // norm-weight gradient (trainable-norm variant only): dw_j = sum_t dH_tj x_tj rstd_t
  if (gr->dw) {
    const int rows = static_cast<int>(std::max<long long>(64, (T + 65534) / 65535));
    const dim3 grid(static_cast<unsigned>((d / 4 + 255) / 256), static_cast<unsigned>((T + rows - 1) / rows));
    PhaseScope ps(st, PH_DW);
    norm_weight_grad_kernel<<<grid, 256, 0, st>>>(dH, static_cast<const uint16_t*>(X), rstd, gr->dw, T, d, rows);
    CUDA_TRY(cudaGetLastError());
  }
  // Adapter-gradient reductions over T: accumulator rows are the big dimension
  // (M = d or f, MN-major A), columns the rank (N = r, MN-major narrow B).
  const int rbn = r <= 64 ? 64 : 128;
  // S9: dAg = Q_g^T H, dAu = Q_u^T H   ([r x d], written transposed from [d x r] tiles)
  if (dual) {
    DualProblem pr{};
    pr.X = H; pr.ldx = d; pr.P = Q; pr.ldp = 2 * rp; pr.p_cols = 2 * rp; pr.out[0] = gr->dAg; pr.out[1] = gr->dAu;
    TRY(launch_dual(dual_plan(D, DL_RED_GU).sp, &pr, 1, T, d, r, 1.0f, nullptr, 0, part, nullptr, status, st,
                    PH_RED_DA_GU));
  } else {
    GemmArgs a = new_args(status);
    a.mn3d_a = d % 64 == 0;
    if (a.mn3d_a) TRY(map_mn3(&a.maps[0], H, T, d, d, 2));
    else TRY(map_mn(&a.maps[0], H, T, d, d));
    TRY(map_mn(&a.maps[1], Q, T, r, 2 * rp));
    TRY(map_mn(&a.maps[2], static_cast<const char*>(Q) + rp * 2, T, r, 2 * rp));
    set_seg(a, 0, 0, 0, 1, 0, 2, 0, static_cast<int>(T));
    a.M = d; a.N = r; a.bn = rbn; a.tiles_m = (d + BM - 1) / BM; a.tiles_n = 1;
    a.rng[0] = OutRange{gr->dAg, 0, 1, d};
    a.rng[1] = OutRange{gr->dAu, 1, 1, d};
    a.nrng = 2;
    choose_splits(a, T);
    TRY((launch_gemm<1, 1, 2, EPI_ATOMIC>(a, st, PH_RED_DA_GU)));
  }
  // S7b: dBg = dG^T P_g, dBu = dU^T P_u  ([f x r])
  if (!dual) {
    GemmArgs a = new_args(status);
    a.mn3d_a = f % 64 == 0;
    if (a.mn3d_a) {
      TRY(map_mn3(&a.maps[0], dG, T, f, f, 2));
      TRY(map_mn3(&a.maps[1], dU, T, f, f, 2));
    } else {
      TRY(map_mn(&a.maps[0], dG, T, f, f));
      TRY(map_mn(&a.maps[1], dU, T, f, f));
    }
    TRY(map_mn(&a.maps[2], P, T, r, 2 * rp));
    TRY(map_mn(&a.maps[3], static_cast<const char*>(P) + rp * 2, T, r, 2 * rp));
    set_seg(a, 0, 0, 0, 2, 0, -1, 0, static_cast<int>(T));
    set_seg(a, 1, 1, 0, -1, 0, 3, 0, static_cast<int>(T));
    a.M = f; a.N = r; a.bn = rbn; a.tiles_m = (f + BM - 1) / BM; a.tiles_n = 1;
    a.rng[0] = OutRange{gr->dBg, 0, 0, r};
    a.rng[1] = OutRange{gr->dBu, 1, 0, r};
    a.nrng = 2;
    choose_splits(a, T);
    TRY((launch_gemm<1, 1, 2, EPI_ATOMIC>(a, st, PH_RED_DB_GU)));
  }
  // S5c: dBd = dY^T Pd  ([d x r])
  if (!dual) {
    GemmArgs a = new_args(status);
    a.mn3d_a = d % 64 == 0;
    if (a.mn3d_a) TRY(map_mn3(&a.maps[0], dY, T, d, d, 2));
    else TRY(map_mn(&a.maps[0], dY, T, d, d));
    TRY(map_mn(&a.maps[1], Pd, T, r, rp));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, static_cast<int>(T));
    a.M = d; a.N = r; a.bn = rbn; a.tiles_m = (d + BM - 1) / BM; a.tiles_n = 1;
    a.rng[0] = OutRange{gr->dBd, 0, 0, r};
    a.nrng = 1;
    choose_splits(a, T);
    TRY((launch_gemm<1, 1, 1, EPI_ATOMIC>(a, st, PH_RED_DB_D)));
  }
  // S6b: dAd = Qd^T Act  ([r x f], written transposed from [f x r] tiles)
  if (dual) {
    DualProblem pr{};
    pr.X = Act; pr.ldx = f; pr.P = Qd; pr.ldp = rp; pr.p_cols = rp; pr.out[0] = gr->dAd;
    TRY(launch_dual(dual_plan(D, DL_RED_D).sp, &pr, 1, T, f, r, 1.0f, nullptr, 0, part, nullptr, status, st,
                    PH_RED_DA_D));
  } else {
    GemmArgs a = new_args(status);
    a.mn3d_a = f % 64 == 0;
    if (a.mn3d_a) TRY(map_mn3(&a.maps[0], Act, T, f, f, 2));
    else TRY(map_mn(&a.maps[0], Act, T, f, f));
    TRY(map_mn(&a.maps[1], Qd, T, r, rp));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, static_cast<int>(T));
    a.M = f; a.N = r; a.bn = rbn; a.tiles_m = (f + BM - 1) / BM; a.tiles_n = 1;
    a.rng[0] = OutRange{gr->dAd, 0, 1, f};
    a.nrng = 1;
    choose_splits(a, T);
    TRY((launch_gemm<1, 1, 1, EPI_ATOMIC>(a, st, PH_RED_DA_D)));
  }
  return end_call(status, st);
}

int lora_lowrank_proj_noalloc(int64_t T, int32_t K, int32_t r, float scale, const void* X, const void* A,
                              void* P, void* stream) {
  if (T < 1 || T >= (1LL << 31) || K < 8 || r < 8 || r > 128)
    return fail(LORA_ERR_INVALID_ARG, "bad T/K/r (%lld, %d, %d)", (long long)T, K, r);
  if (K % 8 || r % 8) return fail(LORA_ERR_ALIGNMENT, "K and r must be multiples of 8");
  TRY(check_ptrs({X, A, P}));
  const int rp = round_up(r, 16);
  const int splits = proj_splits(T, K);
  const size_t need = static_cast<size_t>(splits) * static_cast<size_t>(T) * rp;
  if (need > kNoAllocScratchFloats)
    return fail(LORA_ERR_UNSUPPORTED,
                "T x rp x splits = %lld x %d x %d fp32 partial sums exceed the %zu-float no-alloc scratch",
                (long long)T, rp, splits, kNoAllocScratchFloats);
  LibSyms ls;
  TRY(lib_syms(&ls));
  float* part = ls.scratch;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Every partial-sum element is overwritten by the split GEMM (all T rows and rp
  // columns of each split), so the scratch needs no clearing between calls.
  GemmArgs a = new_args(ls.status);
  TRY(map_k(&a.maps[0], X, T, K, K, 128));
  TRY(map_k(&a.maps[1], A, r, K, K, rp));
  set_seg(a, 0, 0, 0, 1, 0, -1, 0, K);
  a.M = static_cast<int>(T); a.N = rp; a.bn = rp;
  a.tiles_m = static_cast<int>((T + BM - 1) / BM); a.tiles_n = 1;
  TRY(begin_call(a.status, st));
  TRY((launch_proj<0, 1>(a, T, K, rp, part, P, scale, st, PH_OTHER)));
  return end_call(a.status, st);
}

}  // extern "C"
