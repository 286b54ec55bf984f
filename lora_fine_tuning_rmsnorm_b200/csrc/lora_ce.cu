// Host side of the fused LM-head cross-entropy entry points of liblora_mlp.so
// (lora_ce_workspace_bytes, lora_ce_fwd, lora_ce_bwd).
//
// Forward: one tcgen05 GEMM over logits tiles z = H W^T whose epilogue reduces each tile
// to per-token (max, sum of exponentials) pairs and picks out the label's logit, then a
// row kernel combines them into lse and the loss, and a one-CTA kernel reduces the
// losses.  The logits never leave tensor memory.
// Backward: for each vocabulary chunk, the same GEMM recomputes the chunk's logits and
// its epilogue writes dZ = g' (softmax - onehot) as bf16 for that chunk only; a second
// GEMM accumulates dH += dZ_chunk W_chunk in fp32.  Only [T x chunk] of dZ ever exists.
#include "host.cuh"
#include "ce.cuh"

using namespace lm;
using namespace lm::host;

namespace {

constexpr int kCeDefaultChunk = 32768;

int check_ce_dims(const lora_ce_dims* D) {
  if (!D) return fail(LORA_ERR_INVALID_ARG, "dims is NULL");
  if (D->T < 1 || D->T >= (1LL << 31)) return fail(LORA_ERR_INVALID_ARG, "T = %lld out of range", (long long)D->T);
  if (D->d < 8 || D->V < 8) return fail(LORA_ERR_INVALID_ARG, "d, V must be >= 8");
  if (D->d % 8 || D->V % 8) return fail(LORA_ERR_ALIGNMENT, "d, V must be multiples of 8; got %d %d", D->d, D->V);
  if (D->vocab_chunk < 0 || D->vocab_chunk % 256)
    return fail(LORA_ERR_INVALID_ARG, "vocab_chunk = %d must be 0 or a positive multiple of 256", D->vocab_chunk);
  if (D->reduction != LORA_CE_MEAN && D->reduction != LORA_CE_SUM)
    return fail(LORA_ERR_INVALID_ARG, "reduction must be LORA_CE_MEAN or LORA_CE_SUM");
  return LORA_OK;
}

int ce_chunk(const lora_ce_dims* D) {
  const int c = D->vocab_chunk ? D->vocab_chunk : kCeDefaultChunk;
  return std::min(c, round_up(D->V, 256));
}

struct CeWsLayout {
  size_t status, part, zlab, blk, dZ, total;
  long long nblk;
};
CeWsLayout ce_ws_layout(const lora_ce_dims* D) {
  const size_t T = D->T;
  const size_t nparts = 2 * ((static_cast<size_t>(D->V) + 127) / 128);  // two per N tile of >= 128 columns
  CeWsLayout L{};
  L.nblk = (D->T + kCeThreads - 1) / kCeThreads;
  size_t o = 0;
  L.status = o; o = 256;
  L.part = o; o = up256(o + nparts * T * 8);
  L.zlab = o; o = up256(o + T * 4);
  L.blk = o;  o = up256(o + static_cast<size_t>(L.nblk) * 8);
  L.dZ = o;   o = up256(o + T * static_cast<size_t>(ce_chunk(D)) * 2);
  L.total = o;
  return L;
}

int check_scalar_ptr(const void* p, const char* name) {
  if (!p) return fail(LORA_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % 4) return fail(LORA_ERR_ALIGNMENT, "%s is not 4-byte aligned", name);
  return LORA_OK;
}

}  // namespace

extern "C" {

int lora_ce_workspace_bytes(const lora_ce_dims* dims, size_t* bytes) {
  TRY(check_ce_dims(dims));
  if (!bytes) return fail(LORA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = ce_ws_layout(dims).total;
  return LORA_OK;
}

int lora_ce_fwd(const lora_ce_dims* D, const void* H, const void* W, const int32_t* labels, float* loss_rows,
                float* lse, float* loss, int32_t* n_valid, void* workspace, void* stream) {
  TRY(check_ce_dims(D));
  TRY(check_ptrs({H, W, labels, loss_rows, lse, workspace}));
  TRY(check_scalar_ptr(loss, "loss"));
  TRY(check_scalar_ptr(n_valid, "n_valid"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long T = D->T;
  const int d = D->d, V = D->V;
  const CeWsLayout WL = ce_ws_layout(D);
  int* status = at<int>(workspace, WL.status);
  float2* part = at<float2>(workspace, WL.part);
  float* zlab = at<float>(workspace, WL.zlab);
  float2* blk = at<float2>(workspace, WL.blk);
  TRY(begin_call(status, st));
  int nparts = 0;
  {
    GemmArgs a = new_args(status);
    const TileChoice tcx = pick_tiles(T, V, false);
    const int bn = tcx.bn;
    const int pair = (tcx.pair == 2 && bn >= 32) ? 2 : 1;
    TRY(map_k(&a.maps[0], H, T, d, d, 128));
    TRY(map_k(&a.maps[1], W, V, d, d, bn / pair));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, d);
    // tiles M-fastest: every LM-head tile is read from HBM once and meets all token
    // tiles while it is in L2; H (re-read by every vocabulary tile) is kept in L2
    set_hints(a, HINT_EVICT_LAST, HINT_NONE);
    const int mt = pair == 2 ? pick_mt(T, pair, bn, V, kMtGainCe) : 1;
    a.M = static_cast<int>(T); a.N = V; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (V + bn - 1) / bn;
    a.out[0] = part; a.out[1] = zlab;
    a.ce_labels = labels; a.ce_col0 = 0; a.ce_V = V;
    nparts = 2 * a.tiles_n;
    if (mt == 2) TRY((launch_gemm<0, 0, 1, EPI_CE_LSE, 2, 0, 0, 2>(a, st, PH_CE_LSE)));
    else if (pair == 2) TRY((launch_gemm<0, 0, 1, EPI_CE_LSE, 2>(a, st, PH_CE_LSE)));
    else TRY((launch_gemm<0, 0, 1, EPI_CE_LSE>(a, st, PH_CE_LSE)));
  }
  {
    PhaseScope ps(st, PH_CE_FIN);
    ce_finalize_kernel<<<static_cast<unsigned>(WL.nblk), kCeThreads, 0, st>>>(part, nparts, zlab, labels, T, V,
                                                                             loss_rows, lse, blk);
    CUDA_TRY(cudaGetLastError());
    ce_reduce_kernel<<<1, kCeThreads, 0, st>>>(blk, static_cast<int>(WL.nblk), D->reduction == LORA_CE_MEAN, loss,
                                               n_valid);
    CUDA_TRY(cudaGetLastError());
  }
  return end_call(status, st);
}

int lora_ce_bwd(const lora_ce_dims* D, const void* H, const void* W, const int32_t* labels, const float* lse,
                const int32_t* n_valid, float dloss, float* dH, void* workspace, void* stream) {
  TRY(check_ce_dims(D));
  TRY(check_ptrs({H, W, labels, lse, dH, workspace}));
  TRY(check_scalar_ptr(n_valid, "n_valid"));
  if (!std::isfinite(dloss)) return fail(LORA_ERR_INVALID_ARG, "dloss is not finite");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long T = D->T;
  const int d = D->d, V = D->V, chunk = ce_chunk(D);
  const CeWsLayout WL = ce_ws_layout(D);
  int* status = at<int>(workspace, WL.status);
  void* dZ = at<char>(workspace, WL.dZ);
  TRY(begin_call(status, st));
  for (int v0 = 0; v0 < V; v0 += chunk) {
    const int N = std::min(chunk, V - v0);
    const char* Wc = static_cast<const char*>(W) + static_cast<size_t>(v0) * d * 2;
    // dZ[:, 0:N] = g' (softmax - onehot) of vocabulary columns [v0, v0 + N)
    {
      GemmArgs a = new_args(status);
      const TileChoice tcx = pick_tiles(T, N, false);
      const int bn = tcx.bn;
      const int pair = (tcx.pair == 2 && bn >= 32) ? 2 : 1;
      TRY(map_k(&a.maps[0], H, T, d, d, 128));
      TRY(map_k(&a.maps[1], Wc, N, d, d, bn / pair));
      set_seg(a, 0, 0, 0, 1, 0, -1, 0, d);
      set_hints(a, HINT_EVICT_LAST, HINT_NONE);
      const int mt = pair == 2 ? pick_mt(T, pair, bn, N, kMtGainCe) : 1;
      a.M = static_cast<int>(T); a.N = N; a.bn = bn;
      a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (N + bn - 1) / bn;
      a.out[0] = dZ; a.ld_out = chunk;
      if (mt == 2) TRY(set_epilogue_tma(a, 2, {dZ}, T, N, chunk));
      a.ce_labels = labels; a.ce_lse = lse; a.ce_count = D->reduction == LORA_CE_MEAN ? n_valid : nullptr;
      a.ce_g = dloss; a.ce_col0 = v0; a.ce_V = V;
      if (mt == 2) TRY((launch_gemm<0, 0, 1, EPI_CE_DZ, 2, 0, 0, 2>(a, st, PH_CE_DZ)));
      else if (pair == 2) TRY((launch_gemm<0, 0, 1, EPI_CE_DZ, 2>(a, st, PH_CE_DZ)));
      else TRY((launch_gemm<0, 0, 1, EPI_CE_DZ>(a, st, PH_CE_DZ)));
    }
    // dH (+)= dZ[:, 0:N] W[v0 : v0 + N]   (fp32; the LM head read MN-major)
    {
      GemmArgs a = new_args(status);
      const TileChoice tcx = pick_tiles(T, d, true);
      const int bn = tcx.bn;
      const int pair = (tcx.pair == 2 && bn % 128 == 0) ? 2 : 1;
      TRY(map_k(&a.maps[0], dZ, T, N, chunk, 128));
      a.mn3d_b = d % 64 == 0;
      if (a.mn3d_b) TRY(map_mn3(&a.maps[1], Wc, N, d, d, bn / pair / 64));
      else TRY(map_mn(&a.maps[1], Wc, N, d, d));
      set_seg(a, 0, 0, 0, 1, 0, -1, 0, N);
      const int mt = pair == 2 ? pick_mt(T, pair, bn, d, kMtGainBf16LongK) : 1;  // K = the chunk
      a.M = static_cast<int>(T); a.N = d; a.bn = bn;
      a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (d + bn - 1) / bn;
      a.out[0] = dH; a.ld_out = d;
      a.out_add = v0 > 0;  // with TMA stores: an fp32 add-reduction into the previous chunks' sum
      if (mt == 2) TRY(set_epilogue_tma(a, 2, {dH}, T, d, d, true));
      set_band(a, mt == 2 ? 2 : 4);
      if (mt == 2) TRY((launch_gemm<0, 1, 1, EPI_F32, 2, 0, 0, 2>(a, st, PH_CE_DH)));
      else if (pair == 2) TRY((launch_gemm<0, 1, 1, EPI_F32, 2>(a, st, PH_CE_DH)));
      else TRY((launch_gemm<0, 1, 1, EPI_F32>(a, st, PH_CE_DH)));
    }
  }
  return end_call(status, st);
}

}  // extern "C"
