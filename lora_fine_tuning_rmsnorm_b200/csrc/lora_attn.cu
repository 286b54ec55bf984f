// Host side of the attention-side entry points of liblora_mlp.so: LoRA on the Q/K/V
// projections (with the RMSNorm in front), LoRA on the output projection o_proj, and
// the rotary position embedding of the query / key heads.
#include "host.cuh"

using namespace lm;
using namespace lm::host;

namespace {

// ------------------------------------------------- attention Q/K/V projections
int check_qkv_dims(const lora_qkv_dims* D) {
  if (!D) return fail(LORA_ERR_INVALID_ARG, "dims is NULL");
  if (D->T < 1 || D->T >= (1LL << 31)) return fail(LORA_ERR_INVALID_ARG, "T = %lld out of range", (long long)D->T);
  if (D->d < 8 || D->nq < 8 || D->nkv < 8 || D->r < 1) return fail(LORA_ERR_INVALID_ARG, "d, nq, nkv >= 8, r >= 1");
  if (D->d % 8 || D->nq % 8 || D->nkv % 8 || D->r % 8)
    return fail(LORA_ERR_ALIGNMENT, "d, nq, nkv, r must be multiples of 8; got %d %d %d %d", D->d, D->nq, D->nkv, D->r);
  if (D->d > 65536) return fail(LORA_ERR_UNSUPPORTED, "d = %d > 65536", D->d);
  if (D->r > 128) return fail(LORA_ERR_UNSUPPORTED, "r = %d > 128", D->r);
  return LORA_OK;
}

lora_qkv_ctx_layout qkv_ctx_layout(const lora_qkv_dims* D) {
  const size_t T = D->T, d = D->d, rp = round_up(D->r, 16);
  lora_qkv_ctx_layout L{};
  size_t o = 0;
  L.rstd = o; o = up256(o + T * 4);
  L.H = o;    o = up256(o + T * d * 2);
  L.P = o;    o = up256(o + T * 3 * rp * 2);
  L.total = o;
  L.rp = static_cast<int32_t>(rp);
  return L;
}

// Rank-r streaming launches of the Q/K/V backward (lowrank_dual.cuh): Q_q with dB_q, then
// Q_k, Q_v with dB_k, dB_v (two problems sharing K = nkv), then dA_q, dA_k, dA_v in one
// read of H.  Their arrival counters follow one another in the workspace.
struct QkvDual {
  DualSpec sp;
  int K, nx;
  long long cnt_off;
};
QkvDual qkv_dual(const lora_qkv_dims* D, int which) {
  const DualSpec both = dual_spec_both(D->r);
  const long long c0 = dual_counters(both, D->T, D->nq, 1);
  if (which == 0) return QkvDual{both, D->nq, 1, 0};
  if (which == 1) return QkvDual{both, D->nkv, 2, c0};
  return QkvDual{dual_spec_reduce(D->r, 3), D->d, 1, c0 + dual_counters(both, D->T, D->nkv, 2)};
}

struct QkvWsLayout {
  size_t status, Q, dH, part, cnt, total;
  long long ncnt;
};
QkvWsLayout qkv_ws_layout(const lora_qkv_dims* D) {
  const size_t T = D->T, d = D->d, rp = round_up(D->r, 16);
  QkvWsLayout L{};
  size_t o = 0;
  L.status = o; o = 256;
  L.Q = o;  o = up256(o + T * 3 * rp * 2);   // s (dQ Bq | dK Bk | dV Bv)
  L.dH = o; o = up256(o + T * d * 4);
  size_t part = 0;
  for (long long K : {static_cast<long long>(D->d), static_cast<long long>(D->nq), static_cast<long long>(D->nkv)})
    part = std::max(part, size_t(proj_splits(T, K)) * T * rp);
  for (int i = 0; i < 2; ++i) {  // the single-pass kernels' partial slots (Q rows of 3 rp)
    const QkvDual q = qkv_dual(D, i);
    part = std::max(part, size_t(dual_slots_bound(q.sp, D->T, q.K, q.nx)) * T * 3 * rp);
  }
  L.part = o; o = up256(o + part * 4);
  L.ncnt = qkv_dual(D, 2).cnt_off;
  L.cnt = o; o = up256(o + static_cast<size_t>(L.ncnt) * 4);
  L.total = o;
  return L;
}

// ------------------------------------------------------- o_proj LoRA linear
int check_o_dims(const lora_o_dims* D) {
  if (!D) return fail(LORA_ERR_INVALID_ARG, "dims is NULL");
  if (D->T < 1 || D->T >= (1LL << 31)) return fail(LORA_ERR_INVALID_ARG, "T = %lld out of range", (long long)D->T);
  if (D->n_in < 8 || D->n_out < 8 || D->r < 1) return fail(LORA_ERR_INVALID_ARG, "n_in, n_out >= 8, r >= 1");
  if (D->n_in % 8 || D->n_out % 8 || D->r % 8)
    return fail(LORA_ERR_ALIGNMENT, "n_in, n_out, r must be multiples of 8; got %d %d %d", D->n_in, D->n_out, D->r);
  if (D->r > 128) return fail(LORA_ERR_UNSUPPORTED, "r = %d > 128", D->r);
  return LORA_OK;
}

struct OWsLayout {
  size_t status, Q, part, cnt, total;
  long long ncnt;
};
OWsLayout o_ws_layout(const lora_o_dims* D) {
  const size_t T = D->T, rp = round_up(D->r, 16);
  const DualSpec both = dual_spec_both(D->r);  // Q = s dY Bo with dBo = dY^T P, one read of dY
  OWsLayout L{};
  size_t o = 0;
  L.status = o; o = 256;
  L.Q = o; o = up256(o + T * rp * 2);        // s dY Bo
  size_t part = std::max(size_t(proj_splits(T, D->n_in)), size_t(proj_splits(T, D->n_out))) * T * rp;
  part = std::max(part, size_t(dual_slots_bound(both, D->T, D->n_out, 1)) * T * rp);
  L.part = o; o = up256(o + part * 4);
  L.ncnt = dual_counters(both, D->T, D->n_out, 1);
  L.cnt = o; o = up256(o + static_cast<size_t>(L.ncnt) * 4);
  L.total = o;
  return L;
}
size_t o_ctx_bytes(const lora_o_dims* D) { return up256(size_t(D->T) * round_up(D->r, 16) * 2); }

}  // namespace

extern "C" {

int lora_qkv_ctx_layout_get(const lora_qkv_dims* dims, lora_qkv_ctx_layout* out) {
  TRY(check_qkv_dims(dims));
  if (!out) return fail(LORA_ERR_INVALID_ARG, "out is NULL");
  *out = qkv_ctx_layout(dims);
  return LORA_OK;
}

int lora_qkv_workspace_bytes(const lora_qkv_dims* dims, size_t* bytes) {
  TRY(check_qkv_dims(dims));
  if (!bytes) return fail(LORA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = qkv_ws_layout(dims).total;
  return LORA_OK;
}

int lora_qkv_fwd(const lora_qkv_dims* D, const void* X, const void* rms_w, const lora_qkv_weights* W,
                 const lora_qkv_adapters* A, void* Qo, void* Ko, void* Vo, void* ctx, void* workspace,
                 void* stream) {
  TRY(check_qkv_dims(D));
  if (!W || !A) return fail(LORA_ERR_INVALID_ARG, "weights/adapters is NULL");
  TRY(check_ptrs({X, rms_w, Qo, Ko, Vo, ctx, workspace, W->Wq, W->Wk, W->Wv, A->Aq, A->Bq, A->Ak, A->Bk, A->Av,
                  A->Bv}));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long T = D->T;
  const int d = D->d, r = D->r, rp = round_up(r, 16);
  const lora_qkv_ctx_layout L = qkv_ctx_layout(D);
  const QkvWsLayout WL = qkv_ws_layout(D);
  int* status = at<int>(workspace, WL.status);
  void* H = at<char>(ctx, L.H);
  float* rstd = at<float>(ctx, L.rstd);
  char* P = at<char>(ctx, L.P);
  float* part = at<float>(workspace, WL.part);
  TRY(begin_call(status, st));
  TRY(launch_rms_fwd(st, X, rms_w, H, rstd, T, d, D->eps));
  const void* Wx[3] = {W->Wq, W->Wk, W->Wv};
  const void* Ax[3] = {A->Aq, A->Ak, A->Av};
  const void* Bx[3] = {A->Bq, A->Bk, A->Bv};
  void* Ox[3] = {Qo, Ko, Vo};
  const int nx[3] = {D->nq, D->nkv, D->nkv};
  // P_x = s H A_x^T into columns [x rp, x rp + rp) of P [T x 3rp]
  for (int x = 0; x < 3; ++x) {
    GemmArgs a = new_args(status);
    TRY(map_k(&a.maps[0], H, T, d, d, 128));
    TRY(map_k(&a.maps[1], Ax[x], r, d, d, rp));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, d);
    a.M = static_cast<int>(T); a.N = rp; a.bn = rp;
    a.tiles_m = static_cast<int>((T + BM - 1) / BM); a.tiles_n = 1;
    TRY((launch_proj_into<0>(a, T, d, rp, part, P + static_cast<size_t>(x) * rp * 2, 3LL * rp, D->scale, st,
                             PH_QKV_LOWRANK)));
  }
  // Out_x = H W_x^T + P_x B_x^T: the LoRA term as a K = rp extension of the dense GEMM
  for (int x = 0; x < 3; ++x) {
    GemmArgs a = new_args(status);
    const TileChoice tcx = pick_tiles(T, nx[x], false);
    const int bn = tcx.bn;
    const int pair = (tcx.pair == 2 && bn >= 32) ? 2 : 1;
    TRY(map_k(&a.maps[0], H, T, d, d, 128));
    TRY(map_k(&a.maps[1], Wx[x], nx[x], d, d, bn / pair));
    TRY(map_k(&a.maps[2], P + static_cast<size_t>(x) * rp * 2, T, rp, 3 * rp, 128));
    TRY(map_k(&a.maps[3], Bx[x], nx[x], r, r, bn / pair));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, d);
    set_seg(a, 1, 2, 0, 3, 0, -1, 0, rp);
    const int mt = pair == 2 ? pick_mt(T, pair, bn, nx[x], mt_gain_bf16_stores()) : 1;
    a.M = static_cast<int>(T); a.N = nx[x]; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (nx[x] + bn - 1) / bn;
    a.out[0] = Ox[x]; a.ld_out = nx[x];
    if (mt == 2) TRY(set_epilogue_tma(a, 4, {Ox[x]}, T, nx[x], nx[x]));
    a.stream_out = 1;
    set_band(a, 8 / mt);
    if (mt == 2) TRY((launch_gemm<0, 0, 1, EPI_BF16, 2, 0, 0, 2>(a, st, PH_QKV_GEMM)));
    else if (pair == 2) TRY((launch_gemm<0, 0, 1, EPI_BF16, 2>(a, st, PH_QKV_GEMM)));
    else TRY((launch_gemm<0, 0, 1, EPI_BF16>(a, st, PH_QKV_GEMM)));
  }
  return end_call(status, st);
}

int lora_qkv_bwd(const lora_qkv_dims* D, const void* dQ, const void* dK, const void* dV, const void* X,
                 const void* rms_w, const lora_qkv_weights* W, const lora_qkv_adapters* A, const void* ctx,
                 void* dX, const lora_qkv_grads* gr, void* workspace, void* stream) {
  TRY(check_qkv_dims(D));
  if (!W || !A || !gr) return fail(LORA_ERR_INVALID_ARG, "weights/adapters/grads is NULL");
  TRY(check_ptrs({dQ, dK, dV, X, rms_w, ctx, dX, workspace, W->Wq, W->Wk, W->Wv, A->Aq, A->Bq, A->Ak, A->Bk,
                  A->Av, A->Bv, gr->dAq, gr->dBq, gr->dAk, gr->dBk, gr->dAv, gr->dBv}));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long T = D->T;
  const int d = D->d, r = D->r, rp = round_up(r, 16);
  const lora_qkv_ctx_layout L = qkv_ctx_layout(D);
  const QkvWsLayout WL = qkv_ws_layout(D);
  int* status = at<int>(workspace, WL.status);
  const void* H = at<char>(ctx, L.H);
  const float* rstd = at<float>(ctx, L.rstd);
  const char* P = at<char>(ctx, L.P);
  char* Q = at<char>(workspace, WL.Q);
  float* dH = at<float>(workspace, WL.dH);
  float* part = at<float>(workspace, WL.part);
  const void* dZ[3] = {dQ, dK, dV};
  const void* Wx[3] = {W->Wq, W->Wk, W->Wv};
  const void* Ax[3] = {A->Aq, A->Ak, A->Av};
  const void* Bx[3] = {A->Bq, A->Bk, A->Bv};
  float* dAx[3] = {gr->dAq, gr->dAk, gr->dAv};
  float* dBx[3] = {gr->dBq, gr->dBk, gr->dBv};
  const int nx[3] = {D->nq, D->nkv, D->nkv};
  const int qbn = rp <= 64 ? 64 : 128;
  TRY(begin_call(status, st));
  int* cnt = at<int>(workspace, WL.cnt);
  const bool dual = dual_mode() >= 1;
  // adapter gradients: overwrite semantics -> zero them (and the arrival counters), then
  // accumulate with atomics
  {
    ZeroList z{};
    for (int x = 0; x < 3; ++x) {
      z.p[2 * x] = dAx[x]; z.n[2 * x] = static_cast<long long>(r) * d;
      z.p[2 * x + 1] = dBx[x]; z.n[2 * x + 1] = static_cast<long long>(nx[x]) * r;
    }
    z.p[6] = reinterpret_cast<float*>(cnt); z.n[6] = WL.ncnt;  // int zero = float +0 bits
    PhaseScope ps(st, PH_ZERO);
    zero_grads_kernel<<<296, 256, 0, st>>>(z);
    CUDA_TRY(cudaGetLastError());
  }
  if (dual) {
    // Q_x = s dZ_x B_x into columns [x rp, x rp + rp) of Q [T x 3rp] with dB_x = dZ_x^T P_x,
    // one read of each dZ_x: q alone, then k and v (same width) together
    DualProblem pr[3] = {};
    for (int x = 0; x < 3; ++x) {
      pr[x].X = dZ[x]; pr[x].ldx = nx[x]; pr[x].S[0] = Bx[x];
      pr[x].P = P + static_cast<size_t>(x) * rp * 2; pr[x].ldp = 3 * rp; pr[x].p_cols = r;
      pr[x].out[0] = dBx[x];
    }
    const QkvDual q0 = qkv_dual(D, 0), q1 = qkv_dual(D, 1);
    TRY(launch_dual(q0.sp, &pr[0], 1, T, D->nq, r, D->scale, Q, 3 * rp, part, cnt + q0.cnt_off, status, st,
                    PH_QKV_LOWRANK));
    TRY(launch_dual(q1.sp, &pr[1], 2, T, D->nkv, r, D->scale, Q + static_cast<size_t>(rp) * 2, 3 * rp, part,
                    cnt + q1.cnt_off, status, st, PH_QKV_LOWRANK));
  }
  // Q_x = s dZ_x B_x into columns [x rp, x rp + rp) of Q [T x 3rp]
  for (int x = 0; x < 3 && !dual; ++x) {
    GemmArgs a = new_args(status);
    TRY(map_k(&a.maps[0], dZ[x], T, nx[x], nx[x], 128));
    TRY(map_mn(&a.maps[1], Bx[x], nx[x], r, r));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, nx[x]);
    a.M = static_cast<int>(T); a.N = rp; a.bn = qbn;
    a.tiles_m = static_cast<int>((T + BM - 1) / BM); a.tiles_n = 1;
    TRY((launch_proj_into<1>(a, T, nx[x], rp, part, Q + static_cast<size_t>(x) * rp * 2, 3LL * rp, D->scale, st,
                             PH_QKV_LOWRANK)));
  }
  // dH = dQ Wq + dK Wk + dV Wv + [Q_q | Q_k | Q_v] [Aq; Ak; Av]   (fp32; six K segments)
  {
    GemmArgs a = new_args(status);
    const TileChoice tcx = pick_tiles(T, d, true);
    const int bn = tcx.bn;
    const int pair = (tcx.pair == 2 && bn % 128 == 0) ? 2 : 1;
    a.mn3d_b = d % 64 == 0;
    for (int x = 0; x < 3; ++x) {
      TRY(map_k(&a.maps[2 * x], dZ[x], T, nx[x], nx[x], 128));
      if (a.mn3d_b) {
        TRY(map_mn3(&a.maps[2 * x + 1], Wx[x], nx[x], d, d, bn / pair / 64));
        TRY(map_mn3(&a.maps[7 + x], Ax[x], r, d, d, bn / pair / 64));
      } else {
        TRY(map_mn(&a.maps[2 * x + 1], Wx[x], nx[x], d, d));
        TRY(map_mn(&a.maps[7 + x], Ax[x], r, d, d));
      }
      set_seg(a, x, 2 * x, 0, 2 * x + 1, 0, -1, 0, nx[x]);
    }
    TRY(map_k(&a.maps[6], Q, T, 3 * rp, 3 * rp, 128));
    for (int x = 0; x < 3; ++x) set_seg(a, 3 + x, 6, x * rp, 7 + x, 0, -1, 0, rp);
    // K = nq + 2 nkv (+ 3 rp): long enough that B fetched once per two M tiles pays
    const int mt = pair == 2 ? pick_mt(T, pair, bn, d, kMtGainBf16LongK) : 1;
    a.M = static_cast<int>(T); a.N = d; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (d + bn - 1) / bn;
    a.out[0] = dH; a.ld_out = d;
    if (mt == 2) TRY(set_epilogue_tma(a, 10, {dH}, T, d, d, true));
    set_band(a, mt == 2 ? 2 : 4);
    if (mt == 2) TRY((launch_gemm<0, 1, 1, EPI_F32, 2, 0, 0, 2>(a, st, PH_QKV_DH)));
    else if (pair == 2) TRY((launch_gemm<0, 1, 1, EPI_F32, 2>(a, st, PH_QKV_DH)));
    else TRY((launch_gemm<0, 1, 1, EPI_F32>(a, st, PH_QKV_DH)));
  }
  TRY(launch_rms_bwd(st, dH, X, rms_w, rstd, dX, T, d));
  const int rbn = r <= 64 ? 64 : 128;
  const bool dual_da = dual && qkv_dual(D, 2).sp.n <= 256;  // 3 rp columns fit one MMA (r <= 80)
  if (dual_da) {
    // dA_q, dA_k, dA_v = [Q_q | Q_k | Q_v]^T H in one read of H  ([r x d] each)
    DualProblem pr{};
    pr.X = H; pr.ldx = d; pr.P = Q; pr.ldp = 3 * rp; pr.p_cols = 3 * rp;
    for (int x = 0; x < 3; ++x) pr.out[x] = dAx[x];
    TRY(launch_dual(qkv_dual(D, 2).sp, &pr, 1, T, d, r, 1.0f, nullptr, 0, part, nullptr, status, st,
                    PH_QKV_LOWRANK));
  }
  // dA_x = Q_x^T H  ([r x d], written transposed from [d x r] tiles)
  for (int x = 0; x < 3 && !dual_da; ++x) {
    GemmArgs a = new_args(status);
    a.mn3d_a = d % 64 == 0;
    if (a.mn3d_a) TRY(map_mn3(&a.maps[0], H, T, d, d, 2));
    else TRY(map_mn(&a.maps[0], H, T, d, d));
    TRY(map_mn(&a.maps[1], Q + static_cast<size_t>(x) * rp * 2, T, r, 3 * rp));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, static_cast<int>(T));
    a.M = d; a.N = r; a.bn = rbn; a.tiles_m = (d + BM - 1) / BM; a.tiles_n = 1;
    a.rng[0] = OutRange{dAx[x], 0, 1, d};
    a.nrng = 1;
    choose_splits(a, T);
    TRY((launch_gemm<1, 1, 1, EPI_ATOMIC>(a, st, PH_QKV_LOWRANK)));
  }
  // dB_x = dZ_x^T P_x  ([n_x x r])
  for (int x = 0; x < 3 && !dual; ++x) {
    GemmArgs a = new_args(status);
    a.mn3d_a = nx[x] % 64 == 0;
    if (a.mn3d_a) TRY(map_mn3(&a.maps[0], dZ[x], T, nx[x], nx[x], 2));
    else TRY(map_mn(&a.maps[0], dZ[x], T, nx[x], nx[x]));
    TRY(map_mn(&a.maps[1], P + static_cast<size_t>(x) * rp * 2, T, r, 3 * rp));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, static_cast<int>(T));
    a.M = nx[x]; a.N = r; a.bn = rbn; a.tiles_m = (nx[x] + BM - 1) / BM; a.tiles_n = 1;
    a.rng[0] = OutRange{dBx[x], 0, 0, r};
    a.nrng = 1;
    choose_splits(a, T);
    TRY((launch_gemm<1, 1, 1, EPI_ATOMIC>(a, st, PH_QKV_LOWRANK)));
  }
  return end_call(status, st);
}

// ------------------------------------------------------- o_proj LoRA linear
int lora_o_ctx_bytes(const lora_o_dims* dims, size_t* bytes) {
  TRY(check_o_dims(dims));
  if (!bytes) return fail(LORA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = o_ctx_bytes(dims);
  return LORA_OK;
}

int lora_o_workspace_bytes(const lora_o_dims* dims, size_t* bytes) {
  TRY(check_o_dims(dims));
  if (!bytes) return fail(LORA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = o_ws_layout(dims).total;
  return LORA_OK;
}

int lora_o_fwd(const lora_o_dims* D, const void* X, const void* Wo, const void* Ao, const void* Bo, void* Y, void* ctx,
               void* workspace, void* stream) {
  TRY(check_o_dims(D));
  TRY(check_ptrs({X, Wo, Ao, Bo, Y, ctx, workspace}));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long T = D->T;
  const int n_in = D->n_in, n_out = D->n_out, r = D->r, rp = round_up(r, 16);
  const OWsLayout WL = o_ws_layout(D);
  int* status = at<int>(workspace, WL.status);
  float* part = at<float>(workspace, WL.part);
  TRY(begin_call(status, st));
  // P = s X Ao^T  (rank-r projection, saved for the backward)
  {
    GemmArgs a = new_args(status);
    TRY(map_k(&a.maps[0], X, T, n_in, n_in, 128));
    TRY(map_k(&a.maps[1], Ao, r, n_in, n_in, rp));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, n_in);
    a.M = static_cast<int>(T); a.N = rp; a.bn = rp;
    a.tiles_m = static_cast<int>((T + BM - 1) / BM); a.tiles_n = 1;
    TRY((launch_proj<0, 1>(a, T, n_in, rp, part, ctx, D->scale, st, PH_O_LOWRANK)));
  }
  // Y = X Wo^T + P Bo^T: the LoRA term as a K = rp extension of the dense GEMM
  {
    GemmArgs a = new_args(status);
    const TileChoice tcx = pick_tiles(T, n_out, false);
    const int bn = tcx.bn;
    const int pair = (tcx.pair == 2 && bn >= 32) ? 2 : 1;
    TRY(map_k(&a.maps[0], X, T, n_in, n_in, 128));
    TRY(map_k(&a.maps[1], Wo, n_out, n_in, n_in, bn / pair));
    TRY(map_k(&a.maps[2], ctx, T, rp, rp, 128));
    TRY(map_k(&a.maps[3], Bo, n_out, r, r, bn / pair));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, n_in);
    set_seg(a, 1, 2, 0, 3, 0, -1, 0, rp);
    const int mt = pair == 2 ? pick_mt(T, pair, bn, n_out, mt_gain_bf16_stores()) : 1;
    a.M = static_cast<int>(T); a.N = n_out; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (n_out + bn - 1) / bn;
    a.out[0] = Y; a.ld_out = n_out;
    if (mt == 2) TRY(set_epilogue_tma(a, 4, {Y}, T, n_out, n_out));
    a.stream_out = 1;
    set_band(a, 8 / mt);
    if (mt == 2) TRY((launch_gemm<0, 0, 1, EPI_BF16, 2, 0, 0, 2>(a, st, PH_O_GEMM)));
    else if (pair == 2) TRY((launch_gemm<0, 0, 1, EPI_BF16, 2>(a, st, PH_O_GEMM)));
    else TRY((launch_gemm<0, 0, 1, EPI_BF16>(a, st, PH_O_GEMM)));
  }
  return end_call(status, st);
}

int lora_o_bwd(const lora_o_dims* D, const void* dY, const void* X, const void* Wo, const void* Ao, const void* Bo,
               const void* ctx, void* dX, float* dAo, float* dBo, void* workspace, void* stream) {
  TRY(check_o_dims(D));
  TRY(check_ptrs({dY, X, Wo, Ao, Bo, ctx, dX, dAo, dBo, workspace}));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long T = D->T;
  const int n_in = D->n_in, n_out = D->n_out, r = D->r, rp = round_up(r, 16);
  const OWsLayout WL = o_ws_layout(D);
  int* status = at<int>(workspace, WL.status);
  float* part = at<float>(workspace, WL.part);
  void* Q = at<char>(workspace, WL.Q);
  TRY(begin_call(status, st));
  int* cnt = at<int>(workspace, WL.cnt);
  const bool dual = dual_mode() >= 1;
  {  // overwrite semantics: zero the gradients (and the arrival counters), then accumulate
    ZeroList z{};
    z.p[0] = dAo; z.n[0] = static_cast<long long>(r) * n_in;
    z.p[1] = dBo; z.n[1] = static_cast<long long>(n_out) * r;
    z.p[2] = reinterpret_cast<float*>(cnt); z.n[2] = WL.ncnt;  // int zero = float +0 bits
    PhaseScope ps(st, PH_ZERO);
    zero_grads_kernel<<<148, 256, 0, st>>>(z);
    CUDA_TRY(cudaGetLastError());
  }
  if (dual) {
    // Q = s dY Bo with dBo = dY^T P, one read of dY
    DualProblem pr{};
    pr.X = dY; pr.ldx = n_out; pr.S[0] = Bo; pr.P = ctx; pr.ldp = rp; pr.p_cols = r; pr.out[0] = dBo;
    TRY(launch_dual(dual_spec_both(r), &pr, 1, T, n_out, r, D->scale, Q, rp, part, cnt, status, st, PH_O_LOWRANK));
  } else {
    // Q = s dY Bo
    GemmArgs a = new_args(status);
    TRY(map_k(&a.maps[0], dY, T, n_out, n_out, 128));
    TRY(map_mn(&a.maps[1], Bo, n_out, r, r));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, n_out);
    a.M = static_cast<int>(T); a.N = rp; a.bn = rp <= 64 ? 64 : 128;
    a.tiles_m = static_cast<int>((T + BM - 1) / BM); a.tiles_n = 1;
    TRY((launch_proj<1, 1>(a, T, n_out, rp, part, Q, D->scale, st, PH_O_LOWRANK)));
  }
  // dX = dY Wo + Q Ao  (bf16 out; Wo and Ao read MN-major)
  {
    GemmArgs a = new_args(status);
    const TileChoice tcx = pick_tiles(T, n_in, true);
    const int bn = tcx.bn;
    const int pair = (tcx.pair == 2 && bn % 128 == 0) ? 2 : 1;
    TRY(map_k(&a.maps[0], dY, T, n_out, n_out, 128));
    TRY(map_k(&a.maps[2], Q, T, rp, rp, 128));
    a.mn3d_b = n_in % 64 == 0;
    if (a.mn3d_b) {
      TRY(map_mn3(&a.maps[1], Wo, n_out, n_in, n_in, bn / pair / 64));
      TRY(map_mn3(&a.maps[3], Ao, r, n_in, n_in, bn / pair / 64));
    } else {
      TRY(map_mn(&a.maps[1], Wo, n_out, n_in, n_in));
      TRY(map_mn(&a.maps[3], Ao, r, n_in, n_in));
    }
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, n_out);
    set_seg(a, 1, 2, 0, 3, 0, -1, 0, rp);
    const int mt = pair == 2 ? pick_mt(T, pair, bn, n_in, mt_gain_bf16_stores()) : 1;
    a.M = static_cast<int>(T); a.N = n_in; a.bn = bn;
    a.tiles_m = static_cast<int>((T + BM * pair * mt - 1) / (BM * pair * mt)); a.tiles_n = (n_in + bn - 1) / bn;
    a.out[0] = dX; a.ld_out = n_in;
    if (mt == 2) TRY(set_epilogue_tma(a, 4, {dX}, T, n_in, n_in));
    a.stream_out = 1;
    set_band(a, 8 / mt);
    if (mt == 2) TRY((launch_gemm<0, 1, 1, EPI_BF16, 2, 0, 0, 2>(a, st, PH_O_DX)));
    else if (pair == 2) TRY((launch_gemm<0, 1, 1, EPI_BF16, 2>(a, st, PH_O_DX)));
    else TRY((launch_gemm<0, 1, 1, EPI_BF16>(a, st, PH_O_DX)));
  }
  const int rbn = r <= 64 ? 64 : 128;
  // dAo = Q^T X  ([r x n_in], written transposed from [n_in x r] tiles)
  {
    GemmArgs a = new_args(status);
    a.mn3d_a = n_in % 64 == 0;
    if (a.mn3d_a) TRY(map_mn3(&a.maps[0], X, T, n_in, n_in, 2));
    else TRY(map_mn(&a.maps[0], X, T, n_in, n_in));
    TRY(map_mn(&a.maps[1], Q, T, r, rp));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, static_cast<int>(T));
    a.M = n_in; a.N = r; a.bn = rbn; a.tiles_m = (n_in + BM - 1) / BM; a.tiles_n = 1;
    a.rng[0] = OutRange{dAo, 0, 1, n_in};
    a.nrng = 1;
    choose_splits(a, T);
    TRY((launch_gemm<1, 1, 1, EPI_ATOMIC>(a, st, PH_O_LOWRANK)));
  }
  // dBo = dY^T P  ([n_out x r])
  if (!dual) {
    GemmArgs a = new_args(status);
    a.mn3d_a = n_out % 64 == 0;
    if (a.mn3d_a) TRY(map_mn3(&a.maps[0], dY, T, n_out, n_out, 2));
    else TRY(map_mn(&a.maps[0], dY, T, n_out, n_out));
    TRY(map_mn(&a.maps[1], ctx, T, r, rp));
    set_seg(a, 0, 0, 0, 1, 0, -1, 0, static_cast<int>(T));
    a.M = n_out; a.N = r; a.bn = rbn; a.tiles_m = (n_out + BM - 1) / BM; a.tiles_n = 1;
    a.rng[0] = OutRange{dBo, 0, 0, r};
    a.nrng = 1;
    choose_splits(a, T);
    TRY((launch_gemm<1, 1, 1, EPI_ATOMIC>(a, st, PH_O_LOWRANK)));
  }
  return end_call(status, st);
}

// ------------------------------------------------------- RoPE
int lora_rope(int64_t T, int32_t hq, int32_t hk, int32_t hd, const int32_t* pos, int64_t n_pos, const float* cos_t,
              const float* sin_t, void* Q, void* K, int32_t backward, void* stream) {
  if (T < 1 || T >= (1LL << 31) || hq < 0 || hk < 0 || hq + hk < 1 || n_pos < 1)
    return fail(LORA_ERR_INVALID_ARG, "bad T / head counts / n_pos (%lld, %d, %d, %lld)", (long long)T, hq, hk,
                (long long)n_pos);
  if (hd < 16 || hd % 16) return fail(LORA_ERR_ALIGNMENT, "hd = %d must be a positive multiple of 16", hd);
  if (static_cast<long long>(hq + hk) * (hd / 16) > (1LL << 20)) return fail(LORA_ERR_UNSUPPORTED, "row too wide");
  if (backward != 0 && backward != 1) return fail(LORA_ERR_INVALID_ARG, "backward must be 0 or 1");
  TRY(check_ptrs({pos, cos_t, sin_t}));
  if (hq) TRY(check_ptrs({Q}));
  if (hk) TRY(check_ptrs({K}));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LibSyms ls;
  TRY(lib_syms(&ls));
  TRY(begin_call(ls.status, st));
  const int per_row = (hq + hk) * (hd / 16);
  const int threads = std::min(512, round_up(per_row, 32));
  const long long grid = std::min<long long>(T, static_cast<long long>(sm_count()) * (2048 / threads));
  {
    PhaseScope ps(st, PH_ROPE);
    rope_kernel<<<static_cast<unsigned>(grid), threads, 0, st>>>(
        static_cast<uint16_t*>(Q), static_cast<uint16_t*>(K), pos, cos_t, sin_t, T, hq, hk, hd, n_pos,
        backward ? -1.0f : 1.0f, ls.status);
    CUDA_TRY(cudaGetLastError());
  }
  return end_call(ls.status, st);
}

}  // extern "C"
