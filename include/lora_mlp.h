/*
 * lora_mlp.h — C ABI of the B200 (sm_100a) LoRA-augmented Llama MLP sub-block.
 *
 *   H   = RMSNorm(X; w, eps)                (cached rstd per row)
 *   G   = H Wg^T + s (H Ag^T) Bg^T           U = H Wu^T + s (H Au^T) Bu^T
 *   Act = silu(G) * U                        silu(z) = z * sigmoid(z)
 *   Y   = Act Wd^T + s (Act Ad^T) Bd^T
 * and the hand-derived backward giving dX and the six adapter gradients
 * (W, the norm weight and eps are frozen; no autograd).
 *
 * Sources of the definitions (web pages on Unsloth-style LoRA fine-tuning):
 *   RMSNorm with cached rstd, mean over the true column count, eps inside the sqrt:
 *     "Unsloth提速秘诀：Triton内核如何加速反向传播", §3.2 (FastRMSNorm).
 *   LoRA linear x W^T + (x A^T) B^T * (alpha / r), A [r x in], B [out x r], frozen W:
 *     "Unsloth 深度实战：Triton 内核 + 手写反向传播引擎…", §1.3 (LoRALayer, LinearWithLoRA).
 *   SwiGLU MLP with a hand-written LoRA_MLP autograd that saves only X, e, g, and the
 *   4-bit dequantise-then-matmul path (matmul_lora / fast_dequantize):
 *     "Unsloth — 用手写 Triton kernel 给 HF 微调换心脏", §2.3, §4, §7.
 *   4-bit NormalFloat storage with normal-quantile codes, dequantisation fused with the
 *   matmul: "Unsloth 深度实战…", §1.4; "Unsloth加速原理揭秘：为何训练快5-8倍？", §5.2.
 *
 * Conventions (all entry points):
 *   - Matrices are row-major.  bf16 tensors are passed as `const void*` to 16-bit
 *     elements (IEEE bfloat16 bit patterns); fp32 tensors as float*.
 *   - All pointers are DEVICE pointers (cudaMalloc'd or equivalent) unless stated,
 *     and must be 16-byte aligned.  The caller owns every buffer; the library
 *     allocates no device memory.  Inputs are never written.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call only enqueues work on that stream and returns; it does not
 *     synchronise (except with LORA_MLP_DEBUG=1 in the environment, where each call
 *     synchronises the stream and reports device-side errors).
 *   - Return value 0 (LORA_OK) on success or a negative LORA_ERR_* code; no C++
 *     exception or abort crosses the ABI.  lora_mlp_last_error() then gives a
 *     thread-local message.
 *   - Calls on different streams may run concurrently if their output, ctx and
 *     workspace buffers differ.
 */
#ifndef LORA_MLP_H
#define LORA_MLP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum lora_status {
  LORA_OK = 0,
  LORA_ERR_INVALID_ARG = -1, /* null pointer, non-positive or inconsistent size      */
  LORA_ERR_ALIGNMENT = -2,   /* pointer not 16-B aligned; d, f, r not multiples of 8 */
  LORA_ERR_UNSUPPORTED = -3, /* size outside the supported range (see each call)     */
  LORA_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed (message has text)  */
  LORA_ERR_TIMEOUT = -5      /* a bounded device-side wait gave up (reported by the   */
                             /* call itself in debug mode, else by lora_mlp_status)   */
};

enum lora_wfmt {
  LORA_WFMT_BF16 = 0,    /* frozen Wg, Wu, Wd given as bf16                              */
  LORA_WFMT_4BIT = 1,    /* frozen weights given as 4-bit blockwise codes (qblock = 64)  */
  LORA_WFMT_4BIT_DQ = 2  /* the same codes with double-quantised block constants: 8-bit  */
                         /* codes of the absmax values plus an fp32 scale per 256 of them */
};

/* Problem sizes.  T tokens, hidden d, intermediate f, LoRA rank r.
 * Limits: 1 <= T < 2^31; d, f multiples of 8 with 8 <= d <= 65536, 8 <= f;
 * r a multiple of 8 with 8 <= r <= 128.  scale = alpha / r (any finite value).
 * wfmt = LORA_WFMT_BF16 or LORA_WFMT_4BIT (then qblock must be 64 and d, f
 * multiples of 256; the same for LORA_WFMT_4BIT_DQ).  residual = 1 adds the decoder layer's residual connection
 * around the sub-block ("Unsloth加速原理揭秘", §3.1, the LoRA forward ending in a
 * residual add): Y = X + MLP(RMSNorm(X)) and dX gets + dY; 0 = the sub-block alone. */
typedef struct lora_mlp_dims {
  int64_t T;
  int32_t d, f, r;
  float eps;
  float scale;
  int32_t wfmt;
  int32_t qblock;
  int32_t residual;
} lora_mlp_dims;

/* Frozen base weights, nn.Linear layout (out x in):
 *   Wg, Wu [f x d], Wd [d x f]              bf16       (wfmt = LORA_WFMT_BF16)
 *   Qg, Qu [f*d/2], Qd [d*f/2] bytes        two 4-bit codes per byte, the even element of
 *                                           the row-major matrix in the low nibble
 *   absmax_g, absmax_u [f*d/64], absmax_d [d*f/64]  fp32 per-block absmax
 *   codebook [16] fp32                      code values (wfmt = LORA_WFMT_4BIT)
 * With 4-bit weights the GEMMs copy the codes and absmax into shared memory and
 * expand them to bf16 tiles in-kernel (w = bf16(codebook[idx] * absmax), fp32
 * product rounded once) right before the tensor-core MMA; no bf16 copy of W is
 * ever written to memory.
 * wfmt = LORA_WFMT_4BIT_DQ (double quantisation, "Unsloth 深度实战…", §1.4: the
 * quantisation constants are quantised too) replaces absmax_x by
 *   absmax8_x [n] uint8 and scale2_x [ceil(n / 256)] fp32, n = (block count) = out*in/64:
 *   absmax = fl32(fl32(scale2[i / 256] * k) / 255), k = absmax8[i]
 * (from lora_quantize_absmax8); each call expands them to fp32 in its workspace
 * (3 * n floats) before the GEMMs.
 * Unused members may be NULL.  (The absmax8 / scale2 members were appended after the
 * others; callers of the bf16 and plain 4-bit formats may leave them zero.) */
typedef struct lora_mlp_weights {
  const void* Wg;
  const void* Wu;
  const void* Wd;
  const uint8_t* Qg;
  const uint8_t* Qu;
  const uint8_t* Qd;
  const float* absmax_g;
  const float* absmax_u;
  const float* absmax_d;
  const float* codebook;
  const uint8_t* absmax8_g;
  const uint8_t* absmax8_u;
  const uint8_t* absmax8_d;
  const float* scale2_g;
  const float* scale2_u;
  const float* scale2_d;
} lora_mlp_weights;

/* LoRA adapters, bf16: Ag, Au [r x d]; Bg, Bu [f x r]; Ad [r x f]; Bd [d x r]. */
typedef struct lora_mlp_adapters {
  const void* Ag;
  const void* Bg;
  const void* Au;
  const void* Bu;
  const void* Ad;
  const void* Bd;
} lora_mlp_adapters;

/* Adapter gradients, fp32, same shapes as the adapters.  OVERWRITTEN by the
 * backward (not accumulated).  Sums over T are formed with fp32 atomics, so the
 * last bits may differ between runs.
 * dw [d] fp32: gradient of the norm weight, dw_j = sum_t dH_tj x_tj rstd_t, for a
 * trainable-norm variant ("Unsloth提速秘诀：Triton内核如何加速反向传播", §3.2, the norm
 * kernel's weight operand); NULL = the norm weight is frozen (LoRA) and dw is not
 * computed.  Overwritten, fp32 atomics as above. */
typedef struct lora_mlp_grads {
  float* dAg;
  float* dBg;
  float* dAu;
  float* dBu;
  float* dAd;
  float* dBd;
  float* dw;
} lora_mlp_grads;

/* Byte offsets of the saved-activation context (one caller-owned device buffer,
 * written by lora_mlp_fwd, read by lora_mlp_bwd).  rp = r rounded up to 16.
 *   rstd [T] fp32;  H [T x d] bf16 (normalised input);  G, U, Act [T x f] bf16;
 *   P [T x 2rp] bf16 = s*(H Ag^T | 0 | H Au^T | 0), columns [0,r) and [rp, rp+r);
 *   Pd [T x rp] bf16 = s*(Act Ad^T | 0).
 * Offsets are multiples of 256. */
typedef struct lora_mlp_ctx_layout {
  size_t rstd, H, G, U, Act, P, Pd;
  size_t total;
  int32_t rp;
} lora_mlp_ctx_layout;

/* Saved-context size and layout for `dims`.  Returns LORA_ERR_* on bad dims. */
int lora_mlp_ctx_layout_get(const lora_mlp_dims* dims, lora_mlp_ctx_layout* out);

/* Workspace bytes needed by lora_mlp_fwd / lora_mlp_bwd (one buffer serves both;
 * it holds the backward's dH fp32 [T x d], dG, dU bf16 [T x f], the rank-r
 * projections and, at offset 0, a device status word).  Contents need not be
 * initialised. */
int lora_mlp_workspace_bytes(const lora_mlp_dims* dims, size_t* bytes);

/* Forward.  X [T x d] bf16, rms_w [d] bf16 -> Y [T x d] bf16, and the saved context
 * `ctx` (lora_mlp_ctx_layout_get().total bytes).  `workspace` as above.
 * Errors: INVALID_ARG (null/inconsistent), ALIGNMENT, UNSUPPORTED, CUDA. */
int lora_mlp_fwd(const lora_mlp_dims* dims, const void* X, const void* rms_w,
                 const lora_mlp_weights* W, const lora_mlp_adapters* A, void* Y, void* ctx,
                 void* workspace, void* stream);

/* Backward.  dY [T x d] bf16 plus the forward's X, rms_w, weights, adapters and ctx
 * -> dX [T x d] bf16 and the six fp32 adapter gradients (overwritten).
 * The gradient of <dY, Y>:
 *   dAct = dY Wd + s (dY Bd) Ad;  dG = dAct * U * silu'(G);  dU = dAct * silu(G);
 *   dH = dG Wg + dU Wu + s ((dG Bg) Ag + (dU Bu) Au);  dX = RMSNorm'(dH);
 *   dBg = s dG^T (H Ag^T), dAg = s (dG Bg)^T H, and likewise for u and d. */
int lora_mlp_bwd(const lora_mlp_dims* dims, const void* dY, const void* X, const void* rms_w,
                 const lora_mlp_weights* W, const lora_mlp_adapters* A, const void* ctx,
                 void* dX, const lora_mlp_grads* grads, void* workspace, void* stream);

/* RMSNorm forward alone: H = X * rstd * w, rstd = 1/sqrt(mean(X^2) + eps) in fp32.
 * X, H [T x d] bf16, w [d] bf16, rstd [T] fp32.  d a multiple of 8, <= 65536. */
int lora_rmsnorm_fwd(int64_t T, int32_t d, float eps, const void* X, const void* w, void* H,
                     float* rstd, void* stream);

/* RMSNorm backward alone (weight frozen): dX = rstd * (g - xhat * mean(g * xhat)),
 * g = dH * w, xhat = X * rstd.  dH [T x d] fp32, X [T x d] bf16, w [d] bf16,
 * rstd [T] fp32 (from the forward) -> dX [T x d] bf16. */
int lora_rmsnorm_bwd(int64_t T, int32_t d, const float* dH, const void* X, const void* w,
                     const float* rstd, void* dX, void* stream);

/* ---------------------------------------------------------------------------
 * LoRA on the attention Q/K/V projections (the layer's attention half up to
 * RoPE: "Unsloth — 用手写 Triton kernel 给 HF 微调换心脏", §2.3, RMSNorm kernel then
 * the Q/K/V projection with the LoRA forward written by hand; §7, LoRA_QKV /
 * apply_lora_qkv):
 *   H = RMSNorm(X) (cached rstd);  Q = H Wq^T + s (H Aq^T) Bq^T;  K, V likewise.
 * Backward from dQ, dK, dV: dX and the six adapter gradients (frozen W and norm
 * weight).  Same conventions as the MLP calls (asynchronous, caller-owned buffers,
 * 16-byte aligned pointers, status codes). */
typedef struct lora_qkv_dims {
  int64_t T;            /* tokens, 1 <= T < 2^31                                    */
  int32_t d;            /* hidden size, multiple of 8, 8 <= d <= 65536              */
  int32_t nq, nkv;      /* Q and K/V output features (grouped-query: nkv < nq),    */
                        /* multiples of 8                                          */
  int32_t r;            /* rank, multiple of 8, 8 <= r <= 128                       */
  float eps;
  float scale;          /* s = alpha / r                                            */
} lora_qkv_dims;

/* Wq [nq x d], Wk, Wv [nkv x d] bf16 row-major. */
typedef struct lora_qkv_weights {
  const void* Wq;
  const void* Wk;
  const void* Wv;
} lora_qkv_weights;

/* Aq, Ak, Av [r x d]; Bq [nq x r]; Bk, Bv [nkv x r]; bf16 row-major. */
typedef struct lora_qkv_adapters {
  const void* Aq;
  const void* Bq;
  const void* Ak;
  const void* Bk;
  const void* Av;
  const void* Bv;
} lora_qkv_adapters;

/* fp32, shapes of the adapters, OVERWRITTEN (fp32 atomics over T). */
typedef struct lora_qkv_grads {
  float* dAq;
  float* dBq;
  float* dAk;
  float* dBk;
  float* dAv;
  float* dBv;
} lora_qkv_grads;

/* Saved context: rstd [T] fp32; H [T x d] bf16; P [T x 3rp] bf16 =
 * s (H Aq^T | H Ak^T | H Av^T), each block rp = r rounded up to 16 wide (zero padded).
 * Offsets are multiples of 256. */
typedef struct lora_qkv_ctx_layout {
  size_t rstd, H, P;
  size_t total;
  int32_t rp;
} lora_qkv_ctx_layout;

int lora_qkv_ctx_layout_get(const lora_qkv_dims* dims, lora_qkv_ctx_layout* out);
int lora_qkv_workspace_bytes(const lora_qkv_dims* dims, size_t* bytes);

/* Forward: Q [T x nq], K, V [T x nkv] bf16; writes the context. */
int lora_qkv_fwd(const lora_qkv_dims* dims, const void* X, const void* rms_w, const lora_qkv_weights* W,
                 const lora_qkv_adapters* A, void* Q, void* K, void* V, void* ctx, void* workspace,
                 void* stream);

/* Backward: dQ [T x nq], dK, dV [T x nkv] bf16 in; dX [T x d] bf16 and the grads out.
 * Needs the context of the forward of the same X. */
int lora_qkv_bwd(const lora_qkv_dims* dims, const void* dQ, const void* dK, const void* dV, const void* X,
                 const void* rms_w, const lora_qkv_weights* W, const lora_qkv_adapters* A, const void* ctx,
                 void* dX, const lora_qkv_grads* grads, void* workspace, void* stream);

/* ---------------------------------------------------------------------------
 * LoRA on the attention output projection o_proj: a LoRA linear with no norm in front
 * (o_proj is adapted in every LoRA configuration of the pages: target_modules q_proj,
 * k_proj, v_proj, o_proj, gate_proj, up_proj, down_proj — "【编译】结合 Unsloth 与 🤗 TRL",
 * §三.2; the adapter is the LoRALayer linear of "Unsloth 深度实战…", §1.3):
 *   P = s X Ao^T;  Y = X Wo^T + P Bo^T
 * X [T x n_in] (the attention output, heads x head dim), Wo [n_out x n_in], Ao [r x n_in],
 * Bo [n_out x r], Y [T x n_out], all bf16 row-major; the context holds P [T x rp] bf16
 * (rp = r rounded up to 16, zero padded).  Backward from dY [T x n_out] (frozen Wo):
 *   Q = s dY Bo;  dX = dY Wo + Q Ao (bf16);  dAo = Q^T X, dBo = dY^T P (fp32 [r x n_in],
 *   [n_out x r], OVERWRITTEN, fp32 atomics over T).
 * Limits: 1 <= T < 2^31; n_in, n_out >= 8 and r multiples of 8, r <= 128.  Same conventions
 * as the MLP calls (asynchronous, caller-owned 16-byte aligned device buffers). */
typedef struct lora_o_dims {
  int64_t T;
  int32_t n_in, n_out, r;
  float scale;          /* s = alpha / r */
} lora_o_dims;

int lora_o_ctx_bytes(const lora_o_dims* dims, size_t* bytes);
int lora_o_workspace_bytes(const lora_o_dims* dims, size_t* bytes);
int lora_o_fwd(const lora_o_dims* dims, const void* X, const void* Wo, const void* Ao, const void* Bo, void* Y,
               void* ctx, void* workspace, void* stream);
int lora_o_bwd(const lora_o_dims* dims, const void* dY, const void* X, const void* Wo, const void* Ao,
               const void* Bo, const void* ctx, void* dX, float* dAo, float* dBo, void* workspace, void* stream);

/* ---------------------------------------------------------------------------
 * Rotary position embedding of the query and key heads, in place ("Unsloth — 用手写
 * Triton kernel 给 HF 微调换心脏", §2.3: the RoPE kernel after the Q/K/V projections,
 * writing in place; §4: the backward is the same kernel with the sine negated;
 * "Unsloth加速原理揭秘", §2.2: q and k rotated at their positions by one kernel).
 * Q [T x hq*hd], K [T x hk*hd] bf16 row-major (heads of hd contiguous features, as the
 * Q/K/V projections write them).  Dimension i of a head is paired with i + hd/2:
 *   q_i <- q_i c - q_{i+hd/2} s,   q_{i+hd/2} <- q_{i+hd/2} c + q_i s,
 *   c = cos[pos[t]][i], s = sin[pos[t]][i] (fp32 tables [n_pos x hd/2], row-major),
 * computed in fp32 and rounded once to bf16.  backward = 1 applies the inverse rotation
 * (s negated): the gradient of the forward, in place on dQ, dK.  pos [T] int32 position
 * ids (packed sequences restart them).  hd a multiple of 16; hq or hk may be 0 (that
 * pointer may then be NULL).  A position outside [0, n_pos) leaves its row unchanged and
 * is reported as LORA_ERR_INVALID_ARG (by the call in debug mode, else by
 * lora_mlp_status(NULL, ...)). */
int lora_rope(int64_t T, int32_t hq, int32_t hk, int32_t hd, const int32_t* pos, int64_t n_pos, const float* cos_t,
              const float* sin_t, void* Q, void* K, int32_t backward, void* stream);

/* ---------------------------------------------------------------------------
 * Fused cross-entropy of the language-model head ("Unsloth — 用手写 Triton kernel 给 HF
 * 微调换心脏", §2.3 step 6 and §4: the loss is computed from the final hidden states in
 * chunks and the logits tensor never exists in full; §7, Fast_CrossEntropyLoss):
 *   z = H W^T (never stored), lse_t = log sum_v exp(z_tv),
 *   loss_t = lse_t - z_{t, labels[t]}, or 0 when labels[t] is outside [0, V) (the ignore
 *   index -100 included: the token is left out);
 *   loss = mean of loss_t over the kept tokens (LORA_CE_MEAN; 0 if none) or their sum.
 * Backward for the upstream gradient dloss of the reduced loss (W frozen):
 *   dH_t = dloss' sum_v (softmax(z_t)_v - [v = labels[t]]) W_v,  dloss' = dloss / n_valid
 *   (mean) or dloss (sum); dH_t = 0 for tokens left out.
 * H [T x d] bf16 (final normalised hidden states), W [V x d] bf16 (the LM head), labels
 * [T] int32 (already shifted by the caller), all row-major device memory.  Forward writes
 * loss_rows [T] fp32, lse [T] fp32 (saved for the backward), *loss (fp32) and *n_valid
 * (int32, the kept count); the backward reads lse and n_valid from the forward and writes
 * dH [T x d] fp32 (OVERWRITTEN).  The backward recomputes the logits of vocab_chunk
 * columns at a time and keeps only that chunk's dZ = dloss' (softmax - onehot) in the
 * workspace (bf16 [T x vocab_chunk]).  d, V multiples of 8; vocab_chunk a multiple of
 * 256, 0 = 32768.  loss and n_valid need 4-byte alignment, the rest 16.  The per-token
 * sums are reduced in a fixed order (the loss is deterministic). */
#define LORA_CE_MEAN 0
#define LORA_CE_SUM 1
typedef struct lora_ce_dims {
  int64_t T;
  int32_t d;
  int32_t V;
  int32_t vocab_chunk;
  int32_t reduction;  /* LORA_CE_MEAN or LORA_CE_SUM */
} lora_ce_dims;

int lora_ce_workspace_bytes(const lora_ce_dims* dims, size_t* bytes);
int lora_ce_fwd(const lora_ce_dims* dims, const void* H, const void* W, const int32_t* labels, float* loss_rows,
                float* lse, float* loss, int32_t* n_valid, void* workspace, void* stream);
int lora_ce_bwd(const lora_ce_dims* dims, const void* H, const void* W, const int32_t* labels, const float* lse,
                const int32_t* n_valid, float dloss, float* dH, void* workspace, void* stream);

/* Adapter folded into its frozen weight for export ("Unsloth提速秘诀…", §3.1, "LoRA
 * Update + Weight Merge"; "Unsloth 深度实战", §5.1, the merged 16-bit save):
 *   Wm[o][i] = bf16( W[o][i] + scale * sum_{k<r} B[o][k] A[k][i] )
 * with the sum in fp32 over k = 0..r-1, then one fp32 fma (scale * sum + W), then
 * one rounding to bf16 (RN).
 * W, Wm [rows x cols] bf16 row-major (Wm may equal W: in place); A [r x cols], B
 * [rows x r] bf16 row-major.  cols a multiple of 8, 1 <= r <= 256, pointers 16-byte
 * aligned (B: 2-byte).  Asynchronous on `stream`; nothing is allocated. */
int lora_merge_weights(int64_t rows, int64_t cols, int32_t r, float scale, const void* W, const void* A,
                       const void* B, void* Wm, void* stream);

/* 4-bit blockwise quantisation of a bf16 matrix (flattened row-major, numel a
 * multiple of block = 64): per block absmax = max|w| (fp32); code index
 * idx = #{ i in 0..14 : w > absmax * m_i }, m_i = fl32((c_i + c_{i+1}) / 2), decided
 * exactly (nearest code, ties to the lower index; all-zero block -> 0).  codebook16
 * [16] fp32 ascending.  codes [numel/2] bytes (even element in the low nibble),
 * absmax [numel/64] fp32. */
int lora_quantize_4bit(const void* W, int64_t numel, int32_t block, const float* codebook16,
                       uint8_t* codes, float* absmax, void* stream);

/* Double quantisation of the 4-bit block constants ("Unsloth 深度实战…", §1.4: the
 * quantisation constants are themselves quantised; the pages give no format, so this
 * is a reading): absmax [n] fp32 (>= 0, as lora_quantize_4bit writes it) in blocks of
 * block2 = 256 consecutive values (the last may be shorter); scale2[b] = the block's
 * largest value; codes8[i] = #{ j in 1..255 : 510 absmax[i] > (2j - 1) scale2[b] },
 * i.e. the nearest of the levels scale2 k / 255, ties to the lower one, decided exactly
 * (fp64 products); an all-zero block gives scale2 0 and codes 0.  codes8 [n] bytes,
 * scale2 [ceil(n / 256)] fp32.  Asynchronous; nothing is allocated. */
int lora_quantize_absmax8(const float* absmax, int64_t n, int32_t block2, uint8_t* codes8, float* scale2,
                          void* stream);

/* Plain tensor-core GEMM (the core the fused path is built on), fp32 out:
 *   C[M x N] = A' B'^T,  A' [M x K] = A (a_mn = 0, A row-major [M x K]) or A^T
 *   (a_mn = 1, A row-major [K x M]);  B' [N x K] = B (b_mn = 0, B [N x K]) or B^T
 *   (b_mn = 1, B [K x N]).  M, N, K must be multiples of 8.
 * flags: LORA_GEMM_CTA_PAIR runs 256-row tiles on pairs of SMs (tcgen05
 * cta_group::2; needs a_mn = 0), otherwise one 128-row tile per SM. */
#define LORA_GEMM_CTA_PAIR 1
/* Test of the failure path only: the kernel's copy warp issues no loads and arms no
 * barrier, so the MMA's first bounded wait runs out after LORA_MLP_WAIT_LIMIT_MS; the
 * kernel then records the timeout, frees its tensor memory and returns (C is left
 * unwritten).  Not combinable with LORA_GEMM_CTA_PAIR. */
#define LORA_GEMM_TEST_NO_LOADS 2
int lora_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, int32_t a_mn, const void* B,
                   int32_t b_mn, float* C, int32_t flags, void* stream);

/* Bounded-wait status of the most recent call that used `workspace` (any workspace
 * of this library: its status word sits at offset 0), or, with workspace = NULL, of
 * the most recent lora_gemm_bf16 / lora_lowrank_proj_noalloc / lora_rope call in the
 * current CUDA context.  Every device wait in the kernels has a time limit
 * (LORA_MLP_WAIT_LIMIT_MS in the environment, default 5000 ms); a wait that runs out
 * makes its kernel record a code in the status word, stop its other roles, wait for
 * its own copies and tensor-core operations in flight, free its tensor memory and
 * return, leaving the outputs incomplete.  Each call clears its status word when it
 * is enqueued, so check after every call whose result matters.
 * Synchronises `stream`, then returns LORA_OK, or LORA_ERR_TIMEOUT with the code in
 * *code (may be NULL) and in lora_mlp_last_error() (LORA_ERR_INVALID_ARG for a device-side
 * index input out of range, such as a RoPE position).  With LORA_MLP_DEBUG=1 every call
 * does this check itself before it returns. */
int lora_mlp_status(const void* workspace, int32_t* code, void* stream);

/* Allocation-free rank-r projection.  The pages have no counterpart to this entry
 * point; it exists for callers that cannot allocate device memory themselves, such
 * as a plugin inside a host framework that owns the device memory and hands it only
 * its input and output buffers, so it has nowhere to put a workspace.
 *   P[T x rp] bf16 = scale * X A^T,  X [T x K] bf16, A [r x K] bf16, rp = r rounded up
 *   to 16 (columns [r, rp) are written as 0).  Same result as the projection the
 *   forward stores in the saved context (P there holds scale * H Ag^T at columns
 *   [0, rp)).  K, r multiples of 8, 8 <= r <= 128.
 * The K-split fp32 partial sums go to a fixed 16 MiB array inside the library
 * (4 Mi floats, held on every GPU that loads the library until the process exits);
 * sizes with splits * T * rp above that are rejected with LORA_ERR_UNSUPPORTED.
 * No cudaMalloc/cudaFree or other allocation is made.  The array's device address
 * belongs to one CUDA context, so the first call in each context (the one current
 * on the calling thread: the device's primary context, or a context the caller
 * created) looks it up with cudaGetSymbolAddress and caches it under that context's
 * unique id; make that first call before any stream capture.  The bounded-wait
 * status of the call is kept in a library word of the same context (read it with
 * lora_mlp_status(NULL, ...); debug mode reports it from the call itself).
 * All calls share the array: calls that can overlap on the GPU (different streams,
 * or several host threads) race on it and must be serialised by the caller.  Every
 * partial-sum element is rewritten by each call, so nothing has to be cleared. */
int lora_lowrank_proj_noalloc(int64_t T, int32_t K, int32_t r, float scale, const void* X, const void* A,
                              void* P, void* stream);

/* Per-phase timing.  With timing enabled, every kernel launch of the calls above
 * is bracketed by CUDA events on the caller's stream.  lora_mlp_timing_collect()
 * synchronises those events and returns, per phase id, the summed milliseconds and
 * the number of launches since the previous collect (arrays of LORA_NUM_PHASES). */
#define LORA_NUM_PHASES 28
int lora_mlp_timing_enable(int32_t on);
int lora_mlp_timing_collect(double* ms, int64_t* launches);
const char* lora_mlp_phase_name(int32_t phase);

/* Thread-local description of the last error (never NULL). */
const char* lora_mlp_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* LORA_MLP_H */
