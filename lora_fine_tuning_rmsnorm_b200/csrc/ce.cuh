// Row kernels of the fused cross-entropy: combine the per-tile (max, sum of exponentials)
// partials of each token's logits into its logsumexp and loss, then reduce the losses.
//
// The loss is computed from the final hidden states in chunks and the logits never exist
// in full ("Unsloth — 用手写 Triton kernel 给 HF 微调换心脏", §2.3 step 6 and §4: the fused
// CE loss, the EMPTY_LOGITS placeholder).  Here the logits of a tile live only in tensor
// memory: the GEMM's epilogue leaves two (max, sum) pairs per token and tile (one per
// half of the tile's columns) and the label's logit; these kernels finish the reduction.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace lm {

constexpr int kCeThreads = 256;

// Thread per token: lse = M + log(sum_j s_j exp(m_j - M)), loss = lse - z_label (0 when the
// label is outside [0, V)); per-CTA sums of the losses and of the kept tokens go to blk.
static __global__ void __launch_bounds__(kCeThreads) ce_finalize_kernel(const float2* __restrict__ part, int nparts,
                                                                        const float* __restrict__ zlab,
                                                                        const int* __restrict__ labels, long long T,
                                                                        int V, float* __restrict__ loss_rows,
                                                                        float* __restrict__ lse_out,
                                                                        float2* __restrict__ blk) {
  constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  float loss = 0.f, kept = 0.f;
  if (t < T) {
    float M = -INFINITY;
    for (int j = 0; j < nparts; ++j) M = fmaxf(M, part[static_cast<long long>(j) * T + t].x);
    const float Ms = M * kLog2e;
    float S = 0.f;
    for (int j = 0; j < nparts; ++j) {
      const float2 q = part[static_cast<long long>(j) * T + t];
      if (q.y > 0.f) S += q.y * exp2f(fmaf(q.x, kLog2e, -Ms));
    }
    const float lse = M + log2f(S) * kLn2;
    lse_out[t] = lse;
    const int lab = labels[t];
    if (lab >= 0 && lab < V) {
      loss = lse - zlab[t];
      kept = 1.f;
    }
    loss_rows[t] = loss;
  }
  __shared__ float2 red[kCeThreads / 32];
  float a = loss, b = kept;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = make_float2(a, b);
  __syncthreads();
  if (threadIdx.x == 0) {
    float2 s = make_float2(0.f, 0.f);
    for (int w = 0; w < kCeThreads / 32; ++w) {
      s.x += red[w].x;
      s.y += red[w].y;
    }
    blk[blockIdx.x] = s;
  }
}

// One CTA: the per-CTA sums in a fixed order (deterministic) -> the reduced loss
// (mean over kept tokens, or sum; 0 with no kept token) and the kept count.
static __global__ void __launch_bounds__(kCeThreads) ce_reduce_kernel(const float2* __restrict__ blk, int nblk,
                                                                      int mean, float* __restrict__ loss,
                                                                      int* __restrict__ count) {
  __shared__ double red[kCeThreads][2];
  double a = 0.0, b = 0.0;
  for (int i = threadIdx.x; i < nblk; i += blockDim.x) {
    a += blk[i].x;
    b += blk[i].y;
  }
  red[threadIdx.x][0] = a;
  red[threadIdx.x][1] = b;
  __syncthreads();
  for (int w = kCeThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      red[threadIdx.x][0] += red[threadIdx.x + w][0];
      red[threadIdx.x][1] += red[threadIdx.x + w][1];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double n = red[0][1];
    const int kept = static_cast<int>(n + 0.5);
    *count = kept;
    *loss = static_cast<float>(mean ? (kept ? red[0][0] / n : 0.0) : red[0][0]);
  }
}

}  // namespace lm
