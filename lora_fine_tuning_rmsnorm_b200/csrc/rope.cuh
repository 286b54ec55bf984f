// Rotary position embedding (RoPE) of the query and key heads, in place.
//
// Each decoder layer rotates Q and K right after their projections, writing in place,
// and the backward is the same kernel with the sine negated ("Unsloth — 用手写 Triton
// kernel 给 HF 微调换心脏", §2.3 and §4); the rotation of q and of k at their positions
// share one kernel that looks the cos / sin tables up by position ("Unsloth加速原理揭秘",
// §2.2).  Pairing: dimension i of a head with dimension i + hd/2 (rotate-half):
//     y_i = x_i c - x_{i+hd/2} s,   y_{i+hd/2} = x_{i+hd/2} c + x_i s.
//
// HBM-bound: every element is read and written once (bf16), the tables (fp32, a few
// hundred KB) stay in L2.  A thread takes 8 pairs of one head: two 16-byte vectors in
// and out, 8 cos and 8 sin values; a warp covers 4 heads of hd = 128 contiguously.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace lm {

// One work item: 8 pairs of one head of one token (see above).
struct RopeItem {
  uint4* pa;
  uint4* pb;
  uint4 va, vb;
  float4 c0, c1, s0, s1;
};
__device__ __forceinline__ void rope_load(RopeItem& it, uint16_t* head, int i0, int half, const float* cosT,
                                          const float* sinT, long long p) {
  it.pa = reinterpret_cast<uint4*>(head + i0);
  it.pb = reinterpret_cast<uint4*>(head + i0 + half);
  it.va = *it.pa;
  it.vb = *it.pb;
  const float4* pc = reinterpret_cast<const float4*>(cosT + p * half + i0);
  const float4* ps = reinterpret_cast<const float4*>(sinT + p * half + i0);
  it.c0 = __ldg(pc);
  it.c1 = __ldg(pc + 1);
  it.s0 = __ldg(ps);
  it.s1 = __ldg(ps + 1);
}
__device__ __forceinline__ void rope_apply(const RopeItem& it, float sgn) {
  const float c[8] = {it.c0.x, it.c0.y, it.c0.z, it.c0.w, it.c1.x, it.c1.y, it.c1.z, it.c1.w};
  const float sn[8] = {sgn * it.s0.x, sgn * it.s0.y, sgn * it.s0.z, sgn * it.s0.w,
                       sgn * it.s1.x, sgn * it.s1.y, sgn * it.s1.z, sgn * it.s1.w};
  const uint32_t wa[4] = {it.va.x, it.va.y, it.va.z, it.va.w}, wb[4] = {it.vb.x, it.vb.y, it.vb.z, it.vb.w};
  uint32_t oa[4], ob[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float a0 = bf16lo(wa[k]), a1 = bf16hi(wa[k]), b0 = bf16lo(wb[k]), b1 = bf16hi(wb[k]);
    const float cc0 = c[2 * k], cc1 = c[2 * k + 1], s0k = sn[2 * k], s1k = sn[2 * k + 1];
    oa[k] = pack_bf16x2(fmaf(a0, cc0, -b0 * s0k), fmaf(a1, cc1, -b1 * s1k));
    ob[k] = pack_bf16x2(fmaf(b0, cc0, a0 * s0k), fmaf(b1, cc1, a1 * s1k));
  }
  *it.pa = make_uint4(oa[0], oa[1], oa[2], oa[3]);
  *it.pb = make_uint4(ob[0], ob[1], ob[2], ob[3]);
}

// blockDim.x threads per token row; a CTA walks rows blockIdx.x, + gridDim.x, ...
// (one row's state per thread keeps six 320-thread CTAs resident per SM for the 8B heads).
// sgn = +1 forward, -1 backward (the inverse rotation).
static __global__ void __launch_bounds__(512) rope_kernel(uint16_t* __restrict__ Q, uint16_t* __restrict__ K,
                                                          const int32_t* __restrict__ pos,
                                                          const float* __restrict__ cosT,
                                                          const float* __restrict__ sinT, long long T, int hq,
                                                          int hk, int hd, long long n_pos, float sgn, int* status) {
  const int per_head = hd >> 4;  // work items (8 pairs each) per head
  const int per_row = (hq + hk) * per_head;
  const int half = hd >> 1;
  for (long long t = blockIdx.x; t < T; t += gridDim.x) {
    const long long p = __ldg(pos + t);
    if (p < 0 || p >= n_pos) {
      if (threadIdx.x == 0 && status) atomicCAS(status, 0, kDevBadIndex);
      continue;  // the row is left as it was
    }
    for (int j = threadIdx.x; j < per_row; j += blockDim.x) {
      const int h = j / per_head, i0 = (j - h * per_head) * 8;
      RopeItem it;
      rope_load(it, h < hq ? Q + (t * hq + h) * hd : K + (t * hk + (h - hq)) * hd, i0, half, cosT, sinT, p);
      rope_apply(it, sgn);
    }
  }
}

}  // namespace lm
