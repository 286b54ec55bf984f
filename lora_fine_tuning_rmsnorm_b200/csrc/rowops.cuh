// Row kernels bounded by HBM bandwidth: RMSNorm forward/backward, the 4-bit
// blockwise quantiser, and zero-fill of the fp32 gradient outputs.
//
// RMSNorm ("Unsloth提速秘诀：Triton内核如何加速反向传播", §3.2): one CTA per row,
// 16-byte vector loads held in registers (the row is read once), fp32 sums,
// rstd cached for the backward, the normalised row rounded once to bf16.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace lm {

constexpr int kRowThreads = 128;

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nw = blockDim.x / 32;
  __syncthreads();  // protect `red` from a previous use
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < nw; ++i) s += red[i];
  return s;
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// VPT = 16-byte vectors (8 bf16) per thread; blockDim.x * VPT * 8 >= d; MAXT bounds
// blockDim.x (the common 128-thread launch gets the registers to hold its row unspilled).
template <int VPT, int MAXT>
static __global__ void __launch_bounds__(MAXT) rmsnorm_fwd_kernel(const uint16_t* __restrict__ X,
                                                           const uint16_t* __restrict__ w,
                                                           uint16_t* __restrict__ H,
                                                           float* __restrict__ rstd, int d,
                                                           float eps) {
  __shared__ float red[32];
  const long long row = blockIdx.x;
  const int nvec = d / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(X + row * d);
  uint4 xv[VPT];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int v = threadIdx.x + i * blockDim.x;
    xv[i] = v < nvec ? __ldcs(xr + v) : make_uint4(0, 0, 0, 0);
    float f[8];
    unpack8(xv[i], f);
#pragma unroll
    for (int j = 0; j < 8; ++j) ss = fmaf(f[j], f[j], ss);
  }
  ss = block_sum(ss, red);
  const float rs = rsqrtf(ss / static_cast<float>(d) + eps);
  if (threadIdx.x == 0) rstd[row] = rs;
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  uint4* hr = reinterpret_cast<uint4*>(H + row * d);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int v = threadIdx.x + i * blockDim.x;
    if (v >= nvec) continue;
    float f[8], g[8];
    unpack8(xv[i], f);
    unpack8(__ldg(wr + v), g);
    uint4 o;
    o.x = pack_bf16x2(f[0] * rs * g[0], f[1] * rs * g[1]);
    o.y = pack_bf16x2(f[2] * rs * g[2], f[3] * rs * g[3]);
    o.z = pack_bf16x2(f[4] * rs * g[4], f[5] * rs * g[5]);
    o.w = pack_bf16x2(f[6] * rs * g[6], f[7] * rs * g[7]);
    hr[v] = o;
  }
}

// dX = rstd * (g - xhat * mean(g * xhat)), g = dH * w, xhat = x * rstd.
template <int VPT, int MAXT>
static __global__ void __launch_bounds__(MAXT) rmsnorm_bwd_kernel(const float* __restrict__ dH,
                                                           const uint16_t* __restrict__ X,
                                                           const uint16_t* __restrict__ w,
                                                           const float* __restrict__ rstd,
                                                           const uint16_t* __restrict__ dY,
                                                           uint16_t* __restrict__ dX, int d) {
  __shared__ float red[32];
  const long long row = blockIdx.x;
  const int nvec = d / 8;
  const float rs = rstd[row];
  const float4* hr = reinterpret_cast<const float4*>(dH + row * d);
  const uint4* xr = reinterpret_cast<const uint4*>(X + row * d);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  float g[VPT][8], xh[VPT][8];
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int v = threadIdx.x + i * blockDim.x;
    if (v < nvec) {
      const float4 h0 = __ldcs(hr + 2 * v), h1 = __ldcs(hr + 2 * v + 1);
      float xf[8], wf[8];
      unpack8(__ldcs(xr + v), xf);
      unpack8(__ldg(wr + v), wf);
      const float hh[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        g[i][j] = hh[j] * wf[j];
        xh[i][j] = xf[j] * rs;
        dot = fmaf(g[i][j], xh[i][j], dot);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) g[i][j] = xh[i][j] = 0.f;
    }
  }
  dot = block_sum(dot, red);
  const float c = dot / static_cast<float>(d);
  uint4* dr = reinterpret_cast<uint4*>(dX + row * d);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int v = threadIdx.x + i * blockDim.x;
    if (v >= nvec) continue;
    float o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = rs * (g[i][j] - xh[i][j] * c);
    if (dY) {  // residual connection: the sub-block's input gradient also gets dY
      float yf[8];
      unpack8(__ldcs(reinterpret_cast<const uint4*>(dY + row * d) + v), yf);
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] += yf[j];
    }
    uint4 ov;
    ov.x = pack_bf16x2(o[0], o[1]);
    ov.y = pack_bf16x2(o[2], o[3]);
    ov.z = pack_bf16x2(o[4], o[5]);
    ov.w = pack_bf16x2(o[6], o[7]);
    dr[v] = ov;
  }
}

// One warp per 64-element block: two elements per lane, absmax by warp max,
// code index = number of midpoints the value exceeds (decided exactly: the sign of
// a fused multiply-add w - absmax * m_i is the sign of the exact difference).
static __global__ void quantize4_kernel(const uint16_t* __restrict__ W, long long nblocks,
                                 const float* __restrict__ code, uint8_t* __restrict__ codes,
                                 float* __restrict__ absmax) {
  __shared__ float mid[15];
  if (threadIdx.x < 15) mid[threadIdx.x] = (code[threadIdx.x] + code[threadIdx.x + 1]) * 0.5f;
  __syncthreads();
  const int lane = threadIdx.x % 32;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long b = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
       b < nblocks; b += warps) {
    const uint32_t pair = reinterpret_cast<const uint32_t*>(W + b * 64)[lane];
    const float w0 = bf16lo(pair), w1 = bf16hi(pair);
    float am = fmaxf(fabsf(w0), fabsf(w1));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    int i0 = 0, i1 = 0;
#pragma unroll
    for (int i = 0; i < 15; ++i) {
      i0 += fmaf(-am, mid[i], w0) > 0.f;
      i1 += fmaf(-am, mid[i], w1) > 0.f;
    }
    codes[b * 32 + lane] = static_cast<uint8_t>(i0 | (i1 << 4));
    if (lane == 0) absmax[b] = am;
  }
}

// out[i] = bf16(scale * sum_s part[s * stride + i]) for the K-split partial sums
// of a rank-r projection (deterministic: fixed summation order).
static __global__ void splitk_finalize_kernel(const float* __restrict__ part, int splits, long long stride,
                                       long long n, float scale, uint16_t* __restrict__ out) {
  const long long i4 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i4 >= n) return;
  float4 acc = *reinterpret_cast<const float4*>(part + i4);
  for (int s = 1; s < splits; ++s) {
    const float4 v = *reinterpret_cast<const float4*>(part + s * stride + i4);
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  uint2 o;
  o.x = pack_bf16x2(acc.x * scale, acc.y * scale);
  o.y = pack_bf16x2(acc.z * scale, acc.w * scale);
  *reinterpret_cast<uint2*>(out + i4) = o;
}

// The same sum of K-split partials, written into columns [0, cols) of an output with
// row stride ld_out (a column block of a wider matrix).  cols is a multiple of 4.
static __global__ void splitk_finalize_strided_kernel(const float* __restrict__ part, int splits, long long stride,
                                               long long rows, int cols, long long ld_out, float scale,
                                               uint16_t* __restrict__ out) {
  const long long i4 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i4 >= rows * cols) return;
  float4 acc = *reinterpret_cast<const float4*>(part + i4);
  for (int s = 1; s < splits; ++s) {
    const float4 v = *reinterpret_cast<const float4*>(part + s * stride + i4);
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  const long long row = i4 / cols, col = i4 - row * cols;
  uint2 o;
  o.x = pack_bf16x2(acc.x * scale, acc.y * scale);
  o.y = pack_bf16x2(acc.z * scale, acc.w * scale);
  *reinterpret_cast<uint2*>(out + row * ld_out + col) = o;
}

constexpr int kZeroMax = 8;
struct ZeroList {
  float* p[kZeroMax];  // NULL entries (n = 0) are skipped
  long long n[kZeroMax];
};
static __global__ void zero_grads_kernel(ZeroList z) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (int k = 0; k < kZeroMax; ++k)
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < z.n[k]; i += stride)
      z.p[k][i] = 0.f;
}

// Norm-weight gradient of H = X * rstd * w: dw_j += sum over a chunk of `rows` rows of
// dH_tj * x_tj * rstd_t, added to dw (zeroed by the caller) with fp32 atomics.  A thread
// owns 4 consecutive columns, so every row of dH / X is read coalesced.
static __global__ void __launch_bounds__(256) norm_weight_grad_kernel(const float* __restrict__ dH,
                                                               const uint16_t* __restrict__ X,
                                                               const float* __restrict__ rstd,
                                                               float* __restrict__ dw, long long T, int d,
                                                               int rows) {
  const long long c = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (c >= d) return;
  const long long t0 = static_cast<long long>(blockIdx.y) * rows;
  const long long t1 = t0 + rows < T ? t0 + rows : T;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  for (long long t = t0; t < t1; ++t) {
    const float rs = __ldg(rstd + t);
    const float4 h = __ldcs(reinterpret_cast<const float4*>(dH + t * d + c));
    const uint2 xv = __ldcs(reinterpret_cast<const uint2*>(X + t * d + c));
    a0 = fmaf(h.x * bf16lo(xv.x), rs, a0);
    a1 = fmaf(h.y * bf16hi(xv.x), rs, a1);
    a2 = fmaf(h.z * bf16lo(xv.y), rs, a2);
    a3 = fmaf(h.w * bf16hi(xv.y), rs, a3);
  }
  atomicAdd(dw + c, a0);
  atomicAdd(dw + c + 1, a1);
  atomicAdd(dw + c + 2, a2);
  atomicAdd(dw + c + 3, a3);
}

// Adapter folded into its weight: Wm = bf16(fma(s, sum_k B[o][k] A[k][j], W[o][j])), the sum
// in fp32 over k = 0..r-1.  A thread owns 4 rows x 8 consecutive columns, so each A
// vector it loads serves 4 rows; the B values of the block's rows are shared by all of its
// threads (broadcast loads).  W and Wm may alias: each element is read and written by
// one thread only.
static __global__ void __launch_bounds__(128) merge_weights_kernel(const uint16_t* W, const uint16_t* __restrict__ A,
                                                            const uint16_t* __restrict__ B, uint16_t* Wm,
                                                            long long rows, long long cols, int r, float s) {
  const long long j = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (j >= cols) return;
  for (long long o0 = static_cast<long long>(blockIdx.y) * 4; o0 < rows; o0 += static_cast<long long>(gridDim.y) * 4) {
    float acc[4][8];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[q][e] = 0.f;
    for (int k = 0; k < r; ++k) {
      float a[8];
      unpack8(__ldg(reinterpret_cast<const uint4*>(A + static_cast<long long>(k) * cols + j)), a);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (o0 + q >= rows) break;
        const float b = __uint_as_float(static_cast<uint32_t>(__ldg(B + (o0 + q) * r + k)) << 16);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[q][e] = fmaf(b, a[e], acc[q][e]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (o0 + q >= rows) break;
      const long long off = (o0 + q) * cols + j;
      float w[8];
      unpack8(*reinterpret_cast<const uint4*>(W + off), w);
      uint4 ov;
      ov.x = pack_bf16x2(fmaf(s, acc[q][0], w[0]), fmaf(s, acc[q][1], w[1]));
      ov.y = pack_bf16x2(fmaf(s, acc[q][2], w[2]), fmaf(s, acc[q][3], w[3]));
      ov.z = pack_bf16x2(fmaf(s, acc[q][4], w[4]), fmaf(s, acc[q][5], w[5]));
      ov.w = pack_bf16x2(fmaf(s, acc[q][6], w[6]), fmaf(s, acc[q][7], w[7]));
      *reinterpret_cast<uint4*>(Wm + off) = ov;
    }
  }
}

// Double quantisation of the 4-bit block constants ("Unsloth 深度实战…", §1.4: the
// quantisation constants are quantised as well).  One warp per block of 256 absmax
// values: scale2 = the block's largest value; each value a gets the 8-bit code
// k = #{ j in 1..255 : 510 a > (2j - 1) scale2 } (nearest of the levels scale2 k / 255,
// ties to the lower one), decided exactly: both products are exact in double.
constexpr int kAbsmax8Block = 256;
static __global__ void absmax8_quantize_kernel(const float* __restrict__ absmax, long long n,
                                               uint8_t* __restrict__ codes8, float* __restrict__ scale2) {
  const int lane = threadIdx.x % 32;
  const long long nblk = (n + kAbsmax8Block - 1) / kAbsmax8Block;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long b = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32; b < nblk;
       b += warps) {
    const long long i0 = b * kAbsmax8Block;
    float v[kAbsmax8Block / 32];
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < kAbsmax8Block / 32; ++e) {
      const long long i = i0 + e * 32 + lane;
      v[e] = i < n ? absmax[i] : 0.f;
      mx = fmaxf(mx, v[e]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) scale2[b] = mx;
    const double sd = mx;
#pragma unroll
    for (int e = 0; e < kAbsmax8Block / 32; ++e) {
      const long long i = i0 + e * 32 + lane;
      if (i >= n) continue;
      const double x = 510.0 * static_cast<double>(v[e]);
      int k = 0;
      if (sd > 0.0) {
        k = static_cast<int>(floor((x / sd + 1.0) * 0.5));  // estimate, then settle exactly
        k = k < 0 ? 0 : (k > 255 ? 255 : k);
        while (k < 255 && x > sd * (2 * (k + 1) - 1)) ++k;
        while (k > 0 && !(x > sd * (2 * k - 1))) --k;
      }
      codes8[i] = static_cast<uint8_t>(k);
    }
  }
}

// absmax[i] = scale2[i / 256] * codes8[i] / 255 in fp32, for up to three matrices.
struct Absmax8List {
  const uint8_t* codes[3];
  const float* scale2[3];
  float* out[3];
  long long n[3];
};
static __global__ void absmax8_decode_kernel(Absmax8List L) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (int m = 0; m < 3; ++m)
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < L.n[m]; i += stride)
      L.out[m][i] = L.scale2[m][i / kAbsmax8Block] * static_cast<float>(L.codes[m][i]) / 255.0f;
}

}  // namespace lm
