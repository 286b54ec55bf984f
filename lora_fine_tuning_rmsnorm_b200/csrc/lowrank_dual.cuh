// Both rank-r products of an activation gradient in one read of it.
//
// For an up-projection y = x W^T + P B^T with P = s x A^T (the LoRA form of the
// "Unsloth — 用手写 Triton kernel…" pages, §4: the LoRA linear and its backward), the
// backward needs, from dy = X [T x K]:
//   Q[t, 0:rp] = s * sum_k X[t, k] B[k, 0:r]    (the gradient of the rank-r input, for dA)
//   dB[k, 0:r] =     sum_t X[t, k] P[t, 0:r]    (the gradient of B)
// Both are skinny contractions bounded by reading X once from HBM, one over the columns
// of X and one over its rows.  This kernel streams each [128 x 128] tile of X through
// shared memory once and issues both tcgen05 MMAs on it: the tile is a K-major A operand
// of the Q product (M = rows) and, read as its transpose, an MN-major A operand of the dB
// product (M = columns).  Up to two problems share a launch (gate and up).
//
// Work: units = (row region of R row blocks, problem, column group of 128); CTA i takes
// the contiguous unit range [i U / G, (i + 1) U / G).  Per unit the dB accumulator (TMEM)
// collects the R row blocks and is added to dB with fp32 atomics; the Q accumulators
// (one per row block of the region) collect every column group of the CTA's run of the
// same (region, problem) and are flushed when the run ends.  A run that covers the whole
// row of column groups writes Q directly; otherwise every contributing CTA stores an fp32
// partial in its slot and the last to arrive (an arrival counter per (region, problem))
// sums the slots in slot order, so Q does not depend on arrival order.
//
// CTA = 7 warps: warp 0 copies X, P and B tiles by TMA into a ring, warp 1 owns TMEM and
// issues the Q MMAs from one thread, warp 6 issues the dB MMAs, warps 2..5 drain the
// accumulators (one TMEM lane quarter each).  Every wait is bounded; the epilogue warps agree on each wait's outcome
// through a reducing named barrier, so none is left waiting on a warp that gave up.
#pragma once
#include "gemm_sm100.cuh"

namespace lm {

constexpr int kDualEpiWarps = 4;
constexpr int kDualThreads = 64 + 32 * kDualEpiWarps + 32;  // + the dB MMA warp
constexpr int kDualMaxGrid = 148;   // CTAs per launch at most (one per SM)
constexpr int kDualMaxStages = 6;
constexpr uint32_t kDualXBytes = 2u * 128u * 128u;  // one [128 rows x 128 columns] bf16 tile of X

struct DualArgs {
  CUtensorMap x[2];  // X of problem m: [T x K], K contiguous, box {64, 128}
  CUtensorMap b[2];  // B of problem m: [K x r], r contiguous, box {prow / 2, 128}, prow-byte swizzle
  CUtensorMap p[2];  // P of problem m: [T x r] (row stride ldp), box {prow / 2, 128}, prow-byte swizzle
  int nx;            // problems (1 or 2)
  long long T;       // rows of X
  int K;             // columns of X
  int r, rp, qn;     // rank, padded rank (Q columns per problem), MMA N (16, 32, 64 or 128)
  int prow, patoms;  // P / B tiles: bytes per row (32, 64 or 128 = the swizzle width), atoms of 64 columns
  uint32_t swz;      // their shared-memory swizzle (SmemSwizzle)
  int nsplit;        // accumulators per product (2: independent MMA chains, summed when drained)
  uint32_t tmem_cols;
  int R;             // row blocks of 128 per row region
  int nrb, nc, nreg; // row blocks, column groups of 128, row regions
  long long units;   // nreg * nx * nc
  float scale;       // s, applied to Q only
  float* dB[2];      // [K x r] fp32 per problem, accumulated with atomics (zeroed by the caller)
  uint16_t* Q;       // bf16 [T x ldq]; problem m owns columns [m rp, (m + 1) rp)
  int ldq;
  float* part;       // fp32 partials [slots][T][ldq]
  long long part_slot;
  int* cnt;          // [nreg * nx] arrival counters: zero before the launch, zero after it
  int* status;
  unsigned long long limit_ns;
  uint32_t stage_bytes;  // X tile + P tile + B tile
  int stages;
};

// Unit ranges: CTA i of G owns [dual_lo(i), dual_lo(i + 1)); dual_owner(u) is the CTA
// whose range holds unit u (requires G <= U, so that no range is empty).
__host__ __device__ inline long long dual_lo(long long i, long long U, long long G) { return i * U / G; }
__host__ __device__ inline long long dual_owner(long long u, long long U, long long G) {
  return ((u + 1) * G + U - 1) / U - 1;
}

// Named barrier 1 over the epilogue warps: AND of the threads' predicates / plain sync.
__device__ __forceinline__ int dual_epi_and(int pred) {
  int out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.s32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(pred), "n"(32 * kDualEpiWarps)
      : "memory");
  return out;
}
__device__ __forceinline__ void dual_epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kDualEpiWarps) : "memory");
}

struct DualUnit {
  long long key;  // (region, problem) index = region * nx + problem
  int c, reg, m;
};
__device__ __forceinline__ DualUnit dual_unit(long long u, int nc, int nx) {
  DualUnit d;
  d.key = u / nc;
  d.c = static_cast<int>(u - d.key * nc);
  d.reg = static_cast<int>(d.key / nx);
  d.m = static_cast<int>(d.key - static_cast<long long>(d.reg) * nx);
  return d;
}

// Shared-memory stage: [X: two 16 KB halves of 64 columns, 128 rows, 128-byte swizzled]
// [P: patoms atoms of 128 rows x prow bytes][B: patoms atoms of 128 K rows x prow bytes];
// the P and B rows are exactly the padded rank wide (N = 16 -> 32-byte rows, 32-byte swizzle).
static __device__ __noinline__ void dual_producer(const DualArgs& p, uint8_t* tiles, uint32_t full0, uint32_t empty0,
                                                  const WaitCtl& wc, long long u0, long long u1) {
  const int nstages = p.stages, nc = p.nc, nx = p.nx, R = p.R, nrb = p.nrb, patoms = p.patoms;
  const uint32_t stage_bytes = p.stage_bytes;
  const uint32_t atom = static_cast<uint32_t>(p.prow) * 128u;  // one 128-row atom of the P (or B) tile
  int stage = 0;
  uint32_t phase = 0, issued_mask = 0, issued_par = 0;
  bool ok = true;
  for (long long u = u0; u < u1 && ok; ++u) {
    const DualUnit du = dual_unit(u, nc, nx);
    const CUtensorMap* xm = &p.x[du.m];
    const CUtensorMap* bm = &p.b[du.m];
    const CUtensorMap* pm = &p.p[du.m];
    for (int rl = 0; rl < R; ++rl) {
      const int rb = du.reg * R + rl;
      if (rb >= nrb) break;
      const uint32_t full = full0 + 8 * stage, empty = empty0 + 8 * stage;
      if (!mbar_wait(empty, phase ^ 1, wc, kDevTimeoutProducer)) {
        ok = false;
        break;
      }
      mbar_expect_tx(full, stage_bytes);
      const uint32_t sX = smem_u32(tiles + static_cast<size_t>(stage) * stage_bytes);
      const uint32_t sP = sX + kDualXBytes, sB = sP + patoms * atom;
      const int col = du.c * 128, row = rb * 128;
      tma_load_2d(sX, xm, full, col, row);
      tma_load_2d(sX + 16384, xm, full, col + 64, row);
      for (int a = 0; a < patoms; ++a) {
        tma_load_2d(sP + a * atom, pm, full, a * 64, row);
        tma_load_2d(sB + a * atom, bm, full, a * 64, col);
      }
      issued_mask |= 1u << stage;
      issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
      if (++stage == nstages) {
        stage = 0;
        phase ^= 1;
      }
    }
  }
  if (!ok) {  // aborting: no copy into shared memory may still be in flight
    for (int s = 0; s < nstages; ++s)
      if (issued_mask & (1u << s)) drain_wait(full0 + 8 * s, (issued_par >> s) & 1, wc);
  }
}

// MMA issue, split over two threads of different warps that walk the same stages: ROLE 0
// issues the Q products (and owns the run-level Q hand-off), ROLE 1 the dB products (and
// the per-unit dB hand-off).  Each commits its MMAs of a stage to the stage's empty
// barrier, which counts both.  Small-N MMAs cost a roughly fixed issue time each (about
// 85 cycles at N = 16, measured), so two issuers keep the tensor pipe fed where one could
// not; four (one per accumulator chain) measured slower than two.
template <int ROLE>
static __device__ __noinline__ void dual_mma(const DualArgs& p, uint8_t* tiles, uint32_t full0, uint32_t empty0,
                                             uint32_t dbfull0, uint32_t dbempty0, uint32_t qfull, uint32_t qempty,
                                             uint32_t drain_bar, uint32_t tmem_base, const WaitCtl& wc, long long u0,
                                             long long u1) {
  const int nstages = p.stages, nc = p.nc, nx = p.nx, R = p.R, nrb = p.nrb, qn = p.qn;
  const uint32_t stage_bytes = p.stage_bytes, swz = p.swz, prow = static_cast<uint32_t>(p.prow);
  const uint32_t atom = prow * 128u, pbytes = static_cast<uint32_t>(p.patoms) * atom;
  const uint32_t lbo = p.patoms > 1 ? atom : 0u;  // between 64-column atoms; unused with one atom
  const uint32_t idesc_q = idesc_bf16(128, qn, 0, 1);  // A = X (K-major), B = B (MN-major)
  const uint32_t idesc_b = idesc_bf16(128, qn, 1, 1);  // A = X^T (MN-major), B = P (MN-major)
  const uint32_t tiles_u32 = smem_u32(tiles);
  // TMEM: Q accumulators (rl, s) at (rl * nsplit + s) * qn, dB accumulators (buf, s) after them
  const int nsplit = p.nsplit;
  const uint32_t q_cols = static_cast<uint32_t>(R * nsplit * qn);
  const uint32_t second = nsplit == 1 ? 1u : 0u;  // a second chain continues the first's sum
  constexpr int kKind = ROLE;
  int stage = 0;
  uint32_t phase = 0, it = 0, qrun = 0, started = 0;
  bool ok = true, issued_any = false;
  for (long long u = u0; u < u1 && ok; ++u, ++it) {
    const DualUnit du = dual_unit(u, nc, nx);
    const uint32_t buf = it & 1;
    if (kKind == 0 && (u == u0 || du.c == 0)) {  // a new run of (region, problem): Q accumulators free again
      if (!mbar_wait(qempty, (qrun & 1) ^ 1, wc, kDevTimeoutMma)) {
        ok = false;
        break;
      }
      started = 0;
    }
    if (kKind == 1 && !mbar_wait(dbempty0 + 8 * buf, ((it >> 1) & 1) ^ 1, wc, kDevTimeoutMma)) {
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t db0 = tmem_base + q_cols + buf * nsplit * qn;
    const uint32_t db1 = db0 + (nsplit - 1) * qn;
    for (int rl = 0; rl < R; ++rl) {
      const int rb = du.reg * R + rl;
      if (rb >= nrb) break;
      if (!mbar_wait(full0 + 8 * stage, phase, wc, kDevTimeoutMma)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sX = tiles_u32 + static_cast<uint32_t>(stage) * stage_bytes;
      const uint32_t sP = sX + kDualXBytes, sB = sP + pbytes;
      if (kKind == 0) {
        // Q[rows of block rl] += X_tile B_tile: K = the tile's 128 columns in two halves of 64
        // (B is MN-major: rows = K, a k-step of 16 rows is 16 * prow bytes), one chain per half
        const uint32_t dq0 = tmem_base + static_cast<uint32_t>(rl * nsplit * qn);
        const uint32_t dq1 = dq0 + (nsplit - 1) * qn;
        const uint32_t st_q = (started >> rl) & 1;
        const uint64_t qa0 = sdesc_sw128(sX, 16, 1024), qa1 = sdesc_sw128(sX + 16384, 16, 1024);
        const uint64_t qb0 = sdesc(sB, lbo, 8 * prow, swz), qb1 = sdesc(sB + 64 * prow, lbo, 8 * prow, swz);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          mma_bf16(dq0, qa0 + j * (32 >> 4), qb0 + j * prow, idesc_q, j ? 1u : st_q);
          mma_bf16(dq1, qa1 + j * (32 >> 4), qb1 + j * prow, idesc_q, j ? 1u : (st_q | second));
        }
        started |= 1u << rl;
      } else {
        // dB[columns of the group] += X_tile^T P_tile: K = the tile's 128 rows, one chain per half
        const uint64_t ba = sdesc_sw128(sX, 16384, 1024);
        const uint64_t bb = sdesc(sP, lbo, 8 * prow, swz);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          mma_bf16(db0, ba + j * (2048 >> 4), bb + j * prow, idesc_b, (rl | j) ? 1u : 0u);
          mma_bf16(db1, ba + (j + 4) * (2048 >> 4), bb + (j + 4) * prow, idesc_b, (rl | j) ? 1u : second);
        }
      }
      issued_any = true;
      mma_commit(empty0 + 8 * stage);  // frees the stage once both issuers' MMAs finish
      if (++stage == nstages) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (!ok) break;
    if (kKind == 1) mma_commit(dbfull0 + 8 * buf);
    if (kKind == 0 && (u + 1 == u1 || (u + 1) % nc == 0)) {  // the run ends: Q accumulators ready
      mma_commit(qfull);
      ++qrun;
    }
  }
  if (!ok && issued_any) {  // aborting: the MMAs already issued finish before TMEM is released
    mma_commit(drain_bar);
    drain_wait(drain_bar, 0, wc);
  }
}

static __device__ __noinline__ void dual_epilogue(const DualArgs& p, uint32_t dbfull0, uint32_t dbempty0,
                                                  uint32_t qfull, uint32_t qempty, uint32_t tmem_base,
                                                  volatile int* s_last, const WaitCtl& wc, long long u0,
                                                  long long u1, long long U, long long G) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int q = warp & 3;  // TMEM lane quarter
  const int etid = threadIdx.x - 64;
  const int nc = p.nc, nx = p.nx, R = p.R, nrb = p.nrb, qn = p.qn, r = p.r, rp = p.rp, K = p.K, ldq = p.ldq;
  const int nsplit = p.nsplit;
  const long long T = p.T, part_slot = p.part_slot;
  const float scale = p.scale;
  uint16_t* const Q = p.Q;
  float* const part = p.part;
  const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
  uint32_t it = 0, qrun = 0;
  for (long long u = u0; u < u1; ++u, ++it) {
    const DualUnit du = dual_unit(u, nc, nx);
    const uint32_t buf = it & 1;
    int ok = 1;
    if (lane == 0) ok = mbar_wait(dbfull0 + 8 * buf, (it >> 1) & 1, wc, kDevTimeoutEpilogue) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!dual_epi_and(ok)) break;
    tc_fence_after();
    // dB rows of this lane: column kk of X
    {
      float* const dB = p.dB[du.m];
      const long long kk = static_cast<long long>(du.c) * 128 + 32 * q + lane;
      const uint32_t t0 = lane_base + static_cast<uint32_t>(R * nsplit * qn) + buf * nsplit * qn;
#pragma unroll 1
      for (int c0 = 0; c0 < r; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(t0 + c0, v);
        tmem_wait16(v);
        if (nsplit == 2) {  // the second accumulator (rows 64-127 of each tile)
          uint32_t w[16];
          tmem_ld16(t0 + qn + c0, w);
          tmem_wait16(w);
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) + __uint_as_float(w[e]));
        }
        if (kk < K) {
          float* o = dB + kk * r + c0;
#pragma unroll
          for (int h = 0; h < 4; ++h)
            if (c0 + 4 * h < r)
              atomicAdd(reinterpret_cast<float4*>(o + 4 * h),
                        make_float4(__uint_as_float(v[4 * h]), __uint_as_float(v[4 * h + 1]),
                                    __uint_as_float(v[4 * h + 2]), __uint_as_float(v[4 * h + 3])));
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(dbempty0 + 8 * buf);
    if (!(u + 1 == u1 || (u + 1) % nc == 0)) continue;

    // End of a run of (region, problem): flush the Q accumulators.
    if (lane == 0) ok = mbar_wait(qfull, qrun & 1, wc, kDevTimeoutEpilogue) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!dual_epi_and(ok)) break;
    tc_fence_after();
    ++qrun;
    const long long first = dual_owner(du.key * nc, U, G);
    const long long last = dual_owner(du.key * nc + nc - 1, U, G);
    const int n = static_cast<int>(last - first + 1);
    const long long slot = static_cast<long long>(blockIdx.x) - first;
    const int qcol = du.m * rp;
#pragma unroll 1
    for (int rl = 0; rl < R; ++rl) {
      const int rb = du.reg * R + rl;
      if (rb >= nrb) break;
      const long long t = static_cast<long long>(rb) * 128 + 32 * q + lane;
#pragma unroll 1
      for (int c0 = 0; c0 < rp; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(lane_base + static_cast<uint32_t>(rl * nsplit * qn + c0), v);
        tmem_wait16(v);
        if (nsplit == 2) {  // the second accumulator (columns 64-127 of each tile)
          uint32_t w[16];
          tmem_ld16(lane_base + static_cast<uint32_t>((rl * nsplit + 1) * qn + c0), w);
          tmem_wait16(w);
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) + __uint_as_float(w[e]));
        }
        if (t >= T) continue;
        if (n == 1) {  // the whole row of column groups was this CTA's: Q directly
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            w[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * scale, __uint_as_float(v[2 * e + 1]) * scale);
          uint4* o = reinterpret_cast<uint4*>(Q + t * ldq + qcol + c0);
          o[0] = make_uint4(w[0], w[1], w[2], w[3]);
          o[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
          float4* o = reinterpret_cast<float4*>(part + slot * part_slot + t * ldq + qcol + c0);
#pragma unroll
          for (int h = 0; h < 4; ++h)
            o[h] = make_float4(__uint_as_float(v[4 * h]), __uint_as_float(v[4 * h + 1]),
                               __uint_as_float(v[4 * h + 2]), __uint_as_float(v[4 * h + 3]));
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(qempty);
    if (n == 1) continue;
    // the last of the run's n CTAs to arrive sums the partial slots in slot order
    __threadfence();
    dual_epi_sync();
    if (etid == 0) *s_last = atomicAdd(p.cnt + du.key, 1) == n - 1 ? 1 : 0;
    dual_epi_sync();
    if (!*s_last) continue;
    __threadfence();
    const long long r0 = static_cast<long long>(du.reg) * R * 128;
    const long long r1 = min(T, r0 + static_cast<long long>(R) * 128);
    const int c4n = rp / 4;
    for (long long i = etid; i < (r1 - r0) * c4n; i += 32 * kDualEpiWarps) {
      const long long row = r0 + i / c4n;
      const int c4 = static_cast<int>(i % c4n);
      const long long off = row * ldq + qcol + 4 * c4;
      float4 s4 = __ldcg(reinterpret_cast<const float4*>(part + off));
      for (int j = 1; j < n; ++j) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(part + j * part_slot + off));
        s4.x += x.x; s4.y += x.y; s4.z += x.z; s4.w += x.w;
      }
      *reinterpret_cast<uint2*>(Q + off) =
          make_uint2(pack_bf16x2(s4.x * scale, s4.y * scale), pack_bf16x2(s4.z * scale, s4.w * scale));
    }
    if (etid == 0) p.cnt[du.key] = 0;  // every contributor has arrived: ready for the next launch
  }
}

static __global__ void __launch_bounds__(kDualThreads, 1) lowrank_dual_kernel(const __grid_constant__ DualArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(tiles + static_cast<size_t>(p.stages) * p.stage_bytes);
  const int S = p.stages;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * S;
  const uint32_t dbfull0 = empty0 + 8 * S;
  const uint32_t dbempty0 = dbfull0 + 16;
  const uint32_t qfull = dbempty0 + 16;
  const uint32_t qempty = qfull + 8;
  const uint32_t drain_bar = qempty + 8;  // one per MMA issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_slot + 2);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long U = p.units, G = gridDim.x;
  const long long u0 = dual_lo(blockIdx.x, U, G), u1 = dual_lo(blockIdx.x + 1, U, G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 2);  // both MMA issuers commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(dbfull0 + 8 * b, 1);
      mbar_init(dbempty0 + 8 * b, kDualEpiWarps);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, kDualEpiWarps);
    for (int i = 0; i < 2; ++i) mbar_init(drain_bar + 8 * i, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < 2; ++i) {
      tma_prefetch_desc(&p.x[i]);
      tma_prefetch_desc(&p.b[i]);
      tma_prefetch_desc(&p.p[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, p.limit_ns};

  if (warp == 0) {
    if (lane == 0) dual_producer(p, tiles, full0, empty0, wc, u0, u1);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0)
      dual_mma<0>(p, tiles, full0, empty0, dbfull0, dbempty0, qfull, qempty, drain_bar, tmem_base, wc, u0, u1);
    __syncwarp();
  } else if (warp < 2 + kDualEpiWarps) {
    dual_epilogue(p, dbfull0, dbempty0, qfull, qempty, tmem_base, s_last, wc, u0, u1, U, G);
  } else {
    if (lane == 0)
      dual_mma<1>(p, tiles, full0, empty0, dbfull0, dbempty0, qfull, qempty, drain_bar + 8, tmem_base, wc, u0, u1);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace lm
