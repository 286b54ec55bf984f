// The rank-r products of the LoRA path that stream one large activation X [T x K] past
// a skinny operand, on the tensor cores, reading X once from HBM.
//
// For a LoRA linear y = x W^T + P B^T with P = s x A^T (the LoRA form of the
// "Unsloth — 用手写 Triton kernel…" pages, §4: the LoRA linear and its backward):
//   forward:   P[t, :]   = s * sum_k X[t, k] A[:, k]      (X = the layer input)
//   backward:  Q[t, :]   = s * sum_k X[t, k] B[k, :]      (X = dy, the gradient of the rank-r input)
//              dB[k, :]  =     sum_t X[t, k] P[t, :]      (X = dy)
//              dA[:, k]  =     sum_t Q[t, :] X[t, k]      (X = the layer input)
// Two product kinds cover all four: the "row" product (a sum over the columns of X, one
// output row per row of X: P and Q) and the "column" product (a sum over the rows of X,
// one output row per column of X: dB and dA).  This kernel streams each [128 x 128] tile
// of X through shared memory once and issues tcgen05 MMAs for either product or both:
// the tile is a K-major A operand of the row product (M = rows) and, read as its
// transpose, an MN-major A operand of the column product (M = columns).  The skinny
// operand of the row product is MN-major ([K x r], as B is stored) or K-major (rows of
// [r x K], as A is stored, from one or two matrices stacked); that of the column product
// is MN-major ([T x n]).  Up to two problems (separate X) share a launch.
//
// Work: units = (row region of R row blocks, problem, column group of 128); CTA i takes
// the contiguous unit range [i U / G, (i + 1) U / G).  Per unit the column-product
// accumulator (TMEM) collects the R row blocks and is added to its output with fp32
// atomics; the row-product accumulators (one per row block of the region) collect every
// column group of the CTA's run of the same (region, problem) and are flushed when the
// run ends.  A run that covers the whole row of column groups writes its rows directly;
// otherwise every contributing CTA stores an fp32 partial in its slot and the last to
// arrive (an arrival counter per (region, problem)) sums the slots in slot order, so the
// row product does not depend on arrival order.
//
// CTA = 7 warps: warp 0 copies the tiles by TMA into a ring, warp 1 owns TMEM and issues
// the row-product MMAs from one thread, warp 6 issues the column-product MMAs, warps 2..5
// drain the accumulators (one TMEM lane quarter each).  Every wait is bounded; the
// epilogue warps agree on each wait's outcome through a reducing named barrier, so none
// is left waiting on a warp that gave up.
#pragma once
#include "gemm_sm100.cuh"

namespace lm {

constexpr int kDualEpiWarps = 4;
constexpr int kDualThreads = 64 + 32 * kDualEpiWarps + 32;  // + the column-product MMA warp
constexpr int kDualMaxGrid = 148;                           // CTAs per launch at most (one per SM)
constexpr int kDualMaxStages = 6;
constexpr uint32_t kDualXBytes = 2u * 128u * 128u;  // one [128 rows x 128 columns] bf16 tile of X

struct DualArgs {
  CUtensorMap x[2];     // X of problem m: [T x K], K contiguous, box {64, 128}
  CUtensorMap b[2][2];  // row product, problem m: MN-major [K x r] in b[m][0] (box {prow / 2, 128},
                        // prow-byte swizzle), or K-major rows [r x K] in b[m][i] giving the
                        // operand's rows [i rp, (i + 1) rp) (box {64, rp}, 128-byte swizzle)
  CUtensorMap p[2];     // column product, problem m: MN-major [T x n] (box {prow / 2, 128})
  int nx;               // problems (1 or 2)
  long long T;          // rows of X
  int K;                // columns of X
  int r, rp;            // rank, rank padded to 16
  int n;                // MMA N of both products
  int do_row, do_col;   // products computed
  int row_kmajor, nbk;  // the row product's operand is K-major from nbk maps (else MN-major)
  int qw;               // row-product columns written per problem: problem m owns [m qw, (m + 1) qw)
  int col_trans;        // column product: 0 -> out[m] is [K x r]; 1 -> accumulator column c goes to
                        // row c % rp of the [r x K] matrix out[c / rp] (problem 0 only, up to 3)
  int prow, patoms;     // MN-major skinny tiles: bytes per row (32, 64, 128 = the swizzle width),
                        // 64-column atoms
  uint32_t swz;         // their shared-memory swizzle (SmemSwizzle)
  int nsplit;           // accumulators per product (2: independent MMA chains, summed when drained)
  int rsets;            // row-accumulator sets (2: a run's flush overlaps the next run's MMAs)
  uint32_t tmem_cols;
  int R;                // row blocks of 128 per row region
  int nrb, nc, nreg;    // row blocks, column groups of 128, row regions
  long long units;      // nreg * nx * nc
  float scale;          // applied to the row product only
  float* out[3];        // column-product outputs, fp32, accumulated with atomics (zeroed by the caller)
  uint16_t* Q;          // row-product output, bf16 [T x ldq]
  int ldq;
  float* part;          // fp32 partials [slots][T][ldq]
  long long part_slot;
  int* cnt;             // [nreg * nx] arrival counters: zero before the launch, zero after it
  int* status;
  unsigned long long limit_ns;
  uint32_t stage_bytes;  // X tile + column-product tile + row-product tile
  uint32_t col_off, row_off;  // offsets of the two skinny tiles in a stage
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
__device__ __forceinline__ bool dual_run_end(long long u, long long u1, int nc) {
  return u + 1 == u1 || (u + 1) % nc == 0;
}

// Shared-memory stage: [X: two 16 KB halves of 64 columns, 128 rows, 128-byte swizzled]
// [column-product tile: patoms atoms of 128 rows x prow bytes]
// [row-product tile: MN-major like the above over 128 K rows, or K-major: two halves of
//  64 K, each n rows of 128 bytes].
static __device__ __noinline__ void dual_producer(const DualArgs& p, uint8_t* tiles, uint32_t full0, uint32_t empty0,
                                                  const WaitCtl& wc, long long u0, long long u1) {
  const int nstages = p.stages, nc = p.nc, nx = p.nx, R = p.R, nrb = p.nrb, patoms = p.patoms;
  const int do_row = p.do_row, do_col = p.do_col, row_kmajor = p.row_kmajor, nbk = p.nbk, n = p.n, rp = p.rp;
  const uint32_t stage_bytes = p.stage_bytes, col_off = p.col_off, row_off = p.row_off;
  const uint32_t atom = static_cast<uint32_t>(p.prow) * 128u;  // one 128-row atom of an MN-major tile
  int stage = 0;
  uint32_t phase = 0, issued_mask = 0, issued_par = 0;
  bool ok = true;
  for (long long u = u0; u < u1 && ok; ++u) {
    const DualUnit du = dual_unit(u, nc, nx);
    const CUtensorMap* xm = &p.x[du.m];
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
      const int col = du.c * 128, row = rb * 128;
      tma_load_2d(sX, xm, full, col, row);
      tma_load_2d(sX + 16384, xm, full, col + 64, row);
      if (do_col)
        for (int a = 0; a < patoms; ++a) tma_load_2d(sX + col_off + a * atom, pm, full, a * 64, row);
      if (do_row) {
        if (row_kmajor) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            for (int i = 0; i < nbk; ++i)
              tma_load_2d(sX + row_off + h * n * 128 + i * rp * 128, &p.b[du.m][i], full, col + 64 * h, 0);
        } else {
          for (int a = 0; a < patoms; ++a) tma_load_2d(sX + row_off + a * atom, &p.b[du.m][0], full, a * 64, col);
        }
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
// issues the row products (and owns the run-level hand-off), ROLE 1 the column products
// (and the per-unit hand-off).  Each commits its MMAs of a stage to the stage's empty
// barrier, which counts the active issuers.  Small-N MMAs cost a roughly fixed issue time
// each (about 85 cycles at N = 16, measured), so two issuers keep the tensor pipe fed
// where one could not; four (one per accumulator chain) measured slower than two.
template <int ROLE>
static __device__ __noinline__ void dual_mma(const DualArgs& p, uint8_t* tiles, uint32_t full0, uint32_t empty0,
                                             uint32_t cfull0, uint32_t cempty0, uint32_t rfull, uint32_t rempty,
                                             uint32_t drain_bar, uint32_t tmem_base, const WaitCtl& wc, long long u0,
                                             long long u1) {
  if (ROLE == 0 ? !p.do_row : !p.do_col) return;  // idle issuer
  const int nstages = p.stages, nc = p.nc, nx = p.nx, R = p.R, nrb = p.nrb, n = p.n, row_kmajor = p.row_kmajor;
  const uint32_t stage_bytes = p.stage_bytes, swz = p.swz, prow = static_cast<uint32_t>(p.prow);
  const uint32_t col_off = p.col_off, row_off = p.row_off;
  const uint32_t atom = prow * 128u;
  const uint32_t lbo = p.patoms > 1 ? atom : 0u;  // between 64-column atoms; unused with one atom
  // row product: A = X (K-major), B = the skinny operand (MN- or K-major)
  const uint32_t idesc_r = idesc_bf16(128, n, 0, row_kmajor ? 0 : 1);
  // column product: A = X^T (MN-major), B = the skinny operand (MN-major)
  const uint32_t idesc_c = idesc_bf16(128, n, 1, 1);
  const uint32_t tiles_u32 = smem_u32(tiles);
  // TMEM: row accumulators (set, rl, s) at ((set * R + rl) * nsplit + s) * n, column
  // accumulators (buf, s) after them
  const int nsplit = p.nsplit, rsets = p.rsets;
  const uint32_t rset_cols = static_cast<uint32_t>(R * nsplit * n);
  const uint32_t r_cols = p.do_row ? rsets * rset_cols : 0u;
  const uint32_t second = nsplit == 1 ? 1u : 0u;  // a second chain continues the first's sum
  int stage = 0;
  uint32_t phase = 0, it = 0, run = 0, started = 0;
  bool ok = true, issued_any = false;
  for (long long u = u0; u < u1 && ok; ++u, ++it) {
    const DualUnit du = dual_unit(u, nc, nx);
    const uint32_t buf = it & 1;
    const uint32_t rs = rsets == 2 ? (run & 1) : 0u, rph = rsets == 2 ? ((run >> 1) & 1) : (run & 1);
    if (ROLE == 0 && (u == u0 || du.c == 0)) {  // a new run of (region, problem): its row set is free again
      if (!mbar_wait(rempty + 8 * rs, rph ^ 1, wc, kDevTimeoutMma)) {
        ok = false;
        break;
      }
      started = 0;
    }
    if (ROLE == 1 && !mbar_wait(cempty0 + 8 * buf, ((it >> 1) & 1) ^ 1, wc, kDevTimeoutMma)) {
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t dc0 = tmem_base + r_cols + buf * nsplit * n;
    const uint32_t dc1 = dc0 + (nsplit - 1) * n;
    for (int rl = 0; rl < R; ++rl) {
      const int rb = du.reg * R + rl;
      if (rb >= nrb) break;
      if (!mbar_wait(full0 + 8 * stage, phase, wc, kDevTimeoutMma)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sX = tiles_u32 + static_cast<uint32_t>(stage) * stage_bytes;
      if (ROLE == 0) {
        // rows of block rl += X_tile S_tile: K = the tile's 128 columns in two halves of 64,
        // one accumulator chain per half.  MN-major S: rows = K, a k-step of 16 rows is
        // 16 * prow bytes; K-major S: n rows of 128 bytes per half, a k-step is 32 bytes.
        const uint32_t sS = sX + row_off;
        const uint32_t dr0 = tmem_base + rs * rset_cols + static_cast<uint32_t>(rl * nsplit * n);
        const uint32_t dr1 = dr0 + (nsplit - 1) * n;
        const uint32_t st = (started >> rl) & 1;
        const uint64_t a0 = sdesc_sw128(sX, 16, 1024), a1 = sdesc_sw128(sX + 16384, 16, 1024);
        uint64_t b0, b1;
        uint32_t bstep;
        if (row_kmajor) {
          b0 = sdesc_sw128(sS, 16, 1024);
          b1 = sdesc_sw128(sS + n * 128, 16, 1024);
          bstep = 32 >> 4;
        } else {
          b0 = sdesc(sS, lbo, 8 * prow, swz);
          b1 = sdesc(sS + 64 * prow, lbo, 8 * prow, swz);
          bstep = prow;  // (16 rows * prow bytes) >> 4
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          mma_bf16(dr0, a0 + j * (32 >> 4), b0 + j * bstep, idesc_r, j ? 1u : st);
          mma_bf16(dr1, a1 + j * (32 >> 4), b1 + j * bstep, idesc_r, j ? 1u : (st | second));
        }
        started |= 1u << rl;
      } else {
        // columns of the group += X_tile^T S_tile: K = the tile's 128 rows, one chain per half
        const uint64_t a = sdesc_sw128(sX, 16384, 1024);
        const uint64_t b = sdesc(sX + col_off, lbo, 8 * prow, swz);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          mma_bf16(dc0, a + j * (2048 >> 4), b + j * prow, idesc_c, (rl | j) ? 1u : 0u);
          mma_bf16(dc1, a + (j + 4) * (2048 >> 4), b + (j + 4) * prow, idesc_c, (rl | j) ? 1u : second);
        }
      }
      issued_any = true;
      mma_commit(empty0 + 8 * stage);  // frees the stage once every issuer's MMAs finish
      if (++stage == nstages) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (!ok) break;
    if (ROLE == 1) mma_commit(cfull0 + 8 * buf);
    if (ROLE == 0 && dual_run_end(u, u1, nc)) {  // the run ends: row accumulators ready
      mma_commit(rfull + 8 * rs);
      ++run;
    }
  }
  if (!ok && issued_any) {  // aborting: the MMAs already issued finish before TMEM is released
    mma_commit(drain_bar);
    drain_wait(drain_bar, 0, wc);
  }
}

// 16 accumulator columns [c, c + 16) of this thread's TMEM lane, the nsplit chains summed.
__device__ __forceinline__ void dual_ld16(uint32_t taddr, uint32_t chain_cols, int nsplit, uint32_t (&v)[16]) {
  tmem_ld16(taddr, v);
  tmem_wait16(v);
  if (nsplit == 2) {
    uint32_t w[16];
    tmem_ld16(taddr + chain_cols, w);
    tmem_wait16(w);
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) + __uint_as_float(w[e]));
  }
}

static __device__ __noinline__ void dual_epilogue(const DualArgs& p, uint32_t cfull0, uint32_t cempty0,
                                                  uint32_t rfull, uint32_t rempty, uint32_t tmem_base,
                                                  volatile int* s_last, const WaitCtl& wc, long long u0,
                                                  long long u1, long long U, long long G) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int q = warp & 3;  // TMEM lane quarter
  const int etid = threadIdx.x - 64;
  const int nc = p.nc, nx = p.nx, R = p.R, nrb = p.nrb, n = p.n, r = p.r, rp = p.rp, K = p.K, ldq = p.ldq;
  const int nsplit = p.nsplit, qw = p.qw, do_row = p.do_row, do_col = p.do_col, col_trans = p.col_trans;
  const int rsets = p.rsets;
  const long long T = p.T, part_slot = p.part_slot;
  const float scale = p.scale;
  uint16_t* const Q = p.Q;
  float* const part = p.part;
  const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
  const uint32_t rset_cols = static_cast<uint32_t>(R * nsplit * n);
  const uint32_t r_cols = do_row ? rsets * rset_cols : 0u;
  uint32_t it = 0, run = 0;
  for (long long u = u0; u < u1; ++u, ++it) {
    const DualUnit du = dual_unit(u, nc, nx);
    const uint32_t buf = it & 1;
    int ok = 1;
    if (do_col) {
      if (lane == 0) ok = mbar_wait(cfull0 + 8 * buf, (it >> 1) & 1, wc, kDevTimeoutEpilogue) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!dual_epi_and(ok)) break;
      tc_fence_after();
      // column kk of X: this lane's accumulator row
      const long long kk = static_cast<long long>(du.c) * 128 + 32 * q + lane;
      const uint32_t t0 = lane_base + r_cols + buf * nsplit * n;
      if (!col_trans) {  // out[m][kk, 0:r]: 16 consecutive values of one row -> four vector atomics
        float* const o0 = p.out[du.m];
#pragma unroll 1
        for (int c0 = 0; c0 < r; c0 += 16) {
          uint32_t v[16];
          dual_ld16(t0 + c0, n, nsplit, v);
          if (kk < K) {
            float* o = o0 + kk * r + c0;
#pragma unroll
            for (int h = 0; h < 4; ++h)
              if (c0 + 4 * h < r)
                atomicAdd(reinterpret_cast<float4*>(o + 4 * h),
                          make_float4(__uint_as_float(v[4 * h]), __uint_as_float(v[4 * h + 1]),
                                      __uint_as_float(v[4 * h + 2]), __uint_as_float(v[4 * h + 3])));
          }
        }
      } else {
        // out[c / rp][c % rp, kk]: a lane holds one kk; the four lanes of a group hold four
        // consecutive kk, gathered by shuffles into one vector atomic (group lane e % 4
        // issues the one for accumulator column c0 + e)
        const long long kb = kk & ~3LL;
#pragma unroll 1
        for (int c0 = 0; c0 < n; c0 += 16) {
          uint32_t v[16];
          dual_ld16(t0 + c0, n, nsplit, v);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int src = lane & ~3;
            const float x0 = __shfl_sync(0xffffffffu, __uint_as_float(v[e]), src);
            const float x1 = __shfl_sync(0xffffffffu, __uint_as_float(v[e]), src + 1);
            const float x2 = __shfl_sync(0xffffffffu, __uint_as_float(v[e]), src + 2);
            const float x3 = __shfl_sync(0xffffffffu, __uint_as_float(v[e]), src + 3);
            const int c = c0 + e, o = c / rp, j = c - o * rp;
            if ((lane & 3) == (e & 3) && j < r && o < 3 && kb < K) {
              float* dst = p.out[o];
              if (dst) atomicAdd(reinterpret_cast<float4*>(dst + static_cast<long long>(j) * K + kb),
                                 make_float4(x0, x1, x2, x3));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(cempty0 + 8 * buf);
    }
    if (!do_row || !dual_run_end(u, u1, nc)) continue;

    // End of a run of (region, problem): flush the row accumulators.
    const uint32_t rs = rsets == 2 ? (run & 1) : 0u, rph = rsets == 2 ? ((run >> 1) & 1) : (run & 1);
    if (lane == 0) ok = mbar_wait(rfull + 8 * rs, rph, wc, kDevTimeoutEpilogue) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!dual_epi_and(ok)) break;
    tc_fence_after();
    ++run;
    const long long first = dual_owner(du.key * nc, U, G);
    const long long last = dual_owner(du.key * nc + nc - 1, U, G);
    const int nparts = static_cast<int>(last - first + 1);
    const long long slot = static_cast<long long>(blockIdx.x) - first;
    const int qcol = du.m * qw;
#pragma unroll 1
    for (int rl = 0; rl < R; ++rl) {
      const int rb = du.reg * R + rl;
      if (rb >= nrb) break;
      const long long t = static_cast<long long>(rb) * 128 + 32 * q + lane;
#pragma unroll 1
      for (int c0 = 0; c0 < qw; c0 += 16) {
        uint32_t v[16];
        dual_ld16(lane_base + rs * rset_cols + static_cast<uint32_t>(rl * nsplit * n + c0), n, nsplit, v);
        if (t >= T) continue;
        if (nparts == 1) {  // the whole row of column groups was this CTA's: the output directly
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
    if (lane == 0) mbar_arrive(rempty + 8 * rs);
    if (nparts == 1) continue;
    // the last of the run's CTAs to arrive sums the partial slots in slot order
    __threadfence();
    dual_epi_sync();
    if (etid == 0) *s_last = atomicAdd(p.cnt + du.key, 1) == nparts - 1 ? 1 : 0;
    dual_epi_sync();
    if (!*s_last) continue;
    __threadfence();
    const long long r0 = static_cast<long long>(du.reg) * R * 128;
    const long long r1 = min(T, r0 + static_cast<long long>(R) * 128);
    const int c4n = qw / 4;
    for (long long i = etid; i < (r1 - r0) * c4n; i += 32 * kDualEpiWarps) {
      const long long row = r0 + i / c4n;
      const int c4 = static_cast<int>(i % c4n);
      const long long off = row * ldq + qcol + 4 * c4;
      float4 s4 = __ldcg(reinterpret_cast<const float4*>(part + off));
      for (int j = 1; j < nparts; ++j) {
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
  const uint32_t cfull0 = empty0 + 8 * S;
  const uint32_t cempty0 = cfull0 + 16;
  const uint32_t rfull = cempty0 + 16;   // one per row set
  const uint32_t rempty = rfull + 16;
  const uint32_t drain_bar = rempty + 16;  // one per MMA issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_slot + 2);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long U = p.units, G = gridDim.x;
  const long long u0 = dual_lo(blockIdx.x, U, G), u1 = dual_lo(blockIdx.x + 1, U, G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, p.do_row + p.do_col);  // every active MMA issuer commits
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(cfull0 + 8 * b, 1);
      mbar_init(cempty0 + 8 * b, kDualEpiWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(rfull + 8 * b, 1);
      mbar_init(rempty + 8 * b, kDualEpiWarps);
    }
    for (int i = 0; i < 2; ++i) mbar_init(drain_bar + 8 * i, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int m = 0; m < p.nx; ++m) {
      tma_prefetch_desc(&p.x[m]);
      if (p.do_col) tma_prefetch_desc(&p.p[m]);
      if (p.do_row)
        for (int i = 0; i < (p.row_kmajor ? p.nbk : 1); ++i) tma_prefetch_desc(&p.b[m][i]);
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
      dual_mma<0>(p, tiles, full0, empty0, cfull0, cempty0, rfull, rempty, drain_bar, tmem_base, wc, u0, u1);
    __syncwarp();
  } else if (warp < 2 + kDualEpiWarps) {
    dual_epilogue(p, cfull0, cempty0, rfull, rempty, tmem_base, s_last, wc, u0, u1, U, G);
  } else {
    if (lane == 0)
      dual_mma<1>(p, tiles, full0, empty0, cfull0, cempty0, rfull, rempty, drain_bar + 8, tmem_base, wc, u0, u1);
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
