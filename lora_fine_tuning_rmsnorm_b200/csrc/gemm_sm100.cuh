// Warp-specialised, persistent tcgen05 GEMM for sm_100a with TMA-fed operands,
// TMEM accumulators and fused epilogues.  One kernel template serves every
// contraction of the LoRA-MLP forward/backward:
//
//   D_a[m, n] = sum over segments s feeding accumulator a of
//               sum_k  A_s[m, a_k0 + k] * B_{s,a}[n, b_k0 + k],   k in [0, k_len_s)
//
// A "segment" is a K range with its own A and B tensor maps, so the LoRA rank-r
// term is folded into the same accumulator as one short extra K range
// ([H | s P] x [W | B]^T), and gate/up share one A tile with two accumulators
// (NACC = 2).  Operands are bf16, 128-byte swizzled in shared memory, either
// K-major (x = K innermost) or MN-major (x = M/N innermost); out-of-range boxes
// are zero-filled by TMA, which also pads ragged K tails and rank r to 16.
//
// PAIR = 2 runs the same roles on a cluster of two CTAs that share one 256-row
// tile through tcgen05 cta_group::2: each CTA loads its own 128 rows of A and its
// half of the N columns of B (TMA completions counted on the even CTA's barrier,
// no multicast loads), the even CTA issues the pair MMA, and commits arrive on both
// CTAs' barriers.  This halves the B bytes each SM pulls from L2 per MMA.
//
// CTA = 10 warps: warp 0 issues TMA loads into a `stages`-deep ring, warp 1 owns
// TMEM and issues tcgen05.mma from one thread, warps 2..9 drain the double-
// buffered TMEM accumulators (tcgen05.ld) through the epilogue while the next
// tile's main loop runs (two warps per TMEM lane quarter, alternating 16-column
// chunks).  With 4-bit weights (Q4 = 1) warps 10..17 expand the codes into the bf16
// B tiles and warp 18 fills the code ring.  Tiles are handed out over a persistent
// grid, M-fastest or in bands of group_m row tiles with N swept per band.
#pragma once
#include "ptx.cuh"

namespace lm {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kMaxStages = 8;
constexpr int kMaxSegs = 6;
constexpr int kMaxMaps = 12;
constexpr int kEpiWarps = 8;  // two warps per TMEM lane quarter, alternating 16-column chunks
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr int kDqWarps = 8;  // 4-bit weights: warps that expand codes into bf16 B tiles
constexpr int kDqGroups = 2;  // ... in groups that take alternate stages
constexpr int kCodeRing = 8;  // 4-bit weights: entries of the code ring (codes + absmax of one stage)
// Epilogue staging for TMA stores: per epilogue warp, three [32 rows x 16 columns] bf16 tiles
constexpr int kEpiStageBytes = 3 * 32 * 16 * 2;
// Code-ring entries for MT M tiles per unit (two tiles per unit leave less shared memory)
__host__ __device__ constexpr int code_ring(int mt) { return mt == 2 ? 4 : kCodeRing; }
// 4-bit CTAs add the dequant warps and one warp that fills the code ring
__host__ __device__ constexpr int gemm_threads(int q4) { return kGemmThreads + (q4 ? 32 * kDqWarps + 32 : 0); }

// Shared-memory layout of the 4-bit operand in one CTA (host and device use the same):
// each stage is [A: MT x 16 KB][expanded bf16 B: slots x b_unit]; each of the code_ring(MT)
// code-ring entries is [codes: slots x q_unit][absmax: slots x m_unit] (cr_bytes, 1 KB aligned).
// A unit is one B operand (one accumulator, or one gate/up branch) as held by this CTA:
// `cols` B rows (K-major) or B columns (MN-major) by 64 K, i.e. `cols` 128-byte smem rows.
struct Q4Layout {
  uint32_t b_unit, q_unit, m_unit;
  int slots, cols;
};
__host__ __device__ inline Q4Layout q4_layout(int bn, int pair, int fuse, int b_mn, int nacc) {
  Q4Layout L;
  L.cols = fuse ? bn : bn / pair;
  L.slots = fuse ? (pair == 1 ? 2 : 1) : nacc;
  L.b_unit = static_cast<uint32_t>(L.cols) * 128u;
  L.q_unit = static_cast<uint32_t>(L.cols) * 32u;
  L.m_unit = b_mn ? 1024u : static_cast<uint32_t>(L.cols) * 16u;  // absmax box {4 floats} x rows
  return L;
}

enum Epi : int {
  EPI_F32 = 0,         // out[0] fp32 = acc_a * alpha at column a * out_acc_col (+ split * split_stride)
  EPI_BF16 = 1,        // out[0] bf16 = acc_a * alpha (+ in[0] when set), accumulator a at column a * out_acc_col
  EPI_SWIGLU_FWD = 2,  // acc0 = G, acc1 = U -> out[0] G, out[1] U, out[2] silu(G) * U (bf16)
  EPI_SWIGLU_BWD = 3,  // acc0 = dAct; in[0] G, in[1] U -> out[0] dG, out[1] dU (bf16)
  EPI_ATOMIC = 4,      // accumulator a atomically added into fp32 output rng[a] (split-K reductions)
  EPI_CE_LSE = 5,      // logits tile -> per row and tile half: (max, sum exp(z - max)) into out[0] (float2
                       // [2 tiles_n][M]) and the label's logit into out[1] (float [M]); logits never stored
  EPI_CE_DZ = 6        // logits tile -> dZ = g' (softmax - onehot(label)) as bf16 into out[0] (ld_out)
};

enum Hint : int { HINT_NONE = 0, HINT_EVICT_FIRST = 1, HINT_EVICT_LAST = 2 };

struct Seg {
  int a_map;
  int a_k0;
  int b_map[2];  // -1: this segment does not feed that accumulator
  int b_k0[2];
  int k_len;
  int a_hint, b_hint;  // L2 eviction priority of the A / B loads (Hint)
  int q4;              // 1: B comes from 4-bit codes (b_map = code map, b_am = absmax map)
  int b_am[2];
};

struct OutRange {
  float* out;     // destination of accumulator `acc` (rows m < M, columns n < N)
  int acc;
  int trans;      // 0: out[m * ld + n]; 1: out[n * ld + m]
  long long ld;
};

struct GemmArgs {
  CUtensorMap maps[kMaxMaps];
  Seg seg[kMaxSegs];
  int nseg;
  int M, N;  // valid rows / valid columns per accumulator
  int bn;    // N tile per accumulator (multiple of 16; multiple of 64 when B is MN-major)
  int tiles_m, tiles_n, splits;
  int raster;      // 0: M-fastest tile order; 1: N-fastest; 2: bands of group_m row tiles, N swept per band
  int group_m;
  int mn3d_a, mn3d_b;  // 1: that MN-major operand's maps are 3-D {64, K, MN/64} views (one box per tile)
  int stream_out;  // 1: epilogue stores are streaming (evict-first in L2)
  int k_chunk;  // split-K chunk in elements (multiple of BK) when splits > 1
  int stages;
  uint32_t stage_bytes;
  uint32_t tmem_cols;
  int nbuf;        // accumulator sets in TMEM: 2 (the epilogue drains one while the MMA fills the
                   // other) or 1 (a unit of MT = 2 M tiles fills all 512 columns)
  void* out[3];
  long long ld_out;
  long long split_stride;  // EPI_F32: element offset between the partial sums of K splits
  int out_acc_col;
  float alpha;
  const void* in[2];
  long long ld_in;
  OutRange rng[2];
  int nrng;
  int* status;
  unsigned long long limit_ns;
  const float* codebook;  // 4-bit code values (16 fp32)
  uint32_t cr_bytes;      // 4-bit: bytes of one code-ring entry
  int test_no_loads;      // test of the bounded waits: the producer copies nothing and arms no
                          // barrier, so the MMA's first wait runs out (single-CTA tiles only)
  int out_add;            // EPI_F32: add into the fp32 output instead of overwriting it
  int epi_tma;            // the outputs (SwiGLU: G, U, Act / dG, dU; bf16, fp32 (NACC = 1) and CE dZ: out[0])
                          // leave through shared memory by TMA stores; maps from out_map0, box {16, 32}, no swizzle
  int epi_drain;          // with epi_tma, MT = 2, bf16 out (N tile 256) or SwiGLU fwd (N tile 128): the
                          // epilogue empties TMEM into registers first (see gemm_epilogue)
  int out_map0;
  // cross-entropy epilogues (rows = tokens, columns = vocabulary entries ce_col0 + n)
  const int* ce_labels;   // label of each row; outside [0, ce_V) = left out of the loss
  const float* ce_lse;    // EPI_CE_DZ: logsumexp of each row (from the forward)
  const int* ce_count;    // EPI_CE_DZ: number of kept rows (mean reduction), NULL = sum reduction
  float ce_g;             // EPI_CE_DZ: upstream gradient of the reduced loss
  int ce_col0;            // vocabulary index of this launch's column 0 (vocabulary chunks)
  int ce_V;               // vocabulary size
};

// Tile-scheduling constants, copied out of the launch parameters once per role: every
// inline-asm statement in the role loops clobbers memory, so a field read inside a loop
// would be re-read from the parameter space (through the small constant cache) on every
// iteration, on the critical path from "stage freed" to "copy issued".
struct Sched {
  int tiles_m, tiles_n, splits, raster, group_m, k_chunk, total;
};
__device__ __forceinline__ Sched sched_of(const GemmArgs& p) {
  Sched s;
  s.tiles_m = p.tiles_m;
  s.tiles_n = p.tiles_n;
  s.splits = p.splits;
  s.raster = p.raster;
  s.group_m = p.group_m;
  s.k_chunk = p.k_chunk;
  s.total = p.tiles_m * p.tiles_n * p.splits;
  return s;
}

// Work unit u (a CTA, or a CTA pair when PAIR = 2) -> tile coordinates.
__device__ __forceinline__ void decode_tile(const Sched& p, int t, int& mt, int& nt, int& ks) {
  if (p.raster == 2) {
    // a band of group_m row tiles stays in L2 while the wave sweeps the N tiles
    const int per_split = p.tiles_m * p.tiles_n;
    ks = t / per_split;
    const int u = t - ks * per_split;
    const int g = u / (p.group_m * p.tiles_n);
    const int m_base = g * p.group_m;
    const int gsz = min(p.group_m, p.tiles_m - m_base);
    const int r = u - g * p.group_m * p.tiles_n;
    mt = m_base + r % gsz;
    nt = r / gsz;
  } else if (p.raster == 1) {
    nt = t % p.tiles_n;
    t /= p.tiles_n;
    mt = t % p.tiles_m;
    ks = t / p.tiles_m;
  } else {
    mt = t % p.tiles_m;
    t /= p.tiles_m;
    nt = t % p.tiles_n;
    ks = t / p.tiles_n;
  }
}

// k-block range [lo, hi) of a segment of k_len elements in K split ks.
__device__ __forceinline__ void seg_kb_range(const Sched& p, int k_len, int ks, int& lo, int& hi) {
  const int nkb = (k_len + BK - 1) / BK;
  if (p.splits > 1) {
    const int per = p.k_chunk / BK;
    lo = ks * per;
    hi = min(nkb, lo + per);
  } else {
    lo = 0;
    hi = nkb;
  }
}

// One segment's launch constants in registers (see Sched).
struct SegR {
  int a_map, a_k0, b_map0, b_map1, b_k00, b_k01, k_len, a_hint, b_hint, q4, b_am0, b_am1;
};
__device__ __forceinline__ SegR seg_of(const GemmArgs& p, int s) {
  const Seg& g = p.seg[s];
  return SegR{g.a_map, g.a_k0, g.b_map[0], g.b_map[1], g.b_k0[0], g.b_k0[1], g.k_len, g.a_hint, g.b_hint,
              g.q4, g.b_am[0], g.b_am[1]};
}
__device__ __forceinline__ int seg_bmap(const SegR& g, int a) { return a ? g.b_map1 : g.b_map0; }
__device__ __forceinline__ int seg_bk0(const SegR& g, int a) { return a ? g.b_k01 : g.b_k00; }
__device__ __forceinline__ int seg_bam(const SegR& g, int a) { return a ? g.b_am1 : g.b_am0; }

// Drain wait used after an abort: ignores the abort flag, bounded by the limit.
static __device__ __noinline__ void drain_wait(uint32_t bar, uint32_t parity, const WaitCtl& c) {
  const uint64_t t0 = global_ns();
  while (!mbar_test(bar, parity)) {
    if (global_ns() - t0 > c.limit_ns) {
      if (c.status) atomicCAS(c.status, 0, kDevTimeoutDrain);
      return;
    }
  }
}

// FUSE = 1 (gate/up): the two B operands of a segment are two halves of ONE
// N = 2 * bn MMA (branch 0 -> columns [0, bn), branch 1 -> [bn, 2 bn)), so a k-step
// issues one wide MMA instead of two; with PAIR = 2, CTA rank r loads branch r.
template <int A_MN, int B_MN, int NACC, int PAIR, int FUSE, int Q4, int MT>
__device__ __forceinline__ void gemm_producer(const GemmArgs& p, uint8_t* tiles, uint32_t full0,
                                              uint32_t empty0, const WaitCtl& wc, uint32_t rank) {
  const Sched sc = sched_of(p);
  const int unit0 = blockIdx.x / PAIR, nunits = gridDim.x / PAIR;
  // launch constants in registers (see Sched)
  const int M = p.M, N = p.N, bn = p.bn, nstages = p.stages, nseg = p.nseg;
  const int mn3d_a = p.mn3d_a, mn3d_b = p.mn3d_b, no_loads = p.test_no_loads;
  const uint32_t stage_bytes = p.stage_bytes;
  const CUtensorMap* maps = p.maps;
  const int bnl = bn / PAIR;  // B rows (N) held by this CTA
  int stage = 0;
  uint32_t phase = 0;
  uint32_t issued_mask = 0, issued_par = 0;
  const uint32_t a_bytes = BM * BK * 2;
  const uint32_t b_bytes = static_cast<uint32_t>(bnl) * BK * 2;
  const uint64_t pol_first = policy_evict_first(), pol_last = policy_evict_last();
  bool ok = true;
  for (int t = unit0; t < sc.total && ok; t += nunits) {
    int mt, nt, ks;
    decode_tile(sc, t, mt, nt, ks);
    const int mbase = mt * BM * PAIR * MT, n0 = nt * bn;
    for (int s = 0; s < nseg && ok; ++s) {
      const SegR sg = seg_of(p, s);
      int kb0, kb1;
      seg_kb_range(sc, sg.k_len, ks, kb0, kb1);
      // Bytes landing per stage for CTA rank rr.  Boxes that would lie entirely
      // outside the matrix are skipped: the rows / columns they feed are never stored.
      auto bytes_of = [&](uint32_t rr) -> uint32_t {
        uint32_t by = 0;
#pragma unroll
        for (int h = 0; h < MT; ++h) {  // M tile h of the unit: rows mbase + h * BM * PAIR + ...
          const int m0r = mbase + h * BM * PAIR + static_cast<int>(rr) * BM;
          if (A_MN) by += mn3d_a ? (m0r < M ? 16384u : 0u) : (m0r < M ? 8192u : 0u) + (m0r + 64 < M ? 8192u : 0u);
          else by += (m0r < M ? a_bytes : 0u);
        }
        const int nb0 = FUSE ? n0 : n0 + static_cast<int>(rr) * bnl;
        uint32_t bb = 0;
        if (B_MN) {
          if (mn3d_b) {
            bb = nb0 < N ? b_bytes : 0u;
          } else {
            for (int c = 0; c < bnl / 64; ++c)
              if (nb0 + 64 * c < N) bb += 8192u;
          }
        } else {
          bb = nb0 < N ? b_bytes : 0u;
        }
        if (!(Q4 && sg.q4)) {  // 4-bit B is written by the dequant warps instead
#pragma unroll
          for (int a = 0; a < NACC; ++a)
            if (seg_bmap(sg, a) >= 0) by += bb;
        }
        return by;
      };
      const uint32_t stage_tx = PAIR == 1 ? bytes_of(0) : (rank == 0 ? bytes_of(0) + bytes_of(1) : 0u);
      const int m0 = mbase + static_cast<int>(rank) * BM;
      const int nb0 = FUSE ? n0 : n0 + static_cast<int>(rank) * bnl;
      const CUtensorMap* am = maps + sg.a_map;
      for (int kb = kb0; kb < kb1; ++kb) {
        const uint32_t full = full0 + 8 * stage, empty = empty0 + 8 * stage;
        if (!mbar_wait(empty, phase ^ 1, wc, kDevTimeoutProducer)) {
          ok = false;
          break;
        }
        if (no_loads) {  // nothing issued, nothing armed: no copy can be in flight
          if (++stage == nstages) {
            stage = 0;
            phase ^= 1;
          }
          continue;
        }
        if (stage_tx) mbar_expect_tx(full, stage_tx);
        const uint32_t bar = PAIR == 1 ? full : mapa_shared(full, 0);
        const uint32_t sA = smem_u32(tiles + static_cast<size_t>(stage) * stage_bytes);
        const int k = kb * BK;
        int hint = sg.a_hint;
        auto load = [&](uint32_t dst, const CUtensorMap* m, int x, int y) {
          if (hint == HINT_NONE) {
            if (PAIR == 1) tma_load_2d(dst, m, bar, x, y);
            else tma_load_2d_pair(dst, m, bar, x, y);
          } else {
            const uint64_t pol = hint == HINT_EVICT_LAST ? pol_last : pol_first;
            if (PAIR == 1) tma_load_2d_hint(dst, m, bar, x, y, pol);
            else tma_load_2d_pair_hint(dst, m, bar, x, y, pol);
          }
        };
        // one 3-D box = all 64-column chunks of an MN-major operand tile, K rows [y, y + 64)
        auto load3 = [&](uint32_t dst, const CUtensorMap* m, int y, int z) {
          if (PAIR == 1) tma_load_3d(dst, m, bar, 0, y, z);
          else tma_load_3d_pair(dst, m, bar, 0, y, z);
        };
        if (A_MN && mn3d_a) {
          if (m0 < M) load3(sA, am, sg.a_k0 + k, m0 / 64);
        } else if (A_MN) {
          if (m0 < M) load(sA, am, m0, sg.a_k0 + k);
          if (m0 + 64 < M) load(sA + 8192, am, m0 + 64, sg.a_k0 + k);
        } else {
#pragma unroll
          for (int h = 0; h < MT; ++h)
            if (m0 + h * BM * PAIR < M) load(sA + h * a_bytes, am, sg.a_k0 + k, m0 + h * BM * PAIR);
        }
        hint = sg.b_hint;
        if (Q4 && sg.q4) {
          // 4-bit B: the dequant warps fill the B slots from the code ring
        } else if (FUSE) {
          // branch r fills B rows [r * bn, (r + 1) * bn) of the wide tile; a CTA of a
          // pair holds only its own branch
          const uint32_t sB = sA + MT * a_bytes;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            if (PAIR == 2 && static_cast<uint32_t>(r) != rank) continue;
            const uint32_t dst = PAIR == 2 ? sB : sB + r * bn * BK * 2;
            load(dst, maps + seg_bmap(sg, r), seg_bk0(sg, r) + k, n0);
          }
        } else {
#pragma unroll
          for (int a = 0; a < NACC; ++a) {
            if (seg_bmap(sg, a) < 0) continue;
            const uint32_t sB = sA + MT * a_bytes + a * b_bytes;
            const CUtensorMap* bm = maps + seg_bmap(sg, a);
            if (B_MN && mn3d_b) {
              if (nb0 < N) load3(sB, bm, seg_bk0(sg, a) + k, nb0 / 64);
            } else if (B_MN) {
              for (int c = 0; c < bnl / 64; ++c)
                if (nb0 + 64 * c < N) load(sB + c * 8192, bm, nb0 + 64 * c, seg_bk0(sg, a) + k);
            } else if (nb0 < N) {
              load(sB, bm, seg_bk0(sg, a) + k, nb0);
            }
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
  }
  if (!ok) {
    // Aborting: make sure no TMA write into shared memory is still in flight (the
    // even CTA's full barriers also count the odd CTA's bytes).
    for (int s = 0; s < nstages; ++s) {
      if (!(issued_mask & (1u << s))) continue;
      if (rank == 0) drain_wait(full0 + 8 * s, (issued_par >> s) & 1, wc);
    }
  }
}

template <int A_MN, int B_MN, int NACC, int PAIR, int FUSE, int Q4, int MT>
__device__ __forceinline__ void gemm_mma(const GemmArgs& p, uint8_t* tiles, uint32_t full0,
                                         uint32_t empty0, uint32_t tfull0, uint32_t tempty0,
                                         uint32_t drain_bar, uint32_t tmem_base,
                                         const WaitCtl& wc, uint32_t dq0) {
  const Sched sc = sched_of(p);
  const int total = sc.total;
  const int unit0 = blockIdx.x / PAIR, nunits = gridDim.x / PAIR;
  const uint32_t idesc = idesc_bf16(BM * PAIR, FUSE ? 2 * p.bn : p.bn, A_MN, B_MN);
  const uint32_t a_bytes = BM * BK * 2;
  const uint32_t b_bytes = static_cast<uint32_t>(p.bn / PAIR) * BK * 2;
  const uint32_t tiles_u32 = smem_u32(tiles);
  // launch constants in registers: the asm statements below clobber memory, which would
  // otherwise make the compiler re-read them from the parameter space in the issue loop
  const int nstages = p.stages, nseg = p.nseg, bn = p.bn, nbuf = p.nbuf;
  const uint32_t stage_bytes = p.stage_bytes;
  int stage = 0;
  uint32_t phase = 0;
  uint32_t it = 0;
  bool ok = true, issued_any = false;
  bool ready = false;  // the current stage's full barrier was seen complete by a peek
  for (int t = unit0; t < total && ok; t += nunits, ++it) {
    int mt, nt, ks;
    decode_tile(sc, t, mt, nt, ks);
    const uint32_t buf = nbuf == 2 ? (it & 1) : 0, aphase = nbuf == 2 ? (it >> 1) & 1 : it & 1;
    if (!mbar_wait(tempty0 + 8 * buf, aphase ^ 1, wc, kDevTimeoutMma)) {
      ok = false;
      break;
    }
    tc_fence_after();
    uint32_t started = 0;  // bit h * NACC + a: accumulator a of M tile h has its first product
    for (int s = 0; s < nseg && ok; ++s) {
      const SegR sg = seg_of(p, s);
      int kb0, kb1;
      seg_kb_range(sc, sg.k_len, ks, kb0, kb1);
      const int k_len = sg.k_len;
      uint32_t bmask = 0;  // accumulators this segment feeds
#pragma unroll
      for (int a = 0; a < NACC; ++a)
        if (seg_bmap(sg, a) >= 0) bmask |= 1u << a;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!ready && !mbar_wait(full0 + 8 * stage, phase, wc, kDevTimeoutMma)) {
          ok = false;
          break;
        }
        if (Q4 && !mbar_wait(dq0 + 8 * stage, phase, wc, kDevTimeoutMma)) {  // B tiles expanded (both CTAs)
          ok = false;
          break;
        }
        tc_fence_after();
        const int rem = k_len - kb * BK;
        const uint32_t sA = tiles_u32 + static_cast<uint32_t>(stage) * stage_bytes;
        // Peek at the next stage of the ring (the next tile's first, at a tile's end)
        // while the MMAs below issue: when its copies have landed no wait separates
        // these MMAs from the next ones, and the tensor pipe does not drain between
        // stages.
        {
          const int ns = stage + 1 == nstages ? 0 : stage + 1;
          ready = mbar_peek(full0 + 8 * ns, ns == 0 ? phase ^ 1u : phase);
        }
        // descriptors of k-step 0; later k-steps only move the start address
        // (+32 B in a K-major 128-byte row, +2048 B = 16 rows for MN-major)
        constexpr uint32_t a_step = A_MN ? (2048 >> 4) : (32 >> 4);
        constexpr uint32_t b_step = B_MN ? (2048 >> 4) : (32 >> 4);
#pragma unroll
        for (int h = 0; h < MT; ++h) {  // M tile h: its own A sub-tile and accumulator set
          const uint32_t sAh = sA + h * a_bytes;
          const uint64_t ad0 = A_MN ? sdesc_sw128(sAh, 8192, 1024) : sdesc_sw128(sAh, 16, 1024);
#pragma unroll
          for (int a = 0; a < (FUSE ? 1 : NACC); ++a) {
            if (!((bmask >> a) & 1u)) continue;
            const uint32_t sB = sA + MT * a_bytes + a * b_bytes;
            const uint64_t bd0 = B_MN ? sdesc_sw128(sB, 8192, 1024) : sdesc_sw128(sB, 16, 1024);
            const uint32_t d = tmem_base + buf * (MT * NACC * bn) + h * (NACC * bn) + a * bn;
            const int bit = h * NACC + a;
            const uint32_t acc0 = (started >> bit) & 1;
            if (rem >= BK) {
#pragma unroll
              for (int j = 0; j < BK / 16; ++j) {
                if (PAIR == 1) mma_bf16(d, ad0 + j * a_step, bd0 + j * b_step, idesc, j ? 1u : acc0);
                else mma_bf16_pair(d, ad0 + j * a_step, bd0 + j * b_step, idesc, j ? 1u : acc0);
              }
            } else {
              const int nsteps = (rem + 15) / 16;
              for (int j = 0; j < nsteps; ++j) {
                if (PAIR == 1) mma_bf16(d, ad0 + j * a_step, bd0 + j * b_step, idesc, j ? 1u : acc0);
                else mma_bf16_pair(d, ad0 + j * a_step, bd0 + j * b_step, idesc, j ? 1u : acc0);
              }
            }
            started |= 1u << bit;
            issued_any = true;
          }
        }
        // frees the smem stage (in both CTAs of a pair) once these MMAs finish
        if (PAIR == 1) mma_commit(empty0 + 8 * stage);
        else mma_commit_pair(empty0 + 8 * stage, 0x3);
        if (++stage == nstages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (ok) {  // accumulator ready for the epilogue(s)
      if (PAIR == 1) mma_commit(tfull0 + 8 * buf);
      else mma_commit_pair(tfull0 + 8 * buf, 0x3);
    }
  }
  if (!ok && issued_any) {
    // Aborting: wait for the MMAs already issued before TMEM is released.
    if (PAIR == 1) mma_commit(drain_bar);
    else mma_commit_pair(drain_bar, 0x1);
    drain_wait(drain_bar, 0, wc);
  }
}

template <class V>
__device__ __forceinline__ void st_out(V* ptr, const V& v, int streaming) {
  if (streaming) __stcs(ptr, v);
  else *ptr = v;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
// sigmoid(g) = 1 / (1 + e^-g); for g << 0 the reciprocal of +inf is 0.
__device__ __forceinline__ float sigmoid_f(float g) { return rcp_approx(1.0f + __expf(-g)); }
__device__ __forceinline__ float silu_f(float g) { return g * sigmoid_f(g); }

template <int NACC, int EPI, int PAIR, int MT, int Q4>
__device__ __forceinline__ void gemm_epilogue(const GemmArgs& p, uint32_t tfull0, uint32_t tempty0,
                                              uint32_t tmem_base, const WaitCtl& wc, uint32_t rank,
                                              uint8_t* stage_out) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int q = warp & 3;             // TMEM lane quarter this warp may access
  const int c0 = ((warp - 2) >> 2) * 16;  // first 16-column chunk of this warp; stride 32
  const Sched sc = sched_of(p);
  const int total = sc.total;
  const int unit0 = blockIdx.x / PAIR, nunits = gridDim.x / PAIR;
  // launch constants in registers (see Sched)
  const int bn = p.bn, N = p.N, M = p.M, stream_out = p.stream_out, out_acc_col = p.out_acc_col;
  const int out_add = p.out_add, nrng = p.nrng, nbuf = p.nbuf;
  const float alpha = p.alpha;
  const long long ld_out = p.ld_out, ld_in = p.ld_in, split_stride = p.split_stride;
  void* const out0 = p.out[0];
  void* const out1 = p.out[1];
  void* const out2 = p.out[2];
  const void* const in0 = p.in[0];
  const void* const in1 = p.in[1];
  const int* const ce_labels = p.ce_labels;
  const float* const ce_lse = p.ce_lse;
  const int* const ce_count = p.ce_count;
  const float ce_g = p.ce_g;
  const int ce_col0 = p.ce_col0, ce_V = p.ce_V;
  const int epi_tma = p.epi_tma;
  // whole 16-column pieces of a row go out (come in) as one 32-byte access when aligned
  const bool v8_out = ld_out % 16 == 0 && ((reinterpret_cast<uintptr_t>(out0) | reinterpret_cast<uintptr_t>(out1) |
                                            reinterpret_cast<uintptr_t>(out2)) & 31) == 0;
  const bool v8_in = ld_in % 16 == 0 && ((reinterpret_cast<uintptr_t>(in0) | reinterpret_cast<uintptr_t>(in1)) & 31) == 0;
  const bool v8_f32 = v8_out && ld_out % 8 == 0 && split_stride % 8 == 0 && out_acc_col % 8 == 0;
  const bool v8_bf16 = v8_out && out_acc_col % 16 == 0 && (!in0 || v8_in);
  const CUtensorMap* const out_maps = p.maps + p.out_map0;
  const uint32_t stg = smem_u32(stage_out) + static_cast<uint32_t>(warp - 2) * kEpiStageBytes;  // this warp's
  uint32_t it = 0;
  for (int t = unit0; t < total; t += nunits, ++it) {
    int mt, nt, ks;
    decode_tile(sc, t, mt, nt, ks);
    const uint32_t buf = nbuf == 2 ? (it & 1) : 0, aphase = nbuf == 2 ? (it >> 1) & 1 : it & 1;
    int ok = 1;
    if (lane == 0) ok = mbar_wait(tfull0 + 8 * buf, aphase, wc, kDevTimeoutEpilogue) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) break;
    tc_fence_after();
    const int n0 = nt * bn;
    if constexpr (MT == 2 && !Q4 && ((EPI == EPI_BF16 && NACC == 1) || (EPI == EPI_SWIGLU_FWD && NACC == 2))) {
      if (epi_tma && p.epi_drain) {
        // With one accumulator set, the next unit's main loop waits for this epilogue.  So the
        // warp reads its share of the accumulators out of TMEM into registers, rounded to bf16
        // and packed two to a word, and releases TMEM before it converts and stores them: the
        // stores then run under the next main loop.  epi_drain 2 holds both M tiles (2 x 64
        // words a lane); 1 holds the second only and sends the first out straight from TMEM.
        // A chunk is 16 columns: bf16 out has 8 a tile (N tile 256); SwiGLU has 4 of G and 4 of
        // U a tile (N tile 128 each), and Act = silu(G) U is formed from the rounded G and U.
        constexpr int kChunks = EPI == EPI_BF16 ? 8 : 4;
        const int full = p.epi_drain == 2;
        // the packed words of chunk i of tile h (G's 8 words, then U's 8 for SwiGLU)
        auto read_chunk = [&](int h, int i, uint32_t (&w)[2][8]) {
          const int m0 = (mt * 2 + h) * BM * PAIR + static_cast<int>(rank) * BM;
          const long long row = static_cast<long long>(m0) + 32 * q + lane;
          const uint32_t tbase =
              tmem_base + (static_cast<uint32_t>(32 * q) << 16) + buf * (MT * NACC * bn) + h * (NACC * bn);
#pragma unroll
          for (int a = 0; a < (EPI == EPI_BF16 ? 1 : 2); ++a) {
            const int c = a * bn + c0 + 32 * i;
            uint32_t r[16];
            tmem_ld16(tbase + c, r);
            tmem_wait16(r);
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = EPI == EPI_BF16 ? __uint_as_float(r[e]) * alpha : __uint_as_float(r[e]);
            if (EPI == EPI_BF16 && in0) {  // residual input (bf16, same layout as the output) added in fp32
              const int n = n0 + c;
#pragma unroll
              for (int hh = 0; hh < 2; ++hh)
                if (row < M && n + 8 * hh < N) {
                  const uint4 xv = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in0) +
                                                                       row * ld_in + n + 8 * hh));
                  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    v[8 * hh + 2 * k] += bf16lo(xw[k]);
                    v[8 * hh + 2 * k + 1] += bf16hi(xw[k]);
                  }
                }
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) w[a][k] = pack_bf16x2(v[2 * k], v[2 * k + 1]);
          }
        };
        // chunk i of tile h through the staging tiles and out by TMA stores
        auto emit_chunk = [&](int h, int i, const uint32_t (&w)[2][8]) {
          const int row0 = (mt * 2 + h) * BM * PAIR + static_cast<int>(rank) * BM + 32 * q;
          const int n = n0 + c0 + 32 * i;
          if (lane == 0) bulk_wait_read0();  // the previous chunk's stores have read the staging
          __syncwarp();
          const uint32_t o = stg + static_cast<uint32_t>(lane) * 32u;
          if (EPI == EPI_SWIGLU_FWD) {
            uint32_t pa[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              pa[k] = pack_bf16x2(silu_f(bf16lo(w[0][k])) * bf16lo(w[1][k]), silu_f(bf16hi(w[0][k])) * bf16hi(w[1][k]));
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t a4[4] = {pa[4 * hh], pa[4 * hh + 1], pa[4 * hh + 2], pa[4 * hh + 3]};
              st_shared_v4(o + 2048u + 16u * hh, a4);
            }
          }
#pragma unroll
          for (int a = 0; a < (EPI == EPI_BF16 ? 1 : 2); ++a)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t w4[4] = {w[a][4 * hh], w[a][4 * hh + 1], w[a][4 * hh + 2], w[a][4 * hh + 3]};
              st_shared_v4(o + 1024u * a + 16u * hh, w4);
            }
          fence_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < M && n < N) {
            tma_store_2d(out_maps + 0, stg, n, row0);
            if (EPI == EPI_SWIGLU_FWD) {
              tma_store_2d(out_maps + 1, stg + 1024u, n, row0);
              tma_store_2d(out_maps + 2, stg + 2048u, n, row0);
            }
            bulk_commit();
          }
        };
        uint32_t hold[2][kChunks][2][8];
        if (full) {
#pragma unroll
          for (int i = 0; i < kChunks; ++i) read_chunk(0, i, hold[0][i]);
        } else {
#pragma unroll 1
          for (int i = 0; i < kChunks; ++i) {
            uint32_t w[2][8];
            read_chunk(0, i, w);
            emit_chunk(0, i, w);
          }
        }
#pragma unroll
        for (int i = 0; i < kChunks; ++i) read_chunk(1, i, hold[1][i]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR == 1) mbar_arrive(tempty0 + 8 * buf);
          else mbar_arrive_cluster(mapa_shared(tempty0 + 8 * buf, 0));  // the MMA issuer's barrier
        }
        if (full) {
#pragma unroll
          for (int i = 0; i < kChunks; ++i) emit_chunk(0, i, hold[0][i]);
        }
#pragma unroll
        for (int i = 0; i < kChunks; ++i) emit_chunk(1, i, hold[1][i]);
        continue;
      }
    }
#pragma unroll 1
    for (int h = 0; h < MT; ++h) {  // the unit's M tiles, each with its own accumulator set
    const int m0 = (mt * MT + h) * BM * PAIR + static_cast<int>(rank) * BM;
    const long long row = static_cast<long long>(m0) + 32 * q + lane;
    const bool row_ok = row < M;
    const uint32_t tbase = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + buf * (MT * NACC * bn) + h * (NACC * bn);

    if ((EPI == EPI_F32 || EPI == EPI_BF16) && NACC == 1 && epi_tma) {
      // The warp's 32 rows x 16 columns leave by one TMA store (fp32 with out_add: a TMA
      // add-reduction into the old values) from its staging tile
      const int row0 = m0 + 32 * q;
#pragma unroll 1
      for (int c = c0; c < bn; c += 32) {
        uint32_t r[16];
        tmem_ld16(tbase + c, r);
        tmem_wait16(r);
        const int n = n0 + c;
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
        if (EPI == EPI_F32) {
          const uint32_t o = stg + static_cast<uint32_t>(lane) * 64u;
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const uint32_t w[4] = {__float_as_uint(__uint_as_float(r[4 * h]) * alpha),
                                   __float_as_uint(__uint_as_float(r[4 * h + 1]) * alpha),
                                   __float_as_uint(__uint_as_float(r[4 * h + 2]) * alpha),
                                   __float_as_uint(__uint_as_float(r[4 * h + 3]) * alpha)};
            st_shared_v4(o + 16u * h, w);
          }
        } else {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float v8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v8[e] = __uint_as_float(r[8 * h + e]) * alpha;
            if (in0 && row_ok && n + 8 * h < N) {  // residual input (bf16, same layout as the output)
              const uint4 xv = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in0) +
                                                                   row * ld_in + n + 8 * h));
              v8[0] += bf16lo(xv.x); v8[1] += bf16hi(xv.x); v8[2] += bf16lo(xv.y); v8[3] += bf16hi(xv.y);
              v8[4] += bf16lo(xv.z); v8[5] += bf16hi(xv.z); v8[6] += bf16lo(xv.w); v8[7] += bf16hi(xv.w);
            }
            const uint32_t w[4] = {pack_bf16x2(v8[0], v8[1]), pack_bf16x2(v8[2], v8[3]), pack_bf16x2(v8[4], v8[5]),
                                   pack_bf16x2(v8[6], v8[7])};
            st_shared_v4(stg + static_cast<uint32_t>(lane) * 32u + 16u * h, w);
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < M && n < N) {
          if (EPI == EPI_F32 && out_add) tma_reduce_add_2d(out_maps, stg, n, row0);
          else tma_store_2d(out_maps, stg, n, row0);
          bulk_commit();
        }
      }
    } else if (EPI == EPI_F32 || EPI == EPI_BF16) {
#pragma unroll 1
      for (int a = 0; a < NACC; ++a) {
#pragma unroll 1
        for (int c = c0; c < bn; c += 32) {
          uint32_t r[16];
          tmem_ld16(tbase + a * bn + c, r);
          tmem_wait16(r);
          const int n = n0 + c;
          if (!row_ok) continue;
          if (EPI == EPI_F32) {
            float* o = static_cast<float*>(out0) + ks * split_stride + row * ld_out +
                       a * out_acc_col + n;
            if (v8_f32 && n + 16 <= N) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                uint32_t w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) w[e] = __float_as_uint(__uint_as_float(r[8 * h + e]) * alpha);
                if (out_add) {
                  uint32_t old[8];
                  ld_global_v8(o + 8 * h, old, 1);
#pragma unroll
                  for (int e = 0; e < 8; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) + __uint_as_float(old[e]));
                }
                st_global_v8(o + 8 * h, w, stream_out);
              }
              continue;
            }
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              if (n + 4 * h < N) {
                float4 v = make_float4(__uint_as_float(r[4 * h]) * alpha,
                                       __uint_as_float(r[4 * h + 1]) * alpha,
                                       __uint_as_float(r[4 * h + 2]) * alpha,
                                       __uint_as_float(r[4 * h + 3]) * alpha);
                if (out_add) {
                  const float4 old = *reinterpret_cast<const float4*>(o + 4 * h);
                  v.x += old.x; v.y += old.y; v.z += old.z; v.w += old.w;
                }
                st_out(reinterpret_cast<float4*>(o + 4 * h), v, stream_out);
              }
            }
          } else {
            uint16_t* o = static_cast<uint16_t*>(out0) + row * ld_out + a * out_acc_col + n;
            if (v8_bf16 && n + 16 <= N) {
              float v16[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) v16[e] = __uint_as_float(r[e]) * alpha;
              if (in0) {  // residual input (bf16, same layout as the output) added in fp32
                uint32_t x8[8];
                ld_global_v8(static_cast<const uint16_t*>(in0) + row * ld_in + n, x8, 0);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  v16[2 * j] += bf16lo(x8[j]);
                  v16[2 * j + 1] += bf16hi(x8[j]);
                }
              }
              uint32_t w[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) w[j] = pack_bf16x2(v16[2 * j], v16[2 * j + 1]);
              st_global_v8(o, w, stream_out);
              continue;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (n + 8 * h < N) {
                float v8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = __uint_as_float(r[8 * h + e]) * alpha;
                if (in0) {  // residual input (bf16, same layout as the output) added in fp32
                  float x8[8];
                  const uint4 xv = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in0) +
                                                                       row * ld_in + n + 8 * h));
                  x8[0] = bf16lo(xv.x); x8[1] = bf16hi(xv.x); x8[2] = bf16lo(xv.y); x8[3] = bf16hi(xv.y);
                  x8[4] = bf16lo(xv.z); x8[5] = bf16hi(xv.z); x8[6] = bf16lo(xv.w); x8[7] = bf16hi(xv.w);
#pragma unroll
                  for (int e = 0; e < 8; ++e) v8[e] += x8[e];
                }
                uint4 v;
                v.x = pack_bf16x2(v8[0], v8[1]);
                v.y = pack_bf16x2(v8[2], v8[3]);
                v.z = pack_bf16x2(v8[4], v8[5]);
                v.w = pack_bf16x2(v8[6], v8[7]);
                st_out(reinterpret_cast<uint4*>(o + 8 * h), v, stream_out);
              }
            }
          }
        }
      }
    } else if (EPI == EPI_SWIGLU_FWD && epi_tma) {
      // The warp's 32 rows x 16 columns of G, U and Act go to its staging tiles, then out by
      // three TMA stores (whole 32-byte rows of the box per write instead of a 16-byte piece of
      // 32 different rows per store instruction); boxes are clipped at the tensor's end.
      const int row0 = m0 + 32 * q;
#pragma unroll 1
      for (int c = c0; c < bn; c += 32) {
        uint32_t rg[16], ru[16];
        tmem_ld16(tbase + c, rg);
        tmem_ld16(tbase + bn + c, ru);
        tmem_wait32(rg, ru);
        const int n = n0 + c;
        if (lane == 0) bulk_wait_read0();  // the previous chunk's stores have read the staging tiles
        __syncwarp();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pg[4], pu[4], pa[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float g0 = __uint_as_float(rg[8 * h + 2 * j]), g1 = __uint_as_float(rg[8 * h + 2 * j + 1]);
            const float u0 = __uint_as_float(ru[8 * h + 2 * j]), u1 = __uint_as_float(ru[8 * h + 2 * j + 1]);
            pg[j] = pack_bf16x2(g0, g1);
            pu[j] = pack_bf16x2(u0, u1);
            pa[j] = pack_bf16x2(silu_f(g0) * u0, silu_f(g1) * u1);
          }
          const uint32_t o = stg + static_cast<uint32_t>(lane) * 32u + 16u * h;
          st_shared_v4(o, pg);
          st_shared_v4(o + 1024u, pu);
          st_shared_v4(o + 2048u, pa);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < M && n < N) {
          tma_store_2d(out_maps + 0, stg, n, row0);
          tma_store_2d(out_maps + 1, stg + 1024u, n, row0);
          tma_store_2d(out_maps + 2, stg + 2048u, n, row0);
          bulk_commit();
        }
      }
    } else if (EPI == EPI_SWIGLU_FWD) {
#pragma unroll 1
      for (int c = c0; c < bn; c += 32) {
        uint32_t rg[16], ru[16];
        tmem_ld16(tbase + c, rg);
        tmem_ld16(tbase + bn + c, ru);
        tmem_wait32(rg, ru);
        const int n = n0 + c;
        if (!row_ok) continue;
        const long long off = row * ld_out + n;
        if (v8_out && n + 16 <= N) {
          uint32_t g8[8], u8[8], a8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float g0 = __uint_as_float(rg[2 * j]), g1 = __uint_as_float(rg[2 * j + 1]);
            const float u0 = __uint_as_float(ru[2 * j]), u1 = __uint_as_float(ru[2 * j + 1]);
            g8[j] = pack_bf16x2(g0, g1);
            u8[j] = pack_bf16x2(u0, u1);
            a8[j] = pack_bf16x2(silu_f(g0) * u0, silu_f(g1) * u1);
          }
          st_global_v8(static_cast<uint16_t*>(out0) + off, g8, stream_out);
          st_global_v8(static_cast<uint16_t*>(out1) + off, u8, stream_out);
          st_global_v8(static_cast<uint16_t*>(out2) + off, a8, stream_out);
          continue;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (n + 8 * h >= N) continue;
          uint32_t pg[4], pu[4], pa[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float g0 = __uint_as_float(rg[8 * h + 2 * j]), g1 = __uint_as_float(rg[8 * h + 2 * j + 1]);
            const float u0 = __uint_as_float(ru[8 * h + 2 * j]), u1 = __uint_as_float(ru[8 * h + 2 * j + 1]);
            pg[j] = pack_bf16x2(g0, g1);
            pu[j] = pack_bf16x2(u0, u1);
            pa[j] = pack_bf16x2(silu_f(g0) * u0, silu_f(g1) * u1);
          }
          st_out(reinterpret_cast<uint4*>(static_cast<uint16_t*>(out0) + off + 8 * h), make_uint4(pg[0], pg[1], pg[2], pg[3]), stream_out);
          st_out(reinterpret_cast<uint4*>(static_cast<uint16_t*>(out1) + off + 8 * h), make_uint4(pu[0], pu[1], pu[2], pu[3]), stream_out);
          st_out(reinterpret_cast<uint4*>(static_cast<uint16_t*>(out2) + off + 8 * h), make_uint4(pa[0], pa[1], pa[2], pa[3]), stream_out);
        }
      }
    } else if (EPI == EPI_SWIGLU_BWD) {
#pragma unroll 1
      for (int c = c0; c < bn; c += 32) {
        const int n = n0 + c;
        uint4 gv[2], uv[2];
        if (v8_in && row_ok && n + 16 <= N) {
          uint32_t g8[8], u8[8];
          const long long off = row * ld_in + n;
          ld_global_v8(static_cast<const uint16_t*>(in0) + off, g8, 1);
          ld_global_v8(static_cast<const uint16_t*>(in1) + off, u8, 1);
          gv[0] = make_uint4(g8[0], g8[1], g8[2], g8[3]); gv[1] = make_uint4(g8[4], g8[5], g8[6], g8[7]);
          uv[0] = make_uint4(u8[0], u8[1], u8[2], u8[3]); uv[1] = make_uint4(u8[4], u8[5], u8[6], u8[7]);
        } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (row_ok && n + 8 * h < N) {
            const long long off = row * ld_in + n + 8 * h;
            // G and U are read once here: evict-first, so they do not displace the operand tiles
            gv[h] = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in0) + off));
            uv[h] = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in1) + off));
          } else {
            gv[h] = make_uint4(0, 0, 0, 0);
            uv[h] = make_uint4(0, 0, 0, 0);
          }
        }
        }
        uint32_t r[16];
        tmem_ld16(tbase + c, r);
        tmem_wait16(r);
        if (epi_tma) {
          // dG and dU of the warp's 32 rows x 16 columns leave by two TMA stores (see SwiGLU fwd)
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t gw[4] = {gv[h].x, gv[h].y, gv[h].z, gv[h].w};
            const uint32_t uw[4] = {uv[h].x, uv[h].y, uv[h].z, uv[h].w};
            uint32_t pdg[4], pdu[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float dg[2], du[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const float g = e ? bf16hi(gw[j]) : bf16lo(gw[j]);
                const float u = e ? bf16hi(uw[j]) : bf16lo(uw[j]);
                const float da = __uint_as_float(r[8 * h + 2 * j + e]);
                const float sg = sigmoid_f(g);
                du[e] = da * g * sg;
                dg[e] = da * u * sg * (1.0f + g * (1.0f - sg));
              }
              pdg[j] = pack_bf16x2(dg[0], dg[1]);
              pdu[j] = pack_bf16x2(du[0], du[1]);
            }
            const uint32_t o = stg + static_cast<uint32_t>(lane) * 32u + 16u * h;
            st_shared_v4(o, pdg);
            st_shared_v4(o + 1024u, pdu);
          }
          fence_async_smem();
          __syncwarp();
          const int row0 = m0 + 32 * q;
          if (lane == 0 && row0 < M && n < N) {
            tma_store_2d(out_maps + 0, stg, n, row0);
            tma_store_2d(out_maps + 1, stg + 1024u, n, row0);
            bulk_commit();
          }
          continue;
        }
        if (!row_ok) continue;
        const long long off = row * ld_out + n;
        uint32_t pdg[8], pdu[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t gw[4] = {gv[h].x, gv[h].y, gv[h].z, gv[h].w};
          const uint32_t uw[4] = {uv[h].x, uv[h].y, uv[h].z, uv[h].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float dg[2], du[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float g = e ? bf16hi(gw[j]) : bf16lo(gw[j]);
              const float u = e ? bf16hi(uw[j]) : bf16lo(uw[j]);
              const float da = __uint_as_float(r[8 * h + 2 * j + e]);
              const float sg = sigmoid_f(g);
              du[e] = da * g * sg;
              dg[e] = da * u * sg * (1.0f + g * (1.0f - sg));
            }
            pdg[4 * h + j] = pack_bf16x2(dg[0], dg[1]);
            pdu[4 * h + j] = pack_bf16x2(du[0], du[1]);
          }
        }
        if (v8_out && n + 16 <= N) {
          st_global_v8(static_cast<uint16_t*>(out0) + off, pdg, stream_out);
          st_global_v8(static_cast<uint16_t*>(out1) + off, pdu, stream_out);
          continue;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (n + 8 * h >= N) continue;
          st_out(reinterpret_cast<uint4*>(static_cast<uint16_t*>(out0) + off + 8 * h),
                 make_uint4(pdg[4 * h], pdg[4 * h + 1], pdg[4 * h + 2], pdg[4 * h + 3]), stream_out);
          st_out(reinterpret_cast<uint4*>(static_cast<uint16_t*>(out1) + off + 8 * h),
                 make_uint4(pdu[4 * h], pdu[4 * h + 1], pdu[4 * h + 2], pdu[4 * h + 3]), stream_out);
        }
      }
    } else if (EPI == EPI_ATOMIC) {
#pragma unroll 1
      for (int ri = 0; ri < nrng; ++ri) {
        const OutRange R = p.rng[ri];
#pragma unroll 1
        for (int c = c0; c < bn; c += 32) {
          const int n = n0 + c;
          if (n >= N) break;  // warp-uniform: remaining chunks are padding columns
          uint32_t r[16];
          tmem_ld16(tbase + R.acc * bn + c, r);
          tmem_wait16(r);
          if (!row_ok) continue;
          if (R.trans) {
            // out[n * ld + m]: lanes hold consecutive m -> coalesced across the warp
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (n + j < N) atomicAdd(R.out + static_cast<long long>(n + j) * R.ld + row, __uint_as_float(r[j]) * alpha);
          } else {
            // out[m * ld + n]: 16 consecutive columns of one row -> four 16-byte vector atomics
            float* o = R.out + row * R.ld + n;
#pragma unroll
            for (int h = 0; h < 4; ++h)
              if (n + 4 * h < N)
                atomicAdd(reinterpret_cast<float4*>(o + 4 * h),
                          make_float4(__uint_as_float(r[4 * h]) * alpha, __uint_as_float(r[4 * h + 1]) * alpha,
                                      __uint_as_float(r[4 * h + 2]) * alpha, __uint_as_float(r[4 * h + 3]) * alpha));
          }
        }
      }
    } else if (EPI == EPI_CE_LSE) {
      // Online max / sum of exponentials over this warp's 16-column chunks of the tile:
      // m = running max, s = sum exp(z - m) (base-2 exponentials of pre-scaled values).
      constexpr float kLog2e = 1.4426950408889634f;
      const int lab = row_ok ? __ldg(ce_labels + row) : -1;
      float m = -INFINITY, sum = 0.f, zl = 0.f;
      bool has = false;
#pragma unroll 1
      for (int c = c0; c < bn; c += 32) {
        const int n = n0 + c;
        if (n >= N) break;  // warp-uniform: the rest of the tile is past the vocabulary
        uint32_t r[16];
        tmem_ld16(tbase + c, r);
        tmem_wait16(r);
        if (!row_ok) continue;
        float v[16], cm = -INFINITY;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          v[e] = n + e < N ? __uint_as_float(r[e]) : -INFINITY;
          cm = fmaxf(cm, v[e]);
          if (ce_col0 + n + e == lab) {
            zl = v[e];
            has = true;
          }
        }
        const float mn = fmaxf(m, cm);
        const float ms = mn * kLog2e;
        float acc = sum * exp2f(fmaf(m, kLog2e, -ms));
#pragma unroll
        for (int e = 0; e < 16; ++e) acc += exp2f(fmaf(v[e], kLog2e, -ms));
        sum = acc;
        m = mn;
      }
      if (row_ok) {
        const int half = (warp - 2) >> 2;
        reinterpret_cast<float2*>(out0)[static_cast<long long>(2 * nt + half) * M + row] = make_float2(m, sum);
        if (has) static_cast<float*>(out1)[row] = zl;
      }
    } else if (EPI == EPI_CE_DZ) {
      // dZ = g' (exp(z - lse) - [column == label]); 0 for rows left out of the loss
      constexpr float kLog2e = 1.4426950408889634f;
      const int lab = row_ok ? __ldg(ce_labels + row) : -1;
      const bool keep = lab >= 0 && lab < ce_V;
      float gs = 0.f, l2 = 0.f;
      if (keep) {
        gs = ce_count ? ce_g / static_cast<float>(max(1, __ldg(ce_count))) : ce_g;
        l2 = __ldg(ce_lse + row) * kLog2e;
      }
#pragma unroll 1
      for (int c = c0; c < bn; c += 32) {
        const int n = n0 + c;
        if (n >= N) break;
        uint32_t r[16];
        tmem_ld16(tbase + c, r);
        tmem_wait16(r);
        if (epi_tma) {  // dZ of the warp's 32 rows x 16 columns leaves by one TMA store
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float dz[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int k = 8 * h + 2 * j + e;
                const float pr = exp2f(fmaf(__uint_as_float(r[k]), kLog2e, -l2));
                dz[e] = gs * (pr - (ce_col0 + n + k == lab ? 1.f : 0.f));
              }
              w[j] = pack_bf16x2(dz[0], dz[1]);
            }
            st_shared_v4(stg + static_cast<uint32_t>(lane) * 32u + 16u * h, w);
          }
          fence_async_smem();
          __syncwarp();
          const int row0 = m0 + 32 * q;
          if (lane == 0 && row0 < M) {
            tma_store_2d(out_maps, stg, n, row0);
            bulk_commit();
          }
          continue;
        }
        if (!row_ok) continue;
        uint16_t* o = static_cast<uint16_t*>(out0) + row * ld_out + n;
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float dz[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int k = 2 * j + e;
            const float pr = exp2f(fmaf(__uint_as_float(r[k]), kLog2e, -l2));
            dz[e] = gs * (pr - (ce_col0 + n + k == lab ? 1.f : 0.f));
          }
          w[j] = pack_bf16x2(dz[0], dz[1]);
        }
        if (v8_out && n + 16 <= N) {
          st_global_v8(o, w, stream_out);
          continue;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (n + 8 * h < N) st_out(reinterpret_cast<uint4*>(o + 8 * h), make_uint4(w[4 * h], w[4 * h + 1], w[4 * h + 2], w[4 * h + 3]), stream_out);
      }
    }
    }  // M tiles of the unit
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (PAIR == 1) mbar_arrive(tempty0 + 8 * buf);
      else mbar_arrive_cluster(mapa_shared(tempty0 + 8 * buf, 0));  // the MMA issuer's barrier
    }
  }
  if (epi_tma && lane == 0) bulk_wait0();  // the TMA stores are done before the CTA exits
}

// 4-bit code-ring producer (one thread of the code warp): for every stage of a 4-bit
// segment, copies this CTA's codes and block absmax into the next of kCodeRing ring
// entries once the dequant group that read the entry before has released it.  The copies
// thus run up to kCodeRing stages ahead of the expansion, outside the per-stage loop of
// A copy -> expansion -> MMA -> free.
template <int B_MN, int NACC, int PAIR, int FUSE, int MT>
__device__ __forceinline__ void gemm_code_producer(const GemmArgs& p, uint8_t* ring, uint32_t crfull0,
                                                   uint32_t crempty0, const WaitCtl& wc, uint32_t rank) {
  const Sched sc = sched_of(p);
  // launch constants in registers (see Sched)
  const int bn = p.bn, nseg = p.nseg;
  const uint32_t cr_bytes = p.cr_bytes;
  const CUtensorMap* maps = p.maps;
  const int total = sc.total;
  const int unit0 = blockIdx.x / PAIR, nunits = gridDim.x / PAIR;
  const Q4Layout QL = q4_layout(bn, PAIR, FUSE, B_MN, NACC);
  int e = 0;
  uint32_t phase = 0, issued_mask = 0, issued_par = 0;
  bool ok = true;
  for (int t = unit0; t < total && ok; t += nunits) {
    int mt, nt, ks;
    decode_tile(sc, t, mt, nt, ks);
    const int n0 = nt * bn;
    for (int s = 0; s < nseg && ok; ++s) {
      const SegR sg = seg_of(p, s);
      if (!sg.q4) continue;
      int kb0, kb1;
      seg_kb_range(sc, sg.k_len, ks, kb0, kb1);
      uint32_t code_tx = 0;
      for (int u = 0; u < (FUSE ? 2 : NACC); ++u) {
        if (FUSE && PAIR == 2 && static_cast<uint32_t>(u) != rank) continue;
        if (seg_bmap(sg, u) >= 0) code_tx += QL.q_unit + QL.m_unit;
      }
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(crempty0 + 8 * e, phase ^ 1, wc, kDevTimeoutProducer)) {
          ok = false;
          break;
        }
        const uint32_t bar = crfull0 + 8 * e;
        if (code_tx) mbar_expect_tx(bar, code_tx);
        else mbar_arrive(bar);
        const uint32_t sQ = smem_u32(ring + static_cast<size_t>(e) * cr_bytes);
        const uint32_t sM = sQ + QL.slots * QL.q_unit;
#pragma unroll
        for (int u = 0; u < (FUSE ? 2 : NACC); ++u) {
          if (FUSE && PAIR == 2 && static_cast<uint32_t>(u) != rank) continue;
          if (seg_bmap(sg, u) < 0) continue;
          const int slot = (FUSE && PAIR == 2) ? 0 : u;
          const int nq = FUSE ? n0 : n0 + static_cast<int>(rank) * (bn / PAIR);  // first B row / column here
          const CUtensorMap* qm = &maps[seg_bmap(sg, u)];
          const CUtensorMap* mm = &maps[seg_bam(sg, u)];
          const int kk = seg_bk0(sg, u) + kb * BK;
          if (B_MN) {
            tma_load_2d(sQ + slot * QL.q_unit, qm, bar, nq / 2, kk);
            tma_load_2d(sM + slot * QL.m_unit, mm, bar, (nq / 64) & ~3, kk);
          } else {
            tma_load_2d(sQ + slot * QL.q_unit, qm, bar, kk / 2, nq);
            tma_load_2d(sM + slot * QL.m_unit, mm, bar, (kk / 64) & ~3, nq);
          }
        }
        issued_mask |= 1u << e;
        issued_par = (issued_par & ~(1u << e)) | (phase << e);
        if (++e == code_ring(MT)) {
          e = 0;
          phase ^= 1;
        }
      }
    }
  }
  if (!ok) {  // aborting: no copy into the ring may still be in flight
    for (int i = 0; i < code_ring(MT); ++i)
      if (issued_mask & (1u << i)) drain_wait(crfull0 + 8 * i, (issued_par >> i) & 1, wc);
  }
}

// 4-bit B producer (kDqWarps warps per CTA, in kDqGroups groups that take turns:
// group g expands the stages with running index = g mod kDqGroups, so a thread has a
// whole 64-element row of work per stage it takes and the wait / fence / arrive cost
// is paid once per kDqGroups stages).  For each stage the group waits until the MMA has
// released the stage (its B slot is free) and for the stage's code-ring entry, expands
// every 128-byte B row (one 64-element quantisation
// block: one absmax) into the 128-byte-swizzled bf16 tile, makes the writes visible
// to the tensor core (async proxy) and arrives on the MMA issuer's dq barrier (the
// even CTA's when CTAs are paired).
//
// Expansion of one row: the 16 products bf16(fl32(code_e * absmax)) are formed once
// (fp32 multiply, one rounding, as every element would get alone) and kept as byte
// planes in registers, lo[0..3] / hi[0..3] = low / high bytes of entries 4q..4q+3.
// A code word holds 8 elements' 4-bit indices in nibble order, which is already the
// selector layout of prmt: the low 3 bits pick one of 8 entries from a plane pair,
// bit 3 picks the pair (entries 0..7 or 8..15) through a byte mask.
template <int B_MN, int NACC, int FUSE, int PAIR, int MT>
__device__ __forceinline__ void gemm_dequant(const GemmArgs& p, uint8_t* tiles, const uint8_t* ring,
                                             uint32_t empty0, uint32_t crfull0, uint32_t crempty0,
                                             uint32_t dq0, const float* tab, const WaitCtl& wc, uint32_t rank) {
  constexpr int kGroupWarps = kDqWarps / kDqGroups;
  const int tid = threadIdx.x - kGemmThreads;  // 0 .. 32 * kDqWarps - 1
  const int lane = threadIdx.x % 32;
  const int group = (tid >> 5) / kGroupWarps;
  const int gtid = tid % (32 * kGroupWarps);
  const Sched sc = sched_of(p);
  // launch constants in registers (see Sched)
  const int bn = p.bn, nseg = p.nseg, nstages = p.stages;
  const uint32_t cr_bytes = p.cr_bytes, stage_bytes = p.stage_bytes;
  const int total = sc.total;
  const int unit0 = blockIdx.x / PAIR, nunits = gridDim.x / PAIR;
  const uint32_t a_bytes = BM * BK * 2;
  const Q4Layout QL = q4_layout(bn, PAIR, FUSE, B_MN, NACC);
  const float* code = tab + lane;  // code value e at code[32 * e] (lane-replicated: conflict-free)
  int stage = 0, turn = 0, e = 0;
  uint32_t phase = 0, cphase = 0;
  bool ok = true;
  for (int t = unit0; t < total && ok; t += nunits) {
    int mt, nt, ks;
    decode_tile(sc, t, mt, nt, ks);
    const int n0 = nt * bn;
    for (int s = 0; s < nseg && ok; ++s) {
      const SegR sg = seg_of(p, s);
      int kb0, kb1;
      seg_kb_range(sc, sg.k_len, ks, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (turn == group) {
          // the stage's previous contents consumed by the MMA (B slot free), codes landed
          int w = 1;
          if (lane == 0) {
            w = mbar_wait(empty0 + 8 * stage, phase ^ 1, wc, kDevTimeoutProducer) ? 1 : 0;
            if (w && sg.q4) w = mbar_wait(crfull0 + 8 * e, cphase, wc, kDevTimeoutProducer) ? 1 : 0;
          }
          w = __shfl_sync(0xffffffffu, w, 0);
          if (!w) {
            ok = false;
            break;
          }
          if (sg.q4) {
            uint8_t* base = tiles + static_cast<size_t>(stage) * stage_bytes;
            const uint8_t* sQ = ring + static_cast<size_t>(e) * cr_bytes;
            const float* sM = reinterpret_cast<const float*>(sQ + QL.slots * QL.q_unit);
            const int kk = kb * BK;
            const int chunks = QL.cols >> 6;
            for (int u = 0; u < (FUSE ? 2 : NACC); ++u) {
              if (FUSE && PAIR == 2 && static_cast<uint32_t>(u) != rank) continue;
              if (seg_bmap(sg, u) < 0) continue;
              const int slot = (FUSE && PAIR == 2) ? 0 : u;
              const int nq = FUSE ? n0 : n0 + static_cast<int>(rank) * (bn / PAIR);
              const uint8_t* q = sQ + slot * QL.q_unit;
              const float* am = sM + slot * (QL.m_unit / 4);
              uint8_t* dst = base + MT * a_bytes + slot * QL.b_unit;
              for (int i = gtid; i < QL.cols; i += 32 * kGroupWarps) {
                const uint4* src;
                float sc;
                if (B_MN) {  // row i = (64-column chunk c, K row krow)
                  const int c = i >> 6, krow = i & 63;
                  src = reinterpret_cast<const uint4*>(q + krow * (chunks * 32) + c * 32);
                  sc = am[krow * 4 + ((nq >> 6) & 3) + c];
                } else {     // row i = B row (N index), 64 K elements
                  src = reinterpret_cast<const uint4*>(q + i * 32);
                  sc = am[i * 4 + ((kk >> 6) & 3)];
                }
                const uint4 c0 = src[0], c1 = src[1];
                uint32_t lo[4], hi[4];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                  const uint32_t w0 = pack_bf16x2(code[32 * (4 * g)] * sc, code[32 * (4 * g + 1)] * sc);
                  const uint32_t w1 = pack_bf16x2(code[32 * (4 * g + 2)] * sc, code[32 * (4 * g + 3)] * sc);
                  lo[g] = prmt(w0, w1, 0x6420u);
                  hi[g] = prmt(w0, w1, 0x7531u);
                }
                const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint8_t* row = dst + static_cast<size_t>(i) * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {  // word j = elements 8j .. 8j+7 = 16-byte piece j
                  const uint32_t m8 = (cw[j] >> 3) & 0x11111111u;  // bit 3 of every index
                  uint32_t o[4];
#pragma unroll
                  for (int h = 0; h < 2; ++h) {  // elements 8j + 4h .. 8j + 4h + 3
                    const uint32_t g16 = h ? (cw[j] >> 16) : cw[j];
                    const uint32_t sel = g16 & 0x7777u;
                    const uint32_t msk = prmt(0x0000FF00u, 0u, h ? (m8 >> 16) : m8);  // 0xFF where index >= 8
                    const uint32_t lb = (prmt(lo[0], lo[1], sel) & ~msk) | (prmt(lo[2], lo[3], sel) & msk);
                    const uint32_t hb = (prmt(hi[0], hi[1], sel) & ~msk) | (prmt(hi[2], hi[3], sel) & msk);
                    o[2 * h] = prmt(lb, hb, 0x5140u);
                    o[2 * h + 1] = prmt(lb, hb, 0x7362u);
                  }
                  *reinterpret_cast<uint4*>(row + ((j ^ (i & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
              }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          }
          __syncwarp();
          if (lane == 0) {
            if (sg.q4) mbar_arrive(crempty0 + 8 * e);  // ring entry read: free for the next copy
            if (PAIR == 1) mbar_arrive(dq0 + 8 * stage);
            else mbar_arrive_cluster(mapa_shared(dq0 + 8 * stage, 0));
          }
        }
        if (sg.q4 && ++e == code_ring(MT)) {
          e = 0;
          cphase ^= 1;
        }
        if (++turn == kDqGroups) turn = 0;
        if (++stage == nstages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  }
}

template <int A_MN, int B_MN, int NACC, int EPI, int PAIR, int FUSE, int Q4, int MT>
static __global__ void __launch_bounds__(gemm_threads(Q4), 1) gemm_kernel(const __grid_constant__ GemmArgs p) {
  static_assert(!FUSE || (NACC == 2 && !B_MN), "fused wide MMA: two K-major B halves");
  static_assert(!Q4 || !A_MN, "4-bit B: K-major A");
  static_assert(MT == 1 || (MT == 2 && !A_MN), "two M tiles per unit: K-major A");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = tiles + static_cast<size_t>(p.stages) * p.stage_bytes;  // Q4: code ring
  uint8_t* stage_out = ring + (Q4 ? static_cast<size_t>(code_ring(MT)) * p.cr_bytes : 0);  // epilogue staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage_out + (p.epi_tma ? kEpiWarps * kEpiStageBytes : 0));
  const int S = p.stages;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * S;
  const uint32_t tfull0 = empty0 + 8 * S;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t drain_bar = tempty0 + 16;
  const uint32_t dq0 = drain_bar + 8;             // Q4: per stage, one arrival per warp of the expanding group, per CTA
  const uint32_t crfull0 = dq0 + 8 * S;           // Q4: per ring entry, the code copy (TMA bytes)
  const uint32_t crempty0 = crfull0 + 8 * code_ring(MT);  // Q4: per ring entry, released by the expanding group
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5 + (Q4 ? S + 2 * code_ring(MT) : 0));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* tab = reinterpret_cast<float*>(tmem_slot + 4);  // Q4: code values replicated per lane, [16][32]
  if (Q4)
    for (int i = threadIdx.x; i < 16 * 32; i += blockDim.x) tab[i] = p.codebook[i / 32];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = PAIR == 1 ? 0u : cluster_ctarank();

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(tfull0, 1);
    mbar_init(tfull0 + 8, 1);
    mbar_init(tempty0, kEpiWarps * PAIR);
    mbar_init(tempty0 + 8, kEpiWarps * PAIR);
    mbar_init(drain_bar, 1);
    if (Q4) {
      for (int s = 0; s < S; ++s) mbar_init(dq0 + 8 * s, (kDqWarps / kDqGroups) * PAIR);
      for (int i = 0; i < code_ring(MT); ++i) {
        mbar_init(crfull0 + 8 * i, 1);
        mbar_init(crempty0 + 8 * i, kDqWarps / kDqGroups);
      }
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kMaxMaps; ++i) tma_prefetch_desc(&p.maps[i]);
  }
  if (warp == 1) {
    if (PAIR == 1) {
      tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
      tmem_relinquish();
    } else {
      tmem_alloc_pair(smem_u32(tmem_slot), p.tmem_cols);
      tmem_relinquish_pair();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR == 2) cluster_sync_all();  // peer barriers initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, p.limit_ns};

  if (warp == 0) {
    if (lane == 0) gemm_producer<A_MN, B_MN, NACC, PAIR, FUSE, Q4, MT>(p, tiles, full0, empty0, wc, rank);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0)
      gemm_mma<A_MN, B_MN, NACC, PAIR, FUSE, Q4, MT>(p, tiles, full0, empty0, tfull0, tempty0, drain_bar, tmem_base, wc, dq0);
    __syncwarp();
  } else if (warp < 2 + kEpiWarps) {
    gemm_epilogue<NACC, EPI, PAIR, MT, Q4>(p, tfull0, tempty0, tmem_base, wc, rank, stage_out);
  } else if (Q4 && warp < 2 + kEpiWarps + kDqWarps) {
    gemm_dequant<B_MN, NACC, FUSE, PAIR, MT>(p, tiles, ring, empty0, crfull0, crempty0, dq0, tab, wc, rank);
  } else if (Q4) {
    if (lane == 0) gemm_code_producer<B_MN, NACC, PAIR, FUSE, MT>(p, ring, crfull0, crempty0, wc, rank);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR == 2) cluster_sync_all();  // no CTA leaves while its pair may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    if (PAIR == 1) tmem_dealloc(tmem_base, p.tmem_cols);
    else tmem_dealloc_pair(tmem_base, p.tmem_cols);
  }
}

}  // namespace lm
