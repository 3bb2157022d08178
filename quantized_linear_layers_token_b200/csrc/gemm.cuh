// gemm.cuh -- stages 2 and 3: INT8 tensor-core GEMM (tcgen05, TMEM
// accumulators, TMA-fed shared-memory operands) with the fused INT32->FP16
// dequant and the sparse outlier compensation.
//
// Orientation ("weights as the 128-row operand"): a tile is 128 output
// channels n (the MMA M dimension, TMEM lanes) by BT tokens m (the MMA N
// dimension, TMEM columns).  Decode shapes (M = 1..16) stay on the tensor
// cores with an N = 16 instruction instead of padding tokens to 128.
//
// Work decomposition (persistent, stream-K): every tile is T iterations --
// nk K-steps of 128 INT8 codes, then the compensation steps -- and the
// tiles * T iterations are split evenly over one CTA per SM.  A CTA that
// covers a whole tile finishes it directly.  A CTA that covers part of a
// tile (at most its first and its last segment) stores its exact INT32
// partial sums with plain coalesced stores into one of its two scratch
// slots; the CTA whose contribution completes the tile's T iterations (a
// counter, no waiting) adds the partials of the tile's CTAs in a fixed order
// and runs the epilogue.  The compensation run of a tile is never split, so
// exactly one CTA computes it.  When tiles are plentiful the split points
// snap to whole tiles and no scratch is used.
//
// Pipeline: three shared-memory rings, each with its own producer, so no
// load waits behind another: the staging ring (INT4 formats) takes packed
// weight blocks straight from bulk copies and is released as soon as the
// converters have read a slot; the A ring holds the tensor core's weight
// operand (written by the converters, or copied for the INT8 format and for
// W_O^T) and the X ring its activation (or compensation) operand; both are
// released by tcgen05.commit.
//
// Warp roles:
//   warp 0        X producer: activation tiles (TMA, after the grid
//                 dependency on the previous kernel) and the compensation
//                 operands U hi/lo.
//   warp 1        allocates TMEM (two accumulator buffers when they fit); the
//                 whole warp runs the MMA loop and an elected lane issues
//                 tcgen05.mma and commits.
//   warp 2        weight producer: packed INT4 blocks into the staging ring,
//                 INT8 blocks and W_O^T blocks into the A ring; starts at once
//                 (weights do not depend on the previous kernel).
//   warps 3..     converters (INT4 formats): unpack the staged INT4 codes into
//                 the 128-byte-swizzled K-major INT8 operand (QQQ review,
//                 per-channel GEMM: INT4 -> INT8 by a left shift of 4;
//                 per-group GEMM: INT4 -> FP16, multiply by the folded ratio
//                 g/c, FP16 -> INT8 through the +128/+1024 bit trick done as
//                 one rounding); the first four are also the epilogue warps.
// Epilogue (Quaff notes, decoupled WAQ formula; QQQ review, fused INT32->FP16
// dequant): Y = fp16(a_m * (c'_n * acc + comp)), comp accumulated in fp32 on
// the tensor cores from W_O^T and U = XqO * (s - 1) carried as two fp16
// terms (hi and lo) into the same accumulator.
#pragma once

#include "sm100.cuh"

namespace qlin {

enum : int { kFmtW4PC = 0, kFmtW4G128 = 1, kFmtW8 = 2 };
constexpr int kMaxGrid = 256;  // persistent CTAs per GEMM (>= SMs per GPU)

// Diagnostic builds (-DQLIN_TRACE) record per-CTA clock64 stamps at the
// phase boundaries below into g_trace[cta][16]; normal builds compile the
// stamps away.
// QLIN_STEP(g, k) records per-step events of CTA 0 into g_steps[g][8] (g < 255).  The
// buffer pointers are read once into registers (QLIN_TRACE_INIT) so a stamp
// costs a clock read and a store, not a global load.
#ifdef QLIN_TRACE
__device__ long long* g_trace = nullptr;
__device__ long long* g_steps = nullptr;
#define QLIN_TRACE_INIT                           \
  long long* const qlin_tr = g_trace;             \
  long long* const qlin_st = blockIdx.x == 0 ? g_steps : nullptr;
#define QLIN_STAMP(k)                                                                \
  do {                                                                               \
    if (qlin_tr) qlin_tr[blockIdx.x * 32 + (k)] = static_cast<long long>(clock64()); \
  } while (0)
#define QLIN_STEP(g, k)                                                                       \
  do {                                                                                        \
    if (qlin_st && (g) < 255) qlin_st[(g) * 8 + (k)] = static_cast<long long>(clock64());     \
  } while (0)
// finisher phases of any CTA into g_steps[255][k] (last writer wins)
#define QLIN_FIN(k)                                                                           \
  do {                                                                                        \
    if (g_steps) g_steps[255 * 8 + (k)] = static_cast<long long>(clock64());                  \
  } while (0)
#else
#define QLIN_FIN(k) do { } while (0)
#define QLIN_TRACE_INIT
#define QLIN_STAMP(k) do { } while (0)
#define QLIN_STEP(g, k) do { } while (0)
#endif

// One GEMM problem of a launch (a linear layer at M tokens).  A launch runs
// one problem (qlin_gemm / qlin_forward) or a group of independent problems
// with the same token tile (qlin_forward_grouped): their tiles' iterations
// are concatenated into one space that the persistent CTAs split.
struct GemmProb {
  const uint8_t* codes;     // tiled packed codes (INT4: 8 KiB blocks, INT8: 16 KiB swizzled blocks)
  const uint16_t* rfold;    // g128 ratios r [K/128][N] fp16
  const uint16_t* wot;      // tiled W_O^T (16 KiB swizzled blocks of 128 channels x 64 outliers)
  const float* cscale;      // c_n [N]
  const float* a;           // a_m [M]
  uint16_t* Y;              // [M][N] fp16
  int32_t* acc_debug;       // [M][N] or null
  float cmul;               // INT8 kernel: factor on c_n (1, or 1/16 for per-channel INT4 widened to 16 q)
  int M, N, K, nO;
  int tiles_n, tiles_m;
  int kb;                   // 128-wide K-blocks per tile (ceil(K / 128))
  int nk;                   // main K-steps per tile (ceil(kb / KS))
  int nc;                   // compensation steps per tile
  int ncs;                  // 64-wide outlier slices
  int T;                    // iterations per tile = nk + nc
  int gm;                   // token tiles per raster group (see tile_coords)
  unsigned it0;             // first iteration of this problem in the launch's iteration space
};

// Tile t of a problem -> (channel tile tn, token tile tm).  Token tiles are
// visited in groups of gm, the token tile varying fastest within a group, so
// the CTAs that run at the same time share weight tiles (one HBM read, the
// rest L2 hits) and the group's activations stay in L2.  gm = 1 is the
// channel-tile-fastest order.
__host__ __device__ __forceinline__ void tile_coords(const GemmProb& pr, unsigned t, int& tn, int& tm) {
  const unsigned per = static_cast<unsigned>(pr.gm) * static_cast<unsigned>(pr.tiles_n);
  const unsigned grp = t / per;
  const unsigned w = t - grp * per;
  const int g0 = static_cast<int>(grp) * pr.gm;
  const int gs = pr.tiles_m - g0 < pr.gm ? pr.tiles_m - g0 : pr.gm;
  tm = g0 + static_cast<int>(w % static_cast<unsigned>(gs));
  tn = static_cast<int>(w / static_cast<unsigned>(gs));
}

// Launch-wide arguments.
struct GemmArgs {
  int32_t* ws_acc;      // [2*grid][BT][128] INT32 partial sums of split tiles
  float* ws_comp;       // [2*grid][BT][128] fp32 compensation of split tiles
  unsigned* ws_cnt;     // [grid] iteration counters (zero on entry, left zero)
  int nprob;            // problems in the launch
  int grid;             // persistent CTAs (<= kMaxGrid)
  int split;            // 1: stream-K split points; 0: whole tiles per CTA
  unsigned total;       // iterations of every problem's tiles
  // Cluster split-K (cs > 1, single-problem launches only): the grid is ncl
  // clusters of cs CTAs; cluster c takes tiles c, c + ncl, ...; cluster rank
  // r computes iterations [cb[r], cb[r+1]) of each (cb[cs] = T, the
  // compensation run never cut), and the partials are reduced through
  // distributed shared memory: rank q owns channels [q * 128/cs, (q+1) *
  // 128/cs) of the tile.
  int cs;
  int ncl;
  int cb[9];
  // 1: the weight blocks were written by the previous kernel (INT4 widened
  // once per call), so the weight producer waits on the grid dependency too
  int wdep;
  // bnd[c] = first iteration of CTA c, bnd[grid] = total (computed on the
  // host by gemm_boundaries(); kernel parameters, read from the constant
  // cache).
  unsigned bnd[kMaxGrid + 1];
};

constexpr int kMaxProbs = 32;  // problems per grouped launch

// Kernel parameters: the TMA maps of every problem's activation (Xq) and
// compensation (U) operands, the launch-wide arguments and the problems.
template <int MAXP>
struct alignas(64) GemmParams {
  CUtensorMap tmX[MAXP];
  CUtensorMap tmU[MAXP];
  GemmArgs g;
  GemmProb pr[MAXP];
};

// K-blocks of 128 INT8 codes per pipeline step for a token tile of BT.
__host__ __device__ constexpr int gemm_ks(int BT) { return BT <= 16 ? 4 : (BT <= 64 ? 2 : 1); }

template <int FMT, int BT>
struct GemmCfg {
  static constexpr int kBN = 128;                    // output channels per tile (MMA M)
  // K-blocks of 128 INT8 codes per pipeline step.  Each step costs a few
  // hundred cycles of bookkeeping in the MMA and converter threads whatever
  // its size, so small token tiles (HBM-bound decode) move four blocks per
  // step; large ones are tensor-bound and move one.
  static constexpr int KS = gemm_ks(BT);
  static constexpr bool kW4 = FMT != kFmtW8;
  // INT4 formats: eight converter warps (two per SM sub-partition, so
  // unpacking is not latency-bound) and four epilogue warps of their own,
  // so accumulators drain while later segments are still being converted.
  // INT8: the four warps after the first three are the epilogue.
  static constexpr int kNCW = kW4 ? 8 : 4;          // arrivals on the converter barriers
  static constexpr int kEpiWarp0 = kW4 ? 3 + kNCW : 3;
  // INT8 with 256-token tiles (prefill): the single-buffered accumulator
  // stalls the MMA while a tile drains, so two groups of four epilogue warps
  // take alternate 16-token chunks of whole tiles.
  static constexpr int kEpiGroups = (!kW4 && BT == 256) ? 2 : 1;
  static constexpr int kThreads = 32 * (kEpiWarp0 + 4 * kEpiGroups);
  // Small token tiles load the hi and lo compensation operands in one step
  // (one W_O^T block feeds both); large ones use two passes.
  static constexpr bool kCompFused = BT <= 64;
  // INT4 formats with token tiles up to 64 keep the converted INT8 weight
  // operand in tensor memory (tcgen05.st by the converters, MMA with A in
  // TMEM): no shared-memory round trip for the 16 KiB of INT8 per K-block.
  static constexpr bool kTA = kW4 && BT <= 64;
  static constexpr int kACols = KS * 32;                                 // TMEM columns per A slot
  static constexpr int kABytes = kTA ? 0 : KS * 16384;                   // smem per A slot: KS x (128 x 128 B)
  static constexpr int kXTile = BT * 128;                                // BT x 128 B per K-block
  static constexpr int kXTiles = KS > (kCompFused ? 2 : 1) ? KS : (kCompFused ? 2 : 1);
  static constexpr int kXBytes = (kXTile * kXTiles + 1023) / 1024 * 1024;
  static constexpr int kStgRatio = KS * 8192;                            // g128 ratio rows follow the codes
  static constexpr int kStgBytes = kW4 ? KS * 8192 + (FMT == kFmtW4G128 ? KS * 256 : 0) : 0;
  static constexpr int kCompSlots = kTA ? 2 : 0;                         // W_O^T ring (16 KiB slots)
  // Cluster split-K receive buffer (token tiles up to 64): INT32 partials of
  // the owned channel slice from every rank, [rank][channel][kRecvLd], and the
  // fp32 compensation of the slice from the rank that ran it; rows padded by
  // 4 words so 16-byte reads of consecutive channels hit distinct banks.
  static constexpr bool kCluster = BT <= 64;
  static constexpr int kRecvLd = BT + 4;
  static constexpr int kRecvMain = kCluster ? 128 * kRecvLd * 4 : 0;
  static constexpr int kRecvComp = kCluster ? 64 * kRecvLd * 4 : 0;  // slice <= 64 channels (cs >= 2)
  static constexpr int kRecvBytes = kRecvMain + kRecvComp;
  static constexpr int kSmemLimit = 232448;          // 227 KB per CTA
  static constexpr int kReserve = 1024 + 1024 + 1024 + 2048;  // alignment slack, barriers, boundary table, token scales (x2)
  static constexpr int kYStage = 16 * 128 * 2;                  // one 16-token x 128-channel fp16 chunk of Y
  static constexpr int kBudget = kSmemLimit - kReserve;
  // 256-token tiles: the INT8 format spends shared memory on activation
  // slots (32 KiB each), the INT4 formats on packed-weight staging
  static constexpr int kXSlots =
      KS == 4 ? (FMT == kFmtW4G128 ? 3 : 4) : (BT <= 32 ? 8 : (BT <= 128 || !kW4 ? 4 : 3));
  static constexpr int kASlotsW8 =
      (kBudget - kXSlots * kXBytes - kRecvBytes - 2 * kEpiGroups * kYStage) / (KS * 16384);
  static constexpr int kASlots = kTA ? (BT <= 16 ? 3 : 4)
                                     : (kW4 ? (KS == 2 ? 3 : (BT <= 128 ? 4 : 3)) : (kASlotsW8 > 8 ? 8 : kASlotsW8));
  static constexpr int kStgSlotsFit =
      kW4 ? (kBudget - kASlots * kABytes - kXSlots * kXBytes - kCompSlots * 16384 - kRecvBytes -
             2 * kEpiGroups * kYStage) /
                kStgBytes
          : 0;
  static constexpr int kStgSlots = kStgSlotsFit > 16 ? 16 : kStgSlotsFit;
  static constexpr int kOffA = 0;
  static constexpr int kOffX = kASlots * kABytes;
  static constexpr int kOffComp = kOffX + kXSlots * kXBytes;
  static constexpr int kOffStg = kOffComp + kCompSlots * 16384;
  static constexpr int kOffRecv = kOffStg + kStgSlots * kStgBytes;
  static constexpr int kOffYst = kOffRecv + kRecvBytes;              // two Y staging chunks
  static constexpr int kOffBar = kOffYst + 2 * kEpiGroups * kYStage;
  static constexpr int kOffBnd = kOffBar + 1024;     // stream-K boundary table (<= 256 entries)
  static constexpr int kOffSa = kOffBnd + 1024;      // token scales a[m] of the tile being finished (per group)
  static constexpr int kSmemBytes = kReserve + kOffBar;
  static constexpr uint32_t kTxX = BT * 128;
  static constexpr uint32_t kTxU = (kCompFused ? 2 : 1) * BT * 128;
  // TMEM: accumulators (two buffers of main + compensation columns), then
  // the A slots
  static_assert(!kTA || 2 * 2 * BT + kASlots * kACols <= 512, "TMEM budget");
  static_assert(!kTA || kCompFused, "the TMEM-A variant loads hi and lo compensation rows together");
  static_assert(kASlots >= 2 && kASlots <= 8, "A ring");
  static_assert(kXSlots >= 2 && kXSlots <= 8, "X ring");
  static_assert(!kW4 || (kStgSlots >= 2 && kStgSlots <= 16), "staging ring");
  static_assert(BT % 16 == 0 && BT >= 16 && BT <= 256, "MMA N must be 16..256 in steps of 16");
};

// TMEM columns per accumulator buffer and the number of buffers.
__host__ __device__ inline int tmem_buf_cols(int BT, bool comp) { return comp ? 2 * BT : BT; }
__host__ __device__ inline int tmem_nbuf(int BT, bool comp) { return 2 * tmem_buf_cols(BT, comp) <= 512 ? 2 : 1; }
// Columns to allocate: the accumulator buffers plus `extra` (A slots).
__host__ __device__ inline uint32_t tmem_alloc_cols(int BT, bool comp, int extra) {
  const int need = tmem_nbuf(BT, comp) * tmem_buf_cols(BT, comp) + extra;
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(need)) c <<= 1;
  return c;
}

// First iteration of every CTA (host side; bnd[grid] = total).  Split
// points never fall strictly inside a tile's compensation run; without
// splitting they snap to the nearest tile start.
inline void gemm_boundaries(const GemmProb* pr, int nprob, int grid, int split, unsigned* bnd) {
  long long total = 0;
  for (int p = 0; p < nprob; ++p) total += static_cast<long long>(pr[p].tiles_n) * pr[p].tiles_m * pr[p].T;
  int p = 0;
  for (int c = 0; c <= grid; ++c) {
    if (c == 0 || c == grid) {
      bnd[c] = c == 0 ? 0u : static_cast<unsigned>(total);
      continue;
    }
    long long b = (total * c) / grid;
    while (p + 1 < nprob && b >= static_cast<long long>(pr[p + 1].it0)) ++p;
    const long long T = pr[p].T;
    const long long r = (b - pr[p].it0) % T;
    if (!split) {
      if (r) b += 2 * r >= T ? T - r : -r;  // the nearest tile start
    } else if (r > pr[p].nk) {
      b += T - r;
    }
    if (b > total) b = total;
    bnd[c] = static_cast<unsigned>(b);
  }
  for (int c = 1; c <= grid; ++c)  // monotone after snapping
    if (bnd[c] < bnd[c - 1]) bnd[c] = bnd[c - 1];
}

// Cluster split-K rank ranges of one tile's T iterations (nk K-steps, then
// the compensation run, which one rank runs whole: the last).  The last
// rank also sends the compensation partial, so its load counts `ccost`
// step-equivalents for that run; the cut gives it as many K-steps as keeps
// the largest rank load smallest and splits the rest evenly.  Returns the
// largest load, or a negative value when some rank would get no work.
inline double cluster_bounds(int T, int nk, int cs, double ccost, int* cb) {
  const int nc = T - nk;
  int best_m = -1;
  double best = 0.0;
  for (int m = 0; m <= nk; ++m) {
    const int rest = nk - m;
    if (rest < cs - 1) break;  // every other rank needs at least one K-step
    const double others = static_cast<double>((rest + cs - 2) / (cs - 1));
    const double last = m + (nc > 0 ? ccost : 0.0);
    const double load = others > last ? others : last;
    if (nc == 0 && m == 0) continue;  // without a compensation run the last rank needs K-steps
    if (best_m < 0 || load < best) {
      best_m = m;
      best = load;
    }
  }
  if (best_m < 0) return -1.0;
  const int rest = nk - best_m;
  int b = 0;
  for (int r = 0; r < cs - 1; ++r) {
    cb[r] = b;
    b += rest / (cs - 1) + (r < rest % (cs - 1) ? 1 : 0);
  }
  cb[cs - 1] = b;  // == rest
  cb[cs] = T;
  return best;
}

// The boundary table is copied into shared memory at kernel start (entries
// 0 .. grid-1; entry grid is the total iteration count).
__device__ __forceinline__ unsigned bnd_s(int c, const unsigned* sbnd, const GemmArgs& g) {
  return c < g.grid ? sbnd[c] : g.total;
}

// The CTA whose range contains iteration `it` (binary search of the table).
__device__ __forceinline__ int owner_cta_s(unsigned it, const unsigned* sbnd, const GemmArgs& g) {
  int lo = 0, hi = g.grid - 1;  // invariant: bnd[lo] <= it < bnd[hi + 1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sbnd[mid] <= it) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Scratch slot holding CTA c's partial of the split tile whose first
// iteration is `tfirst`: its first segment if its range starts inside the
// tile, else its last segment.
__device__ __forceinline__ int partial_slot_s(int c, unsigned tfirst, const unsigned* sbnd) {
  return 2 * c + (sbnd[c] < tfirst ? 1 : 0);
}

struct Segment {
  int p;            // problem
  unsigned tile;    // tile within the problem (tn + tiles_n * tm)
  unsigned tfirst;  // first iteration of the tile in the launch's iteration space
  int r0, r1;       // iterations [r0, r1) of the tile
};

// Dequantisation factor c'_n of output channel n: c_n / 16 for per-channel
// INT4 (the operand holds 16 q), c_n for the other formats, times the INT8
// kernel's factor (exact: 1 or 1/16) when it runs on widened INT4 weights.
template <int FMT>
__device__ __forceinline__ float chan_scale(const GemmProb& g, int n) {
  if (n >= g.N) return 0.f;
  const float c = g.cscale[n];
  return FMT == kFmtW4PC ? __fmul_rn(c, 0.0625f) : (FMT == kFmtW8 ? __fmul_rn(c, g.cmul) : c);
}

// Segments of one CTA, in order: a stream-K range of the launch's iteration
// space (crossing problems), or (cluster split-K) the same rank range of
// every cluster tile of the single problem.  The range comes from the CTA
// plan staged in shared memory at start-up, so no role waits on
// kernel-parameter loads for its first segment.
struct SegGen {
  unsigned it, it1;
  int p, u, cid, ncl, ntiles, r0, r1;
  bool cl;
};

// CTA plan (shared memory, written once during setup).
enum : int { kPlanIt0 = 0, kPlanIt1, kPlanR0, kPlanR1, kPlanNcl, kPlanTiles, kPlanWords };

__device__ __forceinline__ SegGen seg_begin(const int* plan, int cid, bool cl) {
  SegGen s;
  s.it = static_cast<unsigned>(plan[kPlanIt0]);
  s.it1 = static_cast<unsigned>(plan[kPlanIt1]);
  s.p = 0;
  s.u = 0;
  s.cid = cid;
  s.ncl = plan[kPlanNcl];
  s.ntiles = plan[kPlanTiles];
  s.r0 = plan[kPlanR0];
  s.r1 = plan[kPlanR1];
  s.cl = cl;
  return s;
}

__device__ __forceinline__ bool seg_next(SegGen& s, Segment& sg, const GemmProb* pr, int nprob) {
  if (s.cl) {
    const int t = s.cid + s.u * s.ncl;
    if (t >= s.ntiles) return false;
    sg.p = 0;
    sg.tile = static_cast<unsigned>(t);
    sg.tfirst = static_cast<unsigned>(t) * static_cast<unsigned>(pr[0].T);
    sg.r0 = s.r0;
    sg.r1 = s.r1;
    ++s.u;
    return true;
  }
  if (s.it >= s.it1) return false;
  while (s.p + 1 < nprob && s.it >= pr[s.p + 1].it0) ++s.p;
  const unsigned T = static_cast<unsigned>(pr[s.p].T);
  const unsigned local = s.it - pr[s.p].it0;
  sg.p = s.p;
  sg.tile = local / T;
  sg.r0 = static_cast<int>(local - sg.tile * T);
  sg.tfirst = pr[s.p].it0 + sg.tile * T;
  const unsigned left = s.it1 - s.it;
  sg.r1 = static_cast<int>(left < T - sg.r0 ? sg.r0 + left : T);
  s.it += sg.r1 - sg.r0;
  return true;
}

// Per-channel INT4 -> INT8 (16*q) for one packed 16-byte chunk (32 codes).
__device__ __forceinline__ void unpack_w4pc(const uint4 w, uint4& o0, uint4& o1) {
  o0.x = (w.x << 4) & 0xF0F0F0F0u;
  o0.y = w.x & 0xF0F0F0F0u;
  o0.z = (w.y << 4) & 0xF0F0F0F0u;
  o0.w = w.y & 0xF0F0F0F0u;
  o1.x = (w.z << 4) & 0xF0F0F0F0u;
  o1.y = w.z & 0xF0F0F0F0u;
  o1.z = (w.w << 4) & 0xF0F0F0F0u;
  o1.w = w.w & 0xF0F0F0F0u;
}

__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// Per-group requantization of 8 codes (one packed word) to INT8:
// q8 = rne(q4 * r).  Each nibble becomes an fp16 by OR-ing it into the
// significand of 1024 (offset by 8 to make it unsigned); the exact q4 (or
// 16*q4) is recovered by one exact subtraction; one fused multiply-add with
// the ratio and 1152 rounds q4*r + 1152 once to an integer in [1025, 1279]
// where the fp16 spacing is 1, so the low byte is q8 + 128.
__device__ __forceinline__ uint2 requant_g128(uint32_t w, __half2 r1, __half2 r16) {
  const uint32_t wx = w ^ 0x88888888u;
  const uint32_t wy = wx >> 8;
  const uint32_t x0 = lop3_and_or(wx, 0x000F000Fu, 0x64006400u);  // 1032 + q[k0],   1032 + q[k0+2]
  const uint32_t x1 = lop3_and_or(wx, 0x00F000F0u, 0x64006400u);  // 1152 + 16q[k0+4], +16q[k0+6]
  const uint32_t x2 = lop3_and_or(wy, 0x000F000Fu, 0x64006400u);  // q[k0+1], q[k0+3]
  const uint32_t x3 = lop3_and_or(wy, 0x00F000F0u, 0x64006400u);  // 16q[k0+5], 16q[k0+7]
  const __half2 c1032 = __half2half2(__ushort_as_half(static_cast<unsigned short>(0x6408)));  // 1032
  const __half2 c1152 = __half2half2(__ushort_as_half(static_cast<unsigned short>(0x6480)));  // 1152
  const __half2 f0 = __hfma2(__hsub2(u32_as_h2(x0), c1032), r1, c1152);
  const __half2 f1 = __hfma2(__hsub2(u32_as_h2(x1), c1152), r16, c1152);
  const __half2 f2 = __hfma2(__hsub2(u32_as_h2(x2), c1032), r1, c1152);
  const __half2 f3 = __hfma2(__hsub2(u32_as_h2(x3), c1152), r16, c1152);
  uint2 o;
  o.x = prmt(h2_as_u32(f0), h2_as_u32(f2), 0x6240u) ^ 0x80808080u;  // q8[k0..k0+3]
  o.y = prmt(h2_as_u32(f1), h2_as_u32(f3), 0x6240u) ^ 0x80808080u;  // q8[k0+4..k0+7]
  return o;
}

// Wait (bounded) for the last phases of a ring that a producer filled, so
// the CTA never exits with copies in flight.
__device__ __forceinline__ void drain_ring(uint64_t* full, int slots, int issued) {
  for (int t = issued - 1; t >= 0 && t >= issued - slots; --t) {
    const int s = t % slots;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(&full[s], static_cast<uint32_t>(t / slots) & 1u, 1000000u) &&
           globaltimer_ns() - t0 < QLIN_DRAIN_NS) {
    }
  }
}

// Prefill with INT4 weights: the packed blocks are widened once per call to
// the INT8 operand layout (16 KiB blocks, 128-byte swizzle) -- the same
// arithmetic as the converter warps (16 q for per-channel codes, the folded
// FP16 requantisation for g128) -- and the INT8 kernel runs on them.  With
// hundreds of token tiles per weight block this replaces a conversion per
// token tile by one.  One CTA per 128 x 128 block, two 16-byte chunks per
// thread.
template <int FMT>
__global__ void __launch_bounds__(256)
widen_w4_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ rfold, int N, int kb,
                uint8_t* __restrict__ out) {
  griddep_launch_dependents();
  const int blk = blockIdx.x;  // tn * kb + k
  const int tn = blk / kb;
  const int k = blk - tn * kb;
  const uint8_t* src = codes + static_cast<size_t>(blk) * 8192;
  uint8_t* dst = out + static_cast<size_t>(blk) * 16384;
  uint4 w[2];
  uint16_t rb[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int c = threadIdx.x + u * 256;
    w[u] = __ldg(reinterpret_cast<const uint4*>(src) + c);
    const int n = tn * 128 + (c >> 2);
    rb[u] = (FMT == kFmtW4G128 && n < N) ? rfold[static_cast<size_t>(k) * N + n] : static_cast<uint16_t>(0);
  }
  griddep_wait();  // the previous kernel in the stream may still read this workspace
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int c = threadIdx.x + u * 256;
    const int row = c >> 2;
    const int part = (c & 3) ^ ((row >> 1) & 3);  // packed chunks are swizzled by row pair
    uint4 o0, o1;
    if (FMT == kFmtW4PC) {
      unpack_w4pc(w[u], o0, o1);
    } else {
      const __half2 r1 = __half2half2(__ushort_as_half(rb[u]));
      const __half2 r16 = __hmul2(r1, __half2half2(__ushort_as_half(static_cast<unsigned short>(0x2C00))));  // * 1/16
      const uint2 a0 = requant_g128(w[u].x, r1, r16);
      const uint2 a1 = requant_g128(w[u].y, r1, r16);
      const uint2 a2 = requant_g128(w[u].z, r1, r16);
      const uint2 a3 = requant_g128(w[u].w, r1, r16);
      o0 = make_uint4(a0.x, a0.y, a1.x, a1.y);
      o1 = make_uint4(a2.x, a2.y, a3.x, a3.y);
    }
    const int sw = row & 7;
    *reinterpret_cast<uint4*>(dst + row * 128 + (((2 * part) ^ sw) << 4)) = o0;
    *reinterpret_cast<uint4*>(dst + row * 128 + (((2 * part + 1) ^ sw) << 4)) = o1;
  }
}

template <int FMT, int BT, int MAXP>
__global__ void __launch_bounds__(GemmCfg<FMT, BT>::kThreads, 1)
gemm_kernel(const __grid_constant__ GemmParams<MAXP> prm) {
  using C = GemmCfg<FMT, BT>;
  const GemmArgs& args = prm.g;
  const GemmProb* const probs = prm.pr;
  const int nprob = MAXP == 1 ? 1 : args.nprob;
  constexpr int P = C::kASlots;
  constexpr int XS = C::kXSlots;
  constexpr int LS = C::kStgSlots > 0 ? C::kStgSlots : 1;
  constexpr int kConvThreads = 32 * C::kNCW;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* sfull = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* sempty = sfull + 16;
  uint64_t* afull = sempty + 16;
  uint64_t* aconv = afull + 8;
  uint64_t* aempty = aconv + 8;
  uint64_t* xfull = aempty + 8;
  uint64_t* xempty = xfull + 8;
  uint64_t* acc_full = xempty + 8;    // [2]
  uint64_t* acc_empty = acc_full + 2; // [2]
  uint64_t* cfull = acc_empty + 2;    // [2] W_O^T ring (TMEM-A variant)
  uint64_t* cempty = cfull + 2;       // [2]
  uint64_t* recv_full = cempty + 2;   // cluster split-K: this CTA's receive buffer is complete
  uint64_t* recv_free = recv_full + 1; // every owner has read this CTA's previous partials
  uint64_t* mma_done = recv_free + 1;   // every tensor-core op the issuer started has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;  // [2]
  int* plan = const_cast<int*>(last_flag + 2);  // [kPlanWords]
  unsigned* sbnd = reinterpret_cast<unsigned*>(smem + C::kOffBnd);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Compensation accumulators are allocated when any problem has outliers.
  bool comp = false;
  for (int q = 0; q < nprob; ++q) comp = comp || probs[q].nO > 0;
  const int bcols = tmem_buf_cols(BT, comp);
  const int nbuf = tmem_nbuf(BT, comp);
  const uint32_t tcols = tmem_alloc_cols(BT, comp, C::kTA ? P * C::kACols : 0);
  const uint32_t a_col0 = static_cast<uint32_t>(nbuf * bcols);  // first TMEM column of the A slots
  const bool cl = args.cs > 1;
  const int crk = cl ? static_cast<int>(cluster_ctarank()) : 0;
  const int cid = cl ? static_cast<int>(cluster_id_x()) : 0;
  // it0 of this CTA's stream-K range (read once more by the epilogue)
  const unsigned it0 = cl ? 0u : args.bnd[blockIdx.x];
  const int slice = 128 / args.cs;  // channels owned per cluster rank
  // bytes arriving in a receive buffer per round: every rank's INT32 slice,
  // plus the compensation slice when the layer has outliers
  const uint32_t recv_bytes =
      static_cast<uint32_t>(128 * BT * 4 + (probs[0].nO > 0 ? slice * BT * 4 : 0));
  QLIN_TRACE_INIT
#ifdef QLIN_TRACE
  if (threadIdx.x == 0 && qlin_tr) qlin_tr[blockIdx.x * 32 + 31] = static_cast<long long>(globaltimer_ns());
#endif
  if (threadIdx.x == 0) QLIN_STAMP(0);

  // warp 0 initialises the barriers, one per lane
  if (warp == 0) {
    if (lane < 16) {
      mbar_init(&sfull[lane], 1);
      mbar_init(&sempty[lane], C::kNCW);  // one arrival per converter warp
    } else if (lane < 24) {
      const int i = lane - 16;
      mbar_init(&afull[i], 1);
      mbar_init(&aconv[i], C::kNCW);
      mbar_init(&aempty[i], 1);
      mbar_init(&xfull[i], 1);
      mbar_init(&xempty[i], 1);
    } else if (lane < 26) {
      const int b = lane - 24;
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128 * C::kEpiGroups);
      mbar_init(&cfull[b], 1);
      mbar_init(&cempty[b], 1);
    } else if (lane == 26) {
      mbar_init(recv_full, 1);
      mbar_init(recv_free, static_cast<uint32_t>(args.cs));
      mbar_init(mma_done, 1);
      *abort_flag = 0;
    }
    fence_barrier_init();
    __syncwarp();
    if (lane == 26 && cl) mbar_arrive_expect_tx(recv_full, recv_bytes);  // round 0
  }
  if (warp == 0 && lane < nprob) {
    tma_prefetch_desc(&prm.tmX[lane]);
    if (probs[lane].nO > 0) tma_prefetch_desc(&prm.tmU[lane]);
  }
  if (warp == 3 && lane == 0) {
    plan[kPlanIt0] = cl ? 0 : static_cast<int>(it0);
    plan[kPlanIt1] = cl ? 0 : static_cast<int>(args.bnd[blockIdx.x + 1]);
    plan[kPlanR0] = cl ? args.cb[crk] : 0;
    plan[kPlanR1] = cl ? args.cb[crk + 1] : 0;
    plan[kPlanNcl] = args.ncl;
    plan[kPlanTiles] = probs[0].tiles_n * probs[0].tiles_m;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Peers' barriers must be initialised before any remote access: arrive
  // now, wait just before the first one (epilogue) or at the end.
  if (cl) cluster_arrive_relaxed();
  bool cl_waited = false;
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) QLIN_STAMP(1);
  // Let the next kernel in the stream start its prologue; it waits for this
  // grid to complete before it touches anything this kernel writes.
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ X producer
    if (lane == 0) {
      griddep_wait();  // activations come from the previous kernel
      QLIN_STAMP(4);
      bool first_x = true;
      SegGen gen = seg_begin(plan, cid, cl);
      Segment sg;
      int g = 0;
      bool ok = true;
      while (ok && seg_next(gen, sg, probs, nprob)) {
        const GemmProb& pr = probs[sg.p];
        const CUtensorMap* tmX = &prm.tmX[sg.p];
        const CUtensorMap* tmU = &prm.tmU[sg.p];
        int tn_, tm_;
        tile_coords(pr, sg.tile, tn_, tm_);
        const int m0 = tm_ * BT;
        for (int r = sg.r0; r < sg.r1; ++r, ++g) {
          const int x = g % XS;
          if (g >= XS && !mbar_wait(&xempty[x], static_cast<uint32_t>(g / XS - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          unsigned char* xb = smem + C::kOffX + x * C::kXBytes;
          QLIN_STEP(g, 0);
          if (first_x) QLIN_STAMP(28);
          if (r < pr.nk) {
            const int kb0 = r * C::KS;
            const int nkb = min(C::KS, pr.kb - kb0);
            mbar_arrive_expect_tx(&xfull[x], static_cast<uint32_t>(nkb) * C::kTxX);
            if (first_x) QLIN_STAMP(29);
            for (int i = 0; i < nkb; ++i) {
              tma_load_2d(xb + i * C::kXTile, tmX, &xfull[x], (kb0 + i) * 128, m0);
              if (first_x && i == 0) QLIN_STAMP(30);
            }
            first_x = false;
            if (g == 0) QLIN_STAMP(19);
          } else {
            const int j = r - pr.nk;
            mbar_arrive_expect_tx(&xfull[x], C::kTxU);
            if (C::kCompFused) {
              tma_load_2d(xb, tmU, &xfull[x], j * 64, m0);                          // hi rows
              tma_load_2d(xb + C::kXTile, tmU, &xfull[x], j * 64, pr.M + m0);     // lo rows
            } else {
              const int lo = j >= pr.ncs ? 1 : 0;  // U rows [0, M) hold hi, [M, 2M) hold lo
              tma_load_2d(xb, tmU, &xfull[x], (j - lo * pr.ncs) * 64, lo * pr.M + m0);
            }
          }
        }
      }
      QLIN_STAMP(5);
      drain_ring(xfull, XS, g);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ weight producer
    if (lane == 0) {
      QLIN_STAMP(25);
      if (args.wdep) griddep_wait();  // widened weights come from the previous kernel
      const uint64_t pol_stream = policy_evict_first();
      uint32_t a_issues[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // loads issued into each A slot
      SegGen gen = seg_begin(plan, cid, cl);
      Segment sg;
      int g = 0, gs = 0, gc = 0;
      bool ok = true;
      while (ok && seg_next(gen, sg, probs, nprob)) {
        if (g == 0) QLIN_STAMP(26);
        const GemmProb& pr = probs[sg.p];
        int tn, tm_;
        tile_coords(pr, sg.tile, tn, tm_);
        const int n0 = tn * C::kBN;
        const uint32_t rb = FMT == kFmtW4G128 ? static_cast<uint32_t>(min(C::kBN, pr.N - n0)) * 2u : 0u;
        for (int r = sg.r0; r < sg.r1; ++r, ++g) {
          if (r < pr.nk && C::kW4) {
            const int ls = gs % LS;
            if (gs >= LS && !mbar_wait(&sempty[ls], static_cast<uint32_t>(gs / LS - 1) & 1u, abort_flag)) {
              ok = false;
              break;
            }
            unsigned char* st = smem + C::kOffStg + ls * C::kStgBytes;
            QLIN_STEP(g, 1);
            const int kb0 = r * C::KS;
            const int nkb = min(C::KS, pr.kb - kb0);
            if (gs == 0) QLIN_STAMP(15);
            mbar_arrive_expect_tx(&sfull[ls], static_cast<uint32_t>(nkb) * (8192u + rb));
            bulk_load_hint(st, pr.codes + (static_cast<size_t>(tn) * pr.kb + kb0) * 8192,
                           static_cast<uint32_t>(nkb) * 8192u, &sfull[ls], pol_stream);
            if (FMT == kFmtW4G128)
              for (int i = 0; i < nkb; ++i)
                bulk_load(st + C::kStgRatio + i * 256, pr.rfold + static_cast<size_t>(kb0 + i) * pr.N + n0, rb,
                          &sfull[ls]);
            if (gs == 0) QLIN_STAMP(2);
            ++gs;
          } else if (C::kTA) {
            // W_O^T block of a compensation step into its own ring, as soon
            // as a slot is free (well ahead of its use)
            const int cs = gc & 1;
            if (gc >= 2 && !mbar_wait(&cempty[cs], static_cast<uint32_t>(gc / 2 - 1) & 1u, abort_flag)) {
              ok = false;
              break;
            }
            const int j = r - pr.nk;
            const int ib = C::kCompFused ? j : (j >= pr.ncs ? j - pr.ncs : j);
            mbar_arrive_expect_tx(&cfull[cs], 16384u);
            bulk_load(smem + C::kOffComp + cs * 16384, pr.wot + (static_cast<size_t>(tn) * pr.ncs + ib) * 8192,
                      16384, &cfull[cs]);
            ++gc;
          } else if (!C::kW4) {
            // INT8 weights and W_O^T blocks into the A ring.  This thread
            // waits on every A slot in order, so a parity wait never runs
            // more than one phase ahead of the ring.  (For the INT4 formats
            // the converters, which move in step with the A ring, issue the
            // W_O^T copies instead.)
            const int p = g % P;
            if (g >= P && !mbar_wait(&aempty[p], static_cast<uint32_t>(g / P - 1) & 1u, abort_flag)) {
              ok = false;
              break;
            }
            unsigned char* ab = smem + C::kOffA + p * C::kABytes;
            QLIN_STEP(g, 1);
            if (r < pr.nk) {
              const int kb0 = r * C::KS;
              const int nkb = min(C::KS, pr.kb - kb0);
              mbar_arrive_expect_tx(&afull[p], static_cast<uint32_t>(nkb) * 16384u);
              bulk_load_hint(ab, pr.codes + (static_cast<size_t>(tn) * pr.kb + kb0) * 16384,
                             static_cast<uint32_t>(nkb) * 16384u, &afull[p], pol_stream);
            } else {
              const int j = r - pr.nk;
              const int ib = C::kCompFused ? j : (j >= pr.ncs ? j - pr.ncs : j);
              mbar_arrive_expect_tx(&afull[p], 16384u);
              bulk_load(ab, pr.wot + (static_cast<size_t>(tn) * pr.ncs + ib) * 8192, 16384, &afull[p]);
            }
            ++a_issues[p];
          }
        }
      }
      QLIN_STAMP(3);
      if (C::kW4) drain_ring(sfull, LS, gs);
      if (C::kTA) drain_ring(cfull, 2, gc);
      for (int p = 0; p < P; ++p) {  // outstanding A-ring copies
        if (!a_issues[p]) continue;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(&afull[p], (a_issues[p] - 1) & 1u, 1000000u) &&
               globaltimer_ns() - t0 < QLIN_DRAIN_NS) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and its waits; one elected lane issues
    // each step's tensor-core instructions and commits (issued from a
    // converged warp, a narrow MMA costs about a third of the cycles it
    // costs from a lone lane).
    {
      constexpr uint32_t idesc_main = idesc_s8_s32(128, BT);
      constexpr uint32_t idesc_comp = idesc_f16_f32(128, BT);
      // Descriptors of ring slot 0; the start-address field counts 16-byte
      // units, so slot i adds i * slot_bytes / 16 and a 32-byte K-slice adds
      // 2 (shared addresses stay below 2^18, so the field never carries).
      const uint64_t adesc0 = sdesc_k_sw128(smem_u32(smem + C::kOffA));
      const uint64_t xdesc0 = sdesc_k_sw128(smem_u32(smem + C::kOffX));
      const uint64_t cdesc0 = sdesc_k_sw128(smem_u32(smem + C::kOffComp));
      int gm = 0, gc = 0;       // TMEM-A variant: main steps (A ring) and compensation steps (W_O^T ring)
      uint32_t conv_phase = 0;  // per A slot: parity of the next converter phase
      uint32_t full_phase = 0;  // per A slot: parity of the next copy phase
      SegGen gen = seg_begin(plan, cid, cl);
      Segment sg;
      int g = 0, seg = 0;
      bool ok = true;
      bool issued = false;  // any tcgen05.mma started (drained before TMEM is freed)
      while (ok && seg_next(gen, sg, probs, nprob)) {
        const GemmProb& pr = probs[sg.p];
        const int buf = seg % nbuf;
        const int use = seg / nbuf;
        if (use > 0 && !warp_wait(&acc_empty[buf], static_cast<uint32_t>(use - 1) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dmain = tmem + static_cast<uint32_t>(buf * bcols);
        const uint32_t dcomp = dmain + BT;
        for (int r = sg.r0; r < sg.r1; ++r, ++g) {
          const int p = g % P;
          const int x = g % XS;
          const bool main_step = r < pr.nk;
          if (!warp_wait(&xfull[x], static_cast<uint32_t>(g / XS) & 1u, abort_flag)) { ok = false; break; }
          QLIN_STEP(g, 5);
          if (C::kTA) {
            const uint64_t bd = xdesc0 + static_cast<uint64_t>(x * (C::kXBytes >> 4));
            if (main_step) {
              const int pa = gm % P;
              if (!warp_wait(&aconv[pa], static_cast<uint32_t>(gm / P) & 1u, abort_flag)) { ok = false; break; }
              if (g == 0) QLIN_STAMP(8);
              QLIN_STEP(g, 6);
              tc_fence_after();
              issued = true;
              const uint32_t at = tmem + a_col0 + static_cast<uint32_t>(pa * C::kACols);
              const int nkb = min(C::KS, pr.kb - r * C::KS);
              if (elect_one()) {
                mma_i8_ta(dmain, at, bd, idesc_main, r > sg.r0 ? 1u : 0u);
                mma_i8_ta(dmain, at + 8, bd + 2, idesc_main, 1u);
                mma_i8_ta(dmain, at + 16, bd + 4, idesc_main, 1u);
                mma_i8_ta(dmain, at + 24, bd + 6, idesc_main, 1u);
#pragma unroll
                for (int i = 1; i < C::KS; ++i) {
                  if (i < nkb) {
                    const uint32_t ai = at + static_cast<uint32_t>(i * 32);
                    const uint64_t bi = bd + static_cast<uint64_t>(i * (C::kXTile >> 4));
                    mma_i8_ta(dmain, ai, bi, idesc_main, 1u);
                    mma_i8_ta(dmain, ai + 8, bi + 2, idesc_main, 1u);
                    mma_i8_ta(dmain, ai + 16, bi + 4, idesc_main, 1u);
                    mma_i8_ta(dmain, ai + 24, bi + 6, idesc_main, 1u);
                  }
                }
                mma_commit(&aempty[pa]);
              }
              __syncwarp();
              ++gm;
            } else {
              const int cs = gc & 1;
              if (!warp_wait(&cfull[cs], static_cast<uint32_t>(gc / 2) & 1u, abort_flag)) { ok = false; break; }
              if (g == 0) QLIN_STAMP(8);
              QLIN_STEP(g, 6);
              tc_fence_after();
              issued = true;
              const uint64_t ad = cdesc0 + static_cast<uint64_t>(cs * (16384 >> 4));
              const uint32_t acc0 = ((r == pr.nk) || (r == sg.r0)) ? 0u : 1u;
              if (elect_one()) {
                mma_f16(dcomp, ad, bd, idesc_comp, acc0);
                mma_f16(dcomp, ad + 2, bd + 2, idesc_comp, 1u);
                mma_f16(dcomp, ad + 4, bd + 4, idesc_comp, 1u);
                mma_f16(dcomp, ad + 6, bd + 6, idesc_comp, 1u);
                const uint64_t bd2 = bd + (C::kXTile >> 4);  // lo rows (fused hi + lo)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_f16(dcomp, ad + 2 * kk, bd2 + 2 * kk, idesc_comp, 1u);
                mma_commit(&cempty[cs]);
              }
              __syncwarp();
              ++gc;
            }
            if (elect_one()) mma_commit(&xempty[x]);
            __syncwarp();
            QLIN_STEP(g, 7);
            continue;
          }
          if (main_step && C::kW4) {
            if (!warp_wait(&aconv[p], (conv_phase >> p) & 1u, abort_flag)) { ok = false; break; }
            conv_phase ^= 1u << p;
          } else {
            if (!warp_wait(&afull[p], (full_phase >> p) & 1u, abort_flag)) { ok = false; break; }
            full_phase ^= 1u << p;
          }
          if (g == 0) QLIN_STAMP(8);
          QLIN_STEP(g, 6);
          tc_fence_after();
          issued = true;
          const uint64_t ad = adesc0 + static_cast<uint64_t>(p * (C::kABytes >> 4));
          const uint64_t bd = xdesc0 + static_cast<uint64_t>(x * (C::kXBytes >> 4));
          if (elect_one()) {
            if (main_step) {
              const int nkb = min(C::KS, pr.kb - r * C::KS);
              mma_i8(dmain, ad, bd, idesc_main, r > sg.r0 ? 1u : 0u);
              mma_i8(dmain, ad + 2, bd + 2, idesc_main, 1u);
              mma_i8(dmain, ad + 4, bd + 4, idesc_main, 1u);
              mma_i8(dmain, ad + 6, bd + 6, idesc_main, 1u);
#pragma unroll
              for (int i = 1; i < C::KS; ++i) {
                if (i < nkb) {
                  const uint64_t ai = ad + static_cast<uint64_t>(i * 1024);
                  const uint64_t bi = bd + static_cast<uint64_t>(i * (C::kXTile >> 4));
                  mma_i8(dmain, ai, bi, idesc_main, 1u);
                  mma_i8(dmain, ai + 2, bi + 2, idesc_main, 1u);
                  mma_i8(dmain, ai + 4, bi + 4, idesc_main, 1u);
                  mma_i8(dmain, ai + 6, bi + 6, idesc_main, 1u);
                }
              }
            } else {
              const uint32_t acc0 = ((r == pr.nk) || (r == sg.r0)) ? 0u : 1u;
              mma_f16(dcomp, ad, bd, idesc_comp, acc0);
              mma_f16(dcomp, ad + 2, bd + 2, idesc_comp, 1u);
              mma_f16(dcomp, ad + 4, bd + 4, idesc_comp, 1u);
              mma_f16(dcomp, ad + 6, bd + 6, idesc_comp, 1u);
              if (C::kCompFused) {
                const uint64_t bd2 = bd + (C::kXTile >> 4);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_f16(dcomp, ad + 2 * kk, bd2 + 2 * kk, idesc_comp, 1u);
              }
            }
            mma_commit(&aempty[p]);
            mma_commit(&xempty[x]);
          }
          __syncwarp();
          QLIN_STEP(g, 7);
        }
        if (!ok) break;
        if (elect_one()) mma_commit(&acc_full[buf]);
        __syncwarp();
        ++seg;
      }
      QLIN_STAMP(9);
      // Every MMA issued has completed before TMEM is freed: normally the
      // epilogue's accumulator waits already saw that, but after a wait gave
      // up nothing else does, so wait here (fixed limit) either way.
      if (issued) {
        if (elect_one()) mma_commit(mma_done);
        __syncwarp();
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(mma_done, 0u, 1000000u) && globaltimer_ns() - t0 < QLIN_DRAIN_NS) {
        }
      }
    }
    __syncwarp();
  } else {
    const int ctid = threadIdx.x - 96;
    const bool epi = warp >= C::kEpiWarp0;
    // The epilogue threads keep the boundary table in shared memory (read
    // after the epilogue's first named barrier).
    if (epi && !cl && warp < C::kEpiWarp0 + 4)
      for (int i = threadIdx.x - 32 * C::kEpiWarp0; i < args.grid; i += 128) sbnd[i] = args.bnd[i];
    // ------------------------------------------------------------ converters
    if (C::kTA && !epi) {
      // One thread per weight row: warp w may only reach TMEM lanes
      // 32*(w % 4) .. +31, so the two warps of a lane quarter split the
      // step's K-blocks (even / odd).  Each thread reads its row's 64 packed
      // bytes of a block (swizzled chunks: conflict-free), widens them to
      // 128 INT8 codes in registers and stores 32 TMEM columns.
      const int qd = warp & 3;
      const int half = (warp - 3) >> 2;
      const int row = qd * 32 + lane;
      const int sw = (row >> 1) & 3;
      const uint32_t tlane = tmem + (static_cast<uint32_t>(qd * 32) << 16) + a_col0;
      SegGen gen = seg_begin(plan, cid, cl);
      Segment sg;
      int gm = 0, gs = 0;
      bool ok = true;
      while (ok && seg_next(gen, sg, probs, nprob)) {
        const GemmProb& pr = probs[sg.p];
        for (int r = sg.r0; r < sg.r1 && r < pr.nk; ++r) {
          const int ls = gs % LS;
          if (!mbar_wait(&sfull[ls], static_cast<uint32_t>(gs / LS) & 1u, abort_flag)) { ok = false; break; }
          if (gs == 0 && ctid == 0) QLIN_STAMP(6);
          const int pa = gm % P;
          if (gm >= P && !mbar_wait(&aempty[pa], static_cast<uint32_t>(gm / P - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const unsigned char* stg = smem + C::kOffStg + ls * C::kStgBytes;
          const int nkb = min(C::KS, pr.kb - r * C::KS);
          for (int blk = half; blk < nkb; blk += 2) {
            const unsigned char* src = stg + blk * 8192 + row * 64;
            uint32_t o[32];
            if (FMT == kFmtW4PC) {
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const uint4 w = *reinterpret_cast<const uint4*>(src + ((c ^ sw) << 4));
                uint4 o0, o1;
                unpack_w4pc(w, o0, o1);
                o[8 * c + 0] = o0.x; o[8 * c + 1] = o0.y; o[8 * c + 2] = o0.z; o[8 * c + 3] = o0.w;
                o[8 * c + 4] = o1.x; o[8 * c + 5] = o1.y; o[8 * c + 6] = o1.z; o[8 * c + 7] = o1.w;
              }
            } else {
              const uint16_t rbits = reinterpret_cast<const uint16_t*>(stg + C::kStgRatio + blk * 256)[row];
              const __half2 r1 = __half2half2(__ushort_as_half(rbits));
              const __half2 r16 = __hmul2(r1, __half2half2(__ushort_as_half(static_cast<unsigned short>(0x2C00))));  // * 1/16
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const uint4 w = *reinterpret_cast<const uint4*>(src + ((c ^ sw) << 4));
                const uint2 a0 = requant_g128(w.x, r1, r16);
                const uint2 a1 = requant_g128(w.y, r1, r16);
                const uint2 a2 = requant_g128(w.z, r1, r16);
                const uint2 a3 = requant_g128(w.w, r1, r16);
                o[8 * c + 0] = a0.x; o[8 * c + 1] = a0.y; o[8 * c + 2] = a1.x; o[8 * c + 3] = a1.y;
                o[8 * c + 4] = a2.x; o[8 * c + 5] = a2.y; o[8 * c + 6] = a3.x; o[8 * c + 7] = a3.y;
              }
            }
            tmem_st32(tlane + static_cast<uint32_t>(pa * C::kACols + blk * 32), o);
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&sempty[ls]);  // staging slot consumed
            mbar_arrive(&aconv[pa]);   // A slot written
          }
          if (ctid == 0) QLIN_STEP(gs, 4);
          ++gm;
          ++gs;
        }
      }
      if (ctid == 0) QLIN_STAMP(7);
    } else if (C::kW4 && !epi) {
      uint32_t a_issues[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // W_O^T copies issued into each A slot (ctid 0)
      SegGen gen = seg_begin(plan, cid, cl);
      Segment sg;
      int g = 0, gs = 0;
      bool ok = true;
      while (ok && seg_next(gen, sg, probs, nprob)) {
        const GemmProb& pr = probs[sg.p];
        int tn, tm_;
        tile_coords(pr, sg.tile, tn, tm_);
        for (int r = sg.r0; r < sg.r1; ++r, ++g) {
          const int p = g % P;
          if (r >= pr.nk) {
            // compensation step: the W_O^T block goes into the A slot once
            // the tensor core has released it
            if (g >= P && !mbar_wait(&aempty[p], static_cast<uint32_t>(g / P - 1) & 1u, abort_flag)) {
              ok = false;
              break;
            }
            if (ctid == 0) {
              const int j = r - pr.nk;
              const int ib = C::kCompFused ? j : (j >= pr.ncs ? j - pr.ncs : j);
              mbar_arrive_expect_tx(&afull[p], 16384u);
              bulk_load(smem + C::kOffA + p * C::kABytes, pr.wot + (static_cast<size_t>(tn) * pr.ncs + ib) * 8192,
                        16384, &afull[p]);
              ++a_issues[p];
            }
            continue;
          }
          const int ls = gs % LS;
          if (!mbar_wait(&sfull[ls], static_cast<uint32_t>(gs / LS) & 1u, abort_flag)) { ok = false; break; }
          if (gs == 0 && ctid == 0) QLIN_STAMP(6);
          if (ctid == 0) QLIN_STEP(g, 2);
          if (g >= P && !mbar_wait(&aempty[p], static_cast<uint32_t>(g / P - 1) & 1u, abort_flag)) { ok = false; break; }
          if (ctid == 0) QLIN_STEP(g, 3);
          const unsigned char* stg = smem + C::kOffStg + ls * C::kStgBytes;
          unsigned char* A0 = smem + C::kOffA + p * C::kABytes;
          const int nchunk = min(C::KS, pr.kb - r * C::KS) * 512;  // 16-byte packed chunks this step
          // Token tiles >= 128 move one K-block per step: 512 chunks, at
          // most two per thread.  Both chunks (and their ratios) are loaded
          // before any operand store: the compiler cannot prove the staging
          // and operand rings disjoint, so an interleaved load would wait for
          // the previous store.
          static_assert(!C::kW4 || C::kTA || C::KS == 1, "shared-memory operand path converts one K-block per step");
          uint4 wpre[2];
          uint16_t rpre[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int c = ctid + u * kConvThreads;
            wpre[u] = c < nchunk ? *reinterpret_cast<const uint4*>(stg + c * 16) : make_uint4(0u, 0u, 0u, 0u);
            rpre[u] = (FMT == kFmtW4G128 && c < nchunk)
                          ? reinterpret_cast<const uint16_t*>(stg + C::kStgRatio)[(c >> 2) & 127]
                          : static_cast<uint16_t>(0);
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int c = ctid + u * kConvThreads;
            if (c >= nchunk) break;
            const int row = (c >> 2) & 127;
            const int part = (c & 3) ^ ((row >> 1) & 3);  // staged chunks are swizzled by row
            unsigned char* A = A0;
            const uint4 w = wpre[u];
            uint4 o0, o1;
            if (FMT == kFmtW4PC) {
              unpack_w4pc(w, o0, o1);
            } else {
              const __half2 r1 = __half2half2(__ushort_as_half(rpre[u]));
              const __half2 r16 = __hmul2(r1, __half2half2(__ushort_as_half(static_cast<unsigned short>(0x2C00))));  // * 1/16
              const uint2 a0 = requant_g128(w.x, r1, r16);
              const uint2 a1 = requant_g128(w.y, r1, r16);
              const uint2 a2 = requant_g128(w.z, r1, r16);
              const uint2 a3 = requant_g128(w.w, r1, r16);
              o0 = make_uint4(a0.x, a0.y, a1.x, a1.y);
              o1 = make_uint4(a2.x, a2.y, a3.x, a3.y);
            }
            const int sw = row & 7;
            *reinterpret_cast<uint4*>(A + row * 128 + (((2 * part) ^ sw) << 4)) = o0;
            *reinterpret_cast<uint4*>(A + row * 128 + (((2 * part + 1) ^ sw) << 4)) = o1;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&sempty[ls]);  // staging slot consumed
            mbar_arrive(&aconv[p]);    // A slot written
          }
          if (ctid == 0) QLIN_STEP(g, 4);
          ++gs;
        }
      }
      if (ctid == 0) {
        QLIN_STAMP(7);
        for (int p = 0; p < P; ++p) {  // outstanding W_O^T copies
          if (!a_issues[p]) continue;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait_sleep(&afull[p], (a_issues[p] - 1) & 1u, 1000000u) &&
                 globaltimer_ns() - t0 < QLIN_DRAIN_NS) {
          }
        }
      }
    }
    // ------------------------------------------------------------ epilogue
    if (epi) {
      const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
      const int nl = quad * 32 + lane;
      const int grp = (warp - C::kEpiWarp0) >> 2;  // epilogue group (two for 256-token INT8 tiles)
      const int gbar = 1 + grp;                    // its named barrier
      griddep_wait();  // a[] comes from the previous kernel
      // Partially covered tiles (at most the first and the last segment):
      // their counters and the finishing work run after every segment's
      // TMEM has been drained, so the mainloop never waits on them.
      unsigned pend_tile[2] = {0u, 0u};  // first iteration of each pending tile
      int pend_prob[2] = {0, 0};
      unsigned pend_loc[2] = {0u, 0u};   // its index within its problem
      int pend_add[2] = {0, 0};
      int npend = 0;
      SegGen gen = seg_begin(plan, cid, cl);
      Segment sg;
      int seg = 0;
      int ycnt = 0;  // Y chunks handed to TMA stores (two staging buffers alternate)
      float* sa_t = reinterpret_cast<float*>(smem + C::kOffSa + grp * 1024);
      while (seg_next(gen, sg, probs, nprob)) {
        const GemmProb& pr = probs[sg.p];
        const int buf = seg % nbuf;
        const int use = seg / nbuf;
        // everything that depends only on the tile is read before waiting for
        // its accumulator (the loads complete behind the mainloop)
        int tn, tm;
        tile_coords(pr, sg.tile, tn, tm);
        const int n = tn * C::kBN + nl;
        const int m0 = tm * BT;
        const int mvalid = min(BT, pr.M - m0);
        const bool pcomp = pr.nO > 0;  // this problem has outliers
        const bool has_main = sg.r0 < pr.nk;
        const bool has_comp = pcomp && sg.r1 == pr.T && sg.r0 <= pr.nk;
        const bool whole = sg.r0 == 0 && sg.r1 == pr.T;
        const float cn = chan_scale<FMT>(pr, n);
        float a_own = 0.f, cn_own = 0.f;  // cluster split-K: the owned slice's scales
        if (cl) {
          cn_own = chan_scale<FMT>(pr, tn * C::kBN + crk * slice + (nl % slice));
          if (nl < mvalid) a_own = pr.a[m0 + nl];
        }
        bool ok = mbar_wait(&acc_full[buf], static_cast<uint32_t>(use) & 1u, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (seg == 0 && nl == 0) QLIN_STAMP(10);
        tc_fence_after();
        if (grp > 0 && (cl || !whole)) {
          // the second group only shares whole tiles
          tc_fence_before();
          mbar_arrive(&acc_empty[buf]);
          ++seg;
          continue;
        }
        const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * bcols);
        const int my_slot = whole ? 0 : 2 * static_cast<int>(blockIdx.x) + (it0 < sg.tfirst ? 1 : 0);
        int32_t* pacc = args.ws_acc + static_cast<size_t>(my_slot) * BT * 128;
        float* pcmp = args.ws_comp + static_cast<size_t>(my_slot) * BT * 128;
        // cluster split-K: channel nl goes to owner rank nl / slice
        uint32_t r_main = 0, r_comp = 0, r_bar = 0;
        if (cl) {
          if (!cl_waited) {
            cluster_wait();
            cl_waited = true;
          }
          const int q = nl / slice;
          const int c = nl - q * slice;
          r_main = mapa_shared(smem_u32(smem + C::kOffRecv + ((crk * slice + c) * C::kRecvLd) * 4), q);
          r_comp = mapa_shared(smem_u32(smem + C::kOffRecv + C::kRecvMain + (c * C::kRecvLd) * 4), q);
          r_bar = mapa_shared(smem_u32(recv_full), q);
          // the owners have read this CTA's previous round
          if (seg > 0) ok = mbar_wait_cluster(recv_free, static_cast<uint32_t>(seg - 1) & 1u, abort_flag) && ok;
          ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
        }
        if (!cl && whole) {
          // token scales of the tile, staged once per group
          named_bar_sync(gbar, 128);
          for (int j = nl; j < BT; j += 128) sa_t[j] = j < mvalid ? pr.a[m0 + j] : 0.f;
          named_bar_sync(gbar, 128);
          if (seg == 0 && nl == 0) QLIN_STAMP(16);
        }
#pragma unroll 1
        for (int c0 = 0; c0 < BT; c0 += 16) {
          if (!cl && c0 >= mvalid) break;
          if (C::kEpiGroups > 1 && whole && ((c0 >> 4) & 1) != grp) continue;  // the other group's chunk
          uint32_t acc[16], cmp[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) { acc[j] = 0u; cmp[j] = 0u; }
          if (ok) {
            if (has_main) tmem_ld16(trow + c0, acc);
            if (has_comp) tmem_ld16(trow + BT + c0, cmp);
            tmem_ld_wait();
          }
          if (cl) {
            // every token column goes out (fixed byte count per round)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              st_async_v4(r_main + (c0 + 4 * i) * 4,
                          make_uint4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]), r_bar);
              if (has_comp)
                st_async_v4(r_comp + (c0 + 4 * i) * 4,
                            make_uint4(cmp[4 * i], cmp[4 * i + 1], cmp[4 * i + 2], cmp[4 * i + 3]), r_bar);
            }
          } else if (whole) {
            // 16 tokens x 128 channels of Y, transposed through shared
            // memory (written with thread = channel, read back with 16-byte
            // row segments) and stored with coalesced 16-byte stores.  Two
            // staging buffers alternate, so one barrier per chunk suffices:
            // the next write of a buffer comes after the barrier that
            // follows every thread's reads of it.
            const int b = ycnt & 1;
            uint16_t* ys = reinterpret_cast<uint16_t*>(smem + C::kOffYst + (grp * 2 + b) * C::kYStage);
            // the 16 token scales into registers before any staging store
            // (the compiler cannot prove the two shared arrays disjoint, so
            // interleaved loads would each wait for the previous store)
            float sc[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const float4 t = *reinterpret_cast<const float4*>(sa_t + c0 + 4 * q4);
              sc[4 * q4] = t.x; sc[4 * q4 + 1] = t.y; sc[4 * q4 + 2] = t.z; sc[4 * q4 + 3] = t.w;
            }
            uint16_t yh[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float v = __fmul_rn(cn, static_cast<float>(static_cast<int32_t>(acc[j])));
              if (pcomp) v = __fadd_rn(v, __uint_as_float(cmp[j]));
              yh[j] = __half_as_ushort(__float2half_rn(__fmul_rn(sc[j], v)));
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) ys[j * 128 + nl] = yh[j];
            if (pr.acc_debug) {
              for (int j = 0; j < 16; ++j)
                if (c0 + j < mvalid && n < pr.N)
                  pr.acc_debug[static_cast<size_t>(m0 + c0 + j) * pr.N + n] = static_cast<int32_t>(acc[j]);
            }
            named_bar_sync(gbar, 128);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int idx = nl + h * 128;  // 16 rows x 16 segments of 8 channels
              const int j = idx >> 4;
              const int n8 = tn * C::kBN + (idx & 15) * 8;
              if (c0 + j < mvalid && n8 < pr.N)
                *reinterpret_cast<uint4*>(pr.Y + static_cast<size_t>(m0 + c0 + j) * pr.N + n8) =
                    *reinterpret_cast<const uint4*>(ys + j * 128 + (idx & 15) * 8);
            }
            if (seg == 0 && nl == 0 && c0 == 0) QLIN_STAMP(17);
            ++ycnt;
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (c0 + j < mvalid) {
                const size_t o = static_cast<size_t>(c0 + j) * 128 + nl;
                pacc[o] = static_cast<int32_t>(acc[j]);
                if (has_comp) pcmp[o] = __uint_as_float(cmp[j]);
              }
            }
          }
        }
        if (seg == 0 && nl == 0) QLIN_STAMP(18);
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);  // TMEM buffer may be reused
        if (cl) {
          // Owner of channels [crk * slice, +slice): sum every rank's INT32
          // partial in rank order (exact), add the compensation, dequantize.
          // Thread t takes channel t % slice and token quads t / slice,
          // + cs, ...
          const int c = nl % slice;
          const int n_own = tn * C::kBN + crk * slice + c;
          float* sa = reinterpret_cast<float*>(smem + C::kOffSa);  // token scales of this tile
          if (nl < BT) sa[nl] = a_own;
          if (nl == 0 && seg == 0) QLIN_STAMP(23);
          ok = mbar_wait_cluster(recv_full, static_cast<uint32_t>(seg) & 1u, abort_flag) && ok;
          if (nl == 0 && seg == 0) QLIN_STAMP(12);
          ok = __all_sync(0xffffffffu, ok);
          named_bar_sync(1, 128);  // token scales staged
          const unsigned char* rb = smem + C::kOffRecv;
          // Thread t has token quads t / slice + k * cs, taken four at a
          // time: the group's shared-memory reads all happen before its
          // stores to Y (the compiler would otherwise order each read after
          // the preceding stores).
          constexpr int kG = 4;
          for (int k0 = 0; nl / slice + k0 * args.cs < BT / 4; k0 += kG) {
            int4 sum[kG];
            float4 cp[kG];
            float scl[kG][4];
#pragma unroll
            for (int k = 0; k < kG; ++k) {
              sum[k] = make_int4(0, 0, 0, 0);
              cp[k] = make_float4(0.f, 0.f, 0.f, 0.f);
              scl[k][0] = scl[k][1] = scl[k][2] = scl[k][3] = 0.f;
              const int jq = nl / slice + (k0 + k) * args.cs;
              if (jq < BT / 4) {
                for (int r = 0; r < args.cs; ++r) {
                  const int4 v = *reinterpret_cast<const int4*>(rb + ((r * slice + c) * C::kRecvLd + 4 * jq) * 4);
                  sum[k].x += v.x; sum[k].y += v.y; sum[k].z += v.z; sum[k].w += v.w;
                }
                if (pcomp) cp[k] = *reinterpret_cast<const float4*>(rb + C::kRecvMain + (c * C::kRecvLd + 4 * jq) * 4);
                const float4 t = *reinterpret_cast<const float4*>(sa + 4 * jq);
                scl[k][0] = t.x; scl[k][1] = t.y; scl[k][2] = t.z; scl[k][3] = t.w;
              }
            }
#pragma unroll
            for (int k = 0; k < kG; ++k) {
              const int jq = nl / slice + (k0 + k) * args.cs;
              if (jq >= BT / 4) break;
              const int s4[4] = {sum[k].x, sum[k].y, sum[k].z, sum[k].w};
              const float p4[4] = {cp[k].x, cp[k].y, cp[k].z, cp[k].w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int j = 4 * jq + i;
                if (ok && j < mvalid && n_own < pr.N) {
                  float v = __fmul_rn(cn_own, static_cast<float>(s4[i]));
                  if (pcomp) v = __fadd_rn(v, p4[i]);
                  const float y = __fmul_rn(scl[k][i], v);
                  pr.Y[static_cast<size_t>(m0 + j) * pr.N + n_own] = __half_as_ushort(__float2half_rn(y));
                  if (pr.acc_debug) pr.acc_debug[static_cast<size_t>(m0 + j) * pr.N + n_own] = s4[i];
                }
              }
            }
          }
          named_bar_sync(1, 128);  // every read of the receive buffer is done
          if (nl == 0 && cid + (seg + 1) * args.ncl < pr.tiles_n * pr.tiles_m) {
            mbar_arrive_expect_tx(recv_full, recv_bytes);  // next round
            for (int r = 0; r < args.cs; ++r) mbar_arrive_remote(mapa_shared(smem_u32(recv_free), r));
          }
        }
        if (!cl && !whole && npend < 2) {
          pend_tile[npend] = sg.tfirst;
          pend_prob[npend] = sg.p;
          pend_loc[npend] = sg.tile;
          pend_add[npend] = sg.r1 - sg.r0;
          ++npend;
        }
        ++seg;
      }
      if (nl == 0) QLIN_STAMP(11);
      if (npend > 0) {
        // Count this CTA's contributions (CTA barrier, then one thread's
        // acq_rel fence and atomic: the release covers every epilogue
        // thread's partial stores).  The CTA whose addition completes a
        // tile's T iterations finishes it.
        named_bar_sync(1, 128);
        if (nl == 0) {
          fence_acq_rel_gpu();
          bool any = false;
          for (int q = 0; q < npend; ++q) {
            const int c_lo = owner_cta_s(pend_tile[q], sbnd, args);
            const unsigned old = atom_add_relaxed_gpu(&args.ws_cnt[c_lo], static_cast<unsigned>(pend_add[q]));
            const bool last = old + static_cast<unsigned>(pend_add[q]) == static_cast<unsigned>(probs[pend_prob[q]].T);
            last_flag[q] = last ? 1 : 0;
            any = any || last;
          }
          if (any) fence_acq_rel_gpu();  // acquire the other contributors' partials
        }
        named_bar_sync(1, 128);
        if (nl == 0) QLIN_STAMP(12);
        for (int q = 0; q < npend; ++q) {
          if (!last_flag[q]) continue;
          const GemmProb& pr = probs[pend_prob[q]];
          const bool pcomp = pr.nO > 0;
          const unsigned tile = pend_loc[q];
          const unsigned first_it = pend_tile[q];
          const int c_lo = owner_cta_s(first_it, sbnd, args);
          const int c_hi = owner_cta_s(first_it + pr.T - 1, sbnd, args);
          int tn, tm;
          tile_coords(pr, tile, tn, tm);
          const int m0 = tm * BT;
          const int mvalid = min(BT, pr.M - m0);
          if (nl == 0) QLIN_STAMP(16 + 4 * q);
          // Thread t owns channels 4*(t % 32) .. +3, so a warp covers one
          // 128-channel row of the tile; warp w takes rows w, w + 4, ...
          // Every partial of those rows (and the token scales) is gathered
          // into the idle rings with cp.async, all copies in flight at once;
          // each thread then reduces exactly the elements it copied, and the
          // finished row goes out as one 256-byte store per warp.
          const int cg = nl & 31;
          const int wq = nl >> 5;
          const int n4 = tn * C::kBN + 4 * cg;
          const bool live = n4 < pr.N;
          float c4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) c4[i] = chan_scale<FMT>(pr, n4 + i);
          int nctr = 0;
          for (int c = c_lo; c <= c_hi; ++c) nctr += bnd_s(c, sbnd, args) != bnd_s(c + 1, sbnd, args) ? 1 : 0;
          const int blocks = nctr + (pcomp ? 1 : 0);
          int rows = C::kOffBar / (blocks * 512 + 4);
          rows = rows > 4 ? rows & ~3 : rows;
          int32_t* fin = reinterpret_cast<int32_t*>(smem);
          // kernel parameters used per row, held in registers (the stores
          // below would otherwise force reloads of the parameter block)
          uint16_t* const Yp = pr.Y;
          int32_t* const accd = pr.acc_debug;
          const size_t ldy = static_cast<size_t>(pr.N);
          for (int j0 = 0; j0 < mvalid; j0 += rows) {
            const int rr = min(rows, mvalid - j0);
            float* fa = reinterpret_cast<float*>(fin + static_cast<size_t>(blocks) * rr * 128);
            int qq = 0;
            for (int c = c_lo; c <= c_hi; ++c) {
              if (bnd_s(c, sbnd, args) == bnd_s(c + 1, sbnd, args)) continue;
              const int32_t* src = args.ws_acc + (static_cast<size_t>(partial_slot_s(c, first_it, sbnd)) * BT + j0) * 128 + 4 * cg;
              for (int j = wq; j < rr; j += 4) cp_async16(fin + (static_cast<size_t>(qq) * rr + j) * 128 + 4 * cg, src + j * 128);
              ++qq;
            }
            if (pcomp) {
              const float* src = args.ws_comp + (static_cast<size_t>(partial_slot_s(c_hi, first_it, sbnd)) * BT + j0) * 128 + 4 * cg;
              for (int j = wq; j < rr; j += 4) cp_async16(fin + (static_cast<size_t>(nctr) * rr + j) * 128 + 4 * cg, src + j * 128);
            }
            if (cg == 0)
              for (int j = wq; j < rr; j += 4) cp_async4(fa + j, pr.a + m0 + j0 + j);
            cp_async_wait_all();
            __syncwarp();  // lane 0's token scales
            if (nl == 0 && j0 == 0) QLIN_STAMP(17 + 4 * q);
            // four rows per thread at a time, contributors unrolled, so the
            // shared-memory loads are independent of one another
            for (int jb = wq; jb < rr; jb += 16) {
              int4 sum[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) sum[i] = make_int4(0, 0, 0, 0);
#pragma unroll 2
              for (int k = 0; k < nctr; ++k) {
                const int32_t* blk = fin + static_cast<size_t>(k) * rr * 128 + 4 * cg;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  if (jb + 4 * i < rr) {
                    const int4 v = *reinterpret_cast<const int4*>(blk + (jb + 4 * i) * 128);
                    sum[i].x += v.x; sum[i].y += v.y; sum[i].z += v.z; sum[i].w += v.w;
                  }
                }
              }
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int j = jb + 4 * i;
                if (j >= rr) break;
                float4 cp = make_float4(0.f, 0.f, 0.f, 0.f);
                if (pcomp) cp = *reinterpret_cast<const float4*>(fin + (static_cast<size_t>(nctr) * rr + j) * 128 + 4 * cg);
                const float am = fa[j];
                const int s4[4] = {sum[i].x, sum[i].y, sum[i].z, sum[i].w};
                const float p4[4] = {cp.x, cp.y, cp.z, cp.w};
                float y[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  float v = __fmul_rn(c4[e], static_cast<float>(s4[e]));
                  if (pcomp) v = __fadd_rn(v, p4[e]);
                  y[e] = __fmul_rn(am, v);
                }
                if (live) {
                  uint2 hv;
                  hv.x = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(y[0]))) |
                         (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(y[1]))) << 16);
                  hv.y = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(y[2]))) |
                         (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(y[3]))) << 16);
                  *reinterpret_cast<uint2*>(Yp + static_cast<size_t>(m0 + j0 + j) * ldy + n4) = hv;
                  if (accd) *reinterpret_cast<int4*>(accd + static_cast<size_t>(m0 + j0 + j) * ldy + n4) = sum[i];
                }
              }
              if (nl == 0 && q == 0 && j0 == 0 && jb < 112) QLIN_STAMP(24 + jb / 16);
            }
            __syncwarp();  // the warp's shared rows are reused by the next chunk
          }
          if (nl == 0) args.ws_cnt[c_lo] = 0u;
          if (nl == 0) QLIN_STAMP(18 + 4 * q);
        }
        if (nl == 0) QLIN_STAMP(13);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (cl) {  // no CTA leaves while a peer may still touch its shared memory
    if (!cl_waited) cluster_wait();
    cluster_arrive();
    cluster_wait();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
  if (threadIdx.x == 0) QLIN_STAMP(14);
}

}  // namespace qlin
