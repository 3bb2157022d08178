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
// Pipeline: two shared-memory rings.  The staging ring (INT4 formats) holds
// packed weight tiles straight from TMA and is released as soon as the
// converters have read a slot, so many of them can be in flight; the operand
// ring holds what the tensor core reads (the INT8 weight operand written by
// the converters, or by TMA for the INT8 format, and the activation or
// compensation tiles) and is released by tcgen05.commit.
//
// Warp roles:
//   warp 0        operand producer: activation tiles (after the grid
//                 dependency on the previous kernel), INT8 weight tiles,
//                 compensation operands (W_O^T tile, U hi/lo tiles).
//   warp 1        allocates TMEM (two accumulator buffers when they fit); one
//                 lane issues tcgen05.mma and commits.
//   warp 2        staging producer (INT4 formats): packed weights and the
//                 g128 ratio row; starts at once (weights do not depend on
//                 the previous kernel).
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
#ifdef QLIN_TRACE
__device__ long long* g_trace = nullptr;
#define QLIN_STAMP(k)                                                            \
  do {                                                                           \
    if (g_trace) g_trace[blockIdx.x * 16 + (k)] = static_cast<long long>(clock64()); \
  } while (0)
#else
#define QLIN_STAMP(k) do { } while (0)
#endif

struct GemmArgs {
  const float* cscale;  // c_n [N]
  const float* a;       // a_m [M]
  uint16_t* Y;          // [M][N] fp16
  int32_t* acc_debug;   // [M][N] or null
  int32_t* ws_acc;      // [2*grid][BT][128] INT32 partial sums of split tiles
  float* ws_comp;       // [2*grid][BT][128] fp32 compensation of split tiles
  unsigned* ws_cnt;     // [grid] iteration counters (zero on entry, left zero)
  int M, N, K, nO;
  int tiles_n, tiles_m;
  int nk;               // main K-steps per tile
  int nc;               // compensation steps per tile
  int ncs;              // 64-wide outlier slices
  int T;                // iterations per tile = nk + nc
  int grid;             // persistent CTAs (<= kMaxGrid)
  int split;            // 1: stream-K split points; 0: whole tiles per CTA
  // bnd[c] = first iteration of CTA c, bnd[grid] = tiles * T (computed on
  // the host by gemm_boundary(); kernel parameters, read from the constant
  // cache).
  unsigned bnd[kMaxGrid + 1];
};

template <int FMT, int BT>
struct GemmCfg {
  static constexpr int kBN = 128;                    // output channels per tile (MMA M)
  static constexpr int kBK = 128;                    // INT8 elements of K per stage (one swizzle row)
  static constexpr bool kW4 = FMT != kFmtW8;
  static constexpr int kNCW = FMT == kFmtW4G128 ? 8 : 4;  // converter warps (>= 4: epilogue)
  static constexpr int kThreads = 96 + 32 * kNCW;
  // Small token tiles load the hi and lo compensation operands in one stage
  // (one W_O^T tile feeds both); large ones use two passes.
  static constexpr bool kCompFused = BT <= 64;
  // operand slot: A (128 x 128 B), B (BT x 128 B), B2 (U lo, fused compensation)
  static constexpr int kOffA = 0;
  static constexpr int kOffB = 16384;
  static constexpr int kOffB2 = kOffB + BT * 128;
  static constexpr int kOpBytes = (kOffB2 + (kCompFused ? BT * 128 : 0) + 1023) / 1024 * 1024;
  // staging slot: packed INT4 (128 x 64 B) + g128 ratios (128 fp16)
  static constexpr int kStgBytes = kW4 ? 8192 + (FMT == kFmtW4G128 ? 256 : 0) : 0;
  static constexpr int kSmemLimit = 232448;   // 227 KB per CTA
  static constexpr int kReserve = 1024 + 768; // alignment slack + barriers
  static constexpr int kBudget = kSmemLimit - kReserve;
  static constexpr int kOpSlotsFit = kBudget / kOpBytes;
  static constexpr int kOpSlots = kW4 ? (BT <= 128 ? 4 : 3) : (kOpSlotsFit > 8 ? 8 : kOpSlotsFit);
  static constexpr int kStgSlotsFit = kW4 ? (kBudget - kOpSlots * kOpBytes) / kStgBytes : 0;
  static constexpr int kStgSlots = kStgSlotsFit > 16 ? 16 : kStgSlotsFit;
  static constexpr int kOffStg = kOpSlots * kOpBytes;
  static constexpr int kOffBar = kOffStg + kStgSlots * kStgBytes;
  static constexpr int kSmemBytes = kReserve + kOffBar;
  // TMA transaction bytes
  static constexpr uint32_t kTxStg = kW4 ? kStgBytes : 0;
  static constexpr uint32_t kTxMainOp = (kW4 ? 0 : 16384) + BT * 128;
  static constexpr uint32_t kTxComp = 16384 + (kCompFused ? 2 : 1) * BT * 128;
  static_assert(kOpSlots >= 2, "operand ring too small");
  static_assert(!kW4 || kStgSlots >= 2, "staging ring too small");
  static_assert(BT % 16 == 0 && BT >= 16 && BT <= 256, "MMA N must be 16..256 in steps of 16");
  static_assert(kOpSlots <= 8 && kStgSlots <= 16, "barrier area");
};

// TMEM columns per accumulator buffer and the number of buffers.
__host__ __device__ inline int tmem_buf_cols(int BT, bool comp) { return comp ? 2 * BT : BT; }
__host__ __device__ inline int tmem_nbuf(int BT, bool comp) { return 2 * tmem_buf_cols(BT, comp) <= 512 ? 2 : 1; }
__host__ __device__ inline uint32_t tmem_alloc_cols(int BT, bool comp) {
  const int need = tmem_nbuf(BT, comp) * tmem_buf_cols(BT, comp);
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(need)) c <<= 1;
  return c;
}

// First iteration owned by CTA c (host side; c == grid gives the total).
// Split points never fall strictly inside a tile's compensation run.
inline unsigned gemm_boundary(int c, long long tiles, int T, int nk, int grid, int split) {
  const long long I = tiles * T;
  if (c <= 0) return 0;
  if (c >= grid) return static_cast<unsigned>(I);
  if (!split) return static_cast<unsigned>(((tiles * c) / grid) * T);
  long long b = (I * c) / grid;
  const long long r = b % T;
  if (r > nk) b += T - r;
  return static_cast<unsigned>(b);
}

// The CTA whose range contains iteration `it` (binary search of the table).
__device__ __forceinline__ int owner_cta(unsigned it, const GemmArgs& g) {
  int lo = 0, hi = g.grid - 1;  // invariant: bnd[lo] <= it < bnd[hi + 1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (g.bnd[mid] <= it) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Scratch slot holding CTA c's partial of split tile `tile`: its first
// segment if its range starts inside the tile, else its last segment.
__device__ __forceinline__ int partial_slot(int c, unsigned tile, const GemmArgs& g) {
  return 2 * c + (g.bnd[c] < tile * static_cast<unsigned>(g.T) ? 1 : 0);
}

struct Segment {
  unsigned tile;
  int r0, r1;  // iterations [r0, r1) of the tile
};

__device__ __forceinline__ bool next_segment(unsigned& it, unsigned it1, const GemmArgs& g, Segment& sg) {
  if (it >= it1) return false;
  const unsigned T = static_cast<unsigned>(g.T);
  sg.tile = it / T;
  sg.r0 = static_cast<int>(it - sg.tile * T);
  const unsigned left = it1 - it;
  sg.r1 = static_cast<int>(left < T - sg.r0 ? sg.r0 + left : T);
  it += sg.r1 - sg.r0;
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
    while (!mbar_try_wait(&full[s], static_cast<uint32_t>(t / slots) & 1u) && globaltimer_ns() - t0 < QLIN_WAIT_NS) {
    }
  }
}

template <int FMT, int BT>
__global__ void __launch_bounds__(GemmCfg<FMT, BT>::kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
            const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmWO,
            const __grid_constant__ CUtensorMap tmU, const __grid_constant__ GemmArgs args) {
  using C = GemmCfg<FMT, BT>;
  constexpr int P = C::kOpSlots;
  constexpr int LS = C::kStgSlots;
  constexpr int kConvThreads = 32 * C::kNCW;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* ofull = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* oconv = ofull + 8;
  uint64_t* oempty = oconv + 8;
  uint64_t* sfull = oempty + 8;
  uint64_t* sempty = sfull + 16;
  uint64_t* acc_full = sempty + 16;   // [2]
  uint64_t* acc_empty = acc_full + 2; // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;  // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool comp = args.nO > 0;
  const int bcols = tmem_buf_cols(BT, comp);
  const int nbuf = tmem_nbuf(BT, comp);
  const uint32_t tcols = tmem_alloc_cols(BT, comp);
  const unsigned it0 = args.bnd[blockIdx.x];
  const unsigned it1 = args.bnd[blockIdx.x + 1];
#ifdef QLIN_TRACE
  if (threadIdx.x == 0 && g_trace) g_trace[blockIdx.x * 16 + 15] = static_cast<long long>(globaltimer_ns());
#endif
  if (threadIdx.x == 0) QLIN_STAMP(0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < P; ++s) {
      mbar_init(&ofull[s], 1);
      mbar_init(&oconv[s], kConvThreads);
      mbar_init(&oempty[s], 1);
    }
    for (int s = 0; s < LS; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], kConvThreads);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    if (!C::kW4) tma_prefetch_desc(&tmW);
    if (comp) {
      tma_prefetch_desc(&tmWO);
      tma_prefetch_desc(&tmU);
    }
  }
  if (warp == 2 && lane == 0 && C::kW4) {
    tma_prefetch_desc(&tmW);
    if (FMT == kFmtW4G128) tma_prefetch_desc(&tmR);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) QLIN_STAMP(1);
  // Let the next kernel in the stream start its prologue; it waits for this
  // grid to complete before it touches anything this kernel writes.
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ operand producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      // part 0: expect the slot's bytes and load the weight side (INT8
      // weights or W_O^T); part 1: the activation side; 2: both.
      auto issue = [&](const Segment& sg, int r, int p, int part) {
        unsigned char* op = smem + p * C::kOpBytes;
        const int tn = static_cast<int>(sg.tile % args.tiles_n);
        const int tm = static_cast<int>(sg.tile / args.tiles_n);
        const int n0 = tn * C::kBN, m0 = tm * BT;
        if (r < args.nk) {
          const int k0 = r * C::kBK;
          if (part != 1) {
            mbar_arrive_expect_tx(&ofull[p], C::kTxMainOp);
            if (!C::kW4) tma_load_2d_hint(op + C::kOffA, &tmW, &ofull[p], k0, n0, pol_stream);
          }
          if (part != 0) tma_load_2d(op + C::kOffB, &tmX, &ofull[p], k0, m0);
        } else {
          const int j = r - args.nk;
          int i0, y;
          if (C::kCompFused) {
            i0 = j * 64;
            y = m0;
          } else {
            const int lo = j >= args.ncs ? 1 : 0;  // U rows [0, M) hold hi, [M, 2M) hold lo
            i0 = (j - lo * args.ncs) * 64;
            y = lo * args.M + m0;
          }
          if (part != 1) {
            mbar_arrive_expect_tx(&ofull[p], C::kTxComp);
            tma_load_2d(op + C::kOffA, &tmWO, &ofull[p], i0, n0);
          }
          if (part != 0) {
            tma_load_2d(op + C::kOffB, &tmU, &ofull[p], i0, y);
            if (C::kCompFused) tma_load_2d(op + C::kOffB2, &tmU, &ofull[p], i0, args.M + m0);
          }
        }
      };
      // pass 1: weight side of the first P iterations (independent of the
      // previous kernel), then wait for the grid dependency.
      int pre = 0;
      {
        unsigned ita = it0;
        Segment sa;
        while (pre < P && next_segment(ita, it1, args, sa))
          for (int r = sa.r0; r < sa.r1 && pre < P; ++r, ++pre) issue(sa, r, pre, 0);
      }
      griddep_wait();
      QLIN_STAMP(4);
      unsigned it = it0;
      Segment sg;
      int g = 0;
      bool ok = true;
      while (ok && next_segment(it, it1, args, sg)) {
        for (int r = sg.r0; r < sg.r1; ++r, ++g) {
          const int p = g % P;
          if (g < P) {
            issue(sg, r, p, 1);
          } else {
            if (!mbar_wait(&oempty[p], static_cast<uint32_t>(g / P - 1) & 1u, abort_flag)) { ok = false; break; }
            issue(sg, r, p, 2);
          }
        }
      }
      QLIN_STAMP(5);
      drain_ring(ofull, P, g > pre ? g : pre);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ staging producer
    if (lane == 0 && C::kW4) {
      const uint64_t pol_stream = policy_evict_first();
      unsigned it = it0;
      Segment sg;
      int gs = 0;
      bool ok = true;
      while (ok && next_segment(it, it1, args, sg)) {
        const int n0 = static_cast<int>(sg.tile % args.tiles_n) * C::kBN;
        const int rend = sg.r1 < args.nk ? sg.r1 : args.nk;
        for (int r = sg.r0; r < rend; ++r, ++gs) {
          const int ls = gs % LS;
          if (gs >= LS && !mbar_wait(&sempty[ls], static_cast<uint32_t>(gs / LS - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          unsigned char* st = smem + C::kOffStg + ls * C::kStgBytes;
          mbar_arrive_expect_tx(&sfull[ls], C::kTxStg);
          tma_load_2d_hint(st, &tmW, &sfull[ls], r * (C::kBK / 2), n0, pol_stream);
          if (FMT == kFmtW4G128) tma_load_2d(st + 8192, &tmR, &sfull[ls], n0, r);
          if (gs == 0) QLIN_STAMP(2);
        }
      }
      QLIN_STAMP(3);
      drain_ring(sfull, LS, gs);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_main = idesc_s8_s32(128, BT);
      constexpr uint32_t idesc_comp = idesc_f16_f32(128, BT);
      uint32_t conv_phase = 0;  // one parity bit per operand slot
      unsigned it = it0;
      Segment sg;
      int g = 0, seg = 0;
      bool ok = true;
      while (ok && next_segment(it, it1, args, sg)) {
        const int buf = seg % nbuf;
        const int use = seg / nbuf;
        if (use > 0 && !mbar_wait(&acc_empty[buf], static_cast<uint32_t>(use - 1) & 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t dmain = tmem + static_cast<uint32_t>(buf * bcols);
        const uint32_t dcomp = dmain + BT;
        for (int r = sg.r0; r < sg.r1; ++r, ++g) {
          const int p = g % P;
          const bool main_step = r < args.nk;
          if (!mbar_wait(&ofull[p], static_cast<uint32_t>(g / P) & 1u, abort_flag)) { ok = false; break; }
          if (g == 0) QLIN_STAMP(8);
          if (main_step && C::kW4) {
            if (!mbar_wait(&oconv[p], (conv_phase >> p) & 1u, abort_flag)) { ok = false; break; }
            conv_phase ^= 1u << p;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + p * C::kOpBytes + C::kOffA);
          const uint32_t b_addr = smem_u32(smem + p * C::kOpBytes + C::kOffB);
          if (main_step) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_i8(dmain, sdesc_k_sw128(a_addr + 32 * kk), sdesc_k_sw128(b_addr + 32 * kk), idesc_main,
                     (r > sg.r0 || kk > 0) ? 1u : 0u);
          } else {
            const bool first = (r == args.nk) || (r == sg.r0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16(dcomp, sdesc_k_sw128(a_addr + 32 * kk), sdesc_k_sw128(b_addr + 32 * kk), idesc_comp,
                      (!first || kk > 0) ? 1u : 0u);
            if (C::kCompFused) {
              const uint32_t b2_addr = smem_u32(smem + p * C::kOpBytes + C::kOffB2);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_f16(dcomp, sdesc_k_sw128(a_addr + 32 * kk), sdesc_k_sw128(b2_addr + 32 * kk), idesc_comp, 1u);
            }
          }
          mma_commit(&oempty[p]);
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
        ++seg;
      }
      QLIN_STAMP(9);
    }
    __syncwarp();
  } else {
    const int ctid = threadIdx.x - 96;
    // ------------------------------------------------------------ converters
    if (C::kW4) {
      unsigned it = it0;
      Segment sg;
      int g = 0, gs = 0;
      bool ok = true;
      while (ok && next_segment(it, it1, args, sg)) {
        for (int r = sg.r0; r < sg.r1; ++r, ++g) {
          if (r >= args.nk) continue;
          const int p = g % P;
          const int ls = gs % LS;
          if (!mbar_wait(&sfull[ls], static_cast<uint32_t>(gs / LS) & 1u, abort_flag)) { ok = false; break; }
          if (gs == 0 && ctid == 0) QLIN_STAMP(6);
          if (g >= P && !mbar_wait(&oempty[p], static_cast<uint32_t>(g / P - 1) & 1u, abort_flag)) { ok = false; break; }
          const unsigned char* stg = smem + C::kOffStg + ls * C::kStgBytes;
          unsigned char* A = smem + p * C::kOpBytes + C::kOffA;
#pragma unroll 2
          for (int c = ctid; c < 512; c += kConvThreads) {
            const int row = c >> 2;
            const int part = c & 3;
            const uint4 w = *reinterpret_cast<const uint4*>(stg + c * 16);
            uint4 o0, o1;
            if (FMT == kFmtW4PC) {
              unpack_w4pc(w, o0, o1);
            } else {
              const uint16_t rb = reinterpret_cast<const uint16_t*>(stg + 8192)[row];
              const __half2 r1 = __half2half2(__ushort_as_half(rb));
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
          mbar_arrive(&sempty[ls]);  // staging slot consumed
          fence_proxy_async_smem();
          mbar_arrive(&oconv[p]);
          ++gs;
        }
      }
      if (ctid == 0) QLIN_STAMP(7);
    }
    // ------------------------------------------------------------ epilogue
    if (warp < 7) {
      const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
      const int nl = quad * 32 + lane;
      griddep_wait();  // a[] comes from the previous kernel
      // Partially covered tiles (at most the first and the last segment):
      // their counters and the finishing work run after every segment's
      // TMEM has been drained, so the mainloop never waits on them.
      unsigned pend_tile[2] = {0u, 0u};
      int pend_add[2] = {0, 0};
      int npend = 0;
      unsigned it = it0;
      Segment sg;
      int seg = 0;
      while (next_segment(it, it1, args, sg)) {
        const int buf = seg % nbuf;
        const int use = seg / nbuf;
        bool ok = mbar_wait(&acc_full[buf], static_cast<uint32_t>(use) & 1u, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (seg == 0 && nl == 0) QLIN_STAMP(10);
        tc_fence_after();
        const int tn = static_cast<int>(sg.tile % args.tiles_n);
        const int tm = static_cast<int>(sg.tile / args.tiles_n);
        const int n = tn * C::kBN + nl;
        const int m0 = tm * BT;
        const int mvalid = min(BT, args.M - m0);
        const bool has_main = sg.r0 < args.nk;
        const bool has_comp = comp && sg.r1 == args.T && sg.r0 <= args.nk;
        const bool whole = sg.r0 == 0 && sg.r1 == args.T;
        const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * bcols);
        const float cn = n < args.N ? (FMT == kFmtW4PC ? __fmul_rn(args.cscale[n], 0.0625f) : args.cscale[n]) : 0.f;
        const int my_slot = whole ? 0 : partial_slot(static_cast<int>(blockIdx.x), sg.tile, args);
        int32_t* pacc = args.ws_acc + static_cast<size_t>(my_slot) * BT * 128;
        float* pcmp = args.ws_comp + static_cast<size_t>(my_slot) * BT * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < BT; c0 += 16) {
          if (c0 >= mvalid) break;
          uint32_t acc[16], cmp[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) { acc[j] = 0u; cmp[j] = 0u; }
          if (ok) {
            if (has_main) tmem_ld16(trow + c0, acc);
            if (has_comp) tmem_ld16(trow + BT + c0, cmp);
            tmem_ld_wait();
          }
          if (whole) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int m = m0 + c0 + j;
              if (c0 + j < mvalid && n < args.N) {
                float v = __fmul_rn(cn, static_cast<float>(static_cast<int32_t>(acc[j])));
                if (comp) v = __fadd_rn(v, __uint_as_float(cmp[j]));
                const float y = __fmul_rn(args.a[m], v);
                args.Y[static_cast<size_t>(m) * args.N + n] = __half_as_ushort(__float2half_rn(y));
                if (args.acc_debug) args.acc_debug[static_cast<size_t>(m) * args.N + n] = static_cast<int32_t>(acc[j]);
              }
            }
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
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);  // TMEM buffer may be reused
        if (!whole && npend < 2) {
          pend_tile[npend] = sg.tile;
          pend_add[npend] = sg.r1 - sg.r0;
          ++npend;
        }
        ++seg;
      }
      if (nl == 0) QLIN_STAMP(11);
      if (npend > 0) {
        __threadfence();
        named_bar_sync(1, 128);
        if (nl == 0) {
          for (int q = 0; q < npend; ++q) {
            const int c_lo = owner_cta(pend_tile[q] * static_cast<unsigned>(args.T), args);
            const unsigned old = atomicAdd(&args.ws_cnt[c_lo], static_cast<unsigned>(pend_add[q]));
            last_flag[q] = (old + static_cast<unsigned>(pend_add[q]) == static_cast<unsigned>(args.T)) ? 1 : 0;
          }
        }
        named_bar_sync(1, 128);
        if (nl == 0) QLIN_STAMP(12);
        for (int q = 0; q < npend; ++q) {
          if (!last_flag[q]) continue;
          __threadfence();
          const unsigned tile = pend_tile[q];
          const unsigned first_it = tile * static_cast<unsigned>(args.T);
          const int c_lo = owner_cta(first_it, args);
          const int c_hi = owner_cta(first_it + args.T - 1, args);
          const int tn = static_cast<int>(tile % args.tiles_n);
          const int tm = static_cast<int>(tile / args.tiles_n);
          const int n = tn * C::kBN + nl;
          const int m0 = tm * BT;
          const int mvalid = min(BT, args.M - m0);
          const float cn = n < args.N ? (FMT == kFmtW4PC ? __fmul_rn(args.cscale[n], 0.0625f) : args.cscale[n]) : 0.f;
          const float* ccmp = args.ws_comp + static_cast<size_t>(partial_slot(c_hi, tile, args)) * BT * 128;
          // rows in groups of 8, contributors in groups of 4: 32 independent loads in flight
          for (int j0 = 0; j0 < mvalid; j0 += 8) {
            int32_t av[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) av[r] = 0;
            for (int cb = c_lo; cb <= c_hi; cb += 4) {
              int32_t v[4][8];
#pragma unroll
              for (int cc = 0; cc < 4; ++cc) {
                const int c = cb + cc;
                const bool live = c <= c_hi && args.bnd[c] != args.bnd[c + 1];
                const int32_t* src = args.ws_acc + static_cast<size_t>(live ? partial_slot(c, tile, args) : 0) * BT * 128;
#pragma unroll
                for (int r = 0; r < 8; ++r)
                  v[cc][r] = (live && j0 + r < mvalid) ? __ldcg(src + static_cast<size_t>(j0 + r) * 128 + nl) : 0;
              }
#pragma unroll
              for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                for (int r = 0; r < 8; ++r) av[r] += v[cc][r];
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              const int j = j0 + r;
              if (j < mvalid && n < args.N) {
                const int m = m0 + j;
                float vv = __fmul_rn(cn, static_cast<float>(av[r]));
                if (comp) vv = __fadd_rn(vv, __ldcg(ccmp + static_cast<size_t>(j) * 128 + nl));
                const float y = __fmul_rn(args.a[m], vv);
                args.Y[static_cast<size_t>(m) * args.N + n] = __half_as_ushort(__float2half_rn(y));
                if (args.acc_debug) args.acc_debug[static_cast<size_t>(m) * args.N + n] = av[r];
              }
            }
          }
          if (nl == 0) args.ws_cnt[c_lo] = 0u;
          if (nl == 0) QLIN_STAMP(13);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
  if (threadIdx.x == 0) QLIN_STAMP(14);
}

}  // namespace qlin
