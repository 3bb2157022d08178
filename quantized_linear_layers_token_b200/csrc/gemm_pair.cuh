// gemm_pair.cuh -- stages 2 and 3 for many-token calls on two SMs at a time.
//
// The INT8 contraction of a 256-channel x 256-token tile is one tensor-core
// operation of 256 rows shared by a pair of CTAs (a 2-CTA cluster,
// tcgen05 cta_group::2): each CTA loads its own 128 weight rows and its own
// 128 tokens of every K-block into its shared memory, the even CTA issues
// tcgen05.mma.cta_group::2 over both halves, and each CTA's tensor memory
// receives the accumulator of its 128 channels for all 256 tokens.  Per SM
// and K-block that is 16 KB of weights and 16 KB of activations (against
// 16 + 32 KB when one CTA computes a 128 x 256 tile alone), which is what
// bounds the single-CTA kernel on many-token calls: the operand stream from
// L2 into each SM.  No load is multicast: every CTA loads its own halves.
//
// Operands are INT8: the INT8 weight format, or INT4 weights widened once
// per call (16 q per-channel, q8 for g128; gemm.cuh).  The compensation of
// the outlier channels (the Quaff term X_hat[:,O] (s_O - 1) W_O) runs
// after the K-blocks of a tile as kind::f16 pair operations of W_O^T x U
// (hi and lo passes) into a second accumulator; the epilogue computes
// Y = fp16(a_m (c'_n acc + comp)) exactly as the single-CTA kernel does.
//
// Roles per CTA (both CTAs of a pair run all of them, the MMA only in the
// even CTA):
//   warp 0        producer: per step one TMA load of the weight (or W_O^T)
//                 block rows and one of the activation (or U) rows, both
//                 counted on the even CTA's full barrier; waits for its own
//                 empty barrier (released by the pair's MMA commit).
//   warp 1        tensor memory allocation (both CTAs, cta_group::2); in the
//                 even CTA the whole warp runs the MMA loop and an elected
//                 lane issues the pair MMAs and commits.
//   warps 2..9    epilogue, two groups of four warps taking alternate
//                 16-token chunks of the CTA's 128 x 256 accumulator into an
//                 fp16 output tile in shared memory; each warp then arrives
//                 on the even CTA's accumulator-empty barrier (so the next
//                 tile's products start), and one thread writes the output
//                 tile with a TMA store that runs under them.
#pragma once

#include "gemm.cuh"

namespace qlin {

constexpr int kPairStage = 32768;  // per CTA and step: 16 KB weight rows + 16 KB token rows
constexpr int kPairEpiWarps = 8;
constexpr int kMaxPairs = 128;     // pairs in one launch (stream-K boundary table)

// FMT = kFmtW8: the INT8 weight rows arrive by TMA (the INT8 format, or INT4
// widened ahead of the GEMM).  FMT = kFmtW4PC / kFmtW4G128: the packed INT4
// blocks arrive in a staging ring and eight converter warps per CTA widen
// them into the stage's weight rows (the arithmetic of widen_w4_kernel).
template <int FMT>
struct PairCfg {
  static constexpr bool kConv = FMT != kFmtW8;
  static constexpr int S = kConv ? 4 : 5;             // stages of weight + token rows
  static constexpr int LS = kConv ? 3 : 0;            // staging slots of packed blocks
  static constexpr int kStgBytes = 8192 + 256;        // packed block + the g128 ratio row
  static constexpr int kOffStg = S * kPairStage;
  static constexpr int kOffY = kOffStg + (LS * kStgBytes + 1023) / 1024 * 1024;  // output tile
  static constexpr int kOffBar = kOffY + 256 * 128 * 2;
  static constexpr int kOffSa = kOffBar + 256;
  static constexpr int kSmem = kOffSa + 1024 + 1024;  // + alignment slack
  static constexpr int kConvWarps = kConv ? 8 : 0;
  static constexpr int kThreads = 32 * (2 + kPairEpiWarps + kConvWarps);
  static_assert(kSmem <= 232448, "pair kernel shared memory above 227 KB");
};

struct PairArgs {
  const uint8_t* codes;      // packed INT4 blocks (converting kernels)
  const uint16_t* rfold;     // g128 ratios r [K/128][N]
  const float* cscale;
  float cmul;         // factor on c_n (1, or 1/16 for per-channel INT4 widened to 16 q)
  const float* a;
  uint16_t* Y;
  int32_t* acc_debug;
  int M, N, nO;
  int kb;             // 128-wide K-blocks
  int ntn;            // 128-channel tiles of the weights
  int ncs;            // 64-wide outlier slices
  int T;              // steps per tile: kb + 2 ncs
  int tiles_n2;       // 256-channel pair tiles
  int tiles_m;        // 256-token tiles
  int gm;             // raster group of token tiles
  int tiles;          // tiles_n2 * tiles_m
  int ncl;            // clusters (pairs) in the grid
  // Stream-K tail: tiles [0, dp) are whole tiles, pair c taking c, c + ncl,
  // ...; the steps of tiles [dp, tiles) are split in contiguous ranges,
  // pair c taking [bnd[c], bnd[c + 1]) of them (bnd[ncl] = their total).
  // Tiles split across pairs leave INT32 partials in ws_acc slots
  // [2 * pair + (first segment of its range ? 0 : 1)][CTA][256 tokens][128
  // channels], and the range holding a tile's compensation steps (never
  // split, always the first segment of that range) leaves it, fp32, in
  // ws_comp [pair][CTA][256][128]; ws_cnt counts each split tile's finished
  // steps per CTA, and the range whose steps complete the count sums the
  // partials and writes Y.
  int dp;
  int32_t* ws_acc;
  float* ws_comp;
  unsigned* ws_cnt;   // [tiles - dp][2], zero between launches
  unsigned bnd[kMaxPairs + 1];
};

struct alignas(64) PairParams {
  CUtensorMap tmA;   // weight blocks as rows of 128 bytes: [ntn * kb * 128][128]
  CUtensorMap tmX;   // Xq int8 [M][K], 128 x 128 boxes, 128-byte swizzle
  CUtensorMap tmU;   // U fp16 [2M][nOp], 64 x 128 boxes, 128-byte swizzle
  CUtensorMap tmWo;  // W_O^T blocks as rows of 128 bytes: [ntn * ncs * 128][128]
  CUtensorMap tmY;   // Y fp16 [M][N], 128 x 256 boxes (stores)
  PairArgs g;
};

__device__ __forceinline__ void pair_tile_coords(const PairArgs& g, int t, int& tn2, int& tm) {
  const int per = g.gm * g.tiles_n2;
  const int grp = t / per;
  const int w = t - grp * per;
  const int g0 = grp * g.gm;
  const int gs = g.tiles_m - g0 < g.gm ? g.tiles_m - g0 : g.gm;
  tm = g0 + w % gs;
  tn2 = w / gs;
}

// One unit of a pair's work: steps [r0, r1) of tile t.
struct PairSeg {
  int t;
  int r0, r1;
  int slot;  // partial slot, or -1 for a whole tile
  int sk;    // index of the tile among the split tail (t - dp), -1 for whole tiles before it
};
struct PairGen {
  int t;
  unsigned it, it1;
};
__device__ __forceinline__ PairGen pair_begin(const PairArgs& g, int cid) {
  PairGen s;
  s.t = cid;
  s.it = g.bnd[cid];
  s.it1 = g.bnd[cid + 1];
  return s;
}
__device__ __forceinline__ bool pair_next(const PairArgs& g, int cid, PairGen& s, PairSeg& w) {
  if (s.t < g.dp) {
    w.t = s.t;
    w.r0 = 0;
    w.r1 = g.T;
    w.slot = -1;
    w.sk = -1;
    s.t += g.ncl;
    return true;
  }
  if (s.it >= s.it1) return false;
  const unsigned T = static_cast<unsigned>(g.T);
  const unsigned i = s.it / T;
  const unsigned r0 = s.it - i * T;
  const unsigned left = s.it1 - s.it;
  const unsigned r1 = left < T - r0 ? r0 + left : T;
  w.t = g.dp + static_cast<int>(i);
  w.r0 = static_cast<int>(r0);
  w.r1 = static_cast<int>(r1);
  w.sk = static_cast<int>(i);
  w.slot = (r0 == 0 && r1 == T) ? -1 : 2 * cid + (s.it == g.bnd[cid] ? 0 : 1);
  s.it += r1 - r0;
  return true;
}
// Pair whose range holds step `it` of the split tail (bnd[c] <= it < bnd[c + 1]).
__device__ __forceinline__ int pair_owner(const PairArgs& g, unsigned it) {
  int lo = 0, hi = g.ncl - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (g.bnd[mid] <= it) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int FMT>
__global__ void __launch_bounds__(PairCfg<FMT>::kThreads, 1) gemm_pair_kernel(const __grid_constant__ PairParams prm) {
  using C = PairCfg<FMT>;
  const PairArgs& g = prm.g;
  constexpr int S = C::S;
  constexpr int LS = C::LS > 0 ? C::LS : 1;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);  // [S] (the even CTA's are used)
  uint64_t* empty = full + S;                                        // [S] (each CTA's own)
  uint64_t* aready = empty + S;                                      // [S] converted rows (the even CTA's)
  uint64_t* sfull = aready + S;                                      // [LS] staging (each CTA's own)
  uint64_t* sempty = sfull + LS;                                     // [LS]
  uint64_t* acc_full = sempty + LS;                                  // each CTA's own
  uint64_t* acc_empty = acc_full + 1;                                // the even CTA's
  uint64_t* mma_done = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* fin_flag = abort_flag + 1;  // epilogue: this CTA completes the split tile
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int crk = static_cast<int>(cluster_ctarank());
  const int cid = static_cast<int>(cluster_id_x());
  const bool leader = crk == 0;
  const bool comp = g.nO > 0;
  QLIN_TRACE_INIT

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      if (C::kConv) mbar_init(&aready[s], 2 * C::kConvWarps);
    }
    for (int s = 0; s < C::LS; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], C::kConvWarps);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kPairEpiWarps);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 1) {
    if (!C::kConv) tma_prefetch_desc(&prm.tmA);
    tma_prefetch_desc(&prm.tmX);
    if (comp) {
      tma_prefetch_desc(&prm.tmU);
      tma_prefetch_desc(&prm.tmWo);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();  // both CTAs' barriers exist before either touches the other's
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      griddep_wait();  // Xq, U and widened weights come from the previous kernels
      const uint32_t lfull0 = mapa_shared(smem_u32(&full[0]), 0);
      int gi = 0;
      bool ok = true;
      PairGen gen = pair_begin(g, cid);
      PairSeg sg;
      while (ok && pair_next(g, cid, gen, sg)) {
        int tn2, tm;
        pair_tile_coords(g, sg.t, tn2, tm);
        const int ctile = 2 * tn2 + crk;    // this CTA's 128 channels
        const int m0 = tm * 256 + crk * 128;  // this CTA's 128 tokens
        for (int r = sg.r0; r < sg.r1; ++r, ++gi) {
          const int s = gi % S;
          if (gi >= S && !mbar_wait(&empty[s], static_cast<uint32_t>(gi / S - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          const bool conv = C::kConv && r < g.kb;  // weight rows from the converters
          if (leader) mbar_arrive_expect_tx(&full[s], conv ? 2u * 16384u : 2u * kPairStage);
          QLIN_STEP(gi, 0);
          unsigned char* A = smem + s * kPairStage;
          unsigned char* X = A + 16384;
          const uint32_t lb = lfull0 + static_cast<uint32_t>(8 * s);
          if (conv) {
            tma_load_2d_pair(X, &prm.tmX, lb, r * 128, m0);  // weight rows: converters
          } else if (r < g.kb) {
            tma_load_2d_pair(A, &prm.tmA, lb, 0, (ctile * g.kb + r) * 128);
            tma_load_2d_pair(X, &prm.tmX, lb, r * 128, m0);
          } else {
            const int j = r - g.kb;
            const int lo = j >= g.ncs ? 1 : 0;  // U rows [0, M) hold hi, [M, 2M) hold lo
            const int ib = j - lo * g.ncs;
            tma_load_2d_pair(A, &prm.tmWo, lb, 0, (ctile * g.ncs + ib) * 128);
            tma_load_2d_pair(X, &prm.tmU, lb, ib * 64, lo * g.M + m0);
          }
        }
      }
      // every stage this CTA filled has been consumed by the pair's MMAs (so
      // its copies have landed) before the CTA can leave
      for (int t = gi - 1; t >= 0 && t >= gi - S; --t) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(&empty[t % S], static_cast<uint32_t>(t / S) & 1u, 1000000u) &&
               globaltimer_ns() - t0 < QLIN_DRAIN_NS) {
        }
      }
    } else if (C::kConv && lane == 1) {
      // staging producer: the packed blocks (and g128 ratio rows) of the
      // main steps, as far ahead as the staging ring allows, independent of
      // the stage ring (lane 0)
      int gs = 0;
      bool ok = true;
      PairGen gen = pair_begin(g, cid);
      PairSeg sg;
      while (ok && pair_next(g, cid, gen, sg)) {
        int tn2, tm;
        pair_tile_coords(g, sg.t, tn2, tm);
        const int ctile = 2 * tn2 + crk;
        const int n0 = ctile * 128;
        const uint32_t rb = FMT == kFmtW4G128 ? static_cast<uint32_t>(max(0, min(128, g.N - n0))) * 2u : 0u;
        // the odd CTA of the last pair tile may lie past the weights (an odd
        // number of channel tiles): nothing to load, its rows are never stored
        const bool have = ctile < g.ntn;
        const int r1 = min(sg.r1, g.kb);
        for (int r = sg.r0; r < r1; ++r, ++gs) {
          const int ls = gs % LS;
          if (gs >= LS && !mbar_wait(&sempty[ls], static_cast<uint32_t>(gs / LS - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          unsigned char* st = smem + C::kOffStg + ls * C::kStgBytes;
          mbar_arrive_expect_tx(&sfull[ls], have ? 8192u + rb : 0u);
          if (have) {
            bulk_load(st, g.codes + (static_cast<size_t>(ctile) * g.kb + r) * 8192, 8192u, &sfull[ls]);
            if (rb) bulk_load(st + 8192, g.rfold + static_cast<size_t>(r) * g.N + n0, rb, &sfull[ls]);
          }
        }
      }
      drain_ring(sfull, LS, gs);  // the converters consume every copy unless aborted
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ pair MMA (even CTA)
    // The leader's whole warp runs the loop and its waits; an elected lane
    // issues the pair instructions and commits.
    if (leader) {
      constexpr uint32_t idesc_main = idesc_s8_s32(256, 256);
      constexpr uint32_t idesc_comp = idesc_f16_f32(256, 256);
      const uint64_t adesc0 = sdesc_k_sw128(smem_u32(smem));
      const uint64_t bdesc0 = sdesc_k_sw128(smem_u32(smem + 16384));
      int gi = 0, ti = 0;
      bool ok = true, issued = false;
      PairGen gen = pair_begin(g, cid);
      PairSeg sg;
      for (; ok && pair_next(g, cid, gen, sg); ++ti) {
        if (ti > 0 && !warp_agree(mbar_wait_cluster(acc_empty, static_cast<uint32_t>(ti - 1) & 1u, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int r = sg.r0; r < sg.r1; ++r, ++gi) {
          const int s = gi % S;
          if (!warp_wait(&full[s], static_cast<uint32_t>(gi / S) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          QLIN_STEP(gi, 1);
          if (C::kConv && !warp_agree(mbar_wait_cluster_poll(&aready[s], static_cast<uint32_t>(gi / S) & 1u, abort_flag))) {
            ok = false;
            break;
          }
          QLIN_STEP(gi, 5);
          tc_fence_after();
          issued = true;
          const uint64_t ad = adesc0 + static_cast<uint64_t>(s * (kPairStage >> 4));
          const uint64_t bd = bdesc0 + static_cast<uint64_t>(s * (kPairStage >> 4));
          if (elect_one()) {
            if (r < g.kb) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_i8_pair(tmem, ad + 2 * k, bd + 2 * k, idesc_main, (r > sg.r0 || k > 0) ? 1u : 0u);
            } else {
              const int j = r - g.kb;
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_f16_pair(tmem + 256, ad + 2 * k, bd + 2 * k, idesc_comp, (j > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit_pair(&empty[s], 0x3);
          }
          __syncwarp();
          QLIN_STEP(gi, 7);
        }
        if (!ok) break;
        if (elect_one()) mma_commit_pair(acc_full, 0x3);
        __syncwarp();
      }
      // every pair MMA has completed before tensor memory can be freed
      if (issued) {
        if (elect_one()) mma_commit_pair(mma_done, 0x1);
        __syncwarp();
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(mma_done, 0u, 1000000u) && globaltimer_ns() - t0 < QLIN_DRAIN_NS) {
        }
      }
    }
    __syncwarp();
  } else if (warp >= 2 + kPairEpiWarps) {
    // ------------------------------------------------------------ converters
    // Thread ct widens half a weight row per step: packed chunks 2h, 2h+1
    // (64 inputs) of row ct / 2 into INT8 chunks 4h .. 4h+3 of the stage's
    // weight rows (128-byte swizzle), then every warp arrives on the even
    // CTA's converted-rows barrier of the stage.  Compensation steps carry
    // W_O^T rows from TMA: the warps only arrive.
    if (C::kConv) {
      const int ct = threadIdx.x - 32 * (2 + kPairEpiWarps);
      const int row = ct >> 1, hh = ct & 1;
      const uint32_t lready0 = mapa_shared(smem_u32(&aready[0]), 0);
      int gi = 0, gs = 0;
      bool ok = true;
      PairGen gen = pair_begin(g, cid);
      PairSeg sg;
      while (ok && pair_next(g, cid, gen, sg)) {
        int tn2, tm;
        pair_tile_coords(g, sg.t, tn2, tm);
        const int n = (2 * tn2 + crk) * 128 + row;
        for (int r = sg.r0; r < sg.r1; ++r, ++gi) {
          const int s = gi % S;
          if (gi >= S) ok = mbar_wait(&empty[s], static_cast<uint32_t>(gi / S - 1) & 1u, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          if (ct == 0) QLIN_STEP(gi, 2);
          if (r < g.kb) {
            const int ls = gs % LS;
            ok = __all_sync(0xffffffffu, mbar_wait(&sfull[ls], static_cast<uint32_t>(gs / LS) & 1u, abort_flag));
            if (!ok) break;
            if (ct == 0) QLIN_STEP(gi, 3);
            const unsigned char* st = smem + C::kOffStg + ls * C::kStgBytes;
            const int sw4 = (row >> 1) & 3;  // packed chunks are swizzled by row pair
            const uint4 w0 = *reinterpret_cast<const uint4*>(st + row * 64 + (((2 * hh) ^ sw4) << 4));
            const uint4 w1 = *reinterpret_cast<const uint4*>(st + row * 64 + (((2 * hh + 1) ^ sw4) << 4));
            uint4 o[4];
            if (FMT == kFmtW4PC) {
              unpack_w4pc(w0, o[0], o[1]);
              unpack_w4pc(w1, o[2], o[3]);
            } else {
              // a channel past N has zero codes and no ratio loaded: ratio 0
              const uint16_t rbits = n < g.N ? reinterpret_cast<const uint16_t*>(st + 8192)[row] : uint16_t(0);
              const __half2 r1 = __half2half2(__ushort_as_half(rbits));
              const __half2 r16 = __hmul2(r1, __half2half2(__ushort_as_half(static_cast<unsigned short>(0x2C00))));
              const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
              uint2 a[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) a[i] = requant_g128(wv[i], r1, r16);
#pragma unroll
              for (int i = 0; i < 4; ++i) o[i] = make_uint4(a[2 * i].x, a[2 * i].y, a[2 * i + 1].x, a[2 * i + 1].y);
            }
            unsigned char* A = smem + s * kPairStage;
            const int sw = row & 7;
#pragma unroll
            for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4*>(A + row * 128 + (((4 * hh + i) ^ sw) << 4)) = o[i];
            fence_proxy_async_smem();  // the tensor core reads these rows next
            __syncwarp();
            if (lane == 0) mbar_arrive(&sempty[ls]);
            if (ct == 0) QLIN_STEP(gi, 4);
            ++gs;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(lready0 + static_cast<uint32_t>(8 * s));
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Each tile's output goes to shared memory first; the accumulator is
    // released as soon as it has been read, and one TMA store per tile
    // writes the output while the next tile's products run.
    const int ep = warp - 2;
    const int grp = ep >> 2;
    const int quad = warp & 3;  // TMEM lanes 32*quad .. +31
    const int nl = quad * 32 + lane;
    const bool issuer = ep == 0 && lane == 0;
    float* sa = reinterpret_cast<float*>(smem + C::kOffSa);       // a_m of the tile's 256 tokens
    uint16_t* ys = reinterpret_cast<uint16_t*>(smem + C::kOffY);  // [256 tokens][128 channels]
    const uint32_t lempty = mapa_shared(smem_u32(acc_empty), 0);
    griddep_wait();  // a[] comes from the previous kernel
    int ti = 0;
    bool ok = true;
    PairGen gen = pair_begin(g, cid);
    PairSeg sg;
    for (; pair_next(g, cid, gen, sg); ++ti) {
      int tn2, tm;
      pair_tile_coords(g, sg.t, tn2, tm);
      const int ctile = 2 * tn2 + crk;
      const int n = ctile * 128 + nl;
      const int m0 = tm * 256;
      const int mvalid = min(256, g.M - m0);
      const bool part = sg.slot >= 0;
      const bool has_main = sg.r0 < g.kb;           // the range holds K-blocks of the tile
      const bool has_comp = comp && sg.r1 == g.T;  // ... and its compensation (never split)
      float cn = 0.f;
      if (n < g.N) cn = __fmul_rn(g.cscale[n], g.cmul);
      if (issuer) bulk_wait_group_read0();  // the previous tile's store has read the output buffer
      named_bar_sync(1, 256);
      {
        const int j = ep * 32 + lane;
        sa[j] = j < mvalid ? g.a[m0 + j] : 0.f;
      }
      named_bar_sync(1, 256);
      if (ok) ok = mbar_wait(acc_full, static_cast<uint32_t>(ti) & 1u, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
      // partial of a split tile: this CTA's slot, [token][channel]
      const size_t pslot = part ? (static_cast<size_t>(sg.slot) * 2 + crk) * 256 * 128 : 0;
#pragma unroll 1
      for (int c0 = grp * 16; c0 < mvalid; c0 += 32) {
        uint32_t acc[16], cmp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) { acc[j] = 0u; cmp[j] = 0u; }
        if (ok) {
          if (has_main) tmem_ld16(trow + c0, acc);
          if (has_comp) tmem_ld16(trow + 256 + c0, cmp);
          tmem_ld_wait();
        }
        if (part) {
          int32_t* pa = g.ws_acc + pslot + static_cast<size_t>(c0) * 128 + nl;
#pragma unroll
          for (int j = 0; j < 16; ++j) pa[j * 128] = static_cast<int32_t>(acc[j]);
          if (has_comp) {  // only a range's first segment can hold a compensation: one slot per pair
            float* pc = g.ws_comp + (static_cast<size_t>(cid) * 2 + crk) * 256 * 128 + static_cast<size_t>(c0) * 128 + nl;
#pragma unroll
            for (int j = 0; j < 16; ++j) pc[j * 128] = __uint_as_float(cmp[j]);
          }
          continue;
        }
        float sc[16];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float4 v = *reinterpret_cast<const float4*>(sa + c0 + 4 * q4);
          sc[4 * q4] = v.x; sc[4 * q4 + 1] = v.y; sc[4 * q4 + 2] = v.z; sc[4 * q4 + 3] = v.w;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float v = __fmul_rn(cn, static_cast<float>(static_cast<int32_t>(acc[j])));
          if (comp) v = __fadd_rn(v, __uint_as_float(cmp[j]));
          ys[(c0 + j) * 128 + nl] = __half_as_ushort(__float2half_rn(__fmul_rn(sc[j], v)));
        }
        if (g.acc_debug && n < g.N)
          for (int j = 0; j < 16; ++j)
            if (c0 + j < mvalid) g.acc_debug[static_cast<size_t>(m0 + c0 + j) * g.N + n] = static_cast<int32_t>(acc[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(acc_empty);
        else mbar_arrive_remote(lempty);
      }
      if (part) {
        // Count this CTA's steps of the split tile (CTA barrier, then one
        // thread's release fence and atomic: the release covers every
        // epilogue thread's partial stores); the range whose steps complete
        // the tile sums every contributor's partial and writes the output.
        named_bar_sync(1, 256);
        if (ep == 0 && lane == 0) {
          fence_acq_rel_gpu();
          const unsigned add = static_cast<unsigned>(sg.r1 - sg.r0);
          const unsigned old = atom_add_relaxed_gpu(&g.ws_cnt[sg.sk * 2 + crk], add);
          const bool last = old + add == static_cast<unsigned>(g.T);
          if (last) fence_acq_rel_gpu();  // acquire the other contributors' partials
          *fin_flag = last ? 1 : 0;
        }
        named_bar_sync(1, 256);
        if (!*fin_flag) continue;
        const unsigned ts = static_cast<unsigned>(sg.sk) * static_cast<unsigned>(g.T);
        const int c_lo = pair_owner(g, ts);
        const int c_hi = pair_owner(g, ts + static_cast<unsigned>(g.T) - 1u);
#pragma unroll 1
        for (int c0 = grp * 16; c0 < mvalid; c0 += 32) {
          int32_t sum[16];
          float cp[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) { sum[j] = 0; cp[j] = 0.f; }
          for (int c = c_lo; c <= c_hi; ++c) {
            if (g.bnd[c] == g.bnd[c + 1]) continue;  // an empty range
            const int slot = 2 * c + (g.bnd[c] < ts ? 1 : 0);
            const int32_t* src = g.ws_acc + (static_cast<size_t>(slot) * 2 + crk) * 256 * 128 + static_cast<size_t>(c0) * 128 + nl;
            int32_t v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __ldcg(src + j * 128);
#pragma unroll
            for (int j = 0; j < 16; ++j) sum[j] += v[j];
          }
          if (comp) {
            // the range holding the tile's last step holds its whole compensation
            const float* src = g.ws_comp + (static_cast<size_t>(c_hi) * 2 + crk) * 256 * 128 + static_cast<size_t>(c0) * 128 + nl;
#pragma unroll
            for (int j = 0; j < 16; ++j) cp[j] = __ldcg(src + j * 128);
          }
          float sc[16];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 v = *reinterpret_cast<const float4*>(sa + c0 + 4 * q4);
            sc[4 * q4] = v.x; sc[4 * q4 + 1] = v.y; sc[4 * q4 + 2] = v.z; sc[4 * q4 + 3] = v.w;
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float v = __fmul_rn(cn, static_cast<float>(sum[j]));
            if (comp) v = __fadd_rn(v, cp[j]);
            ys[(c0 + j) * 128 + nl] = __half_as_ushort(__float2half_rn(__fmul_rn(sc[j], v)));
          }
          if (g.acc_debug && n < g.N)
            for (int j = 0; j < 16; ++j)
              if (c0 + j < mvalid) g.acc_debug[static_cast<size_t>(m0 + c0 + j) * g.N + n] = sum[j];
        }
        if (ep == 0 && lane == 0) g.ws_cnt[sg.sk * 2 + crk] = 0u;  // zero for the next launch
      }
      fence_proxy_async_smem();  // the output rows are read by the bulk copy next
      named_bar_sync(1, 256);
      if (issuer && ctile * 128 < g.N) {
        tma_store_2d(&prm.tmY, ys, ctile * 128, m0);
        bulk_commit_group();
      }
    }
    if (issuer) bulk_wait_group_all();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its pair may still signal or read it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace qlin
