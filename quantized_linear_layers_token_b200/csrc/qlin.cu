// qlin.cu -- the C ABI declared in include/qlin.h: host-side validation,
// TMA descriptor encoding, launch selection.  All kernels live in the
// headers included below so the library is one translation unit (the device
// error word needs no relocatable device code).
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "qlin.h"
#include "act_quant.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "backward.cuh"
#include "gptq.cuh"
#include "offq.cuh"
#include "pack.cuh"
#include "smooth.cuh"

using namespace qlin;

namespace {

thread_local char t_last_error[512] = "";

qlin_status fail(qlin_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return st;
}

#define QLIN_CUDA_TRY(expr)                                                                    \
  do {                                                                                         \
    cudaError_t e_ = (expr);                                                                   \
    if (e_ != cudaSuccess)                                                                     \
      return fail(QLIN_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_));              \
  } while (0)

#define QLIN_LAUNCH_CHECK(what)                                                                \
  do {                                                                                         \
    cudaError_t e_ = cudaGetLastError();                                                       \
    if (e_ != cudaSuccess) return fail(QLIN_ERR_CUDA, "%s launch failed: %s", what,           \
                                       cudaGetErrorString(e_));                                \
  } while (0)

constexpr size_t kAlign = 256;
size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int pad8(int n) { return (n + 7) / 8 * 8; }

qlin_status check_shape(int32_t K, int32_t N, int32_t fmt, int32_t nO) {
  if (fmt != QLIN_W4_PERCHANNEL && fmt != QLIN_W4_G128 && fmt != QLIN_W8_PERCHANNEL)
    return fail(QLIN_ERR_ARG, "unknown weight format %d", fmt);
  if (K <= 0 || N <= 0 || nO < 0) return fail(QLIN_ERR_ARG, "negative or zero size K=%d N=%d n_outlier=%d", K, N, nO);
  if (K % 32 != 0 || K > 65536) return fail(QLIN_ERR_SHAPE, "K=%d must be a multiple of 32, at most 65536", K);
  if (N % 16 != 0) return fail(QLIN_ERR_SHAPE, "N=%d must be a multiple of 16", N);
  if (fmt == QLIN_W4_G128 && K % 128 != 0) return fail(QLIN_ERR_SHAPE, "g128 needs K %% 128 == 0 (K=%d)", K);
  if (nO > K || nO > 4096) return fail(QLIN_ERR_SHAPE, "n_outlier=%d must be <= min(K, 4096)", nO);
  return QLIN_OK;
}

struct Layout {
  size_t codes, chan, group, fold, oidx, wot, wmax, total;
};

Layout weights_layout(int32_t K, int32_t N, int32_t fmt, int32_t nO) {
  Layout L{};
  size_t off = 0;
  const size_t tiles_n = (N + 127) / 128, kb = (K + 127) / 128, ib = (nO + 63) / 64;
  const size_t codes_b = tiles_n * kb * ((fmt == QLIN_W8_PERCHANNEL) ? 16384 : 8192);
  L.codes = off; off = round_up(off + codes_b, kAlign);
  L.chan = off; off = round_up(off + size_t(N) * 4, kAlign);
  const size_t gb = (fmt == QLIN_W4_G128) ? size_t(K / 128) * N * 2 : 0;
  L.group = off; off = round_up(off + gb, kAlign);
  L.fold = off; off = round_up(off + gb, kAlign);
  L.oidx = off; off = round_up(off + size_t(nO) * 4, kAlign);
  L.wot = off; off = round_up(off + tiles_n * ib * 16384, kAlign);
  L.wmax = off; off = round_up(off + size_t(nO) * 4, kAlign);
  L.total = off;
  return L;
}

qlin_status check_weights(const qlin_weights* w) {
  if (!w) return fail(QLIN_ERR_ARG, "weights descriptor is NULL");
  qlin_status st = check_shape(w->K, w->N, w->fmt, w->n_outlier);
  if (st != QLIN_OK) return st;
  if (w->n_outlier_pad != pad8(w->n_outlier))
    return fail(QLIN_ERR_ARG, "n_outlier_pad=%d must be n_outlier rounded up to 8 (%d)", w->n_outlier_pad, pad8(w->n_outlier));
  if (w->fmt == QLIN_W4_G128 && w->group != 128) return fail(QLIN_ERR_ARG, "g128 format needs group=128");
  if (w->fmt != QLIN_W4_G128 && w->group != 0) return fail(QLIN_ERR_ARG, "per-channel formats need group=0");
  if (!w->codes || !w->chan_scale) return fail(QLIN_ERR_ARG, "codes/chan_scale is NULL");
  if (w->fmt == QLIN_W4_G128 && (!w->group_scale || !w->fold_ratio)) return fail(QLIN_ERR_ARG, "g128 scales are NULL");
  if (w->n_outlier > 0 && (!w->outlier_idx || !w->W_Ot || !w->wmax_O))
    return fail(QLIN_ERR_ARG, "outlier buffers are NULL");
  if (!aligned16(w->codes) || !aligned16(w->chan_scale) || (w->group_scale && !aligned16(w->group_scale)) ||
      (w->fold_ratio && !aligned16(w->fold_ratio)) || (w->W_Ot && !aligned16(w->W_Ot)) ||
      (w->outlier_idx && !aligned16(w->outlier_idx)) || (w->wmax_O && !aligned16(w->wmax_O)))
    return fail(QLIN_ERR_ALIGN, "a weights buffer is not 16-byte aligned");
  return QLIN_OK;
}

// ---------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

qlin_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return fail(QLIN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  return QLIN_OK;
}

// 2-D map over a row-major [outer][inner] array of `esize`-byte elements.
qlin_status make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize, uint64_t inner,
                     uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * static_cast<uint64_t>(esize)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return QLIN_OK;
}

// ---------------------------------------------------------------- launches
// Test and measurement knobs (qlin_debug_set); the defaults are the tuned
// behaviour.  Kernels are launched with programmatic dependent launch, so
// each may start its prologue (and the GEMM its weight stream) while the
// previous kernel in the stream finishes; every kernel waits on the grid
// dependency before it reads what the previous one wrote.
std::atomic<long long> g_knob[11] = {{1}, {1}, {0}, {0}, {256}, {512}, {kFusedMomentumMaxM}, {2000000000LL}, {2}, {0}, {0}};

long long knob(int k) { return g_knob[k].load(std::memory_order_relaxed); }

bool cluster_disabled() { return knob(QLIN_KNOB_CLUSTER) == 0; }

int forced_cluster_size() {
  const long long v = knob(QLIN_KNOB_CLUSTER_SIZE);
  return (v == 2 || v == 4 || v == 8) ? static_cast<int>(v) : 0;
}

bool pdl_enabled() { return knob(QLIN_KNOB_PDL) != 0; }

// `cluster` > 1 launches thread-block clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_kc(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, int cluster,
                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                     Args... args) {
  return launch_kc(kern, grid, block, smem, stream, 1, args...);
}

int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// CTAs a GEMM may use at most (QLIN_KNOB_MAX_CTAS; default all SMs).
int gemm_cta_cap() {
  const long long v = knob(QLIN_KNOB_MAX_CTAS);
  const int sms = sm_count();
  return (v > 0 && v < sms) ? static_cast<int>(v) : sms;
}

// INT4 layers on CTA pairs up to this many tokens convert their codes inside
// the GEMM instead of widening them ahead (QLIN_KNOB_CONVERT_MAX_M; 0 never).
long long convert_max_m() { return knob(QLIN_KNOB_CONVERT_MAX_M); }

// QLIN_KNOB_MAX_TOKEN_TILE = 64 or 128 caps the token tile.
int max_bt() {
  const long long x = knob(QLIN_KNOB_MAX_TOKEN_TILE);
  return (x == 64 || x == 128) ? static_cast<int>(x) : 256;
}

int pick_bt(int M) {
  int bt = 256;
  if (M <= 16) bt = 16;
  else if (M <= 32) bt = 32;
  else if (M <= 64) bt = 64;
  else if (M <= 128) bt = 128;
  return bt < max_bt() ? bt : max_bt();
}

// Work decomposition of one GEMM launch over one or more problems that
// share the token count M (same on the host for workspace sizes and for the
// launch).
struct GemmPlan {
  int bt, grid, split, widen, nprob;
  long long tiles;         // tiles of every problem
  GemmProb pr[kMaxProbs];  // per problem: shape, tiles and iteration offsets (pointers unset)
  size_t acc_off, comp_off, cnt_off, w8_off, total;  // shared scratch (after the problems' U operands)
  size_t u_off[kMaxProbs];                           // each problem's compensation operand U
  // CTA-pair launch (one problem, 256 x 256 tiles): pairs, whole tiles and
  // the stream-K tail's step boundaries, partial slots and tile counters
  int pair_ncl, pair_dp;
  long long pair_sk_tiles;
  size_t pacc_off, pcomp_off, pcnt_off;
  unsigned pair_bnd[kMaxPairs + 1];
};

bool use_pair(const GemmPlan& p, const qlin_weights* w);
template <int FMT>
int pair_max_clusters();

// Work split of a launch on CTA pairs over `tiles` tiles of T steps (the
// last T - kb of them the outlier compensation, never split).  Whole tiles
// in raster order while they fill whole waves; when the last wave would be
// partly empty, the last full wave and the remainder are instead divided by
// steps into one contiguous range per pair (stream-K), so every pair ends
// at about the same time.  With eight or more full waves the empty part of
// the last one is small and tiles stay whole.
void pair_split(GemmPlan& p, long long tiles, int T, int kb, int maxc) {
  if (maxc > kMaxPairs) maxc = kMaxPairs;
  p.pair_sk_tiles = 0;
  for (int c = 0; c <= kMaxPairs; ++c) p.pair_bnd[c] = 0u;
  const long long full = tiles / maxc, rem = tiles % maxc;
  if (knob(QLIN_KNOB_PAIR_SPLIT) == 0 || rem == 0 || full >= 8 || maxc < 2) {
    p.pair_ncl = static_cast<int>(tiles < maxc ? tiles : maxc);
    p.pair_dp = static_cast<int>(tiles);
    return;
  }
  p.pair_ncl = maxc;
  p.pair_dp = static_cast<int>(full >= 1 ? (full - 1) * maxc : 0);
  p.pair_sk_tiles = tiles - p.pair_dp;
  const unsigned long long total = static_cast<unsigned long long>(p.pair_sk_tiles) * T;
  unsigned prev = 0;
  for (int c = 0; c <= p.pair_ncl; ++c) {
    unsigned long long b = total * c / p.pair_ncl;
    const unsigned long long r = b % T;
    if (r > static_cast<unsigned long long>(kb) && r < static_cast<unsigned long long>(T))
      b = (r - kb <= T - r) ? b - (r - kb) : b + (T - r);  // not inside a compensation run
    if (c == p.pair_ncl) b = total;
    unsigned v = static_cast<unsigned>(b);
    if (v < prev) v = prev;
    p.pair_bnd[c] = v;
    prev = v;
  }
}

// From this many tokens the INT4 formats widen their weights once per call
// and run the INT8 kernel (QLIN_KNOB_WIDEN_MIN_M; 0 turns it off).
int widen_min_m() { return static_cast<int>(knob(QLIN_KNOB_WIDEN_MIN_M)); }

GemmPlan plan_gemm_group(int M, const qlin_weights* const* ws, int n) {
  GemmPlan p{};
  p.nprob = n;
  p.bt = pick_bt(M);
  const int ks = gemm_ks(p.bt);
  bool any_outliers = false;
  unsigned it = 0;
  for (int q = 0; q < n; ++q) {
    const qlin_weights* w = ws[q];
    GemmProb& g = p.pr[q];
    g.M = M;
    g.N = w->N;
    g.K = w->K;
    g.nO = w->n_outlier;
    g.tiles_n = (w->N + 127) / 128;
    g.tiles_m = (M + p.bt - 1) / p.bt;
    g.kb = (w->K + 127) / 128;
    g.nk = (g.kb + ks - 1) / ks;
    g.ncs = w->n_outlier > 0 ? (w->n_outlier + 63) / 64 : 0;
    g.nc = (p.bt <= 64) ? g.ncs : 2 * g.ncs;
    g.T = g.nk + g.nc;
    g.gm = 1;
    g.it0 = it;
    it += static_cast<unsigned>(static_cast<long long>(g.tiles_n) * g.tiles_m * g.T);
    p.tiles += static_cast<long long>(g.tiles_n) * g.tiles_m;
    any_outliers = any_outliers || w->n_outlier > 0;
  }
  long long iters = 0;
  for (int q = 0; q < n; ++q) iters += static_cast<long long>(p.pr[q].tiles_n) * p.pr[q].tiles_m * p.pr[q].T;
  const int sms = gemm_cta_cap();
  // Split tiles (stream-K or cluster split-K) when whole tiles would leave
  // SMs idle or badly balanced.  Token tiles of 128/256 have partials of
  // 64-128 KiB, so they split only when there are fewer tiles than SMs.
  // Groups of decode problems split too: their tiles differ in length (K),
  // and only split points give every CTA the same number of iterations.
  p.split = (p.tiles < (p.bt >= 128 ? 1LL : 4LL) * sms || (n > 1 && p.bt <= 64)) ? 1 : 0;
  const long long units = p.split ? iters : p.tiles;
  const int cap = sms < kMaxGrid ? sms : kMaxGrid;
  p.grid = static_cast<int>(units < cap ? units : cap);
  if (p.grid < 1) p.grid = 1;
  // Raster order of many-token problems: the CTAs running at once should
  // share weight tiles and reuse activation tiles from L2.  All token tiles
  // in one group when the INT8 activations (M x K) fit well inside L2, else
  // groups of about sqrt(grid * 128 / BT) token tiles (the size that
  // minimises the activation bytes plus the weight bytes one wave of CTAs
  // touches).
  for (int q = 0; q < n; ++q) {
    GemmProb& g = p.pr[q];
    if (g.tiles_m <= 1) continue;
    const double x_bytes = static_cast<double>(M) * g.K;
    int gm = static_cast<int>(std::lround(std::sqrt(static_cast<double>(p.grid) * 128.0 / p.bt)));
    if (x_bytes <= 48.0 * 1024 * 1024) gm = g.tiles_m;
    g.gm = gm < 1 ? 1 : (gm > g.tiles_m ? g.tiles_m : gm);
  }
  size_t off = 0;
  for (int q = 0; q < n; ++q) {
    p.u_off[q] = off;
    off = round_up(off + (ws[q]->n_outlier > 0 ? size_t(2) * M * ws[q]->n_outlier_pad * 2 : 0), kAlign);
  }
  const size_t slot_bytes = size_t(p.bt) * 128 * 4;
  p.acc_off = off;
  off = round_up(off + (p.split ? size_t(2) * p.grid * slot_bytes : 0), kAlign);
  p.comp_off = off;
  off = round_up(off + (p.split && any_outliers ? size_t(2) * p.grid * slot_bytes : 0), kAlign);
  p.cnt_off = off;
  off = round_up(off + (p.split ? size_t(p.grid) * 4 : 0), kAlign);
  p.widen = (n == 1 && ws[0]->fmt != QLIN_W8_PERCHANNEL && p.bt == 256 && widen_min_m() > 0 && M >= widen_min_m())
                ? 1 : 0;
  p.w8_off = off;
  off = round_up(off + (p.widen ? size_t(p.pr[0].tiles_n) * p.pr[0].kb * 16384 : 0), kAlign);
  p.pair_ncl = 0;
  p.pair_dp = 0;
  p.pair_sk_tiles = 0;
  p.pacc_off = p.pcomp_off = p.pcnt_off = off;
  if (n == 1 && use_pair(p, ws[0])) {
    const GemmProb& q = p.pr[0];
    const bool conv = p.widen && M <= convert_max_m();
    const int maxc = !conv ? pair_max_clusters<kFmtW8>()
                           : (ws[0]->fmt == QLIN_W4_PERCHANNEL ? pair_max_clusters<kFmtW4PC>()
                                                                : pair_max_clusters<kFmtW4G128>());
    const long long tiles = static_cast<long long>((q.tiles_n + 1) / 2) * q.tiles_m;
    pair_split(p, tiles, q.kb + 2 * q.ncs, q.kb, maxc > 0 ? maxc : 1);
    if (p.pair_sk_tiles > 0) {
      const size_t part = size_t(2) * 256 * 128 * 4;  // one slot: both CTAs' 128 channels x 256 tokens
      off = round_up(off + size_t(2) * p.pair_ncl * part, kAlign);
      p.pcomp_off = off;
      off = round_up(off + (ws[0]->n_outlier > 0 ? size_t(p.pair_ncl) * part : 0), kAlign);
      p.pcnt_off = off;
      off = round_up(off + size_t(p.pair_sk_tiles) * 2 * 4, kAlign);
    }
  }
  p.total = off;
  return p;
}

GemmPlan plan_gemm(int M, const qlin_weights* w) { return plan_gemm_group(M, &w, 1); }

constexpr int kGroupMaxM = 64;  // token counts a grouped launch takes (decode-sized tiles)

// ---------------------------------------------------------------- GEMM launch
template <int FMT, int BT, int MAXP>
qlin_status launch_gemm_t(GemmParams<MAXP>& prm, cudaStream_t stream) {
  using C = GemmCfg<FMT, BT>;
  auto kern = gemm_kernel<FMT, BT, MAXP>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return fail(QLIN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
  GemmArgs& args = prm.g;
  // Single-problem launches whose token tiles (up to 64) would be split
  // (decode): cluster split-K when it is expected to beat global-memory
  // stream-K.  Costs in units of one pipeline step, fitted to B200
  // measurements of the 7B decode shapes: a cluster round costs its longest
  // rank range plus the exchange of BT x 128 partials through distributed
  // shared memory (about 0.5 / 2 / 7.5 steps at BT = 16 / 32 / 64);
  // stream-K costs its per-CTA iterations plus the global fixup chain
  // (about 7 / 12 / 28 steps).  QLIN_KNOB_CLUSTER_SIZE forces a size.
  if (MAXP == 1 && C::kCluster && args.split && !cluster_disabled()) {
    const GemmProb& g0 = prm.pr[0];
    const double xchg = BT <= 16 ? 0.5 : (BT <= 32 ? 2.0 : 7.5);
    const double fixup = BT <= 16 ? 7.0 : (BT <= 32 ? 12.0 : 28.0);
    const int forced = forced_cluster_size();
    const long long iters = static_cast<long long>(g0.tiles_n) * g0.tiles_m * g0.T;
    const double streamk_cost = static_cast<double>((iters + args.grid - 1) / args.grid) + fixup;
    const long long tiles = static_cast<long long>(g0.tiles_n) * g0.tiles_m;
    static int max_clusters[9] = {-1, -1, -1, -1, -1, -1, -1, -1, -1};  // per cluster size, this instantiation
    int best_cs = 0, best_ncl = 0;
    double best_cost = streamk_cost;
    // compensation run of the last rank: its steps plus sending a BT x slice
    // fp32 partial (about BT / 32 steps at cs = 4)
    for (int cs = 2; cs <= 8; cs *= 2) {
      int cb[9];
      const double ccost = (g0.T - g0.nk) + (g0.nO > 0 ? BT / 32.0 * 4.0 / cs : 0.0);
      const double span = cluster_bounds(g0.T, g0.nk, cs, ccost, cb);
      if (span < 0) continue;
      if (max_clusters[cs] < 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(cs * ((sm_count() + cs - 1) / cs)));
        cfg.blockDim = dim3(C::kThreads);
        cfg.dynamicSmemBytes = C::kSmemBytes;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = static_cast<unsigned>(cs);
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
          cudaGetLastError();
          n = 0;
        }
        max_clusters[cs] = n;
      }
      int ncl = static_cast<int>(max_clusters[cs] < tiles ? max_clusters[cs] : tiles);
      if (ncl * cs > gemm_cta_cap()) ncl = gemm_cta_cap() / cs;
      if (ncl < 1) continue;
      double cost = static_cast<double>((tiles + ncl - 1) / ncl) * (span + xchg);
      if (forced) cost = forced == cs ? -1.0 : 1e30;
      if (cost < best_cost) {
        best_cs = cs;
        best_ncl = ncl;
        best_cost = cost;
      }
    }
    if (best_cs) {
      args.cs = best_cs;
      args.ncl = best_ncl;
      args.grid = best_cs * best_ncl;
      cluster_bounds(g0.T, g0.nk, best_cs,
                     (g0.T - g0.nk) + (g0.nO > 0 ? BT / 32.0 * 4.0 / best_cs : 0.0), args.cb);
    }
  }
  cudaError_t e = launch_kc(kern, dim3(args.grid), dim3(C::kThreads), C::kSmemBytes, stream, args.cs, prm);
  if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "gemm_kernel launch failed: %s", cudaGetErrorString(e));
  return QLIN_OK;
}

// Grouped launches (MAXP > 1) take decode-sized token tiles only (<= 64).
template <int FMT, int MAXP>
qlin_status launch_gemm_fmt(int bt, GemmParams<MAXP>& prm, cudaStream_t stream) {
  switch (bt) {
    case 16: return launch_gemm_t<FMT, 16, MAXP>(prm, stream);
    case 32: return launch_gemm_t<FMT, 32, MAXP>(prm, stream);
    case 64: return launch_gemm_t<FMT, 64, MAXP>(prm, stream);
    default:
      if constexpr (MAXP == 1) {
        if (bt == 128) return launch_gemm_t<FMT, 128, 1>(prm, stream);
        return launch_gemm_t<FMT, 256, 1>(prm, stream);
      } else {
        return fail(QLIN_ERR_SHAPE, "grouped GEMMs take at most %d tokens", kGroupMaxM);
      }
  }
}

// ---------------------------------------------------------------- CTA-pair GEMM (many tokens)
template <int FMT>
int pair_max_clusters() {
  static int n = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    if (cudaFuncSetAttribute(gemm_pair_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PairCfg<FMT>::kSmem) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
      return;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * ((sm_count() + 1) / 2)));
    cfg.blockDim = dim3(PairCfg<FMT>::kThreads);
    cfg.dynamicSmemBytes = PairCfg<FMT>::kSmem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, gemm_pair_kernel<FMT>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      c = 0;
    }
    n = c;
  });
  return n;
}

// Whether a single-problem launch runs on CTA pairs: 256-token tiles with
// INT8 operands (the INT8 format, or INT4 widened once per call); by default
// whenever the operands allow, even with fewer 256 x 256 pair tiles than
// pairs on the GPU (QLIN_KNOB_PAIR_MMA: 0 never, 1 only from one full wave).
bool use_pair(const GemmPlan& p, const qlin_weights* w) {
  const long long mode = knob(QLIN_KNOB_PAIR_MMA);
  if (mode == 0 || p.nprob != 1 || p.bt != 256) return false;
  if (!(w->fmt == QLIN_W8_PERCHANNEL || p.widen)) return false;
  const int ncl = pair_max_clusters<kFmtW8>();
  if (ncl < 1) return false;
  const long long tiles = static_cast<long long>((p.pr[0].tiles_n + 1) / 2) * p.pr[0].tiles_m;
  return mode == 2 ? tiles >= 1 : tiles >= ncl;
}

// FMT = kFmtW8: INT8 weight rows by TMA from `codes8` (the INT8 format, or
// INT4 widened ahead); kFmtW4PC / kFmtW4G128: the layer's packed INT4 codes,
// converted inside the kernel.
template <int FMT>
qlin_status launch_gemm_pair(const GemmPlan& p, const qlin_weights* w, const int8_t* Xq, const float* a, uint16_t* Y,
                             int32_t* acc_debug, char* gws, const uint8_t* codes8, float cmul, cudaStream_t stream) {
  PairParams prm;
  memset(&prm, 0, sizeof(prm));
  PairArgs& g = prm.g;
  const GemmProb& q = p.pr[0];
  const int M = q.M;
  g.codes = static_cast<const uint8_t*>(w->codes);
  g.rfold = w->fold_ratio;
  g.cscale = w->chan_scale;
  g.cmul = cmul;
  g.a = a;
  g.Y = Y;
  g.acc_debug = acc_debug;
  g.M = M;
  g.N = w->N;
  g.nO = w->n_outlier;
  g.kb = q.kb;
  g.ntn = q.tiles_n;
  g.ncs = q.ncs;
  g.T = q.kb + 2 * q.ncs;
  g.tiles_n2 = (q.tiles_n + 1) / 2;
  g.tiles_m = q.tiles_m;
  g.tiles = g.tiles_n2 * g.tiles_m;
  const double x_bytes = static_cast<double>(M) * w->K;
  const int maxc = pair_max_clusters<FMT>();
  if (maxc < 1) return fail(QLIN_ERR_CUDA, "gemm_pair_kernel: no 2-CTA cluster fits");
  int gm = static_cast<int>(std::lround(std::sqrt(static_cast<double>(maxc) * 256.0 / 256.0)));
  if (x_bytes <= 48.0 * 1024 * 1024) gm = g.tiles_m;
  g.gm = gm < 1 ? 1 : (gm > g.tiles_m ? g.tiles_m : gm);
  if (p.pair_ncl < 1 || p.pair_ncl > maxc) return fail(QLIN_ERR_CUDA, "gemm_pair_kernel: plan of %d pairs, %d fit", p.pair_ncl, maxc);
  g.ncl = p.pair_ncl;
  g.dp = p.pair_dp;
  for (int c = 0; c <= kMaxPairs; ++c) g.bnd[c] = p.pair_bnd[c];
  g.ws_acc = reinterpret_cast<int32_t*>(gws + p.pacc_off);
  g.ws_comp = reinterpret_cast<float*>(gws + p.pcomp_off);
  g.ws_cnt = reinterpret_cast<unsigned*>(gws + p.pcnt_off);
  qlin_status st = QLIN_OK;
  if (FMT == kFmtW8) {
    st = make_map(&prm.tmA, codes8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 128,
                  static_cast<uint64_t>(q.tiles_n) * q.kb * 128, 128, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != QLIN_OK) return st;
  }
  st = make_map(&prm.tmX, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->K, M, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QLIN_OK) return st;
  if (w->n_outlier > 0) {
    st = make_map(&prm.tmU, gws + p.u_off[0], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, w->n_outlier_pad,
                  2 * static_cast<uint64_t>(M), 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != QLIN_OK) return st;
    st = make_map(&prm.tmWo, w->W_Ot, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 128,
                  static_cast<uint64_t>(q.tiles_n) * q.ncs * 128, 128, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != QLIN_OK) return st;
  }
  st = make_map(&prm.tmY, Y, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, w->N, M, 128, 256, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != QLIN_OK) return st;
  cudaError_t e = launch_kc(gemm_pair_kernel<FMT>, dim3(static_cast<unsigned>(2 * g.ncl)),
                            dim3(PairCfg<FMT>::kThreads), PairCfg<FMT>::kSmem, stream, 2, prm);
  if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "gemm_pair_kernel launch failed: %s", cudaGetErrorString(e));
  return QLIN_OK;
}

// One GEMM launch over the problems of a plan.  Per problem q: weights
// ws[q], the INT8 activations Xq[q], token scales a[q], output Y[q] and
// (optional) acc_debug[q]; `gws` is the scratch laid out by the plan (each
// problem's U, then the shared split-K slots and counters).
template <int MAXP>
qlin_status launch_gemm_group(const GemmPlan& p, const qlin_weights* const* ws, const int8_t* const* Xq,
                              const float* const* a, uint16_t* const* Y, int32_t* const* acc_debug, char* gws,
                              cudaStream_t stream) {
  qlin_status st = get_encoder();
  if (st != QLIN_OK) return st;
  static_assert(sizeof(GemmParams<MAXP>) <= 32000, "kernel parameter space");
  GemmParams<MAXP> prm;
  memset(&prm, 0, sizeof(prm));
  GemmArgs& args = prm.g;
  const int M = p.pr[0].M;
  long long iters = 0;
  for (int q = 0; q < p.nprob; ++q) {
    const qlin_weights* w = ws[q];
    GemmProb& g = prm.pr[q];
    g = p.pr[q];
    g.codes = static_cast<const uint8_t*>(w->codes);
    g.rfold = w->fold_ratio;
    g.wot = w->W_Ot;
    g.cscale = w->chan_scale;
    g.a = a[q];
    g.Y = Y[q];
    g.acc_debug = acc_debug ? acc_debug[q] : nullptr;
    g.cmul = 1.f;
    iters += static_cast<long long>(g.tiles_n) * g.tiles_m * g.T;
    st = make_map(&prm.tmX[q], Xq[q], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->K, M, 128, p.bt,
                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != QLIN_OK) return st;
    if (w->n_outlier > 0) {
      st = make_map(&prm.tmU[q], gws + p.u_off[q], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, w->n_outlier_pad,
                    2 * static_cast<uint64_t>(M), 64, p.bt, CU_TENSOR_MAP_SWIZZLE_128B);
      if (st != QLIN_OK) return st;
    }
  }
  if (iters >= (1LL << 31)) return fail(QLIN_ERR_SHAPE, "problem too large (%lld tile iterations)", iters);
  args.ws_acc = reinterpret_cast<int32_t*>(gws + p.acc_off);
  args.ws_comp = reinterpret_cast<float*>(gws + p.comp_off);
  args.ws_cnt = reinterpret_cast<unsigned*>(gws + p.cnt_off);
  args.nprob = p.nprob;
  args.grid = p.grid;
  args.split = p.split;
  args.total = static_cast<unsigned>(iters);
  args.cs = 1;
  args.ncl = 0;
  args.wdep = p.widen ? 1 : 0;
  gemm_boundaries(prm.pr, p.nprob, p.grid, p.split, args.bnd);
  const int fmt = ws[0]->fmt;
  if (p.widen && MAXP == 1 && use_pair(p, ws[0]) && p.pr[0].M <= convert_max_m()) {
    // INT4 on CTA pairs, converted inside the kernel (no widening pass)
    const qlin_weights* w = ws[0];
    const float cm = fmt == QLIN_W4_PERCHANNEL ? 0.0625f : 1.f;
    return fmt == QLIN_W4_PERCHANNEL
               ? launch_gemm_pair<kFmtW4PC>(p, w, Xq[0], a[0], Y[0], acc_debug ? acc_debug[0] : nullptr, gws, nullptr,
                                            cm, stream)
               : launch_gemm_pair<kFmtW4G128>(p, w, Xq[0], a[0], Y[0], acc_debug ? acc_debug[0] : nullptr, gws,
                                              nullptr, cm, stream);
  }
  if (p.widen) {
    const qlin_weights* w = ws[0];
    uint8_t* w8 = reinterpret_cast<uint8_t*>(gws + p.w8_off);
    const unsigned nblk = static_cast<unsigned>(p.pr[0].tiles_n) * static_cast<unsigned>(p.pr[0].kb);
    const uint8_t* codes = static_cast<const uint8_t*>(w->codes);
    const uint16_t* rf = reinterpret_cast<const uint16_t*>(w->fold_ratio);
    cudaError_t e = fmt == QLIN_W4_PERCHANNEL
                        ? launch_k(widen_w4_kernel<kFmtW4PC>, dim3(nblk), dim3(256), 0, stream, codes, rf, w->N,
                                   p.pr[0].kb, w8)
                        : launch_k(widen_w4_kernel<kFmtW4G128>, dim3(nblk), dim3(256), 0, stream, codes, rf, w->N,
                                   p.pr[0].kb, w8);
    if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "widen_w4_kernel launch failed: %s", cudaGetErrorString(e));
    prm.pr[0].codes = w8;
    prm.pr[0].cmul = fmt == QLIN_W4_PERCHANNEL ? 0.0625f : 1.f;
    if (MAXP == 1 && use_pair(p, w))
      return launch_gemm_pair<kFmtW8>(p, w, Xq[0], a[0], Y[0], acc_debug ? acc_debug[0] : nullptr, gws, w8,
                                      prm.pr[0].cmul, stream);
    return launch_gemm_fmt<kFmtW8, MAXP>(p.bt, prm, stream);
  }
  if (MAXP == 1 && fmt == QLIN_W8_PERCHANNEL && use_pair(p, ws[0]))
    return launch_gemm_pair<kFmtW8>(p, ws[0], Xq[0], a[0], Y[0], acc_debug ? acc_debug[0] : nullptr, gws,
                            static_cast<const uint8_t*>(ws[0]->codes), 1.f, stream);
  switch (fmt) {
    case QLIN_W4_PERCHANNEL: return launch_gemm_fmt<kFmtW4PC, MAXP>(p.bt, prm, stream);
    case QLIN_W4_G128: return launch_gemm_fmt<kFmtW4G128, MAXP>(p.bt, prm, stream);
    default: return launch_gemm_fmt<kFmtW8, MAXP>(p.bt, prm, stream);
  }
}

// Single-problem GEMM launch.
qlin_status launch_gemm(const qlin_weights* w, const int8_t* Xq, const float* a, int M, uint16_t* Y,
                        int32_t* acc_debug, char* gws, cudaStream_t stream) {
  const GemmPlan p = plan_gemm(M, w);
  return launch_gemm_group<1>(p, &w, &Xq, &a, &Y, acc_debug ? &acc_debug : nullptr, gws, stream);
}

// ---------------------------------------------------------------- act quant
// Up to this many tokens the momentum update runs inside the quantization
// kernel (every CTA gathers all rows' outlier values); above it a separate
// column-max kernel gathers them once (QLIN_KNOB_FUSED_MOMENTUM_MAX_M).
int fused_momentum_max_m() { return static_cast<int>(knob(QLIN_KNOB_FUSED_MOMENTUM_MAX_M)); }

constexpr int kQuantSmemMax = 232448 - 1024;  // 227 KB per CTA, less room for the kernel's static shared memory

size_t act_ws_bytes(const qlin_weights* w) {
  return w->n_outlier > 0 ? round_up(size_t(w->n_outlier) * 4 + 4, kAlign) : 0;
}

// Activations of one quantization problem (outputs and scratch per problem).
struct QuantIO {
  const uint16_t* X;
  float* s;
  int8_t* Xq;
  float* a;
  int8_t* XqO;
  uint16_t* U;   // compensation operand (qlin_forward), or null
  void* act_ws;  // outlier column maxima + completion counter (update only)
};

template <int VPT, bool FUSED, int MAXP>
qlin_status launch_quant_v(const QuantGroup<MAXP>& qg, int rows, size_t smem, cudaStream_t stream) {
  auto kern = quant_kernel<VPT, FUSED, MAXP>;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [&] { attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQuantSmemMax); });
  if (attr != cudaSuccess) return fail(QLIN_ERR_CUDA, "quant_kernel attribute: %s", cudaGetErrorString(attr));
  cudaError_t e = launch_k(kern, dim3(rows), dim3(kQuantThreads), smem, stream, qg);
  if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "quant_kernel launch failed: %s", cudaGetErrorString(e));
  return QLIN_OK;
}

template <bool FUSED, int MAXP>
qlin_status launch_quant_f(const QuantGroup<MAXP>& qg, int rows, int vpt, size_t smem, cudaStream_t stream) {
  if (vpt <= 1) return launch_quant_v<1, FUSED, MAXP>(qg, rows, smem, stream);
  if (vpt <= 2) return launch_quant_v<2, FUSED, MAXP>(qg, rows, smem, stream);
  if (vpt <= 4) return launch_quant_v<4, FUSED, MAXP>(qg, rows, smem, stream);
  if (vpt <= 8) return launch_quant_v<8, FUSED, MAXP>(qg, rows, smem, stream);
  return launch_quant_v<16, FUSED, MAXP>(qg, rows, smem, stream);
}

// Stage 1 for one problem or a group (same M): the momentum update (fused
// into the quantization kernel up to the fused-momentum token count, else a
// column-max kernel per problem first), then one quantization launch with a
// CTA per token row of every problem.
template <int MAXP>
qlin_status launch_quant_group(const qlin_weights* const* ws, const QuantIO* io, int n, int M, float gamma,
                               int update, cudaStream_t stream) {
  if (M == 0) return QLIN_OK;
  QuantGroup<MAXP> qg;
  memset(&qg, 0, sizeof(qg));
  qg.gamma = gamma;
  qg.nprob = n;
  bool any_update = false;
  int maxK = 0;
  size_t smem = 0;
  for (int q = 0; q < n; ++q) {
    const qlin_weights* w = ws[q];
    const int K = w->K, nO = w->n_outlier;
    QuantProb& p = qg.pr[q];
    unsigned* cmax = static_cast<unsigned*>(io[q].act_ws);
    p.X = io[q].X;
    p.O = static_cast<const int32_t*>(w->outlier_idx);
    p.s = io[q].s;
    p.Xq = io[q].Xq;
    p.a = io[q].a;
    p.XqO = io[q].XqO;
    p.U = io[q].U;
    p.wmaxO = w->wmax_O;
    p.counter = cmax ? cmax + nO : nullptr;
    p.K = K;
    p.nO = nO;
    p.nOp = w->n_outlier_pad;
    p.M = M;
    p.row0 = q * M;
    any_update = any_update || (update && nO > 0);
    if (K > maxK) maxK = K;
    const size_t sm = size_t(K) * 2 + size_t(nO) * 16;
    if (sm > smem) smem = sm;
  }
  if (smem > size_t(kQuantSmemMax))
    return fail(QLIN_ERR_SHAPE, "K=%d with its outliers needs %zu bytes of shared memory", maxK, smem);
  const int nvec = maxK / 8;
  const int vpt = (nvec + kQuantThreads - 1) / kQuantThreads;
  if (vpt > 16) return fail(QLIN_ERR_SHAPE, "K=%d too large for the quantization kernel", maxK);
  const bool fused = any_update && M <= fused_momentum_max_m();
  if (any_update && !fused) {
    for (int q = 0; q < n; ++q) {
      const qlin_weights* w = ws[q];
      const int nO = w->n_outlier;
      if (nO == 0) continue;
      unsigned* cmax = static_cast<unsigned*>(io[q].act_ws);
      const int grid = (M + kColmaxRows - 1) / kColmaxRows;
      cudaError_t e = launch_k(colmax_kernel, dim3(grid), dim3(256), size_t(nO) * 8, stream, io[q].X, M, w->K,
                               static_cast<const int32_t*>(w->outlier_idx), nO, cmax, 1,
                               static_cast<const float*>(w->wmax_O), io[q].s, gamma, cmax + nO);
      if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "colmax_kernel launch failed: %s", cudaGetErrorString(e));
    }
  }
  const int rows = n * M;
  return fused ? launch_quant_f<true, MAXP>(qg, rows, vpt, smem, stream)
               : launch_quant_f<false, MAXP>(qg, rows, vpt, smem, stream);
}

qlin_status launch_quant(const uint16_t* X, int M, const qlin_weights* w, float* s, float gamma, int update,
                         int8_t* Xq, float* a, int8_t* XqO, uint16_t* U, void* act_ws, cudaStream_t stream) {
  const QuantIO io{X, s, Xq, a, XqO, U, act_ws};
  return launch_quant_group<1>(&w, &io, 1, M, gamma, update, stream);
}

size_t gemm_ws_bytes(int M, const qlin_weights* w) { return M > 0 ? plan_gemm(M, w).total : 0; }

struct FwdLayout {
  size_t act, xq, a, xqo, gemm, total;
};

FwdLayout forward_layout(int M, const qlin_weights* w) {
  FwdLayout L{};
  size_t off = 0;
  L.act = off; off = round_up(off + act_ws_bytes(w), kAlign);
  L.xq = off; off = round_up(off + size_t(M) * w->K, kAlign);
  L.a = off; off = round_up(off + size_t(M) * 4, kAlign);
  L.xqo = off; off = round_up(off + size_t(M) * w->n_outlier, kAlign);
  L.gemm = off; off = round_up(off + gemm_ws_bytes(M, w), kAlign);
  L.total = off;
  return L;
}

// Workspace of a grouped forward: per problem the quantization scratch, Xq,
// a and XqO, then the GEMM launch's scratch (every problem's U and the
// shared split-K slots and counters).
struct GroupLayout {
  size_t act[kMaxProbs], xq[kMaxProbs], a[kMaxProbs], xqo[kMaxProbs];
  size_t gemm, total;
  GemmPlan plan;
};

GroupLayout group_layout(int M, const qlin_weights* const* ws, int n) {
  GroupLayout L{};
  size_t off = 0;
  for (int q = 0; q < n; ++q) {
    const qlin_weights* w = ws[q];
    L.act[q] = off; off = round_up(off + act_ws_bytes(w), kAlign);
    L.xq[q] = off; off = round_up(off + size_t(M) * w->K, kAlign);
    L.a[q] = off; off = round_up(off + size_t(M) * 4, kAlign);
    L.xqo[q] = off; off = round_up(off + size_t(M) * w->n_outlier, kAlign);
  }
  L.plan = plan_gemm_group(M > 0 ? M : 1, ws, n);
  L.gemm = off;
  off = round_up(off + (M > 0 ? L.plan.total : 0), kAlign);
  L.total = off;
  return L;
}

qlin_status check_group(int32_t count, const qlin_weights* const* w, int32_t M) {
  if (count < 1 || count > kMaxProbs) return fail(QLIN_ERR_SHAPE, "count=%d must be in [1, %d]", count, kMaxProbs);
  if (!w) return fail(QLIN_ERR_ARG, "weights array is NULL");
  if (M < 0) return fail(QLIN_ERR_ARG, "M=%d is negative", M);
  if (M > kGroupMaxM) return fail(QLIN_ERR_SHAPE, "M=%d: grouped forwards take at most %d tokens", M, kGroupMaxM);
  for (int q = 0; q < count; ++q) {
    qlin_status st = check_weights(w[q]);
    if (st != QLIN_OK) return fail(st, "problem %d: %s", q, t_last_error);
    if (w[q]->fmt != w[0]->fmt) return fail(QLIN_ERR_ARG, "problem %d: every problem must have the same format", q);
  }
  return QLIN_OK;
}

}  // namespace

// ---------------------------------------------------------------- allocation-free quantization
// Fixed scratch for qlin_quant_act_noalloc: the outlier column maxima and the
// completion counter of the momentum update.  It is a file-scope device
// array, so every GPU that loads this library holds it (4.25 KiB: 1024 + 64
// words) until the process exits, and every call on a device shares the same
// copy.
#define QLIN_NOALLOC_MAX_OUTLIERS 1024
static __device__ __align__(256) unsigned g_noalloc_scratch[QLIN_NOALLOC_MAX_OUTLIERS + 64];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
unsigned* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device.  In host code the
// symbol names a host-side shadow, not device memory, so the address is
// looked up once per device (with that device current) and cached.
qlin_status noalloc_scratch(unsigned** out) {
  int dev = -1;
  QLIN_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(QLIN_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(QLIN_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = static_cast<unsigned*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return QLIN_OK;
}

// ---------------------------------------------------------------- backward
// Work plan of the input gradient: whole 256 x 256 tiles fill complete
// waves of one CTA per SM; when the grid is under two waves, the tiles of
// the ragged last wave are split into tsplit ranges of the channel steps (at
// most 8, at most one range per step) so that wave has as many CTAs as SMs,
// and their fp32 partials go through the workspace.  Without a workspace
// every tile is whole.
struct BwdPlan {
  int ntk, tiles, full, tsplit;
  size_t part_off, cnt_off, bytes;
};

BwdPlan plan_backward(int M, const qlin_weights* w, bool split) {
  BwdPlan p{};
  p.ntk = (w->K + 255) / 256;
  p.tiles = p.ntk * ((M + 255) / 256);
  p.full = p.tiles;
  p.tsplit = 1;
  const int sms = sm_count();
  const int nsteps = (w->N + 63) / 64;
  const int tail = p.tiles % sms;
  // only below two waves: with more, CTAs of different lengths already
  // interleave across the wave boundaries and the partials cost more than
  // the idle SMs of the last wave (measured on 3.5-wave grids)
  if (split && tail > 0 && p.tiles < 2 * sms) {
    int S = sms / tail;
    if (S > 8) S = 8;
    if (S > nsteps) S = nsteps;
    if (S >= 2) {
      p.full = p.tiles - tail;
      p.tsplit = S;
    }
  }
  const int ntail = p.tiles - p.full;
  p.part_off = 0;
  p.cnt_off = round_up(size_t(ntail) * (p.tsplit - 1) * 65536 * 4, kAlign);
  p.bytes = ntail ? round_up(p.cnt_off + size_t(ntail) * 4, kAlign) : 0;
  return p;
}

template <int FMT>
qlin_status launch_backward_t(const CUtensorMap& tm, const BwdArgs& args, cudaStream_t stream) {
  using C = BwdCfg<FMT>;
  auto kern = backward_dx_kernel<FMT>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return fail(QLIN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
  const dim3 grid(static_cast<unsigned>(args.full + (args.ntk * ((args.M + 255) / 256) - args.full) * args.tsplit));
  cudaError_t e = launch_k(kern, grid, dim3(C::kThreads), C::kSmemBytes, stream, tm, args);
  if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "backward_dx_kernel launch failed: %s", cudaGetErrorString(e));
  return QLIN_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* qlin_status_string(qlin_status s) {
  switch (s) {
    case QLIN_OK: return "QLIN_OK";
    case QLIN_ERR_ARG: return "QLIN_ERR_ARG";
    case QLIN_ERR_SHAPE: return "QLIN_ERR_SHAPE";
    case QLIN_ERR_ALIGN: return "QLIN_ERR_ALIGN";
    case QLIN_ERR_WORKSPACE: return "QLIN_ERR_WORKSPACE";
    case QLIN_ERR_CUDA: return "QLIN_ERR_CUDA";
    case QLIN_ERR_TIMEOUT: return "QLIN_ERR_TIMEOUT";
  }
  return "QLIN_UNKNOWN_STATUS";
}

const char* qlin_last_error(void) { return t_last_error; }

qlin_status qlin_weights_bytes(int32_t K, int32_t N, int32_t fmt, int32_t n_outlier, size_t* bytes) {
  if (!bytes) return fail(QLIN_ERR_ARG, "bytes is NULL");
  qlin_status st = check_shape(K, N, fmt, n_outlier);
  if (st != QLIN_OK) return st;
  *bytes = weights_layout(K, N, fmt, n_outlier).total;
  return QLIN_OK;
}

qlin_status qlin_weights_bind(qlin_weights* w, int32_t K, int32_t N, int32_t fmt, int32_t n_outlier, void* base,
                              size_t bytes) {
  if (!w || !base) return fail(QLIN_ERR_ARG, "weights descriptor or base is NULL");
  qlin_status st = check_shape(K, N, fmt, n_outlier);
  if (st != QLIN_OK) return st;
  if (reinterpret_cast<uintptr_t>(base) % kAlign) return fail(QLIN_ERR_ALIGN, "base must be 256-byte aligned");
  Layout L = weights_layout(K, N, fmt, n_outlier);
  if (bytes < L.total) return fail(QLIN_ERR_WORKSPACE, "buffer of %zu bytes < %zu needed", bytes, L.total);
  char* b = static_cast<char*>(base);
  memset(w, 0, sizeof(*w));
  w->K = K;
  w->N = N;
  w->fmt = fmt;
  w->group = fmt == QLIN_W4_G128 ? 128 : 0;
  w->n_outlier = n_outlier;
  w->n_outlier_pad = pad8(n_outlier);
  w->codes = b + L.codes;
  w->chan_scale = reinterpret_cast<float*>(b + L.chan);
  if (fmt == QLIN_W4_G128) {
    w->group_scale = reinterpret_cast<uint16_t*>(b + L.group);
    w->fold_ratio = reinterpret_cast<uint16_t*>(b + L.fold);
  }
  if (n_outlier > 0) {
    w->outlier_idx = reinterpret_cast<int32_t*>(b + L.oidx);
    w->W_Ot = reinterpret_cast<uint16_t*>(b + L.wot);
    w->wmax_O = reinterpret_cast<float*>(b + L.wmax);
  }
  return QLIN_OK;
}

qlin_status qlin_pack_weights(const uint16_t* W, const int32_t* O_host, const qlin_weights* w, void* stream_) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (!W) return fail(QLIN_ERR_ARG, "W is NULL");
  if (!aligned16(W)) return fail(QLIN_ERR_ALIGN, "W is not 16-byte aligned");
  const int K = w->K, N = w->N, nO = w->n_outlier;
  if (nO > 0) {
    if (!O_host) return fail(QLIN_ERR_ARG, "O_host is NULL with n_outlier=%d", nO);
    for (int i = 0; i < nO; ++i) {
      if (O_host[i] < 0 || O_host[i] >= K) return fail(QLIN_ERR_ARG, "O[%d]=%d outside [0, K)", i, O_host[i]);
      if (i > 0 && O_host[i] <= O_host[i - 1]) return fail(QLIN_ERR_ARG, "O is not strictly increasing at %d", i);
    }
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const int threads = 128;
  const int blocks = (N + threads - 1) / threads;
  uint8_t* codes = static_cast<uint8_t*>(w->codes);
  const Layout L = weights_layout(K, N, w->fmt, nO);
  QLIN_CUDA_TRY(cudaMemsetAsync(codes, 0, L.chan - L.codes, stream));  // tile padding is zero
  switch (w->fmt) {
    case QLIN_W4_PERCHANNEL:
      pack_per_channel_kernel<7, true><<<blocks, threads, 0, stream>>>(W, K, N, codes, w->chan_scale);
      break;
    case QLIN_W8_PERCHANNEL:
      pack_per_channel_kernel<127, false><<<blocks, threads, 0, stream>>>(W, K, N, codes, w->chan_scale);
      break;
    default:
      pack_group_kernel<128><<<blocks, threads, 0, stream>>>(W, K, N, codes, w->chan_scale, w->group_scale,
                                                             w->fold_ratio);
  }
  QLIN_LAUNCH_CHECK("pack kernel");
  if (nO > 0) {
    QLIN_CUDA_TRY(cudaMemcpyAsync(w->outlier_idx, O_host, size_t(nO) * 4, cudaMemcpyHostToDevice, stream));
    QLIN_CUDA_TRY(cudaMemsetAsync(w->W_Ot, 0, L.wmax - L.wot, stream));
    pack_outliers_kernel<<<nO, 256, 0, stream>>>(W, N, w->outlier_idx, nO, w->W_Ot, w->wmax_O);
    QLIN_LAUNCH_CHECK("pack_outliers_kernel");
  }
  return QLIN_OK;
}

qlin_status qlin_quant_act_workspace(int32_t M, const qlin_weights* w, size_t* bytes) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (!bytes || M < 0) return fail(QLIN_ERR_ARG, "bad arguments");
  *bytes = act_ws_bytes(w);
  return QLIN_OK;
}

qlin_status qlin_quant_act(const uint16_t* X, int32_t M, const qlin_weights* w, float* s, float gamma,
                           int32_t update_momentum, int8_t* Xq, float* a, int8_t* XqO, void* workspace,
                           size_t ws_bytes, void* stream) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (M < 0) return fail(QLIN_ERR_ARG, "M=%d is negative", M);
  const int nO = w->n_outlier;
  if (M > 0 && (!X || !Xq || !a)) return fail(QLIN_ERR_ARG, "X/Xq/a is NULL");
  if (nO > 0 && M > 0 && (!s || !XqO)) return fail(QLIN_ERR_ARG, "s/XqO is NULL with n_outlier=%d", nO);
  if (!(gamma >= 0.f && gamma <= 1.f)) return fail(QLIN_ERR_ARG, "gamma=%g outside [0, 1]", double(gamma));
  if ((X && !aligned16(X)) || (Xq && !aligned16(Xq)) || (a && !aligned16(a)) || (s && !aligned16(s)) ||
      (XqO && !aligned16(XqO)))
    return fail(QLIN_ERR_ALIGN, "an activation buffer is not 16-byte aligned");
  const size_t need = (update_momentum ? act_ws_bytes(w) : 0);
  if (ws_bytes < need || (need && !workspace)) return fail(QLIN_ERR_WORKSPACE, "workspace %zu < %zu", ws_bytes, need);
  return launch_quant(X, M, w, s, gamma, update_momentum, Xq, a, XqO, nullptr, workspace,
                      static_cast<cudaStream_t>(stream));
}

qlin_status qlin_quant_act_noalloc(const uint16_t* X, int32_t M, const qlin_weights* w, float* s, float gamma,
                                   int32_t update_momentum, int8_t* Xq, float* a, int8_t* XqO, void* stream_) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (M < 0) return fail(QLIN_ERR_ARG, "M=%d is negative", M);
  const int nO = w->n_outlier;
  if (nO > QLIN_NOALLOC_MAX_OUTLIERS)
    return fail(QLIN_ERR_SHAPE, "n_outlier=%d exceeds the %d outlier channels the fixed scratch of "
                "qlin_quant_act_noalloc holds; use qlin_quant_act with a workspace", nO, QLIN_NOALLOC_MAX_OUTLIERS);
  if (M > 0 && (!X || !Xq || !a)) return fail(QLIN_ERR_ARG, "X/Xq/a is NULL");
  if (nO > 0 && M > 0 && (!s || !XqO)) return fail(QLIN_ERR_ARG, "s/XqO is NULL with n_outlier=%d", nO);
  if (!(gamma >= 0.f && gamma <= 1.f)) return fail(QLIN_ERR_ARG, "gamma=%g outside [0, 1]", double(gamma));
  if ((X && !aligned16(X)) || (Xq && !aligned16(Xq)) || (a && !aligned16(a)) || (s && !aligned16(s)) ||
      (XqO && !aligned16(XqO)))
    return fail(QLIN_ERR_ALIGN, "an activation buffer is not 16-byte aligned");
  if (M == 0) return QLIN_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  unsigned* scratch = nullptr;
  if (update_momentum && nO > 0) {
    st = noalloc_scratch(&scratch);
    if (st != QLIN_OK) return st;
    // The scratch keeps whatever the previous call left: clear the maxima
    // and the counter (they must start at zero) before this call uses them.
    QLIN_CUDA_TRY(cudaMemsetAsync(scratch, 0, (size_t(nO) + 1) * sizeof(unsigned), stream));
  }
  return launch_quant(X, M, w, s, gamma, update_momentum, Xq, a, XqO, nullptr, scratch, stream);
}

qlin_status qlin_outlier_colmax(const uint16_t* X, int32_t M, const qlin_weights* w, float* cmax, void* stream_) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (M < 0) return fail(QLIN_ERR_ARG, "M=%d is negative", M);
  const int nO = w->n_outlier;
  if (nO == 0) return QLIN_OK;
  if (!cmax || (M > 0 && !X)) return fail(QLIN_ERR_ARG, "X/cmax is NULL");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  QLIN_CUDA_TRY(cudaMemsetAsync(cmax, 0, size_t(nO) * 4, stream));
  if (M == 0) return QLIN_OK;
  const int grid = (M + kColmaxRows - 1) / kColmaxRows;
  colmax_kernel<<<grid, 256, size_t(nO) * 8, stream>>>(X, M, w->K, w->outlier_idx, nO,
                                                        reinterpret_cast<unsigned*>(cmax), 0, nullptr, nullptr,
                                                        0.f, nullptr);
  QLIN_LAUNCH_CHECK("colmax_kernel");
  return QLIN_OK;
}

qlin_status qlin_momentum_update(const qlin_weights* w, const float* cmax, float* s, float gamma, void* stream) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  const int nO = w->n_outlier;
  if (nO == 0) return QLIN_OK;
  if (!cmax || !s) return fail(QLIN_ERR_ARG, "cmax/s is NULL");
  if (!(gamma >= 0.f && gamma <= 1.f)) return fail(QLIN_ERR_ARG, "gamma=%g outside [0, 1]", double(gamma));
  momentum_kernel<<<(nO + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(cmax, w->wmax_O, s, gamma, nO);
  QLIN_LAUNCH_CHECK("momentum_kernel");
  return QLIN_OK;
}

qlin_status qlin_gemm_workspace(int32_t M, const qlin_weights* w, size_t* bytes) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (!bytes || M < 0) return fail(QLIN_ERR_ARG, "bad arguments");
  *bytes = gemm_ws_bytes(M, w);
  return QLIN_OK;
}

qlin_status qlin_gemm(const qlin_weights* w, const int8_t* Xq, const float* a, const int8_t* XqO, const float* s,
                      int32_t M, uint16_t* Y, int32_t* acc_debug, void* workspace, size_t ws_bytes,
                      void* stream_) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (M < 0) return fail(QLIN_ERR_ARG, "M=%d is negative", M);
  if (M == 0) return QLIN_OK;
  const int nO = w->n_outlier;
  if (!Xq || !a || !Y) return fail(QLIN_ERR_ARG, "Xq/a/Y is NULL");
  if (nO > 0 && (!XqO || !s)) return fail(QLIN_ERR_ARG, "XqO/s is NULL with n_outlier=%d", nO);
  if (!aligned16(Xq) || !aligned16(a) || !aligned16(Y) || (acc_debug && !aligned16(acc_debug)) ||
      (XqO && !aligned16(XqO)) || (s && !aligned16(s)))
    return fail(QLIN_ERR_ALIGN, "a GEMM buffer is not 16-byte aligned");
  const size_t need = gemm_ws_bytes(M, w);
  if (ws_bytes < need || (need && !workspace)) return fail(QLIN_ERR_WORKSPACE, "workspace %zu < %zu", ws_bytes, need);
  if (need && reinterpret_cast<uintptr_t>(workspace) % kAlign)
    return fail(QLIN_ERR_ALIGN, "workspace must be 256-byte aligned");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  char* gws = static_cast<char*>(workspace);
  if (nO > 0) {
    uint16_t* U = reinterpret_cast<uint16_t*>(gws + plan_gemm(M, w).u_off[0]);
    const size_t total = size_t(M) * w->n_outlier_pad;
    comp_operand_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(XqO, s, M, nO,
                                                                                       w->n_outlier_pad, U);
    QLIN_LAUNCH_CHECK("comp_operand_kernel");
  }
  return launch_gemm(w, Xq, a, M, Y, acc_debug, gws, stream);
}

qlin_status qlin_backward_dx_workspace(int32_t M, const qlin_weights* w, size_t* bytes) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (!bytes || M < 0) return fail(QLIN_ERR_ARG, "bad arguments");
  *bytes = M > 0 ? plan_backward(M, w, true).bytes : 0;
  return QLIN_OK;
}

qlin_status qlin_backward_dx(const qlin_weights* w, const uint16_t* dY, int32_t M, const float* s, uint16_t* dX,
                             void* workspace, size_t ws_bytes, void* stream_) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (M < 0) return fail(QLIN_ERR_ARG, "M=%d is negative", M);
  if (M > 65535 * 128) return fail(QLIN_ERR_SHAPE, "M=%d exceeds %d", M, 65535 * 128);
  if (M == 0) return QLIN_OK;
  if (workspace && reinterpret_cast<uintptr_t>(workspace) % kAlign)
    return fail(QLIN_ERR_ALIGN, "workspace must be 256-byte aligned");
  const int nO = w->n_outlier;
  if (!dY || !dX) return fail(QLIN_ERR_ARG, "dY/dX is NULL");
  if (nO > 0 && !s) return fail(QLIN_ERR_ARG, "s is NULL with n_outlier=%d", nO);
  if (!aligned16(dY) || !aligned16(dX) || (s && !aligned16(s)))
    return fail(QLIN_ERR_ALIGN, "a backward buffer is not 16-byte aligned");
  st = get_encoder();
  if (st != QLIN_OK) return st;
  CUtensorMap tm;
  st = make_map(&tm, dY, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, w->N, M, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QLIN_OK) return st;
  BwdArgs args;
  args.codes = static_cast<const uint8_t*>(w->codes);
  args.rfold = w->fold_ratio;
  args.wot = w->W_Ot;
  args.cscale = w->chan_scale;
  args.oidx = w->outlier_idx;
  args.s = s;
  args.dX = dX;
  args.M = M;
  args.N = w->N;
  args.K = w->K;
  args.nO = nO;
  args.kbs = (w->K + 127) / 128;
  args.nib = (nO + 63) / 64;
  args.nsteps = (w->N + 63) / 64;
  // the split plan needs the whole workspace it asks for; with none (or a
  // smaller one) every tile runs whole
  BwdPlan p = plan_backward(M, w, true);
  if (p.bytes && (!workspace || ws_bytes < p.bytes)) p = plan_backward(M, w, false);
  args.ntk = p.ntk;
  args.full = p.full;
  args.tsplit = p.tsplit;
  args.part = p.bytes ? reinterpret_cast<float*>(static_cast<char*>(workspace) + p.part_off) : nullptr;
  args.cnt = p.bytes ? reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + p.cnt_off) : nullptr;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  switch (w->fmt) {
    case QLIN_W4_PERCHANNEL: return launch_backward_t<kFmtW4PC>(tm, args, stream);
    case QLIN_W4_G128: return launch_backward_t<kFmtW4G128>(tm, args, stream);
    default: return launch_backward_t<kFmtW8>(tm, args, stream);
  }
}

qlin_status qlin_forward_workspace(int32_t M, const qlin_weights* w, size_t* bytes) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (!bytes || M < 0) return fail(QLIN_ERR_ARG, "bad arguments");
  *bytes = forward_layout(M, w).total;
  return QLIN_OK;
}

qlin_status qlin_forward(const uint16_t* X, int32_t M, const qlin_weights* w, float* s, float gamma,
                         int32_t update_momentum, uint16_t* Y, void* workspace, size_t ws_bytes, void* stream_) {
  qlin_status st = check_weights(w);
  if (st != QLIN_OK) return st;
  if (M < 0) return fail(QLIN_ERR_ARG, "M=%d is negative", M);
  if (M == 0) return QLIN_OK;
  const int nO = w->n_outlier;
  if (!X || !Y) return fail(QLIN_ERR_ARG, "X/Y is NULL");
  if (nO > 0 && !s) return fail(QLIN_ERR_ARG, "s is NULL with n_outlier=%d", nO);
  if (!(gamma >= 0.f && gamma <= 1.f)) return fail(QLIN_ERR_ARG, "gamma=%g outside [0, 1]", double(gamma));
  if (!aligned16(X) || !aligned16(Y) || (s && !aligned16(s)))
    return fail(QLIN_ERR_ALIGN, "X/Y/s is not 16-byte aligned");
  FwdLayout L = forward_layout(M, w);
  if (ws_bytes < L.total || !workspace) return fail(QLIN_ERR_WORKSPACE, "workspace %zu < %zu", ws_bytes, L.total);
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return fail(QLIN_ERR_ALIGN, "workspace must be 256-byte aligned");
  char* ws = static_cast<char*>(workspace);
  int8_t* Xq = reinterpret_cast<int8_t*>(ws + L.xq);
  float* a = reinterpret_cast<float*>(ws + L.a);
  int8_t* XqO = nO > 0 ? reinterpret_cast<int8_t*>(ws + L.xqo) : nullptr;
  char* gws = ws + L.gemm;
  uint16_t* U = nO > 0 ? reinterpret_cast<uint16_t*>(gws + plan_gemm(M, w).u_off[0]) : nullptr;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  st = launch_quant(X, M, w, s, gamma, update_momentum, Xq, a, XqO, U, ws + L.act, stream);
  if (st != QLIN_OK) return st;
  return launch_gemm(w, Xq, a, M, Y, nullptr, gws, stream);
}

#ifdef QLIN_TRACE
// Diagnostic builds only: point the GEMM's phase stamps at a device buffer
// of [grid][32] int64 (NULL turns them off).
QLIN_API int qlin_trace_set(long long* p) {
  return static_cast<int>(cudaMemcpyToSymbol(qlin::g_trace, &p, sizeof(p)));
}
QLIN_API int qlin_steps_set(long long* p) {
  return static_cast<int>(cudaMemcpyToSymbol(qlin::g_steps, &p, sizeof(p)));
}
#endif

qlin_status qlin_forward_grouped_workspace(int32_t count, const qlin_weights* const* w, int32_t M, size_t* bytes) {
  qlin_status st = check_group(count, w, M);
  if (st != QLIN_OK) return st;
  if (!bytes) return fail(QLIN_ERR_ARG, "bytes is NULL");
  *bytes = group_layout(M, w, count).total;
  return QLIN_OK;
}

qlin_status qlin_forward_grouped(int32_t count, const qlin_weights* const* w, const uint16_t* const* X,
                                 float* const* s, uint16_t* const* Y, int32_t M, float gamma,
                                 int32_t update_momentum, void* workspace, size_t ws_bytes, void* stream_) {
  qlin_status st = check_group(count, w, M);
  if (st != QLIN_OK) return st;
  if (!(gamma >= 0.f && gamma <= 1.f)) return fail(QLIN_ERR_ARG, "gamma=%g outside [0, 1]", double(gamma));
  if (M == 0) return QLIN_OK;
  if (!X || !Y || !s) return fail(QLIN_ERR_ARG, "X/Y/s array is NULL");
  for (int q = 0; q < count; ++q) {
    if (!X[q] || !Y[q]) return fail(QLIN_ERR_ARG, "problem %d: X/Y is NULL", q);
    if (w[q]->n_outlier > 0 && !s[q]) return fail(QLIN_ERR_ARG, "problem %d: s is NULL with n_outlier=%d", q,
                                                  w[q]->n_outlier);
    if (!aligned16(X[q]) || !aligned16(Y[q]) || (s[q] && !aligned16(s[q])))
      return fail(QLIN_ERR_ALIGN, "problem %d: X/Y/s is not 16-byte aligned", q);
    for (int r = 0; r < q; ++r)
      if (Y[r] == Y[q]) return fail(QLIN_ERR_ARG, "problems %d and %d write the same Y", r, q);
  }
  const GroupLayout L = group_layout(M, w, count);
  if (ws_bytes < L.total || !workspace) return fail(QLIN_ERR_WORKSPACE, "workspace %zu < %zu", ws_bytes, L.total);
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return fail(QLIN_ERR_ALIGN, "workspace must be 256-byte aligned");
  char* ws = static_cast<char*>(workspace);
  char* gws = ws + L.gemm;
  QuantIO io[kMaxProbs];
  const int8_t* xq[kMaxProbs];
  const float* av[kMaxProbs];
  uint16_t* yv[kMaxProbs];
  for (int q = 0; q < count; ++q) {
    const bool o = w[q]->n_outlier > 0;
    io[q] = QuantIO{X[q], s[q], reinterpret_cast<int8_t*>(ws + L.xq[q]), reinterpret_cast<float*>(ws + L.a[q]),
                    o ? reinterpret_cast<int8_t*>(ws + L.xqo[q]) : nullptr,
                    o ? reinterpret_cast<uint16_t*>(gws + L.plan.u_off[q]) : nullptr, ws + L.act[q]};
    xq[q] = io[q].Xq;
    av[q] = io[q].a;
    yv[q] = Y[q];
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  st = launch_quant_group<kMaxProbs>(w, io, count, M, gamma, update_momentum, stream);
  if (st != QLIN_OK) return st;
  return launch_gemm_group<kMaxProbs>(L.plan, w, xq, av, yv, nullptr, gws, stream);
}

namespace {
struct GptqLayout {
  size_t st, f, a, total;
};
GptqLayout gptq_layout(int K) {
  GptqLayout L{};
  L.st = 0;
  L.f = round_up(sizeof(GjScratch), kAlign);
  L.a = round_up(L.f + size_t(K) * 8, kAlign);
  L.total = round_up(L.a + size_t(K) * K * 8, kAlign);
  return L;
}
qlin_status check_gptq_shape(int32_t K, int32_t N) {
  if (K < 1 || N < 1) return fail(QLIN_ERR_ARG, "K=%d N=%d must be positive", K, N);
  if (K > 16384) return fail(QLIN_ERR_SHAPE, "K=%d exceeds 16384", K);
  return QLIN_OK;
}
}  // namespace

qlin_status qlin_gptq_workspace(int32_t K, int32_t N, size_t* bytes) {
  qlin_status st = check_gptq_shape(K, N);
  if (st != QLIN_OK) return st;
  if (!bytes) return fail(QLIN_ERR_ARG, "bytes is NULL");
  *bytes = gptq_layout(K).total;
  return QLIN_OK;
}

qlin_status qlin_gptq_quantize(const double* X, int32_t ns, int32_t K, int32_t N, double* W, const double* scale,
                               int32_t qmax, int8_t* codes, double* Hinv, int32_t* singular, void* workspace,
                               size_t ws_bytes, void* stream_) {
  qlin_status st = check_gptq_shape(K, N);
  if (st != QLIN_OK) return st;
  if (ns < 1) return fail(QLIN_ERR_ARG, "ns=%d must be positive", ns);
  if (qmax < 1 || qmax > 127) return fail(QLIN_ERR_ARG, "qmax=%d outside [1, 127]", qmax);
  if (!X || !W || !scale || !codes || !Hinv || !workspace) return fail(QLIN_ERR_ARG, "a GPTQ buffer is NULL");
  if ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(scale) |
       reinterpret_cast<uintptr_t>(Hinv)) & 7u)
    return fail(QLIN_ERR_ALIGN, "fp64 buffers must be 8-byte aligned");
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return fail(QLIN_ERR_ALIGN, "workspace must be 256-byte aligned");
  const GptqLayout L = gptq_layout(K);
  if (ws_bytes < L.total) return fail(QLIN_ERR_WORKSPACE, "workspace %zu < %zu", ws_bytes, L.total);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  char* ws = static_cast<char*>(workspace);
  GjScratch* scr = reinterpret_cast<GjScratch*>(ws + L.st);
  double* f = reinterpret_cast<double*>(ws + L.f);
  double* a = reinterpret_cast<double*>(ws + L.a);
  QLIN_CUDA_TRY(cudaMemsetAsync(scr, 0, sizeof(GjScratch), stream));
  // H = 2 X^T X into the working matrix; the inverse starts as the identity
  const unsigned th = static_cast<unsigned>((K + kHessTile - 1) / kHessTile);
  gptq_hessian_kernel<<<dim3(th, th), 256, 0, stream>>>(X, ns, K, a);
  QLIN_LAUNCH_CHECK("gptq_hessian_kernel");
  const size_t kk = size_t(K) * K;
  gptq_identity_kernel<<<static_cast<unsigned>((kk + 255) / 256), 256, 0, stream>>>(Hinv, K);
  QLIN_LAUNCH_CHECK("gptq_identity_kernel");
  // Gauss-Jordan elimination with partial pivoting: a -> I, Hinv -> H^-1
  const unsigned cb = static_cast<unsigned>((K + 255) / 256);
  const unsigned ex = cb < 4 ? cb : 4;
  for (int c = 0; c < K; ++c) {
    gj_pivot_kernel<<<1, 1024, 0, stream>>>(a, K, c, scr, f);
    gj_swap_scale_kernel<<<cb, 256, 0, stream>>>(a, Hinv, K, c, scr);
    gj_eliminate_kernel<<<dim3(ex, static_cast<unsigned>(K)), 256, 0, stream>>>(a, Hinv, K, c, scr, f);
  }
  QLIN_LAUNCH_CHECK("Gauss-Jordan kernels");
  // column-sequential quantization with compensation on a working copy of H^-1
  QLIN_CUDA_TRY(cudaMemcpyAsync(a, Hinv, kk * 8, cudaMemcpyDeviceToDevice, stream));
  constexpr int kRows = 64;
  for (int i = 0; i < K; ++i) {
    const int rem = K - i - 1;
    const int yw = rem > 0 ? (rem + kRows - 1) / kRows : 1;
    const int yd = rem > 0 ? (rem + kRows - 1) / kRows : 0;
    const int xa = (N + 255) / 256, xd = (rem + 255) / 256;
    const unsigned gx = static_cast<unsigned>(xa > xd ? xa : xd);
    gptq_step_kernel<<<dim3(gx, static_cast<unsigned>(yw + yd)), 256, 0, stream>>>(W, codes, scale, a, K, N, i, qmax,
                                                                                  kRows, yw, scr);
  }
  QLIN_LAUNCH_CHECK("gptq_step_kernel");
  if (singular) QLIN_CUDA_TRY(cudaMemcpyAsync(singular, &scr->singular, 4, cudaMemcpyDeviceToDevice, stream));
  return QLIN_OK;
}

namespace {
struct SmoothLayout {
  size_t cmax, wmax, xall, sv, xh, wh, packed, xq, a, gemm, y, acc, ref, total;
  Layout wl;
};
SmoothLayout smooth_layout(int M, int K, int N) {
  SmoothLayout L{};
  size_t off = 0;
  L.cmax = off; off = round_up(off + size_t(K) * 4, kAlign);
  L.wmax = off; off = round_up(off + size_t(K) * 4, kAlign);
  L.xall = off; off = round_up(off + 16, kAlign);
  L.sv = off; off = round_up(off + size_t(K) * 4, kAlign);
  L.xh = off; off = round_up(off + size_t(M) * K * 2, kAlign);
  L.wh = off; off = round_up(off + size_t(K) * N * 2, kAlign);
  L.wl = weights_layout(K, N, QLIN_W4_PERCHANNEL, 0);
  L.packed = off; off = round_up(off + L.wl.total, kAlign);
  L.xq = off; off = round_up(off + size_t(M) * K, kAlign);
  L.a = off; off = round_up(off + size_t(M) * 4, kAlign);
  qlin_weights w{};
  w.K = K; w.N = N; w.fmt = QLIN_W4_PERCHANNEL; w.n_outlier = 0; w.n_outlier_pad = 0;
  L.gemm = off; off = round_up(off + gemm_ws_bytes(M, &w), kAlign);
  L.y = off; off = round_up(off + size_t(M) * N * 2, kAlign);
  L.acc = off; off = round_up(off + size_t(M) * N * 4, kAlign);
  L.ref = off; off = round_up(off + size_t(M) * N * 4, kAlign);
  L.total = off;
  return L;
}
qlin_status check_smooth(int32_t M, int32_t K, int32_t N, int32_t G) {
  if (M < 1 || G < 1 || G > 64) return fail(QLIN_ERR_ARG, "M=%d must be >= 1 and G=%d in [1, 64]", M, G);
  return check_shape(K, N, QLIN_W4_PERCHANNEL, 0);
}
}  // namespace

qlin_status qlin_smooth_search_workspace(int32_t M, int32_t K, int32_t N, int32_t G, size_t* bytes) {
  qlin_status st = check_smooth(M, K, N, G);
  if (st != QLIN_OK) return st;
  if (!bytes) return fail(QLIN_ERR_ARG, "bytes is NULL");
  *bytes = smooth_layout(M, K, N).total;
  return QLIN_OK;
}

qlin_status qlin_smooth_search(const uint16_t* X, int32_t M, int32_t K, const uint16_t* W, int32_t N, int32_t G,
                               double* loss, int32_t* best, float* s_best, void* workspace, size_t ws_bytes,
                               void* stream_) {
  qlin_status st = check_smooth(M, K, N, G);
  if (st != QLIN_OK) return st;
  if (!X || !W || !loss || !workspace) return fail(QLIN_ERR_ARG, "X/W/loss/workspace is NULL");
  if (!aligned16(X) || !aligned16(W) || (reinterpret_cast<uintptr_t>(loss) & 7u) ||
      (s_best && (reinterpret_cast<uintptr_t>(s_best) & 3u)) || (best && (reinterpret_cast<uintptr_t>(best) & 3u)))
    return fail(QLIN_ERR_ALIGN, "X/W must be 16-byte aligned, loss 8, best and s_best 4");
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return fail(QLIN_ERR_ALIGN, "workspace must be 256-byte aligned");
  const SmoothLayout L = smooth_layout(M, K, N);
  if (ws_bytes < L.total) return fail(QLIN_ERR_WORKSPACE, "workspace %zu < %zu", ws_bytes, L.total);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  char* ws = static_cast<char*>(workspace);
  unsigned* cmax = reinterpret_cast<unsigned*>(ws + L.cmax);
  float* wmax = reinterpret_cast<float*>(ws + L.wmax);
  float* xall = reinterpret_cast<float*>(ws + L.xall);
  float* sv = reinterpret_cast<float*>(ws + L.sv);
  uint16_t* Xh = reinterpret_cast<uint16_t*>(ws + L.xh);
  uint16_t* Wh = reinterpret_cast<uint16_t*>(ws + L.wh);
  int8_t* Xq = reinterpret_cast<int8_t*>(ws + L.xq);
  float* a = reinterpret_cast<float*>(ws + L.a);
  uint16_t* Y = reinterpret_cast<uint16_t*>(ws + L.y);
  int32_t* acc = reinterpret_cast<int32_t*>(ws + L.acc);
  float* ref = reinterpret_cast<float*>(ws + L.ref);
  qlin_weights w{};
  st = qlin_weights_bind(&w, K, N, QLIN_W4_PERCHANNEL, 0, ws + L.packed, L.wl.total);
  if (st != QLIN_OK) return st;
  QLIN_CUDA_TRY(cudaMemsetAsync(cmax, 0, size_t(K) * 4, stream));
  QLIN_CUDA_TRY(cudaMemsetAsync(ws + L.gemm, 0, L.y - L.gemm, stream));  // split-K counters start at zero
  QLIN_CUDA_TRY(cudaMemsetAsync(loss, 0, size_t(G) * 8, stream));
  smooth_colmax_kernel<<<dim3((K + 255) / 256, (M + 63) / 64), 256, 0, stream>>>(X, M, K, cmax);
  smooth_rowmax_kernel<<<K, 256, 0, stream>>>(W, N, wmax);
  smooth_allmax_kernel<<<1, 1024, 0, stream>>>(cmax, K, xall);
  QLIN_LAUNCH_CHECK("smoothing maxima");
  const size_t mk = size_t(M) * K, kn = size_t(K) * N, mn = size_t(M) * N;
  for (int j = 0; j < G; ++j) {
    smooth_factors_kernel<<<(K + 255) / 256, 256, 0, stream>>>(cmax, wmax, xall, K, j, G, sv);
    smooth_apply_x_kernel<<<static_cast<unsigned>((mk + 255) / 256), 256, 0, stream>>>(X, sv, M, K, Xh);
    smooth_apply_w_kernel<<<static_cast<unsigned>((kn + 255) / 256), 256, 0, stream>>>(W, sv, K, N, Wh);
    QLIN_LAUNCH_CHECK("smoothing kernels");
    // the layer's quantizers and integer product on the smoothed tensors
    st = qlin_pack_weights(Wh, nullptr, &w, stream);
    if (st != QLIN_OK) return st;
    st = launch_quant(Xh, M, &w, nullptr, 0.f, 0, Xq, a, nullptr, nullptr, nullptr, stream);
    if (st != QLIN_OK) return st;
    st = launch_gemm(&w, Xq, a, M, Y, acc, ws + L.gemm, stream);
    if (st != QLIN_OK) return st;
    smooth_ref_kernel<<<dim3((N + kRefTile - 1) / kRefTile, (M + kRefTile - 1) / kRefTile), 256, 0, stream>>>(
        X, W, sv, M, K, N, ref);
    smooth_loss_kernel<<<static_cast<unsigned>((mn + 255) / 256), 256, 0, stream>>>(acc, a, w.chan_scale, ref, M,
                                                                                    N, loss + j);
    QLIN_LAUNCH_CHECK("smoothing loss");
  }
  smooth_pick_kernel<<<1, 256, 0, stream>>>(loss, G, cmax, wmax, xall, K, best, s_best);
  QLIN_LAUNCH_CHECK("smooth_pick_kernel");
  return QLIN_OK;
}

// ---------------------------------------------------------------- OffQ
namespace {
// d (+1/-1, d_0 = +1) as a bit mask: bit i set when d_i = -1.
qlin_status offq_signs(const int8_t* d, uint4* out) {
  if (!d) return fail(QLIN_ERR_ARG, "signs is NULL");
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  for (int i = 0; i < 128; ++i) {
    if (d[i] != 1 && d[i] != -1) return fail(QLIN_ERR_ARG, "signs[%d] = %d is not +1 or -1", i, int(d[i]));
    if (d[i] < 0) w[i >> 5] |= 1u << (i & 31);
  }
  if (w[0] & 1u) return fail(QLIN_ERR_ARG, "signs[0] must be +1 (row 0 of D H is all ones)");
  *out = make_uint4(w[0], w[1], w[2], w[3]);
  return QLIN_OK;
}

qlin_status check_offq_shape(int32_t M, int32_t K, int32_t N) {
  if (M < 0 || K <= 0 || N <= 0) return fail(QLIN_ERR_ARG, "bad sizes M=%d K=%d N=%d", M, K, N);
  if (K % 128 || K > 65536) return fail(QLIN_ERR_SHAPE, "OffQ needs K %% 128 == 0 and K <= 65536 (K=%d)", K);
  if (N % 16 || N > 1048576) return fail(QLIN_ERR_SHAPE, "N=%d must be a multiple of 16 and <= 2^20", N);
  return QLIN_OK;
}

size_t offq_codes_size(int32_t K, int32_t N) { return size_t((N + 127) / 128) * (K / 128) * 8192; }
size_t offq_wide_size(int32_t K, int32_t N) { return size_t((N + 127) / 128) * (K / 128) * 16384; }

struct OffqLayout {
  size_t xq = 0, scale = 0, offset = 0, wide = 0, total = 0;
};
OffqLayout offq_layout(int32_t M, int32_t K, int32_t N, bool with_act) {
  OffqLayout L;
  size_t o = 0;
  if (with_act) {
    L.xq = o;
    o = round_up(o + size_t(M) * K, kAlign);
    L.scale = o;
    o = round_up(o + size_t(M) * (K / 128) * 4, kAlign);
    L.offset = o;
    o = round_up(o + size_t(M) * (K / 128) * 4, kAlign);
  }
  L.wide = o;
  L.total = round_up(o + offq_wide_size(K, N), kAlign);
  return L;
}

int offq_gemm_smem_ok() {
  static int ok = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    ok = cudaFuncSetAttribute(offq_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kOffqSmem) ==
         cudaSuccess;
    if (!ok) cudaGetLastError();
  });
  return ok;
}

qlin_status launch_offq_quant(const uint16_t* X, int32_t M, int32_t K, uint4 sg, int8_t* Xq, float* scale,
                              float* offset, cudaStream_t stream) {
  const long long units = static_cast<long long>(M) * (K / 128);
  const long long blocks = (units + kOffqQuantThreads / 4 - 1) / (kOffqQuantThreads / 4);
  if (blocks > 0x7fffffffLL) return fail(QLIN_ERR_SHAPE, "M * K too large");
  cudaError_t e = launch_k(offq_quant_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kOffqQuantThreads), 0,
                           stream, X, M, K, sg, Xq, scale, offset);
  if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "offq_quant_kernel launch failed: %s", cudaGetErrorString(e));
  return QLIN_OK;
}

qlin_status launch_offq_gemm(const int8_t* Xq, const float* scale, const float* offset, int32_t M, int32_t K,
                             int32_t N, const uint8_t* codes, const float* chan_scale, const float* colsum,
                             uint16_t* Y, uint8_t* wide, cudaStream_t stream) {
  qlin_status st = get_encoder();
  if (st != QLIN_OK) return st;
  if (!offq_gemm_smem_ok()) return fail(QLIN_ERR_CUDA, "offq_gemm_kernel: shared memory attribute refused");
  const int kb = K / 128;
  const int tiles_n = (N + 127) / 128;
  const unsigned nblk = static_cast<unsigned>(tiles_n) * static_cast<unsigned>(kb);
  cudaError_t e = launch_k(widen_w4_kernel<kFmtW4PC>, dim3(nblk), dim3(256), 0, stream, codes,
                           static_cast<const uint16_t*>(nullptr), N, kb, wide);
  if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "widen_w4_kernel launch failed: %s", cudaGetErrorString(e));
  OffqParams prm;
  memset(&prm, 0, sizeof(prm));
  OffqArgs& g = prm.g;
  g.scale = scale;
  g.offset = offset;
  g.colsum = colsum;
  g.cscale = chan_scale;
  g.wide = wide;
  g.Y = Y;
  g.M = M;
  g.N = N;
  g.G = kb;
  g.tiles_m = (M + 127) / 128;
  g.tiles = g.tiles_m * tiles_n;
  st = make_map(&prm.tmX, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QLIN_OK) return st;
  const int cap = gemm_cta_cap();
  const int grid = g.tiles < cap ? g.tiles : cap;
  e = launch_k(offq_gemm_kernel, dim3(static_cast<unsigned>(grid)), dim3(kOffqThreads), kOffqSmem, stream, prm);
  if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "offq_gemm_kernel launch failed: %s", cudaGetErrorString(e));
  return QLIN_OK;
}
}  // namespace

qlin_status qlin_offq_codes_bytes(int32_t K, int32_t N, size_t* bytes) {
  qlin_status st = check_offq_shape(0, K, N);
  if (st != QLIN_OK) return st;
  if (!bytes) return fail(QLIN_ERR_ARG, "bytes is NULL");
  *bytes = offq_codes_size(K, N);
  return QLIN_OK;
}

qlin_status qlin_offq_rotate_weights(const uint16_t* W, int32_t K, int32_t N, const int8_t* signs, float* Wr,
                                     void* stream_) {
  qlin_status st = check_offq_shape(0, K, N);
  if (st != QLIN_OK) return st;
  uint4 sg;
  st = offq_signs(signs, &sg);
  if (st != QLIN_OK) return st;
  if (!W || !Wr) return fail(QLIN_ERR_ARG, "W/Wr is NULL");
  if (!aligned16(W) || !aligned16(Wr)) return fail(QLIN_ERR_ALIGN, "W/Wr is not 16-byte aligned");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  offq_rotate_kernel<<<dim3((N + 31) / 32, K / 128), 256, 0, stream>>>(W, K, N, sg, Wr);
  QLIN_LAUNCH_CHECK("offq_rotate_kernel");
  return QLIN_OK;
}

qlin_status qlin_offq_pack(const uint16_t* W, int32_t K, int32_t N, const int8_t* signs, uint8_t* codes,
                           float* chan_scale, float* colsum, float* Wr, void* stream_) {
  qlin_status st = qlin_offq_rotate_weights(W, K, N, signs, Wr, stream_);
  if (st != QLIN_OK) return st;
  if (!codes || !chan_scale || !colsum) return fail(QLIN_ERR_ARG, "codes/chan_scale/colsum is NULL");
  if (!aligned16(codes) || !aligned16(chan_scale) || !aligned16(colsum))
    return fail(QLIN_ERR_ALIGN, "codes/chan_scale/colsum is not 16-byte aligned");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  QLIN_CUDA_TRY(cudaMemsetAsync(codes, 0, offq_codes_size(K, N), stream));  // padding channels stay zero
  offq_pack_kernel<<<(N + 127) / 128, 128, 0, stream>>>(Wr, K, N, codes, chan_scale, colsum);
  QLIN_LAUNCH_CHECK("offq_pack_kernel");
  return QLIN_OK;
}

qlin_status qlin_offq_quant_act(const uint16_t* X, int32_t M, int32_t K, const int8_t* signs, int8_t* Xq,
                                float* scale, float* offset, void* stream_) {
  qlin_status st = check_offq_shape(M, K, 16);
  if (st != QLIN_OK) return st;
  uint4 sg;
  st = offq_signs(signs, &sg);
  if (st != QLIN_OK) return st;
  if (M == 0) return QLIN_OK;
  if (!X || !Xq || !scale || !offset) return fail(QLIN_ERR_ARG, "X/Xq/scale/offset is NULL");
  if (!aligned16(X) || !aligned16(Xq) || (reinterpret_cast<uintptr_t>(scale) & 3u) ||
      (reinterpret_cast<uintptr_t>(offset) & 3u))
    return fail(QLIN_ERR_ALIGN, "X/Xq must be 16-byte aligned, scale/offset 4");
  return launch_offq_quant(X, M, K, sg, Xq, scale, offset, static_cast<cudaStream_t>(stream_));
}

qlin_status qlin_offq_gemm_workspace(int32_t M, int32_t K, int32_t N, size_t* bytes) {
  qlin_status st = check_offq_shape(M, K, N);
  if (st != QLIN_OK) return st;
  if (!bytes) return fail(QLIN_ERR_ARG, "bytes is NULL");
  *bytes = offq_layout(M, K, N, false).total;
  return QLIN_OK;
}

qlin_status qlin_offq_gemm(const int8_t* Xq, const float* scale, const float* offset, int32_t M, int32_t K,
                           int32_t N, const uint8_t* codes, const float* chan_scale, const float* colsum, uint16_t* Y,
                           void* workspace, size_t ws_bytes, void* stream_) {
  qlin_status st = check_offq_shape(M, K, N);
  if (st != QLIN_OK) return st;
  if (M == 0) return QLIN_OK;
  if (!Xq || !scale || !offset || !codes || !chan_scale || !colsum || !Y || !workspace)
    return fail(QLIN_ERR_ARG, "a pointer argument is NULL");
  if (!aligned16(Xq) || !aligned16(codes) || !aligned16(chan_scale) || !aligned16(colsum) || !aligned16(Y) ||
      (reinterpret_cast<uintptr_t>(scale) & 3u) || (reinterpret_cast<uintptr_t>(offset) & 3u))
    return fail(QLIN_ERR_ALIGN, "Xq/codes/chan_scale/colsum/Y must be 16-byte aligned, scale/offset 4");
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return fail(QLIN_ERR_ALIGN, "workspace must be 256-byte aligned");
  const OffqLayout L = offq_layout(M, K, N, false);
  if (ws_bytes < L.total) return fail(QLIN_ERR_WORKSPACE, "workspace %zu < %zu", ws_bytes, L.total);
  uint8_t* wide = static_cast<uint8_t*>(workspace) + L.wide;
  return launch_offq_gemm(Xq, scale, offset, M, K, N, codes, chan_scale, colsum, Y, wide,
                          static_cast<cudaStream_t>(stream_));
}

qlin_status qlin_offq_forward_workspace(int32_t M, int32_t K, int32_t N, size_t* bytes) {
  qlin_status st = check_offq_shape(M, K, N);
  if (st != QLIN_OK) return st;
  if (!bytes) return fail(QLIN_ERR_ARG, "bytes is NULL");
  *bytes = offq_layout(M, K, N, true).total;
  return QLIN_OK;
}

qlin_status qlin_offq_forward(const uint16_t* X, int32_t M, int32_t K, int32_t N, const int8_t* signs,
                              const uint8_t* codes, const float* chan_scale, const float* colsum, uint16_t* Y,
                              void* workspace, size_t ws_bytes, void* stream_) {
  qlin_status st = check_offq_shape(M, K, N);
  if (st != QLIN_OK) return st;
  uint4 sg;
  st = offq_signs(signs, &sg);
  if (st != QLIN_OK) return st;
  if (M == 0) return QLIN_OK;
  if (!X || !codes || !chan_scale || !colsum || !Y || !workspace) return fail(QLIN_ERR_ARG, "a pointer argument is NULL");
  if (!aligned16(X) || !aligned16(codes) || !aligned16(chan_scale) || !aligned16(colsum) || !aligned16(Y))
    return fail(QLIN_ERR_ALIGN, "X/codes/chan_scale/colsum/Y is not 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return fail(QLIN_ERR_ALIGN, "workspace must be 256-byte aligned");
  const OffqLayout L = offq_layout(M, K, N, true);
  if (ws_bytes < L.total) return fail(QLIN_ERR_WORKSPACE, "workspace %zu < %zu", ws_bytes, L.total);
  char* ws = static_cast<char*>(workspace);
  int8_t* Xq = reinterpret_cast<int8_t*>(ws + L.xq);
  float* scale = reinterpret_cast<float*>(ws + L.scale);
  float* offset = reinterpret_cast<float*>(ws + L.offset);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  st = launch_offq_quant(X, M, K, sg, Xq, scale, offset, stream);
  if (st != QLIN_OK) return st;
  return launch_offq_gemm(Xq, scale, offset, M, K, N, codes, chan_scale, colsum, Y,
                          reinterpret_cast<uint8_t*>(ws + L.wide), stream);
}

qlin_status qlin_debug_set(int32_t k, int64_t value, int64_t* previous) {
  if (k < 0 || k > QLIN_KNOB_PAIR_SPLIT) return fail(QLIN_ERR_ARG, "unknown knob %d", k);
  bool ok = true;
  switch (k) {
    case QLIN_KNOB_PDL:
    case QLIN_KNOB_CLUSTER:
    case QLIN_KNOB_PAIR_SPLIT: ok = value == 0 || value == 1; break;
    case QLIN_KNOB_CLUSTER_SIZE: ok = value == 0 || value == 2 || value == 4 || value == 8; break;
    case QLIN_KNOB_MAX_TOKEN_TILE: ok = value == 64 || value == 128 || value == 256; break;
    case QLIN_KNOB_PAIR_MMA: ok = value >= 0 && value <= 2; break;
    default: ok = value >= 0;
  }
  if (!ok) return fail(QLIN_ERR_ARG, "invalid value %lld for knob %d", static_cast<long long>(value), k);
  if (k == QLIN_KNOB_WAIT_NS) {
    const unsigned long long v = static_cast<unsigned long long>(value);
    QLIN_CUDA_TRY(cudaMemcpyToSymbol(qlin::g_wait_ns, &v, sizeof(v)));
  }
  const long long old = g_knob[k].exchange(value);
  if (previous) *previous = old;
  return QLIN_OK;
}

qlin_status qlin_debug_get(int32_t k, int64_t* value) {
  if (k < 0 || k > QLIN_KNOB_PAIR_SPLIT || !value) return fail(QLIN_ERR_ARG, "unknown knob %d or NULL value", k);
  *value = g_knob[k].load();
  return QLIN_OK;
}

qlin_status qlin_poll_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "stream error: %s", cudaGetErrorString(e));
  int flag = 0;
  QLIN_CUDA_TRY(cudaMemcpyFromSymbol(&flag, qlin::g_device_error, sizeof(int)));
  if (flag) {
    const int zero = 0;
    QLIN_CUDA_TRY(cudaMemcpyToSymbol(qlin::g_device_error, &zero, sizeof(int)));
    return fail(QLIN_ERR_TIMEOUT, "a device-side bounded wait gave up (code %d)", flag);
  }
  return QLIN_OK;
}

}  // extern "C"
