// offq.cuh -- OffQ: structured activation outliers absorbed as a per-group
// offset, W4A4 with per-group asymmetric activations.
//
// "OffQ: Taming Structured Outliers in LLM Quantization by Offsetting"
// (technical summary, 方法论: 通过偏移量进行吸收 (Hadamard 旋转) and the
// grouped implementation that follows it): once the offline top-1 PCA step
// has moved the outlier energy of a group of channels into one channel, a
// Hadamard rotation whose first row is all ones turns that channel's value
// into one constant added to every channel of the group; the constant is
// taken up by the offset of a per-group asymmetric low-bit quantizer, and
// the weights carry the inverse rotation so the product is unchanged before
// quantization.
//
// Readings (the summaries fix no precision, normalisation or offset rule):
//   groups of 128 consecutive channels; D H with H the 128 x 128 Sylvester
//   matrix h(i,j) = (-1)^popcount(i & j) and D = diag(d), d_0 = +1 and
//   d_i = +-1 given (so row 0 of D H is all ones);
//   y_g = x_g D H per token and group, unnormalised, in fp64;
//   lo = min y_g, hi = max y_g, sd = (hi - lo) / 15,
//   q = clamp(rne((y - lo) / sd), 0, 15) in fp64 (q = 0 when sd == 0);
//   stored: q (one byte), fp32(sd), fp32(lo);
//   W'_g = (1/128) H D W_g in fp64, then fp32; INT4 per output channel:
//   c_n = max_k |W'[k][n]| / 7, q_w = clamp(rne(W' * (7 / max)), -7, 7) (fp32);
//   y[m][n] = (c_n / 16) sum_g ( sd[m][g] acc_g[m][n] + lo[m][g] colsum_g[n] ),
//   acc_g = sum_{k in g} q[m][k] * 16 q_w[k][n] and colsum_g = sum_{k in g} 16 q_w[k][n].
//
// Exactness of the transform: an fp16 value is an integer multiple of 2^-24
// below 2^16 in magnitude, so a signed sum of up to 128 of them is a
// multiple of 2^-24 below 2^23: at most 47 significant bits.  Every partial
// sum of the fast Walsh-Hadamard butterflies is therefore exact in fp64, and
// the butterfly order gives the bits of any other summation order.
//
// Kernels:
//   offq_quant_kernel    four threads per (token, group), 32 channels each:
//                        signs, in-thread butterflies over strides 1..16,
//                        two shuffle stages for strides 32 and 64, group
//                        min/max, codes.  The quotient (y - lo) / sd is taken
//                        as (y - lo) * (1 / sd) and rounded; only when that
//                        lands within 2^-40 of a half-integer (the two can
//                        then round apart) is the correctly rounded division
//                        done, so every code is rne of the fp64 quotient.
//   offq_rotate_kernel   weights: one CTA per 32 columns of one group, the
//                        128 x 32 block in shared memory as fp64 butterflies.
//   offq_pack_kernel     per-channel INT4 of the rotated weights into the
//                        packed W4 tile layout, plus the per-group column sums.
//   offq_gemm_kernel     per 128-token x 128-channel tile, one INT8 tensor-core
//                        product per 128-wide K-block into its own tensor-memory
//                        accumulator (four in flight); the epilogue promotes
//                        each block with the group's token scale and offset
//                        into fp32 registers, then applies c_n / 16 (eight
//                        epilogue warps of 64 columns, read as two halves
//                        whose loads overlap the other half's promotion).
//                        Each epilogue warp streams its column sums per block
//                        through a private three-slot cp.async ring and
//                        loads the token scales and offsets two blocks ahead,
//                        so no promotion waits on a global load.
#pragma once

#include "gemm.cuh"

namespace qlin {

__device__ __forceinline__ uint32_t sign_word(const uint4& s, int w) {
  return w == 0 ? s.x : (w == 1 ? s.y : (w == 2 ? s.z : s.w));
}

// ------------------------------------------------------------------ activations
constexpr int kOffqQuantThreads = 256;  // 64 (token, group) units of four threads

__global__ void __launch_bounds__(kOffqQuantThreads)
offq_quant_kernel(const uint16_t* __restrict__ X, int M, int K, uint4 sgn, int8_t* __restrict__ Xq,
                  float* __restrict__ scale, float* __restrict__ offset) {
  griddep_launch_dependents();
  const int G = K >> 7;
  const long long unit = static_cast<long long>(blockIdx.x) * (kOffqQuantThreads / 4) + (threadIdx.x >> 2);
  const int part = threadIdx.x & 3;  // channels 32*part .. +31 of the group
  const bool live = unit < static_cast<long long>(M) * G;
  const long long m = live ? unit / G : 0;
  const int g = live ? static_cast<int>(unit - m * G) : 0;
  const size_t base = static_cast<size_t>(m) * K + static_cast<size_t>(g) * 128 + part * 32;
  griddep_wait();  // X may come from the previous kernel; Xq may still be read by it
  uint4 raw[4];
#pragma unroll
  for (int c = 0; c < 4; ++c)
    raw[c] = live ? __ldg(reinterpret_cast<const uint4*>(X + base) + c) : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t sb = sign_word(sgn, part);
  double v[32];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t wd[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int j = 8 * c + e;
      uint16_t h = static_cast<uint16_t>(wd[e >> 1] >> (16 * (e & 1)));
      h ^= static_cast<uint16_t>(((sb >> j) & 1u) << 15);
      v[j] = static_cast<double>(__half2float(__ushort_as_half(h)));
    }
  }
#pragma unroll
  for (int h = 1; h < 32; h <<= 1)
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (!(j & h)) {
        const double a = v[j], b = v[j + h];
        v[j] = __dadd_rn(a, b);
        v[j + h] = __dsub_rn(a, b);
      }
#pragma unroll
  for (int s = 1; s <= 2; s <<= 1)
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const double o = __shfl_xor_sync(0xffffffffu, v[j], s);
      v[j] = (part & s) ? __dsub_rn(o, v[j]) : __dadd_rn(v[j], o);
    }
  double lo = v[0], hi = v[0];
#pragma unroll
  for (int j = 1; j < 32; ++j) {
    lo = v[j] < lo ? v[j] : lo;
    hi = v[j] > hi ? v[j] : hi;
  }
#pragma unroll
  for (int s = 1; s <= 2; s <<= 1) {
    const double ol = __shfl_xor_sync(0xffffffffu, lo, s), oh = __shfl_xor_sync(0xffffffffu, hi, s);
    lo = ol < lo ? ol : lo;
    hi = oh > hi ? oh : hi;
  }
  const double sd = __ddiv_rn(__dsub_rn(hi, lo), 15.0);
  if (live && part == 0) {
    scale[unit] = __double2float_rn(sd);
    offset[unit] = __double2float_rn(lo);
  }
  uint32_t out[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  if (sd > 0.0) {
    const double inv = __drcp_rn(sd);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const double t = __dsub_rn(v[j], lo);  // exact: both are multiples of 2^-24 below 2^23
      double r = __dmul_rn(t, inv);
      const double f = __dsub_rn(__dsub_rn(r, floor(r)), 0.5);
      if (fabs(f) < 0x1p-40) r = __ddiv_rn(t, sd);
      int q = __double2int_rn(r);
      q = q < 0 ? 0 : (q > 15 ? 15 : q);
      out[j >> 2] |= static_cast<uint32_t>(q) << (8 * (j & 3));
    }
  }
  if (live) {
    uint4* dst = reinterpret_cast<uint4*>(Xq + base);
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  }
}

// ------------------------------------------------------------------ weights
// Wr[g*128 + j][n] = fp32((1/128) sum_i h(j,i) d_i W[g*128 + i][n]).
// grid (ceil(N / 32), K / 128), 256 threads.
__global__ void __launch_bounds__(256)
offq_rotate_kernel(const uint16_t* __restrict__ W, int K, int N, uint4 sgn, float* __restrict__ Wr) {
  __shared__ double s[128][33];
  const int g = blockIdx.y;
  const int c = threadIdx.x & 31;
  const int r0 = threadIdx.x >> 5;
  const int n = blockIdx.x * 32 + c;
  for (int i = r0; i < 128; i += 8) {
    double x = 0.0;
    if (n < N) {
      x = static_cast<double>(__half2float(__ushort_as_half(W[static_cast<size_t>(g * 128 + i) * N + n])));
      if ((sign_word(sgn, i >> 5) >> (i & 31)) & 1u) x = -x;
    }
    s[i][c] = x;
  }
  __syncthreads();
  for (int h = 1; h < 128; h <<= 1) {
    for (int p = r0; p < 64; p += 8) {
      const int i0 = (p / h) * 2 * h + (p % h);
      const int i1 = i0 + h;
      const double a = s[i0][c], b = s[i1][c];
      s[i0][c] = __dadd_rn(a, b);
      s[i1][c] = __dsub_rn(a, b);
    }
    __syncthreads();
  }
  if (n < N)
    for (int j = r0; j < 128; j += 8)
      Wr[static_cast<size_t>(g * 128 + j) * N + n] = __double2float_rn(__dmul_rn(s[j][c], 0.0078125));
}

// Per-output-channel INT4 of the rotated fp32 weights (one thread per
// channel; codes into the packed W4 tiles, whose padding the caller
// clears), c_n, and colsum[g][n] = sum over group g of 16 q.
__global__ void offq_pack_kernel(const float* __restrict__ Wr, int K, int N, uint8_t* __restrict__ codes,
                                 float* __restrict__ cscale, float* __restrict__ colsum) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float wmax = 0.f;
  for (int k = 0; k < K; ++k) {
    const float v = fabsf(Wr[static_cast<size_t>(k) * N + n]);
    wmax = v > wmax ? v : wmax;
  }
  cscale[n] = __fdiv_rn(wmax, 7.f);
  const float inv = wmax > 0.f ? __fdiv_rn(7.f, wmax) : 0.f;
  const int KB = K >> 7;
  for (int g = 0; g < KB; ++g) {
    int cs = 0;
    for (int k0 = g * 128; k0 < g * 128 + 128; k0 += 8) {
      int q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        q[j] = rne_clamp(__fmul_rn(Wr[static_cast<size_t>(k0 + j) * N + n], inv), 7);
        cs += q[j];
      }
      *reinterpret_cast<uint32_t*>(codes + w4_tile_offset(n, k0, KB)) = pack8_nibbles(q);
    }
    colsum[static_cast<size_t>(g) * N + n] = static_cast<float>(16 * cs);
  }
}

// ------------------------------------------------------------------ GEMM
constexpr int kOffqStages = 6;
constexpr int kOffqStage = 32768;  // 16 KB token rows (A) + 16 KB weight rows (B)
constexpr int kOffqAccBufs = 4;    // 128-column accumulators in tensor memory
constexpr int kOffqEpiWarps = 8;  // two per TMEM lane quarter, 64 columns each
constexpr int kOffqCols = 128 / (kOffqEpiWarps / 4);
constexpr int kOffqThreads = 32 * (2 + kOffqEpiWarps);
constexpr int kOffqCsSlots = 3;  // per epilogue warp: column sums of 64 channels per K-block
constexpr int kOffqOffCs = kOffqStages * kOffqStage;
constexpr int kOffqOffBar = kOffqOffCs + kOffqEpiWarps * kOffqCsSlots * kOffqCols * 4;
constexpr int kOffqSmem = kOffqOffBar + 256 + 1024;  // barriers + alignment slack

struct OffqArgs {
  const float* scale;    // sd [M][G]
  const float* offset;   // lo [M][G]
  const float* colsum;   // [G][N]
  const float* cscale;   // c_n [N]
  const uint8_t* wide;   // 16 q as INT8 blocks of 128 channels x 128 inputs (16 KiB, swizzled), tn-major
  uint16_t* Y;           // fp16 [M][N]
  int M, N, G;
  int tiles_m, tiles;
};

// sum[J0 + j] += sd * acc[j] + lo * colsum[j] for 32 columns (fp32, the
// offset term first, both fused multiply-adds rounded once).
template <int J0>
__device__ __forceinline__ void offq_promote(const uint32_t (&v)[32], float (&sum)[64], float sd, float lo,
                                             const float4* cs4) {
#pragma unroll
  for (int j4 = 0; j4 < 8; ++j4) {
    const float4 c4 = cs4[j4];
    const float cs[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * j4 + e;
      sum[J0 + j] = __fmaf_rn(sd, __int2float_rn(static_cast<int>(v[j])), __fmaf_rn(lo, cs[e], sum[J0 + j]));
    }
  }
}

struct alignas(64) OffqParams {
  CUtensorMap tmX;  // q int8 [M][K], 128 x 128 boxes, 128-byte swizzle
  OffqArgs g;
};

__global__ void __launch_bounds__(kOffqThreads, 1) offq_gemm_kernel(const __grid_constant__ OffqParams prm) {
  const OffqArgs& g = prm.g;
  constexpr int S = kOffqStages;
  constexpr int B = kOffqAccBufs;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffqOffBar);  // [S]
  uint64_t* empty = full + S;                                         // [S]
  uint64_t* acc_full = empty + S;                                     // [B]
  uint64_t* acc_empty = acc_full + B;                                 // [B]
  uint64_t* mma_done = acc_empty + B;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < B; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kOffqEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 1) tma_prefetch_desc(&prm.tmX);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      griddep_wait();  // q, the widened weights and the scales come from the previous kernels
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < g.tiles; t += gridDim.x) {
        const int tm = t % g.tiles_m, tn = t / g.tiles_m;
        for (int kb = 0; kb < g.G; ++kb, ++it) {
          const int s = it % S;
          if (it >= S && !mbar_wait(&empty[s], static_cast<uint32_t>(it / S - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kOffqStage);
          unsigned char* A = smem + s * kOffqStage;
          tma_load_2d(A, &prm.tmX, &full[s], kb * 128, tm * 128);
          bulk_load(A + 16384, g.wide + (static_cast<size_t>(tn) * g.G + kb) * 16384, 16384, &full[s]);
        }
      }
      drain_ring(full, S, it);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and its waits; an elected lane issues.
    {
      constexpr uint32_t idesc = idesc_s8_s32(128, 128);
      const uint64_t adesc0 = sdesc_k_sw128(smem_u32(smem));
      const uint64_t bdesc0 = sdesc_k_sw128(smem_u32(smem + 16384));
      int it = 0;
      bool ok = true, issued = false;
      for (int t = blockIdx.x; ok && t < g.tiles; t += gridDim.x) {
        for (int kb = 0; kb < g.G; ++kb, ++it) {
          const int s = it % S, b = it % B;
          if (it >= B && !warp_wait(&acc_empty[b], static_cast<uint32_t>(it / B - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (!warp_wait(&full[s], static_cast<uint32_t>(it / S) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issued = true;
          const uint64_t ad = adesc0 + static_cast<uint64_t>(s * (kOffqStage >> 4));
          const uint64_t bd = bdesc0 + static_cast<uint64_t>(s * (kOffqStage >> 4));
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_i8(tmem + 128u * b, ad + 2 * k, bd + 2 * k, idesc, k > 0 ? 1u : 0u);
            mma_commit(&empty[s]);
            mma_commit(&acc_full[b]);
          }
          __syncwarp();
        }
      }
      if (issued) {  // every tensor-core op has completed before tensor memory is freed
        if (elect_one()) mma_commit(mma_done);
        __syncwarp();
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(mma_done, 0u, 1000000u) && globaltimer_ns() - t0 < QLIN_DRAIN_NS) {
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Per K-block the two 32-column halves of this warp's accumulator slice
    // are read alternately with their promotion: the load of one half (or of
    // the next block's first half) is in flight while the other is promoted.
    static_assert(kOffqCols == 64, "the epilogue reads 64 columns as two halves");
    const int ep = warp - 2;
    const int part = ep >> 2;          // columns 64*part .. +63 of each accumulator
    const int quad = warp & 3;         // tensor-memory lanes 32*quad .. +31
    const int row = quad * 32 + lane;  // token within the tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(part * 64);
    float* csr = reinterpret_cast<float*>(smem + kOffqOffCs + ep * kOffqCsSlots * 256);  // this warp's ring
    griddep_wait();
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < g.tiles; t += gridDim.x) {
      const int tm = t % g.tiles_m, tn = t / g.tiles_m;
      const int m = tm * 128 + row;
      const bool mv = m < g.M;
      const int nb = tn * 128 + part * 64;
      // column sums of K-block kb into ring slot kb % 3: 16 lanes x 16 bytes
      // (a lane past N reads an in-range chunk; those columns are not stored)
      const float* csrc = g.colsum + min(nb + 4 * (lane & 15), g.N - 4);
      if (lane < 16) cp_async16(csr + 4 * lane, csrc);
      cp_async_commit();
      if (lane < 16 && g.G > 1) cp_async16(csr + 64 + 4 * lane, csrc + g.N);
      cp_async_commit();
      const float* sdp = g.scale + static_cast<size_t>(mv ? m : 0) * g.G;
      const float* lop = g.offset + static_cast<size_t>(mv ? m : 0) * g.G;
      float sum[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) sum[j] = 0.f;
      // token scale and offset two K-blocks ahead
      float sd1 = mv ? __ldg(sdp) : 0.f, lo1 = mv ? __ldg(lop) : 0.f;
      float sd2 = (mv && g.G > 1) ? __ldg(sdp + 1) : 0.f, lo2 = (mv && g.G > 1) ? __ldg(lop + 1) : 0.f;
      uint32_t v0[32], v1[32];
      {
        const int b = it % B;
        ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[b], static_cast<uint32_t>(it / B) & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        tmem_ld32(trow + 128u * b, v0);
        tmem_ld_wait();
      }
      for (int kb = 0; kb < g.G; ++kb, ++it) {
        const int b = it % B;
        const float sd = sd1, lo = lo1;
        sd1 = sd2;
        lo1 = lo2;
        if (mv && kb + 2 < g.G) {
          sd2 = __ldg(sdp + kb + 2);
          lo2 = __ldg(lop + kb + 2);
        }
        if (lane < 16 && kb + 2 < g.G)
          cp_async16(csr + ((kb + 2) % kOffqCsSlots) * 64 + 4 * lane, csrc + static_cast<size_t>(kb + 2) * g.N);
        cp_async_commit();
        tmem_ld32(trow + 128u * b + 32u, v1);  // second half of this block
        cp_async_wait_group<2>();              // this block's column sums have landed
        __syncwarp();
        const float4* cs4 = reinterpret_cast<const float4*>(csr + (kb % kOffqCsSlots) * 64);
        offq_promote<0>(v0, sum, sd, lo, cs4);
        tmem_ld_wait();  // the block is read: release its accumulator
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
        const bool more = kb + 1 < g.G;
        if (more) {
          const int b1 = (it + 1) % B;
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&acc_full[b1], static_cast<uint32_t>((it + 1) / B) & 1u, abort_flag));
          if (ok) {
            tc_fence_after();
            tmem_ld32(trow + 128u * b1, v0);  // the next block's first half
          }
        }
        offq_promote<32>(v1, sum, sd, lo, cs4 + 8);
        if (more && ok) tmem_ld_wait();
        __syncwarp();  // every lane has read the ring slot before it is refilled
        if (!ok) break;
      }
      cp_async_wait_all();
      __syncwarp();
      if (!ok) break;
      if (mv) {
#pragma unroll
        for (int j8 = 0; j8 < 8; ++j8) {
          const int n = nb + 8 * j8;
          if (n < g.N) {
            const float4 c0 = __ldg(reinterpret_cast<const float4*>(g.cscale + n));
            const float4 c1 = __ldg(reinterpret_cast<const float4*>(g.cscale + n) + 1);
            const float cnv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint32_t h[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float y0 = __fmul_rn(__fmul_rn(cnv[2 * e], 0.0625f), sum[8 * j8 + 2 * e]);
              const float y1 = __fmul_rn(__fmul_rn(cnv[2 * e + 1], 0.0625f), sum[8 * j8 + 2 * e + 1]);
              h[e] = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(y0))) |
                     (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(y1))) << 16);
            }
            *reinterpret_cast<uint4*>(g.Y + static_cast<size_t>(m) * g.N + n) = make_uint4(h[0], h[1], h[2], h[3]);
          }
        }
      }
    }
    cp_async_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace qlin
