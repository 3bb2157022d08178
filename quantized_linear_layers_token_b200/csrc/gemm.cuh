// gemm.cuh -- stages 2 and 3: INT8 tensor-core GEMM (tcgen05, TMEM
// accumulators, TMA-fed shared-memory operands) with the fused INT32->FP16
// dequant and the sparse outlier compensation.
//
// Orientation ("weights as the 128-row operand"): one CTA owns 128 output
// channels n (the MMA M dimension, TMEM lanes) and BT tokens m (the MMA N
// dimension, TMEM columns).  This keeps decode shapes (M = 1..16) on the
// tensor cores with an N = 16 instruction instead of padding tokens to 128.
//
// Warp roles (one CTA per tile):
//   warp 0        TMA producer: weight tile (INT8 codes, or packed INT4 into
//                 a staging buffer), g128 ratio row, activation tile; then the
//                 compensation operands (W_O^T tile, U tile).
//   warp 1        allocates TMEM; one lane issues tcgen05.mma and commits.
//   warps 2..     converters (INT4 formats): unpack the staged INT4 codes into
//                 the 128-byte-swizzled K-major INT8 operand (QQQ review,
//                 per-channel GEMM: INT4 -> INT8 by a left shift of 4;
//                 per-group GEMM: INT4 -> FP16, multiply by the folded ratio
//                 g/c, FP16 -> INT8 through the +128/+1024 bit trick done as
//                 one rounding), then the epilogue (first four warps).
// Epilogue (Quaff notes, decoupled WAQ formula; QQQ review, fused INT32->FP16
// dequant): Y = fp16(a_m * (c'_n * acc + comp)), comp accumulated in fp32 on
// the tensor cores from W_O^T and U = XqO * (s - 1) carried as two fp16
// terms (hi and lo), each its own run of K-steps into the same accumulator.
#pragma once

#include "sm100.cuh"

namespace qlin {

enum : int { kFmtW4PC = 0, kFmtW4G128 = 1, kFmtW8 = 2 };

struct GemmArgs {
  const float* cscale;  // c_n [N]
  const float* a;       // a_m [M]
  uint16_t* Y;          // [M][N] fp16
  int32_t* acc_debug;   // [M][N] or null
  int M, N, K, nO;
};

template <int FMT, int BT>
struct GemmCfg {
  static constexpr int kBN = 128;                    // output channels per CTA (MMA M)
  static constexpr int kBK = 128;                    // INT8 elements of K per stage (one swizzle row)
  static constexpr int kOffA = 0;                    // 128 x 128 B INT8 operand (or W_O^T tile)
  static constexpr int kOffB = 16384;                // BT x 128 B activation operand (or U tile)
  static constexpr int kOffStg = kOffB + BT * 128;   // 128 x 64 B packed INT4 staging
  static constexpr bool kW4 = FMT != kFmtW8;
  static constexpr int kOffR = kOffStg + (kW4 ? 8192 : 0);  // 128 fp16 ratios (g128)
  static constexpr int kRaw = kOffR + (FMT == kFmtW4G128 ? 256 : 0);
  static constexpr int kStageBytes = (kRaw + 1023) / 1024 * 1024;
  static constexpr int kSmemLimit = 232448;           // 227 KB per CTA
  static constexpr int kReserve = 1024 + 256;         // alignment slack + barriers
  static constexpr int kStagesFit = (kSmemLimit - kReserve) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kSmemBytes = kReserve + kStages * kStageBytes;
  static constexpr uint32_t kTxMain = (kW4 ? 8192 : 16384) + (FMT == kFmtW4G128 ? 256 : 0) + BT * 128;
  static constexpr uint32_t kTxComp = 16384 + BT * 128;
  static_assert(kStages >= 2, "tile does not fit in shared memory");
  static_assert(BT % 16 == 0 && BT >= 16 && BT <= 256, "MMA N must be 16..256 in steps of 16");
  static_assert(BT * 256 <= kStages * kStageBytes, "epilogue staging must fit in the stage buffers");
};

__device__ __forceinline__ uint32_t tmem_cols_for(int BT, bool comp) {
  const int need = comp ? 2 * BT : BT;
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(need)) c <<= 1;
  return c;
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

template <int FMT, int BT, int NCW>
__global__ void __launch_bounds__(64 + 32 * NCW, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
            const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmWO,
            const __grid_constant__ CUtensorMap tmU, const GemmArgs args) {
  using C = GemmCfg<FMT, BT>;
  constexpr int S = C::kStages;
  constexpr int kConvThreads = 32 * NCW;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* conv = full + S;
  uint64_t* empty = conv + S;
  uint64_t* accfull = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * C::kBN;
  const int m0 = blockIdx.y * BT;
  const int nk = (args.K + C::kBK - 1) / C::kBK;
  const int ncs = args.nO > 0 ? (args.nO + 63) / 64 : 0;  // 64-wide K-steps over the outliers
  const int nc = 2 * ncs;                                     // hi part, then lo part
  const uint32_t tcols = tmem_cols_for(BT, nc > 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&conv[s], kConvThreads);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accfull, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    if (FMT == kFmtW4G128) tma_prefetch_desc(&tmR);
    if (nc) {
      tma_prefetch_desc(&tmWO);
      tma_prefetch_desc(&tmU);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      int g = 0;
      for (; g < nk + nc; ++g) {
        const int s = g % S;
        const uint32_t r = static_cast<uint32_t>(g / S);
        if (g >= S && !mbar_wait(&empty[s], (r - 1) & 1u, abort_flag)) break;
        unsigned char* st = smem + s * C::kStageBytes;
        if (g < nk) {
          const int k0 = g * C::kBK;
          mbar_arrive_expect_tx(&full[s], C::kTxMain);
          if (FMT == kFmtW8) {
            tma_load_2d_hint(st + C::kOffA, &tmW, &full[s], k0, n0, pol_stream);
          } else {
            tma_load_2d_hint(st + C::kOffStg, &tmW, &full[s], k0 / 2, n0, pol_stream);
          }
          if (FMT == kFmtW4G128) tma_load_2d(st + C::kOffR, &tmR, &full[s], n0, g);
          tma_load_2d(st + C::kOffB, &tmX, &full[s], k0, m0);
        } else {
          const int j = g - nk;
          const int part = j >= ncs ? 1 : 0;  // U rows [0, M) hold hi, [M, 2M) hold lo
          const int i0 = (j - part * ncs) * 64;
          mbar_arrive_expect_tx(&full[s], C::kTxComp);
          tma_load_2d(st + C::kOffA, &tmWO, &full[s], i0, n0);
          tma_load_2d(st + C::kOffB, &tmU, &full[s], i0, part * args.M + m0);
        }
      }
      // Never leave with copies in flight: wait (bounded) for the last
      // stages this thread filled.
      for (int t = g - 1; t >= 0 && t >= g - S; --t) {
        const int s = t % S;
        if (!mbar_wait(&full[s], static_cast<uint32_t>(t / S) & 1u, abort_flag)) {
          // Fall back to a plain bounded wait that ignores the abort flag.
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s], static_cast<uint32_t>(t / S) & 1u) &&
                 globaltimer_ns() - t0 < QLIN_WAIT_NS) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_main = idesc_s8_s32(128, BT);
      constexpr uint32_t idesc_comp = idesc_f16_f32(128, BT);
      for (int g = 0; g < nk + nc; ++g) {
        const int s = g % S;
        const uint32_t r = static_cast<uint32_t>(g / S);
        uint64_t* wbar = (g < nk && C::kW4) ? &conv[s] : &full[s];
        if (!mbar_wait(wbar, r & 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * C::kStageBytes + C::kOffA);
        const uint32_t b_addr = smem_u32(smem + s * C::kStageBytes + C::kOffB);
        if (g < nk) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8(tmem, sdesc_k_sw128(a_addr + 32 * kk), sdesc_k_sw128(b_addr + 32 * kk), idesc_main,
                   (g > 0 || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem + BT, sdesc_k_sw128(a_addr + 32 * kk), sdesc_k_sw128(b_addr + 32 * kk), idesc_comp,
                    (g > nk || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      mma_commit(accfull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ converters
    const int ctid = threadIdx.x - 64;
    if (C::kW4) {
      for (int g = 0; g < nk; ++g) {
        const int s = g % S;
        const uint32_t r = static_cast<uint32_t>(g / S);
        if (!mbar_wait(&full[s], r & 1u, abort_flag)) break;
        unsigned char* st = smem + s * C::kStageBytes;
        const unsigned char* stg = st + C::kOffStg;
        unsigned char* A = st + C::kOffA;
        for (int c = ctid; c < 512; c += kConvThreads) {
          const int row = c >> 2;
          const int part = c & 3;
          const uint4 w = *reinterpret_cast<const uint4*>(stg + c * 16);
          uint4 o0, o1;
          if (FMT == kFmtW4PC) {
            unpack_w4pc(w, o0, o1);
          } else {
            const uint16_t rb = reinterpret_cast<const uint16_t*>(st + C::kOffR)[row];
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
        fence_proxy_async_smem();
        mbar_arrive(&conv[s]);
      }
    }
    // ------------------------------------------------------------ epilogue
    if (warp < 6) {
      const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
      const int nl = quad * 32 + lane;
      const int n = n0 + nl;
      bool ok = mbar_wait(accfull, 0, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const float cn = n < args.N ? (FMT == kFmtW4PC ? __fmul_rn(args.cscale[n], 0.0625f) : args.cscale[n]) : 0.f;
      __half* Ys = reinterpret_cast<__half*>(smem);
      const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BT; c0 += 16) {
        uint32_t acc[16], cmp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) { acc[j] = 0u; cmp[j] = 0u; }
        if (ok) {
          tmem_ld16(trow + c0, acc);
          if (nc) tmem_ld16(trow + BT + c0, cmp);
          tmem_ld_wait();
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = m0 + c0 + j;
          const float am = m < args.M ? args.a[m] : 0.f;
          float v = __fmul_rn(cn, static_cast<float>(static_cast<int32_t>(acc[j])));
          if (nc) v = __fadd_rn(v, __uint_as_float(cmp[j]));
          Ys[(c0 + j) * 128 + nl] = __float2half_rn(__fmul_rn(am, v));
          if (args.acc_debug && m < args.M && n < args.N)
            args.acc_debug[static_cast<size_t>(m) * args.N + n] = static_cast<int32_t>(acc[j]);
        }
      }
      named_bar_sync(1, 128);
      const int et = threadIdx.x - 64;
      for (int idx = et; idx < BT * 16; idx += 128) {
        const int row = idx >> 4;
        const int ch = idx & 15;
        const int m = m0 + row;
        const int n8 = n0 + ch * 8;
        if (m < args.M && n8 < args.N)
          *reinterpret_cast<uint4*>(args.Y + static_cast<size_t>(m) * args.N + n8) =
              *reinterpret_cast<const uint4*>(Ys + row * 128 + ch * 8);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

}  // namespace qlin
