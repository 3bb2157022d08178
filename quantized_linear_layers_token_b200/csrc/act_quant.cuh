// act_quant.cuh -- stage 1: targeted momentum scaling on the outlier
// channels and per-token symmetric INT8 quantization.
//
// Quaff notes, 目标动量缩放: for i in O,
//   beta_i = max(1, sqrt(max_m |X[m,O_i]| / max_n |W[O_i,n]|)),
//   s_i   <- gamma * s_i + (1 - gamma) * beta_i;
// channels outside O keep s = 1, so only |O| values are ever touched.
// The activations the integer GEMM sees are X_hat = X (/) s, quantized per
// token with a symmetric INT8 scale a_m = max_k |x_hat[m,k]| / 127 (QQQ
// review: symmetric activation quantization).
//
// Kernels:
//   colmax_kernel   grid over row blocks; per-CTA maxima of |X[:,O]| in
//                   shared memory, merged with one global atomicMax per
//                   column; with `update` set, the last CTA to finish (a
//                   completion counter, no spinning) applies the momentum
//                   recurrence to s in place and clears its scratch.
//   quant_kernel    one CTA per token: 128-bit loads of the row staged in
//                   shared memory, fp16 |x| row max, RNE codes, 64-bit
//                   stores, outlier codes patched in afterwards; also
//                   emits the compact outlier codes XqO and, when asked, the
//                   fp16 compensation operand U = XqO * (s - 1) as hi + lo.
#pragma once

#include "pack.cuh"

namespace qlin {

constexpr int kColmaxRows = 32;   // rows per CTA of colmax_kernel
constexpr int kQuantThreads = 512;
constexpr int kFusedMomentumMaxM = 64;  // up to this many tokens the update runs inside quant_kernel


__device__ __forceinline__ __half2 u32_as_half2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

__device__ __forceinline__ float block_max(float v, float* red /* >= kQuantThreads / 32 floats */) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) r = fmaxf(r, red[w]);
  return r;
}

// Momentum recurrence in fp32, exactly this association (no contraction).
__device__ __forceinline__ float momentum_step(float s, float gamma, float cmax, float wmax) {
  float beta = 1.f;
  if (wmax > 0.f) {
    const float r = __fsqrt_rn(__fdiv_rn(cmax, wmax));
    beta = r > 1.f ? r : 1.f;
  }
  return __fadd_rn(__fmul_rn(gamma, s), __fmul_rn(__fsub_rn(1.f, gamma), beta));
}

// cmax_bits: fp32 bit patterns of non-negative maxima (ordered like uints).
// With update != 0 the scratch (cmax_bits, counter) must be zero on entry
// and is zero again on exit.
__global__ void colmax_kernel(const uint16_t* __restrict__ X, int M, int K, const int32_t* __restrict__ O,
                              int nO, unsigned* __restrict__ cmax_bits, int update,
                              const float* __restrict__ wmaxO, float* __restrict__ s, float gamma,
                              unsigned* __restrict__ counter) {
  extern __shared__ unsigned char colmax_smem[];
  int* sO = reinterpret_cast<int*>(colmax_smem);
  unsigned* scm = reinterpret_cast<unsigned*>(sO + nO);
  __shared__ int is_last;
  griddep_launch_dependents();
  griddep_wait();
  for (int i = threadIdx.x; i < nO; i += blockDim.x) {
    sO[i] = O[i];
    scm[i] = 0u;
  }
  __syncthreads();
  const int r0 = blockIdx.x * kColmaxRows;
  const int r1 = min(M, r0 + kColmaxRows);
  const int total = (r1 - r0) * nO;
  // eight independent gathers per thread in flight before the merges
  const int stride = static_cast<int>(blockDim.x);
  for (int idx0 = threadIdx.x; idx0 < total; idx0 += 8 * stride) {
    uint16_t hv[8];
    int ii[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int idx = idx0 + u * stride;
      ii[u] = -1;
      hv[u] = 0;
      if (idx < total) {
        const int r = idx / nO;
        const int i = idx - r * nO;
        ii[u] = i;
        hv[u] = X[static_cast<size_t>(r0 + r) * K + sO[i]];
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (ii[u] >= 0) atomicMax(&scm[ii[u]], __float_as_uint(fabsf(h2f(hv[u]))));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nO; i += blockDim.x)
    if (scm[i]) atomicMax(&cmax_bits[i], scm[i]);
  if (!update) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(counter, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int i = threadIdx.x; i < nO; i += blockDim.x) {
    const float cm = __uint_as_float(atomicExch(&cmax_bits[i], 0u));
    s[i] = momentum_step(s[i], gamma, cm, wmaxO[i]);
  }
  if (threadIdx.x == 0) *counter = 0u;
}

// Apply the recurrence from externally reduced maxima (data-parallel use).
__global__ void momentum_kernel(const float* __restrict__ cmax, const float* __restrict__ wmaxO,
                                float* __restrict__ s, float gamma, int nO) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < nO) s[i] = momentum_step(s[i], gamma, cmax[i], wmaxO[i]);
}

__device__ __forceinline__ int lower_bound_sorted(const int* a, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ int quant_code(float xh, float inv) {
  return rne_clamp(__fmul_rn(xh, inv), 127);
}

// Compensation operand for one (token, outlier) pair: u = q * (s - 1) in
// fp32, carried as hi = fp16(u) and lo = fp16(u - hi) (u - hi is exact in
// fp32), so hi + lo matches u to about 2^-22 relative.  A single fp16
// rounding of u is not accurate enough for the 2e-3 output tolerance when
// the outlier terms cancel.
__device__ __forceinline__ uint2 comp_split(int q, float s) {
  const float u = __fmul_rn(static_cast<float>(q), __fsub_rn(s, 1.f));
  const __half hi = __float2half_rn(u);
  const __half lo = __float2half_rn(__fsub_rn(u, __half2float(hi)));
  return make_uint2(__half_as_ushort(hi), __half_as_ushort(lo));
}

// One quantization problem (a layer's activations at M tokens).  A launch
// quantizes one problem or a group of independent problems
// (qlin_forward_grouped); CTA b works on row b - row0 of the problem whose
// rows [row0, row0 + M) contain it.
struct QuantProb {
  const uint16_t* X;     // [M][K] fp16
  const int32_t* O;      // [nO]
  float* s;              // [nO] momentum state
  int8_t* Xq;            // [M][K]
  float* a;              // [M]
  int8_t* XqO;           // [M][nO]
  uint16_t* U;           // [2][M][nOp] compensation operand (hi rows, then lo rows), or null
  const float* wmaxO;    // [nO]
  unsigned* counter;     // completion counter of the fused update (zero on entry, left zero)
  int K, nO, nOp, M, row0;
};

template <int MAXP>
struct QuantGroup {
  float gamma;
  int nprob;
  QuantProb pr[MAXP];
};

// One CTA per token row.  VPT = 8-element vectors per thread
// (K <= 8 * kQuantThreads * VPT).
// FUSED: every CTA also computes the outlier column maxima over all M rows
// of its problem and the momentum update itself (identical in every CTA,
// cheap for small M); the last CTA of the problem to finish writes the new
// state back, after every CTA has read the old one.
// The row is staged in shared memory; the outlier columns' raw values are
// set aside and their slots zeroed, so the row maximum (fp16 |x| maxima,
// exact) and the quantization pass run without per-element outlier checks;
// the outlier codes x_hat = x / s are computed separately and written over
// the zeros after a barrier.  O and max|W_O| do not depend on the previous
// kernel and are read before the grid dependency.
template <int VPT, bool FUSED, int MAXP>
__global__ void __launch_bounds__(kQuantThreads)
quant_kernel(const __grid_constant__ QuantGroup<MAXP> qg) {
  extern __shared__ __align__(16) unsigned char quant_smem[];
  __shared__ float red[kQuantThreads / 32];
  __shared__ int is_last;
  int pi = 0;
  if (MAXP > 1)
    while (pi + 1 < qg.nprob && static_cast<int>(blockIdx.x) >= qg.pr[pi + 1].row0) ++pi;
  const QuantProb& qp = qg.pr[pi];
  const uint16_t* __restrict__ X = qp.X;
  const int K = qp.K, nO = qp.nO, nOp = qp.nOp, M = qp.M;
  const int32_t* __restrict__ O = qp.O;
  float* __restrict__ s = qp.s;
  int8_t* __restrict__ XqO = qp.XqO;
  uint16_t* __restrict__ U = qp.U;
  uint16_t* xs = reinterpret_cast<uint16_t*>(quant_smem);          // [K] this row (outliers zeroed)
  int* sO = reinterpret_cast<int*>(quant_smem + static_cast<size_t>(K) * 2);
  float* sS = reinterpret_cast<float*>(sO + nO);                    // [nO] momentum state
  float* xo = sS + nO;                                              // [nO] raw outlier values of this row
  unsigned* cmx = reinterpret_cast<unsigned*>(xo + nO);             // [nO] fused column maxima (fp32 bits)

  griddep_launch_dependents();
  for (int i = threadIdx.x; i < nO; i += kQuantThreads) {
    sO[i] = O[i];
    if (FUSED) cmx[i] = 0u;
  }
  float wmx = 0.f;  // max|W_O| of outlier threadIdx.x (FUSED, nO <= kQuantThreads handled in the loop below)
  if (FUSED && static_cast<int>(threadIdx.x) < nO) wmx = qp.wmaxO[threadIdx.x];
  griddep_wait();  // X (and s) may come from the previous kernel
  const int m = static_cast<int>(blockIdx.x) - qp.row0;
  const uint4* xv = reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K);
  const int nvec = K >> 3;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int vi = threadIdx.x + j * kQuantThreads;
    if (vi < nvec) reinterpret_cast<uint4*>(xs)[vi] = __ldg(xv + vi);
  }
  for (int i = threadIdx.x; i < nO; i += kQuantThreads) sS[i] = s[i];
  __syncthreads();
  // set the outliers aside (each thread owns distinct columns)
  for (int i = threadIdx.x; i < nO; i += kQuantThreads) {
    const int col = sO[i];
    xo[i] = h2f(xs[col]);
    xs[col] = 0;
  }
  if (FUSED) {
    // column maxima of |X[:, O]| over all M rows: the M * nO gathers are
    // spread over the whole CTA, eight independent loads per thread in
    // flight, merged with shared-memory atomicMax on the fp32 bit patterns
    // (non-negative, so ordered like unsigned integers)
    const int pairs = M * nO;
    for (int p0 = threadIdx.x; p0 < pairs; p0 += 8 * kQuantThreads) {
      uint16_t hv[8];
      int ii[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int p = p0 + u * kQuantThreads;
        ii[u] = -1;
        hv[u] = 0;
        if (p < pairs) {
          const int r = p / nO;
          const int i = p - r * nO;
          ii[u] = i;
          hv[u] = X[static_cast<size_t>(r) * K + sO[i]];
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (ii[u] >= 0) atomicMax(&cmx[ii[u]], __float_as_uint(fabsf(h2f(hv[u]))));
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nO; i += kQuantThreads)
      sS[i] = momentum_step(sS[i], qg.gamma, __uint_as_float(cmx[i]),
                            i == static_cast<int>(threadIdx.x) ? wmx : qp.wmaxO[i]);
  }
  __syncthreads();

  // row maximum: fp16 |x| maxima of the staged row (exact), then the
  // outliers' |x / s| in fp32
  __half2 hm = __float2half2_rn(0.f);
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int vi = threadIdx.x + j * kQuantThreads;
    if (vi < nvec) {
      const uint4 w = reinterpret_cast<const uint4*>(xs)[vi];
      const __half2 m01 = __hmax2(__habs2(u32_as_half2(w.x)), __habs2(u32_as_half2(w.y)));
      const __half2 m23 = __hmax2(__habs2(u32_as_half2(w.z)), __habs2(u32_as_half2(w.w)));
      hm = __hmax2(hm, __hmax2(m01, m23));
    }
  }
  float lmax = fmaxf(__low2float(hm), __high2float(hm));
  for (int i = threadIdx.x; i < nO; i += kQuantThreads) {
    const float f = fabsf(__fdiv_rn(xo[i], sS[i]));
    lmax = f > lmax ? f : lmax;
  }
  const float amax = block_max(lmax, red);
  const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
  if (threadIdx.x == 0) qp.a[m] = __fdiv_rn(amax, 127.f);

  int8_t* qrow = qp.Xq + static_cast<size_t>(m) * K;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int vi = threadIdx.x + j * kQuantThreads;
    if (vi < nvec) {
      const uint4 w = reinterpret_cast<const uint4*>(xs)[vi];
      const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
      int q[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(u32_as_half2(w4[e]));
        q[2 * e] = quant_code(f.x, inv);
        q[2 * e + 1] = quant_code(f.y, inv);
      }
      *reinterpret_cast<uint2*>(qrow + static_cast<size_t>(vi) * 8) = pack8_bytes(q);
    }
  }
  __syncthreads();  // the zero codes at the outlier columns are written before the patch below
  const size_t lo_off = static_cast<size_t>(M) * nOp;  // U holds [2][M][nOp]: hi rows, then lo rows
  for (int i = threadIdx.x; i < nOp; i += kQuantThreads) {
    if (i < nO) {
      const float xh = __fdiv_rn(xo[i], sS[i]);
      const int q = quant_code(xh, inv);
      qrow[sO[i]] = static_cast<int8_t>(q);
      XqO[static_cast<size_t>(m) * nO + i] = static_cast<int8_t>(q);
      if (U) {
        const uint2 hl = comp_split(q, sS[i]);
        U[static_cast<size_t>(m) * nOp + i] = static_cast<uint16_t>(hl.x);
        U[lo_off + static_cast<size_t>(m) * nOp + i] = static_cast<uint16_t>(hl.y);
      }
    } else if (U) {
      U[static_cast<size_t>(m) * nOp + i] = 0;
      U[lo_off + static_cast<size_t>(m) * nOp + i] = 0;
    }
  }
  if (FUSED && nO > 0) {
    if (M == 1) {  // the only reader of the old state
      for (int i = threadIdx.x; i < nO; i += kQuantThreads) s[i] = sS[i];
    } else {
      __syncthreads();
      if (threadIdx.x == 0) is_last = (atomicAdd(qp.counter, 1u) == static_cast<unsigned>(M - 1));
      __syncthreads();
      if (is_last) {
        for (int i = threadIdx.x; i < nO; i += kQuantThreads) s[i] = sS[i];
        if (threadIdx.x == 0) *qp.counter = 0u;
      }
    }
  }
}

// Compensation operand from already quantized outlier codes (qlin_gemm path):
// U[0][m][i] = hi, U[1][m][i] = lo of XqO[m][i] * (s_i - 1); zero in the
// padding columns.
__global__ void comp_operand_kernel(const int8_t* __restrict__ XqO, const float* __restrict__ s, int M,
                                    int nO, int nOp, uint16_t* __restrict__ U) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t total = static_cast<size_t>(M) * nOp;
  if (idx >= total) return;
  const int m = static_cast<int>(idx / nOp);
  const int i = static_cast<int>(idx - static_cast<size_t>(m) * nOp);
  uint2 hl = make_uint2(0u, 0u);
  if (i < nO) hl = comp_split(XqO[static_cast<size_t>(m) * nO + i], s[i]);
  U[idx] = static_cast<uint16_t>(hl.x);
  U[total + idx] = static_cast<uint16_t>(hl.y);
}

}  // namespace qlin
