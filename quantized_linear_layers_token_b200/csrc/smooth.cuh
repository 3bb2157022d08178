// smooth.cuh -- QQQ adaptive smoothing: the threshold search (offline,
// calibration).  QQQ review, section 三 技术架构 -> 自适应平滑: only the
// activation channels with significant outliers are smoothed, the threshold
// sigma is found by a grid search over [0, max|X|], and the smoothing is the
// one that minimises the error of the quantized product on those channels.
//
// For the candidate sigma_j = max|X| * j / G (fp32, this order):
//   T      = { t : max_m |X[m,t]| > sigma_j }
//   s_t    = sqrt(max_m|X[m,t]| / max_n|W[t,n]|) on T (1 if a maximum is 0)
//   Xh     = fp16(X / s) on T, 0 elsewhere;  Wh = fp16(W * s) on T, 0 elsewhere
//   loss_j = sum_{m,n} ( a_m (c_n / 16) acc[m][n] - (X_T W_T)[m][n] )^2
// where (Xq, a) is the layer's per-token INT8 quantization of Xh, (q, c)
// its per-channel INT4 quantization of Wh and acc the exact INT32 product of
// Xq and 16 q.  The quantization and the integer product run through the
// library's own packer, quantization kernel and tcgen05 GEMM; the kernels
// here compute the channel maxima, the smoothed tensors, the unquantized
// reference product on T (fp32 FMA) and the loss (fp64).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qlin {

__device__ __forceinline__ float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// cmax_bits[t] = max_m |X[m,t]| as fp32 bits (zero on entry).  x: columns,
// y: row chunks of 64.
__global__ void smooth_colmax_kernel(const uint16_t* __restrict__ X, int M, int K, unsigned* __restrict__ cmax_bits) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= K) return;
  const int m0 = blockIdx.y * 64, m1 = min(M, m0 + 64);
  float v = 0.f;
  for (int m = m0; m < m1; ++m) v = fmaxf(v, fabsf(half_bits_to_float(X[static_cast<size_t>(m) * K + t])));
  atomicMax(&cmax_bits[t], __float_as_uint(v));
}

// wmax[t] = max_n |W[t,n]|, one CTA of 256 threads per row t.
__global__ void smooth_rowmax_kernel(const uint16_t* __restrict__ W, int N, float* __restrict__ wmax) {
  __shared__ float red[8];
  const uint16_t* row = W + static_cast<size_t>(blockIdx.x) * N;
  float v = 0.f;
  for (int n = threadIdx.x; n < N; n += 256) v = fmaxf(v, fabsf(half_bits_to_float(row[n])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = red[0];
    for (int w = 1; w < 8; ++w) r = fmaxf(r, red[w]);
    wmax[blockIdx.x] = r;
  }
}

// max over the column maxima (one CTA)
__global__ void smooth_allmax_kernel(const unsigned* __restrict__ cmax_bits, int K, float* __restrict__ xall) {
  __shared__ unsigned red[32];
  unsigned v = 0u;
  for (int t = threadIdx.x; t < K; t += blockDim.x) v = max(v, cmax_bits[t]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned r = 0u;
    for (int w = 0; w < static_cast<int>(blockDim.x / 32); ++w) r = max(r, red[w]);
    *xall = __uint_as_float(r);
  }
}

// The smoothing factor of channel t for candidate j: s_t on T, 0 marking a
// channel outside T.
__device__ __forceinline__ float smooth_factor(float cm, float wm, float xall, int j, int G) {
  const float sigma = __fdiv_rn(__fmul_rn(xall, static_cast<float>(j)), static_cast<float>(G));
  if (!(cm > sigma)) return 0.f;
  return (cm > 0.f && wm > 0.f) ? __fsqrt_rn(__fdiv_rn(cm, wm)) : 1.f;
}

__global__ void smooth_factors_kernel(const unsigned* __restrict__ cmax_bits, const float* __restrict__ wmax,
                                      const float* __restrict__ xall, int K, int j, int G, float* __restrict__ sv) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < K) sv[t] = smooth_factor(__uint_as_float(cmax_bits[t]), wmax[t], *xall, j, G);
}

// Xh = fp16(X / s) on T, else 0; Wh = fp16(W * s) on T, else 0.
__global__ void smooth_apply_x_kernel(const uint16_t* __restrict__ X, const float* __restrict__ sv, int M, int K,
                                      uint16_t* __restrict__ Xh) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<size_t>(M) * K) return;
  const float s = sv[idx % K];
  Xh[idx] = s > 0.f ? __half_as_ushort(__float2half_rn(__fdiv_rn(half_bits_to_float(X[idx]), s))) : 0;
}

__global__ void smooth_apply_w_kernel(const uint16_t* __restrict__ W, const float* __restrict__ sv, int K, int N,
                                      uint16_t* __restrict__ Wh) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<size_t>(K) * N) return;
  const float s = sv[idx / N];
  Wh[idx] = s > 0.f ? __half_as_ushort(__float2half_rn(__fmul_rn(half_bits_to_float(W[idx]), s))) : 0;
}

// ref[m][n] = sum over t in T of X[m][t] * W[t][n] (fp32 FMA; 64 x 64 tiles,
// 256 threads of 4 x 4 outputs, K staged 16 at a time).
__global__ void __launch_bounds__(256)
smooth_ref_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ W, const float* __restrict__ sv, int M,
                  int K, int N, float* __restrict__ ref) {
  __shared__ float xs[16][64 + 1];
  __shared__ float ws[16][64];
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  float acc[4][4] = {};
  for (int t0 = 0; t0 < K; t0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int tt = e % 16, mm = e / 16;  // X tile: 64 rows x 16 inputs
      const int t = t0 + tt, m = m0 + mm;
      xs[tt][mm] = (m < M && t < K && sv[t] > 0.f) ? half_bits_to_float(X[static_cast<size_t>(m) * K + t]) : 0.f;
      const int nn = e % 64, tw = e / 64;  // W tile: 16 inputs x 64 outputs
      const int t2 = t0 + tw, n = n0 + nn;
      ws[tw][nn] = (n < N && t2 < K) ? half_bits_to_float(W[static_cast<size_t>(t2) * N + n]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) {
      float a4[4], b4[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) a4[a] = xs[tt][ty * 4 + a];
#pragma unroll
      for (int b = 0; b < 4; ++b) b4[b] = ws[tt][tx * 4 + b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(a4[a], b4[b], acc[a][b]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int m = m0 + ty * 4 + a, n = n0 + tx * 4 + b;
      if (m < M && n < N) ref[static_cast<size_t>(m) * N + n] = acc[a][b];
    }
}

// loss[j] += sum of (a_m (c_n / 16) acc - ref)^2 in fp64 (zero on entry).
__global__ void smooth_loss_kernel(const int32_t* __restrict__ acc, const float* __restrict__ a,
                                   const float* __restrict__ c, const float* __restrict__ ref, int M, int N,
                                   double* __restrict__ loss) {
  __shared__ double red[8];
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  double d2 = 0.0;
  if (idx < static_cast<size_t>(M) * N) {
    const int m = static_cast<int>(idx / N), n = static_cast<int>(idx % N);
    const double y = __dmul_rn(__dmul_rn(static_cast<double>(acc[idx]), static_cast<double>(a[m])),
                               __ddiv_rn(static_cast<double>(c[n]), 16.0));
    const double d = __dsub_rn(y, static_cast<double>(ref[idx]));
    d2 = __dmul_rn(d, d);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) d2 += __shfl_xor_sync(0xffffffffu, d2, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = d2;
  __syncthreads();
  if (threadIdx.x == 0) {
    double r = 0.0;
    for (int w = 0; w < 8; ++w) r += red[w];
    atomicAdd(loss, r);
  }
}

// best = the first candidate of least loss; s_best = its smoothing vector
// (1 outside T).  One CTA.
__global__ void smooth_pick_kernel(const double* __restrict__ loss, int G, const unsigned* __restrict__ cmax_bits,
                                   const float* __restrict__ wmax, const float* __restrict__ xall, int K,
                                   int32_t* __restrict__ best, float* __restrict__ s_best) {
  __shared__ int sb;
  if (threadIdx.x == 0) {
    int b = 0;
    for (int j = 1; j < G; ++j)
      if (loss[j] < loss[b]) b = j;
    sb = b;
    if (best) *best = b;
  }
  __syncthreads();
  if (!s_best) return;
  for (int t = threadIdx.x; t < K; t += blockDim.x) {
    const float s = smooth_factor(__uint_as_float(cmax_bits[t]), wmax[t], *xall, sb, G);
    s_best[t] = s > 0.f ? s : 1.f;
  }
}

}  // namespace qlin
