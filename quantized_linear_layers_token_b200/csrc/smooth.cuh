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

// ref[m][n] = sum over t in T of X[m][t] * W[t][n] (fp32 FMA in input
// order): 128 x 128 tiles, 256 threads of 8 x 8 outputs, 16 inputs per
// stage; the next stage's 16-byte loads go to registers while the current
// stage (shared memory, double-buffered) is used.  K % 32 == 0, N % 16 == 0.
constexpr int kRefTile = 128;
constexpr int kRefK = 16;

__global__ void __launch_bounds__(256)
smooth_ref_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ W, const float* __restrict__ sv,
                  int M, int K, int N, float* __restrict__ ref) {
  __shared__ __align__(16) float xs[2][kRefK][kRefTile];  // [input][token]
  __shared__ __align__(16) float ws[2][kRefK][kRefTile];  // [input][channel]
  const int m0 = blockIdx.y * kRefTile, n0 = blockIdx.x * kRefTile;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;         // 8 tokens x 8 channels each
  const int xr = tid >> 1, xk = (tid & 1) * 8;    // loader: token row, 8 inputs
  const int wk = tid >> 4, wn = (tid & 15) * 8;   // loader: input row, 8 channels
  float xa[8], wb[8];
  auto load = [&](int t0) {
    const int m = m0 + xr;
    const int t = t0 + xk;  // 8 inputs, inside K (K % 16 == 0)
    uint4 xv = make_uint4(0u, 0u, 0u, 0u);
    if (m < M) xv = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + t));
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(sv + t));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(sv + t) + 1);
    const float sm[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int j = 0; j < 8; ++j)
      xa[j] = sm[j] > 0.f ? half_bits_to_float(static_cast<uint16_t>(xw[j >> 1] >> (16 * (j & 1)))) : 0.f;
    const int n = n0 + wn;
    uint4 wv = make_uint4(0u, 0u, 0u, 0u);
    if (n < N) wv = __ldg(reinterpret_cast<const uint4*>(W + static_cast<size_t>(t0 + wk) * N + n));
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) wb[j] = half_bits_to_float(static_cast<uint16_t>(ww[j >> 1] >> (16 * (j & 1))));
  };
  auto store = [&](int b) {
#pragma unroll
    for (int j = 0; j < 8; ++j) xs[b][xk + j][xr] = xa[j];
    *reinterpret_cast<float4*>(&ws[b][wk][wn]) = make_float4(wb[0], wb[1], wb[2], wb[3]);
    *reinterpret_cast<float4*>(&ws[b][wk][wn + 4]) = make_float4(wb[4], wb[5], wb[6], wb[7]);
  };
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  load(0);
  store(0);
  __syncthreads();
  for (int t0 = 0; t0 < K; t0 += kRefK) {
    const int cur = (t0 / kRefK) & 1;
    const bool more = t0 + kRefK < K;
    if (more) load(t0 + kRefK);
#pragma unroll
    for (int k = 0; k < kRefK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&xs[cur][k][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&xs[cur][k][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&ws[cur][k][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&ws[cur][k][tx * 8 + 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
    }
    if (more) store(cur ^ 1);
    __syncthreads();
  }
  const int n = n0 + tx * 8;
  if (n < N) {
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const int m = m0 + ty * 8 + a;
      if (m < M) {
        float* dst = ref + static_cast<size_t>(m) * N + n;
        *reinterpret_cast<float4*>(dst) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
      }
    }
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
