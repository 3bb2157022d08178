// gptq.cuh -- Hessian-compensated weight quantization (offline, before
// packing): QQQ review, section 三 技术架构 -> Hessian补偿.
//
//   H = 2 X^T X                                  (X: calibration activations [ns][K])
//   for i = 0 .. K-1, for every output channel n (column n of W [K][N]):
//     q      = clamp(rne(w_i / scale_n), -qmax, qmax) * scale_n
//     delta  = -(w_i - q) / [H^-1]_ii * (H^-1)[:, i]      applied to w_j, j >= i
//     w_i    = q
//   then H^-1 <- H^-1 - H^-1[:, i] H^-1[i, :] / [H^-1]_ii   (rank-one downdate
//   removing column i from the inverse of the remaining block)
//
// The inverse of H and the downdates do not depend on the weights, so one
// sequence serves every output channel of the layer.  Every step is an
// elementwise fp64 operation done with IEEE round-to-nearest intrinsics and
// no contraction, in the order written above, so the results match a
// sequential CPU evaluation of the same steps bit for bit:
//   gptq_hessian_kernel      H[i][j] = 2 * (sum over t in order of
//                            X[t][i] * X[t][j]); 64 x 64 tiles, samples staged
//                            through shared memory 16 at a time.
//   gj_pivot_kernel          Gauss-Jordan step c: the pivot row (largest
//                            |a[r][c]|, r >= c, first on ties), and the
//                            column of multipliers before the step changes it.
//   gj_swap_scale_kernel     swap rows c and p, divide row c by the pivot.
//   gj_eliminate_kernel      a[r][j] -= f_r * a[c][j] (and the same on the
//                            inverse) for every r != c with f_r != 0.
//   gptq_step_kernel         one column i: the weight updates of every output
//                            channel (y-blocks 0..) and the downdate of the
//                            remaining inverse block (the other y-blocks),
//                            which touch disjoint data.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qlin {

constexpr int kHessTile = 64;

// H = 2 X^T X: one 64 x 64 tile per CTA of 256 threads (4 x 4 elements each).
__global__ void __launch_bounds__(256)
gptq_hessian_kernel(const double* __restrict__ X, int ns, int K, double* __restrict__ H) {
  __shared__ double xi[16][kHessTile];
  __shared__ double xj[16][kHessTile];
  const int i0 = blockIdx.y * kHessTile, j0 = blockIdx.x * kHessTile;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
  for (int t0 = 0; t0 < ns; t0 += 16) {
    for (int e = threadIdx.x; e < 16 * kHessTile; e += 256) {
      const int tt = e / kHessTile, c = e % kHessTile;
      const int t = t0 + tt;
      xi[tt][c] = (t < ns && i0 + c < K) ? X[static_cast<size_t>(t) * K + i0 + c] : 0.0;
      xj[tt][c] = (t < ns && j0 + c < K) ? X[static_cast<size_t>(t) * K + j0 + c] : 0.0;
    }
    __syncthreads();
    const int tn = min(16, ns - t0);
    for (int tt = 0; tt < tn; ++tt) {
      double a4[4], b4[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) a4[a] = xi[tt][ty * 4 + a];
#pragma unroll
      for (int b = 0; b < 4; ++b) b4[b] = xj[tt][tx * 4 + b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = __dadd_rn(acc[a][b], __dmul_rn(a4[a], b4[b]));
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int i = i0 + ty * 4 + a, j = j0 + tx * 4 + b;
      if (i < K && j < K) H[static_cast<size_t>(i) * K + j] = __dmul_rn(2.0, acc[a][b]);
    }
}

// inv = identity
__global__ void gptq_identity_kernel(double* __restrict__ inv, int K) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx < static_cast<size_t>(K) * K) inv[idx] = (idx / K == idx % K) ? 1.0 : 0.0;
}

// GPTQ scratch (device): the pivot row and value of the current step and the
// singular flag (the column of multipliers f[K] follows it in the workspace).
struct GjScratch {
  int pivot;
  int singular;
  double pivot_value;  // a[pivot][c] before the swap (read by every column's thread)
};

// Step c: pivot row p = the first r >= c with the largest |a[r][c]|; the
// multipliers f[r] = the value row r holds in column c once rows c and p are
// swapped (read before the elimination overwrites the column).  One CTA.
__global__ void __launch_bounds__(1024)
gj_pivot_kernel(const double* __restrict__ a, int K, int c, GjScratch* __restrict__ st, double* __restrict__ f) {
  __shared__ double sv[32];
  __shared__ int si[32];
  if (st->singular) return;  // an earlier step failed: leave everything as it is
  double best = -1.0;
  int bi = K;
  for (int r = c + threadIdx.x; r < K; r += blockDim.x) {
    const double v = fabs(a[static_cast<size_t>(r) * K + c]);
    if (v > best) { best = v; bi = r; }  // rows visited in increasing order: the first maximum stays
  }
  // (value, index) reduction: larger value, or equal value and smaller index
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
  }
  if ((threadIdx.x & 31) == 0) { sv[threadIdx.x >> 5] = best; si[threadIdx.x >> 5] = bi; }
  __syncthreads();
  if (threadIdx.x < 32) {
    best = threadIdx.x < blockDim.x / 32 ? sv[threadIdx.x] : -1.0;
    bi = threadIdx.x < blockDim.x / 32 ? si[threadIdx.x] : K;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
    }
    if (threadIdx.x == 0) si[0] = bi;
  }
  __syncthreads();
  const int p = si[0];
  if (p >= K || a[static_cast<size_t>(p) * K + c] == 0.0) {
    if (threadIdx.x == 0) st->singular = 1;
    return;
  }
  if (threadIdx.x == 0) {
    st->pivot = p;
    st->pivot_value = a[static_cast<size_t>(p) * K + c];
  }
  for (int r = threadIdx.x; r < K; r += blockDim.x) {
    const int src = r == p ? c : r;  // after the swap row p holds the old row c
    f[r] = r == c ? 0.0 : a[static_cast<size_t>(src) * K + c];
  }
}

// Swap rows c and p (a: columns >= c, where rows c and p can differ; inv:
// every column), then divide row c by the pivot.  One thread per column.
__global__ void gj_swap_scale_kernel(double* __restrict__ a, double* __restrict__ inv, int K, int c,
                                     const GjScratch* __restrict__ st) {
  if (st->singular) return;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const int p = st->pivot;
  const double piv = st->pivot_value;  // not a[p][c]: the thread of column c may already have swapped it
  double* rc = a + static_cast<size_t>(c) * K;
  double* rp = a + static_cast<size_t>(p) * K;
  double* ic = inv + static_cast<size_t>(c) * K;
  double* ip = inv + static_cast<size_t>(p) * K;
  if (j >= c) {
    const double vc = rc[j], vp = rp[j];
    rc[j] = __ddiv_rn(vp, piv);
    if (p != c) rp[j] = vc;
  }
  const double wc = ic[j], wp = ip[j];
  ic[j] = __ddiv_rn(wp, piv);
  if (p != c) ip[j] = wc;
}

// a[r][j] -= f[r] * a[c][j] (j >= c) and inv[r][j] -= f[r] * inv[c][j] (all
// j) for every r != c whose multiplier is nonzero.  x: columns, y: rows.
__global__ void gj_eliminate_kernel(double* __restrict__ a, double* __restrict__ inv, int K, int c,
                                    const GjScratch* __restrict__ st, const double* __restrict__ f) {
  if (st->singular) return;
  const int r = blockIdx.y;
  if (r == c) return;
  const double fr = f[r];
  if (fr == 0.0) return;
  const double* rc = a + static_cast<size_t>(c) * K;
  const double* ic = inv + static_cast<size_t>(c) * K;
  double* ra = a + static_cast<size_t>(r) * K;
  double* ri = inv + static_cast<size_t>(r) * K;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < K; j += gridDim.x * blockDim.x) {
    if (j >= c) ra[j] = __dsub_rn(ra[j], __dmul_rn(fr, rc[j]));
    ri[j] = __dsub_rn(ri[j], __dmul_rn(fr, ic[j]));
  }
}

// One column i of the compensation.  y-blocks [0, yw): weight updates, one
// thread per output channel n and a range of rows j; y-blocks [yw, ..):
// the downdate of hw[r][c], r, c > i, one thread per column c.
//   W  [K][N] current weights (fp64), hw [K][K] current inverse.
__global__ void gptq_step_kernel(double* __restrict__ W, int8_t* __restrict__ codes, const double* __restrict__ scale,
                                 double* __restrict__ hw, int K, int N, int i, int qmax, int rows_per_block, int yw,
                                 const GjScratch* __restrict__ st) {
  if (st->singular) return;
  const double hii = hw[static_cast<size_t>(i) * K + i];
  if (static_cast<int>(blockIdx.y) < yw) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const double wi = W[static_cast<size_t>(i) * N + n];
    const double sc = scale[n];
    // the grid index is an integer (a rounded zero has no sign), then the
    // grid value is index * scale
    const double t = rint(__ddiv_rn(wi, sc));
    const int ti = t < -qmax ? -qmax : (t > qmax ? qmax : static_cast<int>(t));
    const double q = __dmul_rn(static_cast<double>(ti), sc);
    const double fq = -__ddiv_rn(__dsub_rn(wi, q), hii);
    const int j0 = i + 1 + static_cast<int>(blockIdx.y) * rows_per_block;
    const int j1 = min(K, j0 + rows_per_block);
    for (int j = j0; j < j1; ++j) {
      const size_t o = static_cast<size_t>(j) * N + n;
      W[o] = __dadd_rn(W[o], __dmul_rn(fq, hw[static_cast<size_t>(j) * K + i]));
    }
    if (blockIdx.y == 0) {
      W[static_cast<size_t>(i) * N + n] = q;
      codes[static_cast<size_t>(i) * N + n] = static_cast<int8_t>(ti);
    }
    return;
  }
  const int c = i + 1 + blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= K) return;
  const double rowc = hw[static_cast<size_t>(i) * K + c];
  const int nr = K - i - 1;
  const int ydown = gridDim.y - yw;
  const int per = (nr + ydown - 1) / ydown;
  const int r0 = i + 1 + (static_cast<int>(blockIdx.y) - yw) * per;
  const int r1 = min(K, r0 + per);
  for (int r = r0; r < r1; ++r) {
    const size_t o = static_cast<size_t>(r) * K + c;
    hw[o] = __dsub_rn(hw[o], __ddiv_rn(__dmul_rn(hw[static_cast<size_t>(r) * K + i], rowc), hii));
  }
}

}  // namespace qlin
