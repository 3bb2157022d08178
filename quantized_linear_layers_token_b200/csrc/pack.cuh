// pack.cuh -- weight quantization and packing kernels (offline step).
//
// Quaff notes, 整体框架: the frozen W is quantized once to W_int while the
// rows of the outlier channels, W_O, are kept in full precision.  QQQ review,
// W4A8 GEMM内核: INT4 codes with one scale per output channel, or per group
// of 128 input channels with the group scale divided by the channel scale
// ahead of time (FusedDequantQuant).
//
// One thread owns one output channel n and walks its K inputs twice (scale
// pass, code pass); reads of W[k][*] are coalesced across the threads of a
// warp.  Packing runs once per layer and is not on the timed path.
//
// Packed codes are tile-major so that the GEMM fetches each 128-channel x
// 128-input block with one contiguous bulk copy: block (tn, kb) holds
// channels 128*tn .. +127 (rows) and inputs 128*kb .. +127.  INT4 blocks are
// 128 rows x 64 bytes (8 KiB), 16-byte chunk c of row r at chunk
// c ^ ((r / 2) % 4); INT8 blocks are 128 rows x 128 bytes (16 KiB) stored
// with the tensor core's 128-byte swizzle already applied (16-byte chunk c
// of row r sits at chunk c ^ (r % 8)).  Padding rows and inputs are zero.
#pragma once

#include "sm100.cuh"

namespace qlin {

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }
__device__ __forceinline__ uint16_t f2h_bits(float f) { return __half_as_ushort(__float2half_rn(f)); }

// Round to nearest (ties to even) and clamp to [-qmax, qmax].
__device__ __forceinline__ int rne_clamp(float p, int qmax) {
  const int q = __float2int_rn(p);
  return q < -qmax ? -qmax : (q > qmax ? qmax : q);
}

// Nibble layout of one 32-bit word covering k0..k0+7: byte b holds q[k0+b]
// (low nibble) and q[k0+4+b] (high nibble), so a shift by 4 and a mask give
// the INT8 lanes 16*q of the first half, a mask alone those of the second.
__device__ __forceinline__ uint32_t pack8_nibbles(const int (&q)[8]) {
  uint32_t w = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t byte = (static_cast<uint32_t>(q[b]) & 0xFu) | ((static_cast<uint32_t>(q[4 + b]) & 0xFu) << 4);
    w |= byte << (8 * b);
  }
  return w;
}

__device__ __forceinline__ uint2 pack8_bytes(const int (&q)[8]) {
  uint2 o;
  o.x = (static_cast<uint32_t>(q[0]) & 0xFFu) | ((static_cast<uint32_t>(q[1]) & 0xFFu) << 8) |
        ((static_cast<uint32_t>(q[2]) & 0xFFu) << 16) | ((static_cast<uint32_t>(q[3]) & 0xFFu) << 24);
  o.y = (static_cast<uint32_t>(q[4]) & 0xFFu) | ((static_cast<uint32_t>(q[5]) & 0xFFu) << 8) |
        ((static_cast<uint32_t>(q[6]) & 0xFFu) << 16) | ((static_cast<uint32_t>(q[7]) & 0xFFu) << 24);
  return o;
}

// Byte offset of the 8 codes k0..k0+7 of channel n in the tiled layouts.
// INT4 rows are 64 bytes; the 16-byte chunk c of row r sits at chunk
// c ^ ((r >> 1) & 3) (conflict-free reads with one thread per row).
__device__ __forceinline__ size_t w4_tile_offset(int n, int k0, int KB) {
  const size_t blk = static_cast<size_t>(n >> 7) * KB + (k0 >> 7);
  const int r = n & 127;
  const int byte = (k0 & 127) >> 1;
  return (blk * 128 + r) * 64 + ((((byte >> 4) ^ ((r >> 1) & 3))) << 4) + (byte & 15);
}
__device__ __forceinline__ size_t w8_tile_offset(int n, int k0, int KB) {
  const size_t blk = static_cast<size_t>(n >> 7) * KB + (k0 >> 7);
  const int r = n & 127;
  const int chunk = (k0 & 127) >> 4;
  return (blk * 128 + r) * 128 + ((chunk ^ (r & 7)) << 4) + (k0 & 15);
}

// Symmetric per-output-channel quantization:
//   c_n = wmax_n / qmax,  q = clamp(rne(w * (qmax / wmax_n)), -qmax, qmax)   (fp32)
template <int QMAX, bool W4>
__global__ void pack_per_channel_kernel(const uint16_t* __restrict__ W, int K, int N,
                                        uint8_t* __restrict__ codes, float* __restrict__ cscale) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float wmax = 0.f;
  for (int k = 0; k < K; ++k) {
    const float v = fabsf(h2f(W[static_cast<size_t>(k) * N + n]));
    wmax = v > wmax ? v : wmax;
  }
  const float fq = static_cast<float>(QMAX);
  cscale[n] = __fdiv_rn(wmax, fq);
  const float inv = wmax > 0.f ? __fdiv_rn(fq, wmax) : 0.f;
  for (int k0 = 0; k0 < K; k0 += 8) {
    int q[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) q[j] = rne_clamp(__fmul_rn(h2f(W[static_cast<size_t>(k0 + j) * N + n]), inv), QMAX);
    const int KB = (K + 127) >> 7;
    if (W4) {
      *reinterpret_cast<uint32_t*>(codes + w4_tile_offset(n, k0, KB)) = pack8_nibbles(q);
    } else {
      *reinterpret_cast<uint2*>(codes + w8_tile_offset(n, k0, KB)) = pack8_bytes(q);
    }
  }
}

// Per-group (128 input channels) INT4 with the folded requantization ratio:
//   g = fp16(gmax / 7);  q4 = clamp(rne(w / g), -7, 7)
//   c_n = 7 * max_j g / 127;  r = fp16(g / c_n)
template <int GROUP>
__global__ void pack_group_kernel(const uint16_t* __restrict__ W, int K, int N,
                                  uint8_t* __restrict__ codes, float* __restrict__ cscale,
                                  uint16_t* __restrict__ gscale, uint16_t* __restrict__ rfold) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const int G = K / GROUP;
  float ghmax = 0.f;
  for (int j = 0; j < G; ++j) {
    float gmax = 0.f;
    for (int k = j * GROUP; k < (j + 1) * GROUP; ++k) {
      const float v = fabsf(h2f(W[static_cast<size_t>(k) * N + n]));
      gmax = v > gmax ? v : gmax;
    }
    const uint16_t gh = f2h_bits(__fdiv_rn(gmax, 7.f));
    gscale[static_cast<size_t>(j) * N + n] = gh;
    const float ghf = h2f(gh);
    ghmax = ghf > ghmax ? ghf : ghmax;
  }
  const float cn = __fdiv_rn(__fmul_rn(7.f, ghmax), 127.f);
  cscale[n] = cn;
  for (int j = 0; j < G; ++j) {
    const float ghf = h2f(gscale[static_cast<size_t>(j) * N + n]);
    rfold[static_cast<size_t>(j) * N + n] = cn > 0.f ? f2h_bits(__fdiv_rn(ghf, cn)) : static_cast<uint16_t>(0);
    for (int k0 = j * GROUP; k0 < (j + 1) * GROUP; k0 += 8) {
      int q[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float w = h2f(W[static_cast<size_t>(k0 + t) * N + n]);
        q[t] = ghf > 0.f ? rne_clamp(__fdiv_rn(w, ghf), 7) : 0;
      }
      *reinterpret_cast<uint32_t*>(codes + w4_tile_offset(n, k0, K >> 7)) = pack8_nibbles(q);
    }
  }
}

// Outlier rows: W_Ot holds W[O_i][n] transposed (channel n, outlier i) so
// the compensation operand is K-major for the tensor core, tiled like the
// INT8 codes: block (tn, ib) is channels 128*tn .. +127 by outliers
// 64*ib .. +63 in fp16, 128 bytes per row, 128-byte swizzle applied.
// wmax_O[i] = max_n |W[O_i][n]|.  One CTA per outlier channel; the padding
// is cleared beforehand.
__device__ __forceinline__ size_t wot_tile_index(int n, int i, int IB) {
  const size_t blk = static_cast<size_t>(n >> 7) * IB + (i >> 6);
  const int r = n & 127;
  const int byte = (i & 63) * 2;
  return ((blk * 128 + r) * 128 + (((byte >> 4) ^ (r & 7)) << 4) + (byte & 15)) >> 1;
}

__global__ void pack_outliers_kernel(const uint16_t* __restrict__ W, int N, const int32_t* __restrict__ O,
                                     int nO, uint16_t* __restrict__ W_Ot, float* __restrict__ wmaxO) {
  const int i = blockIdx.x;
  const int IB = (nO + 63) >> 6;
  const uint16_t* row = W + static_cast<size_t>(O[i]) * N;
  float m = 0.f;
  for (int n = threadIdx.x; n < N; n += blockDim.x) {
    const uint16_t v = row[n];
    const float f = fabsf(h2f(v));
    m = f > m ? f : m;
    W_Ot[wot_tile_index(n, i, IB)] = v;
  }
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) wmaxO[i] = m;
  }
}

}  // namespace qlin
