/*
 * qlin_oracle.c -- plain, slow, single-threaded CPU oracle for the
 * outlier-aware quantized linear layer Y = Q(X) . Q(W).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no
 * code, header, table or constant generator with the CUDA library; the two
 * are written independently from the same specification.
 *
 * Sources (page title, section):
 *   [Quaff]  "Quaff: Quantized Parameter-Efficient Fine-Tuning under Outlier
 *            Spatial Stability Hypothesis" (Paper-Notes), sections
 *            "整体框架" (overall framework), "关键设计 / 解耦 WAQ 公式"
 *            (decoupled WAQ formula), "目标动量缩放" (targeted momentum
 *            scaling).
 *   [QQQ]    "QQQ: Quality Quattuor-Bit Quantization for Large Language
 *            Models" (paper review), section 三 "技术架构": "Hessian补偿",
 *            "W4A8 GEMM内核" (per-channel GEMM, per-group GEMM,
 *            FusedDequantQuant, FastFP16toINT8), and section 五's symmetric
 *            quantization column.
 *
 * Every floating-point step below is written out in the order stated so a
 * reader can check it against the pages; fp32 steps use IEEE division and
 * square root and are compiled without contraction (-ffp-contract=off).
 * Readings of points the pages leave open are listed at each function.
 *
 * Parity status: every function here is pinned by a CPU test against an
 * independent fact (brute force, closed form, library routine or exhaustive
 * enumeration); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OQ_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* O1: IEEE-754 binary16, written from the format definition                */
/*     (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits).        */
/* ------------------------------------------------------------------------ */

OQ_EXPORT double oq_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int f = h & 0x3FF;
  double v;
  if (e == 0) {
    v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
  } else if (e == 31) {
    v = f ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

OQ_EXPORT float oq_half_to_float(uint16_t h) { return (float)oq_half_to_double(h); }

/* Round a double to the nearest binary16, ties to even, with subnormals and
 * overflow to infinity.  The quantum of the target binade is a power of two,
 * so x / quantum is exact in double and rint() (default rounding mode:
 * to nearest, ties to even) performs the single rounding. */
OQ_EXPORT uint16_t oq_double_to_half(double x) {
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (isnan(x)) return 0x7E00;
  if (isinf(a)) return sign | 0x7C00;
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2);          /* a = m * 2^e2, m in [0.5, 1) */
  int exp_unb = e2 - 1;   /* a in [2^exp_unb, 2^(exp_unb+1)) */
  if (exp_unb < -14) exp_unb = -14; /* subnormal binade shares quantum 2^-24 */
  double quantum = ldexp(1.0, exp_unb - 10);
  double q = rint(a / quantum); /* integer significand, ties to even */
  /* q may have carried into the next binade (q == 2048). */
  if (q >= 2048.0) {
    q = q / 2.0;
    exp_unb += 1;
  }
  if (exp_unb > 15) return sign | 0x7C00; /* overflow */
  uint16_t bits;
  if (q < 1024.0) {
    /* subnormal (only possible when exp_unb == -14) */
    bits = (uint16_t)q;
  } else {
    bits = (uint16_t)(((exp_unb + 15) << 10) | ((int)q - 1024));
  }
  return sign | bits;
}

/* float -> half: float -> double is exact, so this is one rounding. */
OQ_EXPORT uint16_t oq_float_to_half(float x) { return oq_double_to_half((double)x); }

/* ------------------------------------------------------------------------ */
/* O2: round half to even to an integer                                      */
/* ------------------------------------------------------------------------ */

OQ_EXPORT double oq_rne(double x) { return rint(x); }

static int32_t clampi(double v, int32_t lo, int32_t hi) {
  if (v < lo) return lo;
  if (v > hi) return hi;
  return (int32_t)v;
}

/* ------------------------------------------------------------------------ */
/* O3: weight quantization (offline packer)                                  */
/*                                                                            */
/* W is fp16 [K][N] row-major (Y = X . W; input channel k is row k).          */
/* Codes are returned in the logical layout int8 [K][N].                      */
/* ------------------------------------------------------------------------ */

/* Symmetric per-output-channel quantization to [-qmax, qmax]
 * ([QQQ] section 五: QQQ is symmetric; [QQQ] per-channel GEMM;
 *  [Quaff] INT8 weights).
 *   wmax_n = max_k |W[k][n]|
 *   scale_n = wmax_n / qmax          (fp32, IEEE division)
 *   inv_n   = qmax / wmax_n          (fp32, IEEE division)
 *   q       = clamp(rne(w * inv_n), -qmax, qmax)   (fp32 product)
 * A zero column gets scale 0 and codes 0. */
OQ_EXPORT void oq_quant_weight_per_channel(const uint16_t* W, int K, int N, int qmax,
                                           int8_t* codes, float* scale) {
  const float fq = (float)qmax;
  float* wmax = (float*)calloc((size_t)(N > 0 ? N : 1), sizeof(float));
  float* inv = (float*)calloc((size_t)(N > 0 ? N : 1), sizeof(float));
  /* W is walked row by row (k outer) so every access is sequential; each
   * channel's max and codes are the same values as a channel-by-channel
   * loop gives (max is exact in any order). */
  for (int k = 0; k < K; ++k)
    for (int n = 0; n < N; ++n) {
      float v = fabsf(oq_half_to_float(W[(size_t)k * N + n]));
      if (v > wmax[n]) wmax[n] = v;
    }
  for (int n = 0; n < N; ++n) {
    scale[n] = wmax[n] / fq;
    inv[n] = (wmax[n] > 0.0f) ? (fq / wmax[n]) : 0.0f;
  }
  for (int k = 0; k < K; ++k)
    for (int n = 0; n < N; ++n) {
      float w = oq_half_to_float(W[(size_t)k * N + n]);
      float p = w * inv[n];
      codes[(size_t)k * N + n] = (int8_t)clampi(oq_rne((double)p), -qmax, qmax);
    }
  free(wmax);
  free(inv);
}

/* Per-group (g = 128 along K) symmetric INT4 with per-channel INT8
 * requantization ([QQQ] per-group GEMM; FusedDequantQuant).
 *   gmax[j][n] = max_{k in group j} |W[k][n]|
 *   g_h[j][n]  = fp16_rn( fp32(gmax / 7) )
 *   q4[k][n]   = g_h == 0 ? 0 : clamp(rne( fp32(w / float(g_h)) ), -7, 7)
 *   c_n        = fp32( fp32(7 * max_j float(g_h[j][n])) / 127 )
 *   r_h[j][n]  = c_n == 0 ? 0 : fp16_rn( fp32(float(g_h) / c_n) )
 *                (the group scale divided by the channel scale, folded into
 *                 one factor -- "组缩放除以通道缩放")
 *   q8[k][n]   = rne( q4 * float(r_h) )  -- exact product, one rounding.
 * Reading: codes are [-7, 7] (not [-8, 7]) so that |q8| <= 127 holds; it is
 * asserted here and returned as an error flag (nonzero return).
 * Outputs: q4 int8 [K][N], q8 int8 [K][N], g_h / r_h fp16 bits [K/g][N],
 * c fp32 [N]. */
OQ_EXPORT int oq_quant_weight_group(const uint16_t* W, int K, int N, int group,
                                    int8_t* q4, int8_t* q8, uint16_t* g_h, uint16_t* r_h,
                                    float* c) {
  int bad = 0;
  int G = K / group;
  /* W is walked row by row (k outer) so every access is sequential; every
   * (group, channel) value is the same as a channel-by-channel loop gives. */
  float* gmax = (float*)calloc((size_t)(N > 0 ? N : 1), sizeof(float));
  float* ghmax = (float*)calloc((size_t)(N > 0 ? N : 1), sizeof(float));
  for (int j = 0; j < G; ++j) {
    for (int n = 0; n < N; ++n) gmax[n] = 0.0f;
    for (int k = j * group; k < (j + 1) * group; ++k)
      for (int n = 0; n < N; ++n) {
        float v = fabsf(oq_half_to_float(W[(size_t)k * N + n]));
        if (v > gmax[n]) gmax[n] = v;
      }
    for (int n = 0; n < N; ++n) {
      float gs = gmax[n] / 7.0f;
      uint16_t gh = oq_float_to_half(gs);
      g_h[(size_t)j * N + n] = gh;
      float ghf = oq_half_to_float(gh);
      if (ghf > ghmax[n]) ghmax[n] = ghf;
    }
    for (int k = j * group; k < (j + 1) * group; ++k)
      for (int n = 0; n < N; ++n) {
        float ghf = oq_half_to_float(g_h[(size_t)j * N + n]);
        float w = oq_half_to_float(W[(size_t)k * N + n]);
        int32_t q = 0;
        if (ghf > 0.0f) {
          float t = w / ghf;
          q = clampi(oq_rne((double)t), -7, 7);
        }
        q4[(size_t)k * N + n] = (int8_t)q;
      }
  }
  for (int n = 0; n < N; ++n) {
    float seven_g = 7.0f * ghmax[n];
    c[n] = seven_g / 127.0f;
  }
  for (int j = 0; j < G; ++j) {
    for (int n = 0; n < N; ++n) {
      float ghf = oq_half_to_float(g_h[(size_t)j * N + n]);
      uint16_t rh = 0;
      if (c[n] > 0.0f) {
        float ratio = ghf / c[n];
        rh = oq_float_to_half(ratio);
      }
      r_h[(size_t)j * N + n] = rh;
    }
    for (int k = j * group; k < (j + 1) * group; ++k)
      for (int n = 0; n < N; ++n) {
        double rf = oq_half_to_double(r_h[(size_t)j * N + n]);
        double prod = (double)q4[(size_t)k * N + n] * rf; /* exact in double */
        double q = oq_rne(prod);
        if (q > 127.0 || q < -127.0) bad = 1;
        q8[(size_t)k * N + n] = (int8_t)clampi(q, -127, 127);
      }
  }
  free(gmax);
  free(ghmax);
  return bad;
}

/* Nibble packing of INT4 codes (the pages give no byte layout; this one is
 * chosen so that a left shift by 4 and one mask turn four packed codes into
 * four int8 lanes holding 16*q, the "INT4 -> INT8 by <<4" step of [QQQ]
 * per-channel GEMM).
 * Output row n holds K/2 bytes.  For the 32-bit little-endian word covering
 * k0 .. k0+7 (k0 a multiple of 8), byte b (0..3) has
 *   low nibble  = q[k0 + b]      (two's complement, 4 bits)
 *   high nibble = q[k0 + 4 + b].                                   */
OQ_EXPORT void oq_pack_nibbles(const int8_t* q /*[K][N]*/, int K, int N, uint8_t* out /*[N][K/2]*/) {
  for (int n = 0; n < N; ++n) {
    for (int k0 = 0; k0 < K; k0 += 8) {
      for (int b = 0; b < 4; ++b) {
        uint8_t lo = (uint8_t)(q[(size_t)(k0 + b) * N + n] & 0xF);
        uint8_t hi = (uint8_t)(q[(size_t)(k0 + 4 + b) * N + n] & 0xF);
        out[(size_t)n * (K / 2) + k0 / 2 + b] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
}

/* ------------------------------------------------------------------------ */
/* O4: targeted momentum scaling ([Quaff] 目标动量缩放)                        */
/*   beta_i = max(1, sqrt( max_m |X[m, O_i]| / max_n |W[O_i, n]| ))  i in O  */
/*   s_i   <- gamma * s_i + (1 - gamma) * beta_i                              */
/* Readings: "W_i" is row i of W[K][N] (the weights that multiply input      */
/* channel i); the column max is over the raw X of this step; the state is   */
/* updated first and then used to quantize the same step; a zero weight row  */
/* gives beta = 1.  Arithmetic: fp32, in exactly this association.           */
/* ------------------------------------------------------------------------ */

OQ_EXPORT void oq_outlier_wmax(const uint16_t* W, int K, int N, const int32_t* O, int nO,
                               float* wmaxO) {
  (void)K;
  for (int i = 0; i < nO; ++i) {
    float m = 0.0f;
    for (int n = 0; n < N; ++n) {
      float v = fabsf(oq_half_to_float(W[(size_t)O[i] * N + n]));
      if (v > m) m = v;
    }
    wmaxO[i] = m;
  }
}

OQ_EXPORT void oq_momentum_update(const uint16_t* X, int M, int K, const int32_t* O, int nO,
                                  const float* wmaxO, float gamma, float* s) {
  for (int i = 0; i < nO; ++i) {
    float cmax = 0.0f;
    for (int m = 0; m < M; ++m) {
      float v = fabsf(oq_half_to_float(X[(size_t)m * K + O[i]]));
      if (v > cmax) cmax = v;
    }
    float beta = 1.0f;
    if (wmaxO[i] > 0.0f) {
      float ratio = cmax / wmaxO[i];
      float r = sqrtf(ratio);
      beta = (r > 1.0f) ? r : 1.0f;
    }
    float t1 = gamma * s[i];
    float one_minus = 1.0f - gamma;
    float t2 = one_minus * beta;
    s[i] = t1 + t2;
  }
}

/* ------------------------------------------------------------------------ */
/* O5: per-token symmetric INT8 activation quantization on X_hat = X (/) s   */
/*   x_hat[m,k] = X[m,k] / s_i  if k = O_i, else X[m,k]      (fp32 division)  */
/*   amax_m = max_k |x_hat[m,k]|;  a_m = amax_m / 127;  inv = 127 / amax_m    */
/*   Xq[m,k] = clamp(rne(x_hat * inv), -127, 127);  amax = 0 -> a = 0, 0s.    */
/*   XqO[m,i] = Xq[m, O_i]  (the outlier columns, compacted)                  */
/* ------------------------------------------------------------------------ */

OQ_EXPORT void oq_quant_act(const uint16_t* X, int M, int K, const int32_t* O, int nO,
                            const float* s, int8_t* Xq, float* a, int8_t* XqO) {
  float* xh = (float*)malloc(sizeof(float) * (size_t)K);
  for (int m = 0; m < M; ++m) {
    for (int k = 0; k < K; ++k) xh[k] = oq_half_to_float(X[(size_t)m * K + k]);
    for (int i = 0; i < nO; ++i) xh[O[i]] = xh[O[i]] / s[i];
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
      float v = fabsf(xh[k]);
      if (v > amax) amax = v;
    }
    float am = amax / 127.0f;
    float inv = (amax > 0.0f) ? (127.0f / amax) : 0.0f;
    a[m] = am;
    for (int k = 0; k < K; ++k) {
      float p = xh[k] * inv;
      Xq[(size_t)m * K + k] = (int8_t)clampi(oq_rne((double)p), -127, 127);
    }
    for (int i = 0; i < nO; ++i) XqO[(size_t)m * nO + i] = Xq[(size_t)m * K + O[i]];
  }
  free(xh);
}

/* ------------------------------------------------------------------------ */
/* O6: integer GEMM, int64 accumulation.  acc[m][n] = sum_k Xq[m][k]*B[k][n] */
/* B is the INT8 operand the tensor core sees: 16*q4 for the per-channel W4  */
/* path (the <<4 unpack), q8 for the g128 path, q for W8.                    */
/* Returns nonzero if any sum leaves the int32 range.                        */
/* ------------------------------------------------------------------------ */

OQ_EXPORT int oq_int_gemm(const int8_t* Xq, const int8_t* B, int M, int K, int N, int64_t* acc) {
  int overflow = 0;
  for (int m = 0; m < M; ++m) {
    for (int n = 0; n < N; ++n) {
      int64_t sum = 0;
      for (int k = 0; k < K; ++k) sum += (int64_t)Xq[(size_t)m * K + k] * (int64_t)B[(size_t)k * N + n];
      if (sum > INT32_MAX || sum < INT32_MIN) overflow = 1;
      acc[(size_t)m * N + n] = sum;
    }
  }
  return overflow;
}

/* Same as oq_int_gemm for a subset of rows (rows[r] indexes Xq's rows). */
OQ_EXPORT int oq_int_gemm_rows(const int8_t* Xq, const int8_t* B, int K, int N,
                               const int32_t* rows, int R, int64_t* acc) {
  int overflow = 0;
  for (int r = 0; r < R; ++r) {
    const int8_t* xr = Xq + (size_t)rows[r] * K;
    for (int n = 0; n < N; ++n) {
      int64_t sum = 0;
      for (int k = 0; k < K; ++k) sum += (int64_t)xr[k] * (int64_t)B[(size_t)k * N + n];
      if (sum > INT32_MAX || sum < INT32_MIN) overflow = 1;
      acc[(size_t)r * N + n] = sum;
    }
  }
  return overflow;
}

/* Same sums as oq_int_gemm_rows with the operand stored transposed,
 * Bt[n][k] = B[k][n], so each output channel's K codes are contiguous (the
 * same products added in the same k order; integer sums are exact). */
OQ_EXPORT int oq_int_gemm_rows_nk(const int8_t* Xq, const int8_t* Bt, int K, int N,
                                  const int32_t* rows, int R, int64_t* acc) {
  int overflow = 0;
  for (int r = 0; r < R; ++r) {
    const int8_t* xr = Xq + (size_t)rows[r] * K;
    for (int n = 0; n < N; ++n) {
      const int8_t* bn = Bt + (size_t)n * K;
      int64_t sum = 0;
      for (int k = 0; k < K; ++k) sum += (int64_t)xr[k] * (int64_t)bn[k];
      if (sum > INT32_MAX || sum < INT32_MIN) overflow = 1;
      acc[(size_t)r * N + n] = sum;
    }
  }
  return overflow;
}

/* ------------------------------------------------------------------------ */
/* O7: fp64 dequant epilogue plus the sparse compensation term              */
/* ([Quaff] 解耦 WAQ 公式: Y = X_hat W + X_hat[:,O] (s_O - 1) W_O, with the  */
/*  main term computed from pre-quantized weights).                          */
/*   y[m][n] = acc[m][n] * a_m * cscale_n                                    */
/*           + a_m * sum_i XqO[m][i] * (s_i - 1) * W[O_i][n]                 */
/* cscale_n is the scale of the operand codes (c_n / 16 for the per-channel  */
/* W4 path, c_n otherwise).  W_O stays in fp16 ("全精度").  Reading: the     */
/* compensation uses the same quantized activations as the main term.        */
/* rows[r] selects which rows of a / XqO the r-th row of acc belongs to.      */
/* ------------------------------------------------------------------------ */

OQ_EXPORT void oq_dequant(const int64_t* acc, const float* a, const float* cscale,
                          const int8_t* XqO, const float* s, const uint16_t* W, int N,
                          const int32_t* O, int nO, const int32_t* rows, int R, double* y) {
  for (int r = 0; r < R; ++r) {
    int m = rows[r];
    double am = (double)a[m];
    for (int n = 0; n < N; ++n) {
      double main_t = (double)acc[(size_t)r * N + n] * am * (double)cscale[n];
      double comp = 0.0;
      for (int i = 0; i < nO; ++i) {
        double sm1 = (double)s[i] - 1.0;
        comp += (double)XqO[(size_t)m * nO + i] * sm1 * oq_half_to_double(W[(size_t)O[i] * N + n]);
      }
      y[(size_t)r * N + n] = main_t + am * comp;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Input gradient for fine-tuning ([Quaff] 损失函数 / 训练策略: back-          */
/* propagation through the standard straight-through estimator).             */
/* Reading: under the estimator the quantizers are identities for the        */
/* gradient, so the layer is the linear map X -> (X / s) W_eff, where W_eff   */
/* holds the dequantized weights cscale_n * B[k][n] and, on the outlier rows  */
/* k = O_i, also the compensation term (s_i - 1) * W[O_i][n] of the          */
/* decoupled formula.  Its input gradient is                                 */
/*   dX[m][k] = ( sum_n dY[m][n] * W_eff[k][n] ) / s_k,   s_k = 1 off O.      */
/* fp64 throughout; dY is fp16 bits [M][N], B is the INT8 operand [K][N].     */
/* ------------------------------------------------------------------------ */

OQ_EXPORT void oq_backward_dx(const uint16_t* dY, int M, int N, int K, const int8_t* B, const float* cscale,
                              const uint16_t* W, const int32_t* O, int nO, const float* s, double* dX) {
  int* slot = (int*)malloc(sizeof(int) * (size_t)(K > 0 ? K : 1));
  for (int k = 0; k < K; ++k) slot[k] = -1;
  for (int i = 0; i < nO; ++i) slot[O[i]] = i;
  double* dy = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
  for (int m = 0; m < M; ++m) {
    for (int n = 0; n < N; ++n) dy[n] = oq_half_to_double(dY[(size_t)m * N + n]);
    for (int k = 0; k < K; ++k) {
      double g = 0.0;
      for (int n = 0; n < N; ++n) g += dy[n] * ((double)cscale[n] * (double)B[(size_t)k * N + n]);
      double sk = 1.0;
      if (slot[k] >= 0) {
        const int i = slot[k];
        sk = (double)s[i];
        double c = 0.0;
        for (int n = 0; n < N; ++n) c += dy[n] * oq_half_to_double(W[(size_t)O[i] * N + n]);
        g += (sk - 1.0) * c;
      }
      dX[(size_t)m * K + k] = g / sk;
    }
  }
  free(dy);
  free(slot);
}

/* ------------------------------------------------------------------------ */
/* FastFP16toINT8 ([QQQ] FastFP16toINT8优化): add 128 to move the value into  */
/* [0, 255], add 1024 so the eight bits of the UINT8 land in the low bits of */
/* the FP16 significand, then read them out of the bit pattern.              */
/* Two readings of "add 128, then add 1024":                                  */
/*   two_add:  t = fp16(fp16(v + 128) + 1024)     (two roundings)             */
/*   single:   t = fp16(v + 1152)                  (one rounding)             */
/* Both return the low byte XOR 0x80 as the int8 code, and the high byte of  */
/* t in *hi.                                                                  */
/* ------------------------------------------------------------------------ */

OQ_EXPORT int8_t oq_fast_fp16_to_int8_single(uint16_t v, uint8_t* hi) {
  double x = oq_half_to_double(v);
  uint16_t t = oq_double_to_half(x + 1152.0); /* exact sum in double, one rounding */
  if (hi) *hi = (uint8_t)(t >> 8);
  return (int8_t)((uint8_t)(t & 0xFF) ^ 0x80);
}

OQ_EXPORT int8_t oq_fast_fp16_to_int8_two_add(uint16_t v, uint8_t* hi) {
  double x = oq_half_to_double(v);
  uint16_t t1 = oq_double_to_half(x + 128.0);
  uint16_t t = oq_double_to_half(oq_half_to_double(t1) + 1024.0);
  if (hi) *hi = (uint8_t)(t >> 8);
  return (int8_t)((uint8_t)(t & 0xFF) ^ 0x80);
}

/* ------------------------------------------------------------------------ */
/* O9: GPTQ-style Hessian compensation ([QQQ] Hessian补偿), oracle only.     */
/*   H_F = 2 X_F^T X_F                                                        */
/*   delta_F = -(w_i - Q(w_i)) / [H_F^-1]_ii * (H_F^-1)[:, i]                  */
/* Columns are quantized in order 0..d-1; after column i the inverse of the   */
/* remaining block is obtained by the rank-one downdate                       */
/*   Hinv <- Hinv - Hinv[:, i] Hinv[i, :] / Hinv[i][i].                       */
/* Q is round-to-nearest-even on the grid step `scale` clamped to +-qmax.     */
/* X is [n_samples][d] (double), w is [d] (double, updated in place to the   */
/* quantized values), Hinv_out receives the inverse of H before any update.   */
/* Returns nonzero if H is not positive definite (Cholesky-free Gauss-Jordan  */
/* inverse hits a zero pivot).                                                */
/* ------------------------------------------------------------------------ */

static int invert_sym(double* A, int d, double* inv) {
  /* Gauss-Jordan with partial pivoting on a copy. */
  double* a = (double*)malloc(sizeof(double) * d * d);
  memcpy(a, A, sizeof(double) * d * d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) inv[i * d + j] = (i == j) ? 1.0 : 0.0;
  for (int c = 0; c < d; ++c) {
    int p = c;
    for (int r = c + 1; r < d; ++r)
      if (fabs(a[r * d + c]) > fabs(a[p * d + c])) p = r;
    if (a[p * d + c] == 0.0) {
      free(a);
      return 1;
    }
    if (p != c) {
      for (int j = 0; j < d; ++j) {
        double t = a[c * d + j]; a[c * d + j] = a[p * d + j]; a[p * d + j] = t;
        t = inv[c * d + j]; inv[c * d + j] = inv[p * d + j]; inv[p * d + j] = t;
      }
    }
    double piv = a[c * d + c];
    for (int j = 0; j < d; ++j) {
      a[c * d + j] /= piv;
      inv[c * d + j] /= piv;
    }
    for (int r = 0; r < d; ++r) {
      if (r == c) continue;
      double f = a[r * d + c];
      if (f == 0.0) continue;
      for (int j = 0; j < d; ++j) {
        a[r * d + j] -= f * a[c * d + j];
        inv[r * d + j] -= f * inv[c * d + j];
      }
    }
  }
  free(a);
  return 0;
}

OQ_EXPORT int oq_gptq_hessian(const double* X, int ns, int d, double* H) {
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int t = 0; t < ns; ++t) acc += X[t * d + i] * X[t * d + j];
      H[i * d + j] = 2.0 * acc;
    }
  return 0;
}

/* One compensation step on column i: returns delta (length d) given the
 * current inverse Hinv of the not-yet-quantized block (entries of already
 * quantized columns are ignored by the caller). */
OQ_EXPORT void oq_gptq_delta(const double* w, const double* Hinv, int d, int i, double q_i,
                             double* delta) {
  double f = -(w[i] - q_i) / Hinv[i * d + i];
  for (int j = 0; j < d; ++j) delta[j] = f * Hinv[j * d + i];
}

/* Rank-one downdate that removes column i from the inverse of the remaining
 * block: Hinv <- Hinv - Hinv[:, i] Hinv[i, :] / Hinv[i][i]. */
OQ_EXPORT void oq_gptq_downdate(double* Hinv, int d, int i) {
  double piv = Hinv[i * d + i];
  double* col = (double*)malloc(sizeof(double) * d);
  double* row = (double*)malloc(sizeof(double) * d);
  for (int j = 0; j < d; ++j) { col[j] = Hinv[j * d + i]; row[j] = Hinv[i * d + j]; }
  for (int r = 0; r < d; ++r)
    for (int c = 0; c < d; ++c) Hinv[r * d + c] -= col[r] * row[c] / piv;
  free(col);
  free(row);
}

OQ_EXPORT int oq_gptq_quantize(const double* X, int ns, int d, double* w, double scale, int qmax,
                               double* Hinv_out, double* deltas /* [d][d] or NULL */) {
  double* H = (double*)malloc(sizeof(double) * d * d);
  double* Hinv = (double*)malloc(sizeof(double) * d * d);
  double* delta = (double*)malloc(sizeof(double) * d);
  oq_gptq_hessian(X, ns, d, H);
  if (invert_sym(H, d, Hinv)) {
    free(H); free(Hinv); free(delta);
    return 1;
  }
  if (Hinv_out) memcpy(Hinv_out, Hinv, sizeof(double) * d * d);
  for (int i = 0; i < d; ++i) {
    double q = (double)clampi(oq_rne(w[i] / scale), -qmax, qmax) * scale;
    oq_gptq_delta(w, Hinv, d, i, q, delta);
    for (int j = i; j < d; ++j) w[j] += delta[j];
    w[i] = q; /* delta_i = q - w_i up to rounding; keep the grid value exactly */
    if (deltas) memcpy(deltas + (size_t)i * d, delta, sizeof(double) * d);
    oq_gptq_downdate(Hinv, d, i);
  }
  free(H); free(Hinv); free(delta);
  return 0;
}

/* The same compensation for a whole layer: W is [d][N] (input channel i is
 * row i, output channel n is column n) and every output channel is the
 * weight vector w of oq_gptq_quantize with its own grid step scale[n].  H,
 * its inverse and the downdate sequence do not depend on w, so they are
 * computed once and shared; each column goes through exactly the steps of
 * oq_gptq_quantize (quantize column i, delta from column i of the current
 * inverse, update the not-yet-quantized entries, keep the grid value).
 * codes[i][n] receives the integer grid index clamp(rne(w_i / scale_n)).
 * Returns nonzero if H is singular. */
OQ_EXPORT int oq_gptq_quantize_layer(const double* X, int ns, int d, int N, double* W, const double* scale,
                                     int qmax, int8_t* codes, double* Hinv_out) {
  double* H = (double*)malloc(sizeof(double) * d * d);
  double* Hinv = (double*)malloc(sizeof(double) * d * d);
  double* w = (double*)malloc(sizeof(double) * d);
  double* delta = (double*)malloc(sizeof(double) * d);
  oq_gptq_hessian(X, ns, d, H);
  if (invert_sym(H, d, Hinv)) {
    free(H); free(Hinv); free(w); free(delta);
    return 1;
  }
  if (Hinv_out) memcpy(Hinv_out, Hinv, sizeof(double) * d * d);
  for (int i = 0; i < d; ++i) {
    for (int n = 0; n < N; ++n) {
      for (int j = 0; j < d; ++j) w[j] = W[(size_t)j * N + n];
      int32_t c = clampi(oq_rne(w[i] / scale[n]), -qmax, qmax);
      double q = (double)c * scale[n];
      oq_gptq_delta(w, Hinv, d, i, q, delta);
      for (int j = i; j < d; ++j) W[(size_t)j * N + n] = w[j] + delta[j];
      W[(size_t)i * N + n] = q;
      codes[(size_t)i * N + n] = (int8_t)c;
    }
    oq_gptq_downdate(Hinv, d, i);
  }
  free(H); free(Hinv); free(w); free(delta);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* QQQ adaptive smoothing ([QQQ] 自适应平滑), the threshold search.          */
/* Readings (the page's formulas are partly garbled):                       */
/*  - the smoothed channels are T(sigma) = { t : max_m |X[m,t]| > sigma }    */
/*    (only channels with significant outliers are smoothed);               */
/*  - s_t = sqrt(max_m|X[m,t]| / max_n|W[t,n]|) on T, 1 elsewhere (the       */
/*    migration strength 1/2; 1 when a maximum is 0);                        */
/*  - the smoothed tensors are rounded to fp16 before quantization:          */
/*    Xh[m,t] = fp16(X[m,t] / s_t), Wh[t,n] = fp16(W[t,n] * s_t) on T, and   */
/*    0 off T, so Q(X_T / s) and Q(W_T * s) are the layer's own quantizers   */
/*    (per-token INT8, per-channel INT4) applied to the T parts;            */
/*  - loss(sigma) = sum_{m,n} ( a_m c'_n acc[m][n] - (X_T W_T)[m][n] )^2     */
/*    in fp64, acc the integer product of the codes;                         */
/*  - sigma_j = max|X| * j / G for j = 0 .. G-1 (the grid over               */
/*    [0, max|X|]); the search returns the first j of least loss.            */
/* X fp16 [M][K], W fp16 [K][N]; loss [G]; returns the best index.           */
/* ------------------------------------------------------------------------ */
OQ_EXPORT int oq_smooth_search(const uint16_t* X, int M, int K, const uint16_t* W, int N, int G, double* loss) {
  float* cmax = (float*)calloc((size_t)K, sizeof(float));
  float* wmax = (float*)calloc((size_t)K, sizeof(float));
  float* sv = (float*)malloc(sizeof(float) * (size_t)K);
  uint16_t* Xh = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)M * K);
  uint16_t* Wh = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)K * N);
  int8_t* xq = (int8_t*)malloc((size_t)M * K);
  float* a = (float*)malloc(sizeof(float) * (size_t)M);
  int8_t* wq = (int8_t*)malloc((size_t)K * N);
  float* c = (float*)malloc(sizeof(float) * (size_t)N);
  float xall = 0.0f;
  for (int m = 0; m < M; ++m)
    for (int t = 0; t < K; ++t) {
      float v = fabsf(oq_half_to_float(X[(size_t)m * K + t]));
      if (v > cmax[t]) cmax[t] = v;
      if (v > xall) xall = v;
    }
  for (int t = 0; t < K; ++t)
    for (int n = 0; n < N; ++n) {
      float v = fabsf(oq_half_to_float(W[(size_t)t * N + n]));
      if (v > wmax[t]) wmax[t] = v;
    }
  int best = 0;
  for (int j = 0; j < G; ++j) {
    float sigma = xall * (float)j / (float)G;
    for (int t = 0; t < K; ++t) {
      int in_t = cmax[t] > sigma;
      float st = 1.0f;
      if (in_t && cmax[t] > 0.0f && wmax[t] > 0.0f) st = sqrtf(cmax[t] / wmax[t]);
      sv[t] = in_t ? st : 0.0f;  /* 0 marks a channel outside T */
    }
    for (int m = 0; m < M; ++m)
      for (int t = 0; t < K; ++t)
        Xh[(size_t)m * K + t] = sv[t] > 0.0f ? oq_float_to_half(oq_half_to_float(X[(size_t)m * K + t]) / sv[t]) : 0;
    for (int t = 0; t < K; ++t)
      for (int n = 0; n < N; ++n)
        Wh[(size_t)t * N + n] = sv[t] > 0.0f ? oq_float_to_half(oq_half_to_float(W[(size_t)t * N + n]) * sv[t]) : 0;
    oq_quant_act(Xh, M, K, NULL, 0, NULL, xq, a, NULL);
    oq_quant_weight_per_channel(Wh, K, N, 7, wq, c);
    double L = 0.0;
    for (int m = 0; m < M; ++m)
      for (int n = 0; n < N; ++n) {
        int64_t acc = 0;
        double ref = 0.0;
        for (int t = 0; t < K; ++t) {
          acc += (int64_t)xq[(size_t)m * K + t] * (int64_t)(16 * wq[(size_t)t * N + n]);
          if (sv[t] > 0.0f)
            ref += oq_half_to_double(X[(size_t)m * K + t]) * oq_half_to_double(W[(size_t)t * N + n]);
        }
        double y = (double)acc * (double)a[m] * ((double)c[n] / 16.0);
        double d = y - ref;
        L += d * d;
      }
    loss[j] = L;
    if (L < loss[best]) best = j;
  }
  free(cmax); free(wmax); free(sv); free(Xh); free(Wh); free(xq); free(a); free(wq); free(c);
  return best;
}

/* ------------------------------------------------------------------------ */
/* OffQ: outliers absorbed as an offset ([OffQ] 方法: 通过偏移量进行吸收     */
/* (Hadamard 旋转), 分组实现).  Readings (the pages fix no precision or      */
/* normalisation):                                                          */
/*  - groups of 128 consecutive channels (K % 128 == 0); the activations    */
/*    are taken after the offline top-1 PCA rotation, the outlier of a      */
/*    group in its first channel;                                           */
/*  - the partially random Hadamard matrix is D H, H the 128 x 128 Sylvester */
/*    matrix h(i, j) = (-1)^popcount(i & j) and D = diag(d) with d_0 = 1     */
/*    and d_i = +-1 given (seeded): its first row is all ones, so a value   */
/*    in channel 0 adds the same amount to every transformed channel;       */
/*  - y_g = x_g (D H) for each token and group, unnormalised (exact in fp64: */
/*    sums of +-fp16 values); the 1/128 of the inverse goes to the weights;  */
/*  - per (token, group) asymmetric INT4 with the group minimum as the     */
/*    offset ("absorbed into the zero point"): lo = min y, hi = max y,      */
/*    sd = (hi - lo) / 15, q = clamp(rne((y - lo) / sd), 0, 15), all in      */
/*    fp64, so y ~ q sd + lo; stored: q (0..15), fp32(sd) and fp32(lo); a    */
/*    constant group (hi == lo) gets sd = 0 and q = 0;                       */
/*  - weights: W'_g = (1/128) H D W_g (so y_g W'_g = x_g W_g), fp64 then     */
/*    fp32, quantized per output channel to INT4 like the W4A8 layer, with  */
/*    the operand B = 16 q and its per-group column sums kept for the        */
/*    offset term: y_m W' = sum_g c'_n (sd acc_g + lo colsum_g).             */
/* ------------------------------------------------------------------------ */
static int hsign(int i, int j) { return __builtin_popcount((unsigned)(i & j)) & 1 ? -1 : 1; }

OQ_EXPORT void oq_offq_transform(const uint16_t* X, int M, int K, const int8_t* d, double* Y) {
  for (int m = 0; m < M; ++m)
    for (int g = 0; g < K / 128; ++g)
      for (int j = 0; j < 128; ++j) {
        double acc = 0.0;
        for (int i = 0; i < 128; ++i)
          acc += oq_half_to_double(X[(size_t)m * K + g * 128 + i]) * (double)d[i] * (double)hsign(i, j);
        Y[(size_t)m * K + g * 128 + j] = acc;
      }
}

OQ_EXPORT void oq_offq_quant_act(const uint16_t* X, int M, int K, const int8_t* d, int8_t* Xq, float* scale,
                                 float* offset) {
  const int G = K / 128;
  double* y = (double*)malloc(sizeof(double) * (size_t)M * K);
  oq_offq_transform(X, M, K, d, y);
  for (int m = 0; m < M; ++m)
    for (int g = 0; g < G; ++g) {
      const double* yg = y + (size_t)m * K + g * 128;
      double lo = yg[0], hi = yg[0];
      for (int j = 1; j < 128; ++j) {
        if (yg[j] < lo) lo = yg[j];
        if (yg[j] > hi) hi = yg[j];
      }
      const double sd = (hi - lo) / 15.0;
      scale[(size_t)m * G + g] = (float)sd;
      offset[(size_t)m * G + g] = (float)lo;
      for (int j = 0; j < 128; ++j)
        Xq[(size_t)m * K + g * 128 + j] = (int8_t)(sd > 0.0 ? clampi(oq_rne((yg[j] - lo) / sd), 0, 15) : 0);
    }
  free(y);
}

OQ_EXPORT void oq_offq_rotate_weights(const uint16_t* W, int K, int N, const int8_t* d, float* Wr) {
  for (int g = 0; g < K / 128; ++g)
    for (int n = 0; n < N; ++n)
      for (int j = 0; j < 128; ++j) {
        double acc = 0.0;
        for (int i = 0; i < 128; ++i)
          acc += (double)hsign(j, i) * (double)d[i] * oq_half_to_double(W[(size_t)(g * 128 + i) * N + n]);
        Wr[(size_t)(g * 128 + j) * N + n] = (float)(acc / 128.0);
      }
}

/* Per-output-channel symmetric quantization of fp32 weights (the rule of
 * oq_quant_weight_per_channel on fp32 input). */
OQ_EXPORT void oq_quant_weight_per_channel_f32(const float* W, int K, int N, int qmax, int8_t* codes, float* scale) {
  const float fq = (float)qmax;
  float* wmax = (float*)calloc((size_t)(N > 0 ? N : 1), sizeof(float));
  for (int k = 0; k < K; ++k)
    for (int n = 0; n < N; ++n) {
      float v = fabsf(W[(size_t)k * N + n]);
      if (v > wmax[n]) wmax[n] = v;
    }
  for (int n = 0; n < N; ++n) scale[n] = wmax[n] / fq;
  for (int k = 0; k < K; ++k)
    for (int n = 0; n < N; ++n) {
      float inv = (wmax[n] > 0.0f) ? (fq / wmax[n]) : 0.0f;
      float p = W[(size_t)k * N + n] * inv;
      codes[(size_t)k * N + n] = (int8_t)clampi(oq_rne((double)p), -qmax, qmax);
    }
  free(wmax);
}

/* y[r][n] = cscale[n] * sum_g (scale[m][g] * acc_g[m][n] + offset[m][g] *
 * colsum_g[n]) in fp64, acc_g = sum_{k in g} Xq[m][k] Bt[n][k] and colsum_g
 * = sum_{k in g} Bt[n][k] exact (int64); m = rows[r]. */
OQ_EXPORT void oq_offq_gemm_rows(const int8_t* Xq, const float* scale, const float* offset, const int8_t* Bt,
                                 const float* cscale, int K, int N, const int32_t* rows, int R, double* y) {
  const int G = K / 128;
  for (int r = 0; r < R; ++r) {
    const int m = rows[r];
    for (int n = 0; n < N; ++n) {
      double sum = 0.0;
      for (int g = 0; g < G; ++g) {
        int64_t acc = 0, cs = 0;
        for (int k = g * 128; k < (g + 1) * 128; ++k) {
          acc += (int64_t)Xq[(size_t)m * K + k] * (int64_t)Bt[(size_t)n * K + k];
          cs += (int64_t)Bt[(size_t)n * K + k];
        }
        sum += (double)scale[(size_t)m * G + g] * (double)acc + (double)offset[(size_t)m * G + g] * (double)cs;
      }
      y[(size_t)r * N + n] = sum * (double)cscale[n];
    }
  }
}

OQ_EXPORT int oq_invert(const double* A, int d, double* inv) {
  double* a = (double*)malloc(sizeof(double) * d * d);
  memcpy(a, A, sizeof(double) * d * d);
  int r = invert_sym(a, d, inv);
  free(a);
  return r;
}
