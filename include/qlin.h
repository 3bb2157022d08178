/*
 * qlin.h -- C ABI of the B200 (sm_100a) outlier-aware quantized linear layer
 *
 *     Y = Q(X) . Q(W)
 *       = a (.) [ c' (.) (Xq . B) ]  +  a (.) [ XqO . diag(s_O - 1) . W_O ]
 *
 * Three stages run on the GPU:
 *   1. per-token symmetric INT8 activation quantization on X_hat = X (/) s,
 *      where s is the targeted momentum scale kept only on the outlier
 *      channel set O ("Quaff: Quantized Parameter-Efficient Fine-Tuning under
 *      Outlier Spatial Stability Hypothesis", sections 目标动量缩放 and
 *      整体框架);
 *   2. an INT8 tensor-core GEMM whose weight operand comes from one of three
 *      packed formats -- INT4 per output channel unpacked to INT8 by a left
 *      shift of 4, INT4 with g=128 group scales requantized to INT8 through
 *      the folded group/channel ratio, or plain INT8 per channel ("QQQ:
 *      Quality Quattuor-Bit Quantization for Large Language Models", section
 *      W4A8 GEMM内核: per-channel GEMM, per-group GEMM, FusedDequantQuant,
 *      FastFP16toINT8);
 *   3. a fused INT32 -> FP16 dequant epilogue that adds the sparse outlier
 *      compensation term X_hat[:,O] (s_O - 1) W_O (Quaff notes, section
 *      关键设计, decoupled WAQ formula).
 *
 * Conventions for every entry point
 *   - "device" pointers are CUDA device memory owned by the caller; "host"
 *     pointers are ordinary host memory owned by the caller.  The library
 *     never allocates, frees or retains memory and keeps no state across
 *     calls other than a per-thread last-error string and one device error
 *     word (see qlin_poll_device_status).
 *   - fp16 values are IEEE binary16 bit patterns (uint16_t).
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Every call only enqueues work on `stream` and returns without
 *     synchronizing; argument errors are detected on the host before anything
 *     is enqueued and leave all buffers untouched.
 *   - Matrices are row-major with dense rows (no padding) unless stated.
 *   - Device pointers must be 16-byte aligned (QLIN_ERR_ALIGN otherwise).
 *   - Shapes: K % 32 == 0, N % 16 == 0, 32 <= K <= 65536, N >= 16; for the
 *     g128 format K % 128 == 0; 0 <= n_outlier <= min(K, 4096).
 *   - Workspaces: buffers whose size comes from the matching *_workspace
 *     call.  A workspace must be zero-filled before its first use (for
 *     example with cudaMemsetAsync); every successful call leaves it
 *     zero-filled again in the parts that must start at zero, so it can be
 *     reused by later calls on the same stream without clearing.  Calls that
 *     share a workspace must not overlap on the GPU.
 *   - No entry point is thread-hostile; concurrent calls on different
 *     streams must use different outputs and workspaces.
 */
#ifndef QLIN_H_
#define QLIN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLIN_API __attribute__((visibility("default")))
#else
#define QLIN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLIN_OK = 0,
  QLIN_ERR_ARG = 1,       /* null pointer, negative size, bad O (not sorted/unique/in range), bad fmt */
  QLIN_ERR_SHAPE = 2,     /* shape outside the supported set listed above */
  QLIN_ERR_ALIGN = 3,     /* a device pointer is not 16-byte aligned */
  QLIN_ERR_WORKSPACE = 4, /* workspace smaller than the *_workspace size */
  QLIN_ERR_CUDA = 5,      /* a CUDA runtime / driver call or a launch failed */
  QLIN_ERR_TIMEOUT = 6    /* a bounded device-side wait gave up (see qlin_poll_device_status) */
} qlin_status;

typedef enum {
  QLIN_W4_PERCHANNEL = 0, /* INT4 codes in [-7,7], one fp32 scale per output channel */
  QLIN_W4_G128 = 1,       /* INT4 codes in [-7,7] per group of 128 input channels, requantized to INT8 */
  QLIN_W8_PERCHANNEL = 2  /* INT8 codes in [-127,127], one fp32 scale per output channel */
} qlin_wfmt;

/* Packed weights of one linear layer with K input and N output channels.
 * Plain descriptor: every pointer is device memory owned by the caller, and
 * qlin_weights_bind() can carve all of them out of one allocation.
 *
 *   codes        Tile-major, one contiguous block per (channel tile tn,
 *                input tile kb) of 128 output channels x 128 input channels,
 *                blocks ordered tn-major: block (tn, kb) starts at
 *                (tn * ceil(K/128) + kb) * block_bytes.  Row r of a block is
 *                channel 128*tn + r; channels >= N and inputs >= K are zero.
 *                W4 formats: 8192-byte blocks, 64 bytes per row.  In the
 *                32-bit little-endian word of a row that covers inputs
 *                k0..k0+7, byte b (0..3) holds q[k0+b] in its low nibble and
 *                q[k0+4+b] in its high nibble (two's complement); then
 *                (word << 4) & 0xF0F0F0F0 holds the INT8 lanes 16*q[k0..k0+3]
 *                and word & 0xF0F0F0F0 the lanes 16*q[k0+4..k0+7].  The
 *                16-byte chunk c (inputs 32c..32c+31 of the tile) of row r
 *                sits at chunk c ^ ((r / 2) % 4) of that row, so one thread
 *                per row can read a block without shared-memory bank
 *                conflicts.
 *                W8 format: 16384-byte blocks, 128 bytes per row, stored with
 *                the tensor core's 128-byte swizzle: the 16-byte chunk c
 *                (inputs 16c..16c+15 of the tile) of row r sits at chunk
 *                c ^ (r % 8) of that row.
 *   chan_scale   c_n, fp32 [N].  Per-channel formats: c_n = max_k|W[k][n]| / qmax
 *                (qmax = 7 or 127).  g128: c_n = 7 * max_j g[j][n] / 127.
 *   group_scale  g128 only: g[j][n] = fp16(max_{k in group j}|W[k][n]| / 7), fp16 [K/128][N].
 *   fold_ratio   g128 only: r[j][n] = fp16(g[j][n] / c_n), fp16 [K/128][N].
 *   outlier_idx  O, int32 [n_outlier], strictly increasing, in [0, K).
 *   W_Ot         The outlier rows of W kept in fp16 ("full precision"),
 *                transposed and tiled: one 16384-byte block per (channel
 *                tile tn, outlier tile ib) of 128 channels x 64 outliers,
 *                ordered tn-major; row r holds W[O_i][128*tn + r] for
 *                i = 64*ib .. 64*ib+63 (128 bytes) with the same 128-byte
 *                swizzle as the W8 codes; padding is zero.
 *   wmax_O       fp32 [n_outlier]: max_n |W[O_i][n]| (the weight side of beta).
 */
typedef struct {
  int32_t K;
  int32_t N;
  int32_t fmt;           /* qlin_wfmt */
  int32_t group;         /* 128 for QLIN_W4_G128, else 0 */
  int32_t n_outlier;     /* |O| */
  int32_t n_outlier_pad; /* n_outlier rounded up to a multiple of 8 (row stride of the
                            compensation operand in the GEMM workspace) */
  void* codes;
  float* chan_scale;
  uint16_t* group_scale;
  uint16_t* fold_ratio;
  int32_t* outlier_idx;
  uint16_t* W_Ot;
  float* wmax_O;
} qlin_weights;

/* Human-readable name of a status code (static string). */
QLIN_API const char* qlin_status_string(qlin_status status);

/* Description of the last error returned on the calling host thread
 * (static thread-local buffer, valid until the next call on that thread). */
QLIN_API const char* qlin_last_error(void);

/* Bytes needed to hold all packed buffers of a layer (each sub-buffer
 * aligned to 256 bytes).  Host-only; enqueues nothing. */
QLIN_API qlin_status qlin_weights_bytes(int32_t K, int32_t N, int32_t fmt, int32_t n_outlier,
                               size_t* bytes);

/* Fill `w` with the shape fields and sub-buffer pointers carved out of the
 * device allocation [base, base + bytes).  Host-only; enqueues nothing and
 * does not touch the memory.  base must be 256-byte aligned. */
QLIN_API qlin_status qlin_weights_bind(qlin_weights* w, int32_t K, int32_t N, int32_t fmt,
                              int32_t n_outlier, void* base, size_t bytes);

/* Quantize and pack one layer's weights (offline step of both pages: Quaff
 * quantizes the frozen W to W_int and keeps the outlier rows W_O in full
 * precision; QQQ stores INT4 codes with per-channel or per-group scales and
 * folds the group scale by the channel scale).
 *   W       device fp16 [K][N] (row k = input channel k).
 *   O_host  host int32 [w->n_outlier], strictly increasing, in [0, K); read
 *           during the call only.  May be NULL when n_outlier == 0.
 *   w       bound descriptor (qlin_weights_bind) whose buffers are written.
 * Codes: per-channel q = clamp(rne(w * (qmax / wmax_n)), -qmax, qmax) in
 * fp32; g128 q4 = clamp(rne(w / g), -7, 7) and the INT8 operand
 * q8 = rne(q4 * r) with one rounding. */
QLIN_API qlin_status qlin_pack_weights(const uint16_t* W, const int32_t* O_host, const qlin_weights* w,
                              void* stream);

/* Workspace for qlin_quant_act (holds the outlier column maxima and a
 * completion counter).  0 when n_outlier == 0. */
QLIN_API qlin_status qlin_quant_act_workspace(int32_t M, const qlin_weights* w, size_t* bytes);

/* Stage 1: targeted momentum update and per-token INT8 quantization.
 *   X        device fp16 [M][K] activations (token-major).
 *   s        device fp32 [n_outlier] momentum state, read and (when
 *            update_momentum != 0) updated in place:
 *              beta_i = max(1, sqrt(max_m|X[m,O_i]| / wmax_O[i]))   (1 if wmax_O[i] == 0)
 *              s_i   <- gamma * s_i + (1 - gamma) * beta_i          (fp32, this association)
 *            then the updated s quantizes this same X.
 *   Xq       device int8 [M][K]: clamp(rne(x_hat * (127 / amax_m)), -127, 127),
 *            x_hat[m,k] = X[m,k] / s_i for k = O_i, else X[m,k].
 *   a        device fp32 [M]: amax_m / 127 (0 for an all-zero token).
 *   XqO      device int8 [M][n_outlier]: Xq[m, O_i] (may be NULL when n_outlier == 0).
 * M may be 0 (nothing is enqueued). */
QLIN_API qlin_status qlin_quant_act(const uint16_t* X, int32_t M, const qlin_weights* w, float* s,
                           float gamma, int32_t update_momentum, int8_t* Xq, float* a,
                           int8_t* XqO, void* workspace, size_t ws_bytes, void* stream);

/* qlin_quant_act without a workspace argument, for callers that cannot
 * allocate device memory: code running inside a host framework that owns all
 * GPU memory and forbids cudaMalloc once it has started (a plugin of an
 * inference server, a custom pool), or a latency-bound loop that must not
 * allocate because cudaMalloc may synchronize the device and take unbounded
 * time.  The pages have no counterpart to this entry point; it only changes
 * where the momentum update's scratch lives.
 * Same arguments and results as qlin_quant_act.  The scratch (outlier column
 * maxima and a completion counter) is a fixed array inside the library
 * (4.25 KiB on every GPU that loads it: 1024 + 64 32-bit words, held until
 * the process exits), so:
 *   - n_outlier must be <= 1024, else QLIN_ERR_SHAPE and nothing is enqueued;
 *   - no memory is allocated or freed; the call clears the part of the
 *     scratch it uses with cudaMemsetAsync on `stream` before its kernels;
 *   - every call on a device shares that one scratch: calls whose work
 *     overlaps on the GPU (different streams, or different host threads)
 *     race and may produce wrong momentum updates; serialize them;
 *   - the first call on each device looks up the scratch's device address
 *     (cudaGetSymbolAddress with that device current) and caches it; make
 *     that first call before any stream capture. */
QLIN_API qlin_status qlin_quant_act_noalloc(const uint16_t* X, int32_t M, const qlin_weights* w, float* s,
                                            float gamma, int32_t update_momentum, int8_t* Xq, float* a,
                                            int8_t* XqO, void* stream);

/* Data-parallel split of the momentum update, for callers that shard tokens
 * across GPUs and must keep one s on every replica: qlin_outlier_colmax
 * writes cmax[i] = max_m |X[m, O_i]| (device fp32 [n_outlier]) over this
 * GPU's tokens; the caller reduces cmax with MAX across ranks; then
 * qlin_momentum_update applies the recurrence above to s in place, and
 * qlin_quant_act(..., update_momentum = 0, ...) quantizes. */
QLIN_API qlin_status qlin_outlier_colmax(const uint16_t* X, int32_t M, const qlin_weights* w, float* cmax,
                                void* stream);
QLIN_API qlin_status qlin_momentum_update(const qlin_weights* w, const float* cmax, float* s, float gamma,
                                 void* stream);

/* Workspace for qlin_gemm at token count M. */
QLIN_API qlin_status qlin_gemm_workspace(int32_t M, const qlin_weights* w, size_t* bytes);

/* Stages 2 and 3: INT8 tensor-core GEMM with fused dequant + compensation.
 *   Xq, a, XqO, s  as produced by qlin_quant_act (s is the state used to
 *                  quantize; only read).
 *   Y         device fp16 [M][N]:
 *               Y[m][n] = fp16( a_m * ( c'_n * acc[m][n] + comp[m][n] ) )
 *               acc[m][n]  = sum_k Xq[m][k] * B[k][n] (exact int32), B the
 *                            INT8 operand (16*q, q8 or q);
 *               c'_n       = c_n / 16 (W4 per-channel) or c_n;
 *               comp[m][n] = sum_i XqO[m][i] * (s_i - 1) * W_Ot[n][i], with
 *                            each product u = XqO*(s-1) formed in fp32 and
 *                            carried as fp16(u) + fp16(u - fp16(u)), the sum
 *                            accumulated in fp32 on the tensor cores.
 *   acc_debug NULL, or device int32 [M][N] receiving acc (for parity checks).
 * Y must not alias any input. */
QLIN_API qlin_status qlin_gemm(const qlin_weights* w, const int8_t* Xq, const float* a, const int8_t* XqO,
                      const float* s, int32_t M, uint16_t* Y, int32_t* acc_debug,
                      void* workspace, size_t ws_bytes, void* stream);

/* Workspace for qlin_forward at token count M (holds Xq, a, XqO and the
 * scratch of the two stages). */
QLIN_API qlin_status qlin_forward_workspace(int32_t M, const qlin_weights* w, size_t* bytes);

/* The whole layer: qlin_quant_act followed by qlin_gemm on one stream, with
 * the compensation operand produced directly by the quantization kernel. */
QLIN_API qlin_status qlin_forward(const uint16_t* X, int32_t M, const qlin_weights* w, float* s,
                         float gamma, int32_t update_momentum, uint16_t* Y, void* workspace,
                         size_t ws_bytes, void* stream);

/* Several independent layers in one pass: stage 1 of every problem in one
 * quantization launch, then stages 2 and 3 of every problem in one
 * persistent GEMM launch whose CTAs stream the problems' weights back to
 * back, so the per-launch start-up, the first weight bytes' latency and
 * each problem's split-K reduction and epilogue overlap the other problems'
 * weight streaming.  For decode-sized token counts, where a single layer's
 * weights take a few microseconds to stream: independent projections of
 * one input (q / k / v, gate / up), or many adapters or experts.  Problem q
 * computes exactly what qlin_forward(X[q], M, w[q], s[q], gamma,
 * update_momentum, Y[q], ...) computes (the same arithmetic, bit for bit).
 *   count     1 .. 32 problems; every w[q] has the same format.
 *   w, X, s, Y  host arrays of `count` pointers: packed weights, device X
 *             fp16 [M][K_q], device momentum state fp32 [n_outlier_q] (may
 *             be NULL for a problem without outliers), device Y fp16
 *             [M][N_q]; distinct Y buffers.
 *   M         0 .. 64 tokens, the same for every problem (QLIN_ERR_SHAPE above).
 *   workspace one buffer for the group, of qlin_forward_grouped_workspace
 *             bytes, 256-byte aligned, zero-filled before its first use
 *             and left that way. */
QLIN_API qlin_status qlin_forward_grouped_workspace(int32_t count, const qlin_weights* const* w, int32_t M,
                                                    size_t* bytes);
QLIN_API qlin_status qlin_forward_grouped(int32_t count, const qlin_weights* const* w, const uint16_t* const* X,
                                          float* const* s, uint16_t* const* Y, int32_t M, float gamma,
                                          int32_t update_momentum, void* workspace, size_t ws_bytes, void* stream);

/* Input gradient of the layer for fine-tuning (Quaff notes, 损失函数 /
 * 训练策略: the quantizers are passed by the standard straight-through
 * estimator, so the gradient is that of the decoupled layer of 解耦 WAQ 公式
 * before rounding):
 *   dX[m][k]     = sum_n dY[m][n] Weff[k][n]
 *   Weff[k][n]   = c'_n B[k][n]                                 k not in O
 *   Weff[O_i][n] = (c'_n B[O_i][n] + (s_i - 1) W_O[i][n]) / s_i
 * with B, c'_n the forward's INT8 operand and channel factor (16 q and c_n/16
 * for per-channel INT4, the requantized q8 and c_n for g128, q and c_n for
 * INT8) and W_O the fp16 outlier rows kept in `W_Ot`.  The frozen quantized
 * weights get no gradient.
 *   dY  fp16 [M][N] row-major, device.
 *   s   fp32 [n_outlier], device: the scales of the forward pass whose
 *       gradient this is (ignored and may be NULL when n_outlier = 0).
 *   dX  fp16 [M][K] row-major, device, fully overwritten.
 *   workspace  optional (NULL, or smaller than qlin_backward_dx_workspace):
 *       with it, the tiles of an incomplete last wave of SMs are split along
 *       the reduction and their fp32 partials pass through it; it must be
 *       zero-filled before its first use and is left that way.
 * Arithmetic: Weff is rounded to fp16 (the outlier rows after blending in
 * fp32), products are summed in fp32 on the tensor cores (split tiles add
 * their fp32 partials), dX is rounded to fp16 once.  M = 0 is a no-op; M
 * above 65535 * 128 returns QLIN_ERR_SHAPE; pointers must be 16-byte aligned
 * and the workspace 256-byte aligned (QLIN_ERR_ALIGN). */
QLIN_API qlin_status qlin_backward_dx_workspace(int32_t M, const qlin_weights* w, size_t* bytes);
QLIN_API qlin_status qlin_backward_dx(const qlin_weights* w, const uint16_t* dY, int32_t M, const float* s,
                                      uint16_t* dX, void* workspace, size_t ws_bytes, void* stream);

/* Hessian-compensated quantization of a layer's weights (offline, before
 * packing; "QQQ: Quality Quattuor-Bit Quantization for Large Language
 * Models", section 三 技术架构 -> Hessian补偿): with H = 2 X^T X over the
 * calibration activations, the input channels i = 0 .. K-1 are quantized in
 * order and each one's rounding error is compensated on the channels not
 * yet quantized,
 *   q_n      = clamp(rne(W[i][n] / scale[n]), -qmax, qmax) * scale[n]
 *   W[j][n] += -(W[i][n] - q_n) / [H^-1]_ii * [H^-1]_ji     (j > i)
 *   W[i][n]  = q_n,
 * after which H^-1 loses row and column i by the rank-one downdate
 * H^-1 <- H^-1 - H^-1[:, i] H^-1[i, :] / [H^-1]_ii.  H^-1 is H's inverse by
 * Gauss-Jordan elimination with partial pivoting (the first row of largest
 * magnitude).  Every step is an fp64 operation rounded to nearest, in this
 * order, without fused multiply-adds, so the results do not depend on the
 * GPU's work split.
 *   X        device fp64 [ns][K] calibration activations (ns >= 1).
 *   W        device fp64 [K][N] (input channel i is row i), overwritten with
 *            the quantized values codes * scale.
 *   scale    device fp64 [N] grid step of each output channel.
 *   qmax     1 .. 127 (7 for INT4, 127 for INT8).
 *   codes    device int8 [K][N]: clamp(rne(w / scale)) of each step.
 *   Hinv     device fp64 [K][K]: H^-1 before any downdate.
 *   singular device int32 (may be NULL): 1 if a pivot of H was zero (H is
 *            singular; W, codes and Hinv are then undefined), else 0.
 *   workspace  qlin_gptq_workspace bytes (one K x K fp64 matrix and a
 *            little scratch), 256-byte aligned; no zero-fill needed.
 * K <= 16384.  The call enqueues 4 K + 3 small kernels on `stream`. */
QLIN_API qlin_status qlin_gptq_workspace(int32_t K, int32_t N, size_t* bytes);
QLIN_API qlin_status qlin_gptq_quantize(const double* X, int32_t ns, int32_t K, int32_t N, double* W,
                                        const double* scale, int32_t qmax, int8_t* codes, double* Hinv,
                                        int32_t* singular, void* workspace, size_t ws_bytes, void* stream);

/* QQQ adaptive smoothing, the threshold search (offline calibration; "QQQ:
 * Quality Quattuor-Bit Quantization for Large Language Models", section 三
 * 技术架构 -> 自适应平滑): only activation channels with significant
 * outliers are smoothed, and the threshold sigma comes from a grid search
 * over [0, max|X|] minimising the quantized product's error on those
 * channels.  For j = 0 .. G-1, sigma_j = max|X| * j / G (fp32) and
 *   T      = { t : max_m |X[m][t]| > sigma_j }
 *   s_t    = sqrt(max_m |X[m][t]| / max_n |W[t][n]|) on T (1 if a maximum is 0)
 *   Xh     = fp16(X / s), Wh = fp16(W * s) on T, 0 elsewhere
 *   loss_j = sum_{m,n} (a_m (c_n / 16) acc[m][n] - sum_{t in T} X[m][t] W[t][n])^2
 * where (Xq, a) = qlin_quant_act of Xh (no outliers), (q, c) = the W4A8
 * per-channel packing of Wh and acc = Xq . 16 q exactly (qlin_gemm); the
 * reference product is summed in fp32, the loss in fp64 (its summation
 * order is not fixed: repeated calls may differ in the last bits).
 *   X       device fp16 [M][K] calibration activations; W device fp16 [K][N].
 *   loss    device fp64 [G], overwritten.
 *   best    device int32 (may be NULL): the first j of least loss.
 *   s_best  device fp32 [K] (may be NULL): s of that candidate, 1 off T.
 *   workspace  qlin_smooth_search_workspace bytes, 256-byte aligned (no
 *           zero-fill needed).
 * Shapes: as the W4A8 per-channel layer (K % 32 == 0, N % 16 == 0), M >= 1,
 * 1 <= G <= 64. */
QLIN_API qlin_status qlin_smooth_search_workspace(int32_t M, int32_t K, int32_t N, int32_t G, size_t* bytes);
QLIN_API qlin_status qlin_smooth_search(const uint16_t* X, int32_t M, int32_t K, const uint16_t* W, int32_t N,
                                        int32_t G, double* loss, int32_t* best, float* s_best, void* workspace,
                                        size_t ws_bytes, void* stream);

/* OffQ: W4A4 with per-group asymmetric activations whose offset absorbs the
 * structured outliers ("OffQ: Taming Structured Outliers in LLM Quantization
 * by Offsetting", technical summary, 方法论: 通过偏移量进行吸收 (Hadamard
 * 旋转) and its grouped implementation).  After the offline top-1 PCA step
 * has concentrated a group's outlier energy in one channel, the rotation
 * D H (first row all ones) spreads it as one constant over the group, and
 * that constant becomes the group's offset (zero point).  The readings this
 * library takes where the summaries are silent:
 *   - groups of 128 consecutive input channels (K % 128 == 0);
 *   - H the 128 x 128 Sylvester matrix h(i,j) = (-1)^popcount(i & j),
 *     D = diag(signs), signs[i] = +1 or -1 with signs[0] = +1 (host int8
 *     [128], read during the call; QLIN_ERR_ARG otherwise);
 *   - activations, per token m and group g: y = x_g D H unnormalised and
 *     exact (fp64), lo = min y, hi = max y, sd = (hi - lo) / 15,
 *     q = clamp(rne((y - lo) / sd), 0, 15) taken in fp64 (q = 0 when
 *     sd == 0); so y ~ q sd + lo;
 *   - weights, per group: W' = (1/128) H D W_g in fp64 then fp32, then
 *     symmetric INT4 per output channel in fp32: c_n = max_k|W'[k][n]| / 7,
 *     q_w = clamp(rne(W' * (7 / max)), -7, 7);
 *   - output: Y[m][n] = fp16( (c_n / 16) * sum_g ( sd[m][g] acc_g[m][n]
 *     + lo[m][g] colsum_g[n] ) ), acc_g = sum_{k in g} q[m][k] 16 q_w[k][n]
 *     (exact INT32 per K-block on the tensor cores) and colsum_g[n] =
 *     sum_{k in g} 16 q_w[k][n]; the sum over groups is fp32 (two fused
 *     multiply-adds per group, in group order).
 * Shapes: 128 <= K <= 65536 with K % 128 == 0; N % 16 == 0; M >= 0 (M == 0
 * enqueues nothing).  Non-finite activations give unspecified codes. */

/* Bytes of the packed OffQ codes of a K x N layer: the W4 per-channel tile
 * layout of qlin_weights.codes (ceil(N/128) * K/128 blocks of 8 KiB). */
QLIN_API qlin_status qlin_offq_codes_bytes(int32_t K, int32_t N, size_t* bytes);

/* Wr = the rotated weights, fp32 [K][N] (device), from W fp16 [K][N]
 * (device): Wr[128g + j][n] = fp32((1/128) sum_i h(j,i) signs[i] W[128g + i][n]),
 * bit-exact (the sums are exact in fp64). */
QLIN_API qlin_status qlin_offq_rotate_weights(const uint16_t* W, int32_t K, int32_t N, const int8_t* signs,
                                              float* Wr, void* stream);

/* Offline packing: rotates W into Wr (device fp32 [K][N], caller-owned
 * scratch that keeps the rotated weights) and quantizes it.
 *   codes       device, qlin_offq_codes_bytes bytes (cleared, then written).
 *   chan_scale  device fp32 [N]: c_n.
 *   colsum      device fp32 [K/128][N]: colsum_g[n] (integers, exact). */
QLIN_API qlin_status qlin_offq_pack(const uint16_t* W, int32_t K, int32_t N, const int8_t* signs, uint8_t* codes,
                                    float* chan_scale, float* colsum, float* Wr, void* stream);

/* Activation side: X device fp16 [M][K] -> Xq device int8 [M][K] (codes
 * 0..15, one per byte), scale = fp32(sd) and offset = fp32(lo), device fp32
 * [M][K/128].  Bit-exact. */
QLIN_API qlin_status qlin_offq_quant_act(const uint16_t* X, int32_t M, int32_t K, const int8_t* signs, int8_t* Xq,
                                         float* scale, float* offset, void* stream);

/* The GEMM from quantized activations: Y device fp16 [M][N] as above.  The
 * workspace (qlin_offq_gemm_workspace bytes, 256-byte aligned, no
 * zero-fill needed) receives the codes widened to INT8 (16 q_w) once per
 * call. */
QLIN_API qlin_status qlin_offq_gemm_workspace(int32_t M, int32_t K, int32_t N, size_t* bytes);
QLIN_API qlin_status qlin_offq_gemm(const int8_t* Xq, const float* scale, const float* offset, int32_t M, int32_t K,
                                    int32_t N, const uint8_t* codes, const float* chan_scale, const float* colsum,
                                    uint16_t* Y, void* workspace, size_t ws_bytes, void* stream);

/* qlin_offq_quant_act then qlin_offq_gemm, the intermediates in the
 * workspace (qlin_offq_forward_workspace bytes, 256-byte aligned). */
QLIN_API qlin_status qlin_offq_forward_workspace(int32_t M, int32_t K, int32_t N, size_t* bytes);
QLIN_API qlin_status qlin_offq_forward(const uint16_t* X, int32_t M, int32_t K, int32_t N, const int8_t* signs,
                                       const uint8_t* codes, const float* chan_scale, const float* colsum,
                                       uint16_t* Y, void* workspace, size_t ws_bytes, void* stream);

/* Test and measurement hooks.  The library reads no environment variables:
 * a process that wants a non-default work split, launch mode or wait limit
 * (the test suite forcing each split-K variant, a measurement isolating one
 * mechanism, a failure-detection test) sets it here.  Settings are global to
 * the process, take effect from the next call that launches work, and are
 * not meant for production use; the defaults are what the library is tuned
 * and tested with.
 *   QLIN_KNOB_PDL             1 (default): kernels are chained with
 *                             programmatic dependent launch; 0: plain
 *                             stream-ordered launches.
 *   QLIN_KNOB_CLUSTER         1 (default): decode GEMMs may split tiles over
 *                             thread-block clusters; 0: global stream-K only.
 *   QLIN_KNOB_CLUSTER_SIZE    0 (default): cluster size from the cost model;
 *                             2, 4 or 8: that size whenever it is valid.
 *   QLIN_KNOB_MAX_CTAS        0 (default): one persistent GEMM CTA per SM;
 *                             n > 0: at most n.
 *   QLIN_KNOB_MAX_TOKEN_TILE  256 (default); 64 or 128 cap the GEMM's token tile.
 *   QLIN_KNOB_WIDEN_MIN_M     512 (default): from this token count INT4
 *                             weights are widened to INT8 once per call; 0: never.
 *   QLIN_KNOB_FUSED_MOMENTUM_MAX_M  64 (default): up to this token count the
 *                             momentum update runs inside the quantization kernel
 *                             (every CTA gathers the outlier columns of all rows);
 *                             above it one column-maximum launch per problem
 *                             precedes the quantization.
 *   QLIN_KNOB_CONVERT_MAX_M   0 (default): INT4 layers on CTA pairs up to this
 *                             token count convert their codes inside the GEMM
 *                             (eight converter warps per CTA) instead of
 *                             widening them to INT8 ahead of it; 0: always widen.
 *   QLIN_KNOB_PAIR_MMA        2 (default): 256-token tiles with INT8 operands run
 *                             on CTA pairs (one 256-row tensor-core operation
 *                             per pair) whenever the operands allow; 1: only
 *                             when there is a full wave of 256 x 256 tiles;
 *                             0: never.
 *   QLIN_KNOB_PAIR_SPLIT      0 (default): launches on CTA pairs take whole
 *                             tiles; 1: when such a launch would leave its
 *                             last wave of tiles partly empty (and has fewer
 *                             than eight full waves), its last full wave and
 *                             the remainder are divided by K-steps across all
 *                             pairs, and the pairs that share a tile sum their
 *                             INT32 partials in the workspace (exact: the
 *                             result does not depend on the split; measured
 *                             slower than whole tiles on the bench shapes).
 *   QLIN_KNOB_WAIT_NS         2000000000 (default): limit in ns of every
 *                             device-side pipeline wait, after which the kernel
 *                             gives up, sets the device error word and unwinds
 *                             (QLIN_ERR_TIMEOUT from qlin_poll_device_status).
 *                             It is a device variable: set it with the device
 *                             concerned current, between calls.  After a
 *                             timeout, the workspaces and outputs of the calls
 *                             that gave up are undefined; zero-fill the
 *                             workspaces before reusing them.
 * qlin_debug_set stores `value` (QLIN_ERR_ARG for an unknown knob or an
 * invalid value) and, when `previous` is not NULL, returns the old value
 * there; qlin_debug_get reads a knob. */
typedef enum {
  QLIN_KNOB_PDL = 0,
  QLIN_KNOB_CLUSTER = 1,
  QLIN_KNOB_CLUSTER_SIZE = 2,
  QLIN_KNOB_MAX_CTAS = 3,
  QLIN_KNOB_MAX_TOKEN_TILE = 4,
  QLIN_KNOB_WIDEN_MIN_M = 5,
  QLIN_KNOB_FUSED_MOMENTUM_MAX_M = 6,
  QLIN_KNOB_WAIT_NS = 7,
  QLIN_KNOB_PAIR_MMA = 8,
  QLIN_KNOB_CONVERT_MAX_M = 9,
  QLIN_KNOB_PAIR_SPLIT = 10
} qlin_knob;

QLIN_API qlin_status qlin_debug_set(int32_t knob, int64_t value, int64_t* previous);
QLIN_API qlin_status qlin_debug_get(int32_t knob, int64_t* value);

/* Synchronizes `stream`, then reports and clears the device error word that
 * kernels set when a bounded wait gives up: QLIN_ERR_TIMEOUT if it was set,
 * QLIN_ERR_CUDA if the stream reported an error, else QLIN_OK. */
QLIN_API qlin_status qlin_poll_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QLIN_H_ */
