/*
 * qr.h -- C ABI of the B200 online W4A4 rotated linear layer.
 *
 * The layer computes, for activations X [M x K] and weights W [N x K]
 * (fp16, row-major, W stored output-major as in Y = X W^T):
 *
 *     Y = fp16( dequant( Q(X R) . Q(W R^{-T})^T ) + X_out W_out^T )
 *
 * where R is a rotation (full or block-diagonal Walsh-Hadamard, the
 * grouped sequency-ordered Walsh rotation, or a Kronecker affine transform
 * with per-channel scaling), Q is symmetric per-row 4-bit quantization and
 * X_out, W_out are the QUIK fp16 outlier columns.
 *
 * Sources, by page title and section:
 *   - "QuaRot & SpinQuant" reading notes, §1 Computational Invariance and
 *     §2 Quarot: weights are rotated offline, activations online, so that
 *     the rotated product equals the original one.
 *   - "QUIK：LLM上的一种4-bit推理方法", QUIK量化 §1 (workflow: outlier
 *     columns kept fp16, per-token quantization of the rest, INT4 GEMM with
 *     INT32 accumulation, dequant to fp16, outlier product added) and §3
 *     (outliers chosen by column infinity-norm).
 *   - "LLM量化新篇章：4-bit权重激活量化几乎无损！FlatQuant的平坦之道",
 *     §2.3 方法概述 (Kronecker-decomposed affine transform, per-channel
 *     scaling, clipping) and §3 量化设置 (per-token / per-channel symmetric).
 *   - "Grouped Sequency-arranged Rotation: Optimizing Rotation
 *     Transformation for Quantization for Free", abstract and 方法详解
 *     (block-diagonal sequency-ordered Walsh blocks).
 *   - "SpinQuant: LLM Quantization with Learned Rotations" review
 *     discussion, Q1/A1 (min-max quantizer onto +-(2^(N-1)-1)).
 *
 * Conventions shared by every call:
 *   - Every array pointer is a DEVICE pointer unless stated otherwise; the
 *     caller allocates and owns every buffer.  No call allocates memory.
 *   - fp16 arrays are passed as uint16_t (IEEE binary16 bit patterns).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and operate on the device that is current.
 *   - Argument errors return before any launch and write nothing.  A failed
 *     launch returns QR_ERR_CUDA.  Faults inside a kernel surface as usual
 *     CUDA errors at the next synchronization.
 *   - Kernels that wait on barriers bound every wait; if a wait ever runs out
 *     (a library bug, not a user error) the kernel records a code in a
 *     per-device status word, abandons its work and returns; read it with
 *     qr_device_status().
 *   - 4-bit codes are two's-complement nibbles, two per byte, element 2j in
 *     the low nibble, rows of K_p/2 bytes (K_p from qr_packed_k).  Codes lie
 *     in [-7, 7].  Scales are fp32, one per row.
 */
#ifndef QR_H_
#define QR_H_

#include <stdint.h>

#if defined(__GNUC__)
#define QR_API __attribute__((visibility("default")))
#else
#define QR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                      /* cudaStream_t is struct CUstream_st* */
typedef struct CUstream_st* qr_stream;

typedef enum {
  QR_OK = 0,
  QR_ERR_INVALID_ARG = 1,    /* null pointer, negative or inconsistent size */
  QR_ERR_UNSUPPORTED = 2,    /* a size or kind outside what the kernels handle */
  QR_ERR_ALIGNMENT = 3,      /* a pointer or leading dimension is misaligned */
  QR_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  QR_ERR_DEVICE = 5          /* a kernel recorded an error (qr_device_status) */
} qr_status;

typedef enum {
  QR_ROT_NONE = 0,           /* quantize the (outlier-free, padded) row as is */
  QR_ROT_HADAMARD = 1,       /* block-diagonal Sylvester Hadamard, H_b/sqrt(b) */
  QR_ROT_GSR = 2,            /* block-diagonal sequency-ordered Walsh, Wal_b/sqrt(b) */
  QR_ROT_KRON = 3            /* x -> (x op c) (P1 kron P2): vec(P1^T mat(x) P2) */
} qr_rot_kind;

typedef enum {
  QR_CHAN_DIVIDE = 0,        /* activation side: x_k / c_k  */
  QR_CHAN_MULTIPLY = 1       /* weight side:     w_k * c_k  */
} qr_chan_mode;

/* What is done to a row before it is quantized.  Host struct; the arrays it
 * points to are device arrays that must stay valid until the call's work on
 * the stream has finished. */
typedef struct {
  int32_t kind;              /* qr_rot_kind */
  int32_t block;             /* HADAMARD, GSR: block size b, a power of two,
                                1 <= b <= 16384 (GSR: 2 <= b <= 256);
                                ignored otherwise */
  const float* p1;           /* KRON: row-major n1 x n1 */
  int32_t n1;
  const float* p2;           /* KRON: row-major n2 x n2 */
  int32_t n2;                /* KRON: n1, n2 multiples of 4, n1 + n2 <= 192,
                                n1*n2 % 128 == 0 */
  const float* chan_scale;   /* KRON: per-channel scale c [n1*n2], or NULL */
  int32_t chan_mode;         /* qr_chan_mode: how chan_scale is applied */
  float clip_ratio;          /* alpha in (0, 1]: s = alpha*absmax/7, codes
                                clamped to +-7 (1.0 = plain min-max) */
  const int8_t* signs;       /* HADAMARD, GSR: the random-sign diagonal D of a
                                randomized Hadamard, R = D B (rows become
                                (x .* d) B; "random Hadamard rotations", SpinQuant
                                review, reviewer brBn W2/A2): int8 [K_p] of +-1,
                                8-byte aligned, applied after the outlier split
                                and padding; NULL = no signs.  Must be NULL for
                                the other kinds.  The weight side takes the same
                                descriptor (D B is orthogonal). */
} qr_rotation;

/* ABI version of this header (bumped on any change to the entry points;
 * 3 added the 8-bit calls and qr_check_wait_timeout, 4 the FP4 calls, 5
 * qr_w4a4_linear_fused, 6 qr_w4a4_linear_fused_noalloc). */
#define QR_ABI_VERSION 6
QR_API int32_t qr_abi_version(void);

/* Human-readable name of a status code (static string). */
QR_API const char* qr_status_string(qr_status status);

/* Width K_p of the rotated, quantized part of a row of K columns of which
 * n_out are fp16 outliers: the other K - n_out columns, zero-padded to a
 * multiple of max(b, 128) (HADAMARD, GSR) or of 128 (NONE); for KRON,
 * K - n_out must equal n1*n2.  The zero padding changes neither the scale
 * nor any dot product (the QUIK page's split plus the orthogonality of R).
 * Returns -1 if the descriptor or sizes are invalid.  Host-only. */
QR_API int64_t qr_packed_k(const qr_rotation* rot, int64_t K, int32_t n_out);

/* Online activation path (QuaRot §2 online rotation; QUIK §1 per-token
 * quantization of the non-outlier columns; FlatQuant §2.3 fused transform
 * and quantization).  For each row m of X:
 *   x_out[m, j] = X[m, outlier_idx[j]]                       (fp16 copy)
 *   x = X[m, kept columns] zero-padded to K_p, x' = rotate(x)
 *   scales[m] = alpha * max|x'| / 7   (0 for an all-zero row)
 *   codes[m, k] = clamp(round_half_even(x'[k] / scales[m]), -7, 7), packed
 *
 *  rot          host descriptor (activation side: chan_mode DIVIDE)
 *  X            fp16 [M x ldx], ldx >= K
 *  outlier_idx  int32 [n_out], strictly ascending in [0, K); may be NULL
 *               when n_out == 0.  Out-of-range entries are skipped by the
 *               kernel (their x_out column reads as zero), never read
 *               out of bounds.
 *  codes        uint8 [M x K_p/2] (row stride K_p/2 bytes), 16-byte aligned
 *  scales       fp32 [M]
 *  x_out        fp16 [M x n_out] (row stride n_out), NULL iff n_out == 0
 *  x_rot_debug  fp32 [M x K_p] rotated rows before quantization, or NULL
 * Errors: INVALID_ARG (null/negative/inconsistent, clip_ratio outside (0,1]),
 * UNSUPPORTED (block, n1/n2 outside the limits above, K_p > 32768, or with
 * outliers K > 32768 or n_out > 8192), ALIGNMENT (codes not 16-byte
 * aligned). */
QR_API qr_status qr_rotate_quant(const qr_rotation* rot, const uint16_t* X, int64_t M,
                          int64_t K, int64_t ldx, const int32_t* outlier_idx,
                          int32_t n_out, uint8_t* codes, float* scales,
                          uint16_t* x_out, float* x_rot_debug, qr_stream stream);

/* Offline weight path (QuaRot §2 stage 1: rotate the weights in full
 * precision, then quantize them; SpinQuant review W2/A2: R1/R2 merged into
 * the weights; QUIK §1: weight columns permuted to match the outliers).
 * Same as qr_rotate_quant applied to the rows of W with the weight-side
 * descriptor rot_w: for HADAMARD/GSR it equals the activation descriptor;
 * for KRON it holds P1^{-T}, P2^{-T} (see qr_invert_transpose) and the same
 * c with chan_mode MULTIPLY, so that X' W'^T = X W^T.
 *  W            fp16 [N x ldw], ldw >= K
 *  w_codes      uint8 [N x K_p/2], 16-byte aligned;  w_scales fp32 [N]
 *  w_out        fp16 [N x n_out], NULL iff n_out == 0
 *  w_rot_debug  fp32 [N x K_p] or NULL
 * Errors as qr_rotate_quant. */
QR_API qr_status qr_pack_weights(const qr_rotation* rot_w, const uint16_t* W, int64_t N,
                          int64_t K, int64_t ldw, const int32_t* outlier_idx,
                          int32_t n_out, uint8_t* w_codes, float* w_scales,
                          uint16_t* w_out, float* w_rot_debug, qr_stream stream);

/* The W4A4 linear (QUIK §4: the INT4 x INT4 product on integer tensor cores
 * with INT32 accumulation, dequantized to fp16, plus the fp16 outlier
 * product; FlatQuant §3: per-token x per-channel symmetric scales):
 *   acc[m, n] = sum_k qa[m, k] qw[n, k]                      (exact int32)
 *   Y[m, n]   = fp16( acc * a_scales[m] * w_scales[n]
 *                     + sum_j x_out[m, j] w_out[n, j] )      (fp32 math)
 *  a_codes   uint8 [M x K_p/2], w_codes uint8 [N x K_p/2], both 16-byte
 *            aligned; K_p % 128 == 0, K_p <= 65536
 *  x_out     fp16 [M x n_out], w_out fp16 [N x n_out] (NULL iff n_out == 0),
 *            16-byte aligned, n_out % 8 == 0
 *  Y         fp16 [M x ldy], ldy >= N
 *  acc_debug int32 [M x N] (row stride N), or NULL
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT as above. */
QR_API qr_status qr_w4a4_linear(const uint8_t* a_codes, const float* a_scales,
                         const uint8_t* w_codes, const float* w_scales,
                         int64_t M, int64_t N, int64_t K_p,
                         const uint16_t* x_out, const uint16_t* w_out, int32_t n_out,
                         uint16_t* Y, int64_t ldy, int32_t* acc_debug,
                         qr_stream stream);

/* The decode step in one kernel (FlatQuant "模型架构": the online transform
 * and the quantization fused into the kernel that consumes them; QUIK
 * "性能分析": the separate quantization and dequantization passes are why
 * measured speedups trail the ideal).  Computes exactly what
 * qr_rotate_quant (or qr_rotate_quant_asym when a_zeros != NULL) followed by
 * qr_w4a4_linear (or qr_w4a4_linear_asym) computes, with the same codes,
 * scales and outlier copy and the same Y bit for bit, in one launch: the
 * kernel first rotates and quantizes the M token rows, writes a_codes,
 * a_scales (a_zeros) and x_out, meets all of its CTAs at a grid-wide
 * barrier, then runs the decode GEMM on them.
 *  rot, X, M, K, ldx, outlier_idx, n_out: as qr_rotate_quant, with
 *            1 <= M <= 64 and a NONE, HADAMARD or GSR rotation
 *  w_codes, w_scales, w_out, N: the packed weights, as qr_w4a4_linear;
 *            w_sums [N] (qr_weight_code_sums) with a_zeros, else ignored
 *  a_codes, a_scales, a_zeros, x_out: outputs, as qr_rotate_quant(_asym);
 *            the GEMM phase reads them back
 *  Y         fp16 [M x ldy], ldy >= N
 *  sync      two uint32 words of device memory, 8-byte aligned, that the
 *            caller sets to zero once before the first call; every call
 *            that completes leaves the first word zero again (the second
 *            counts calls).  Calls that share `sync` must not run at the
 *            same time (one stream, or ordered streams).
 * The CTAs of the launch must all be resident at once; when the device
 * cannot hold them (or K_p does not fit the kernel's row buffer) the call
 * returns UNSUPPORTED without launching, and the two-call path applies.
 * A barrier wait that runs out records QR_DEV_TIMEOUT_GRID_SYNC in the
 * device status word.
 * Errors: INVALID_ARG, UNSUPPORTED (M > 64, KRON, sizes), ALIGNMENT (as the
 * two calls; sync not 8-byte aligned), CUDA. */
QR_API qr_status qr_w4a4_linear_fused(const qr_rotation* rot, const uint16_t* X, int64_t M,
                                      int64_t K, int64_t ldx, const int32_t* outlier_idx,
                                      int32_t n_out, const uint8_t* w_codes, const float* w_scales,
                                      const int32_t* w_sums, const uint16_t* w_out, int64_t N,
                                      uint8_t* a_codes, float* a_scales, int32_t* a_zeros,
                                      uint16_t* x_out, uint16_t* Y, int64_t ldy, uint32_t* sync,
                                      qr_stream stream);

/* qr_w4a4_linear_fused without caller scratch.  The pages have no
 * counterpart: this is a convenience form of the call above for callers
 * that want only Y.  The token rows' codes, scales, zero points and outlier
 * copy and the two grid-barrier words live in a scratch array of the
 * library itself, one per device (a __device__ array found with
 * cudaGetSymbolAddress; no memory is allocated).  The barrier words start at
 * zero when the library loads and every completed call leaves the count at
 * zero again.  All calls on one device share this scratch, so two calls
 * that may run at the same time (different streams, or different host
 * threads) race: order them on one stream.
 *  arguments as qr_w4a4_linear_fused, without a_codes, a_scales, a_zeros,
 *  x_out and sync; asym != 0 selects asymmetric activations (w_sums then
 *  required)
 * Errors: as qr_w4a4_linear_fused; UNSUPPORTED also for sizes above the
 * scratch's capacity: M > 64, K_p > 32768 or n_out > 8192. */
QR_API qr_status qr_w4a4_linear_fused_noalloc(const qr_rotation* rot, const uint16_t* X,
                                              int64_t M, int64_t K, int64_t ldx,
                                              const int32_t* outlier_idx, int32_t n_out,
                                              const uint8_t* w_codes, const float* w_scales,
                                              const int32_t* w_sums, const uint16_t* w_out,
                                              int64_t N, int32_t asym, uint16_t* Y, int64_t ldy,
                                              qr_stream stream);

/* ----------------------------------------------------------------------
 * 8-bit layers ("QUIK：LLM上的一种4-bit推理方法", QUIK量化, results: the
 * LLaMA-2 down_proj stays in INT8 with its outlier count raised in
 * proportion to its input width, round(256 K / 4096) = 688 for K = 11008;
 * QUIK-8B runs every layer in INT8).  The same steps as the 4-bit calls with
 * the symmetric quantizer on 8 bits: scales = alpha * max|x'| / 127, codes =
 * clamp(round_half_even(x' / s), -127, 127), one int8 per code, rows of K_p
 * bytes (K_p from qr_packed_k, as for 4 bits).
 *
 * qr_rotate_quant8 / qr_pack_weights8: arguments and errors as
 * qr_rotate_quant / qr_pack_weights, with codes int8 [rows x K_p] (16-byte
 * aligned); Kronecker descriptors are UNSUPPORTED.
 * qr_w8a8_linear: as qr_w4a4_linear for int8 codes [M x K_p] and
 * [N x K_p] (16-byte aligned, K_p % 128 == 0, K_p <= 65536):
 *   acc[m, n] = sum_k qa[m, k] qw[n, k]   (exact int32: |acc| <= 127^2 K_p)
 *   Y[m, n]   = fp16(acc * a_scales[m] * w_scales[n] + X_out[m] . W_out[n]) */
QR_API qr_status qr_rotate_quant8(const qr_rotation* rot, const uint16_t* X, int64_t M, int64_t K,
                                  int64_t ldx, const int32_t* outlier_idx, int32_t n_out,
                                  int8_t* codes, float* scales, uint16_t* x_out,
                                  float* x_rot_debug, qr_stream stream);
QR_API qr_status qr_pack_weights8(const qr_rotation* rot_w, const uint16_t* W, int64_t N,
                                  int64_t K, int64_t ldw, const int32_t* outlier_idx,
                                  int32_t n_out, int8_t* w_codes, float* w_scales,
                                  uint16_t* w_out, float* w_rot_debug, qr_stream stream);
QR_API qr_status qr_w8a8_linear(const int8_t* a_codes, const float* a_scales,
                                const int8_t* w_codes, const float* w_scales, int64_t M,
                                int64_t N, int64_t K_p, const uint16_t* x_out,
                                const uint16_t* w_out, int32_t n_out, uint16_t* Y, int64_t ldy,
                                int32_t* acc_debug, qr_stream stream);

/* ----------------------------------------------------------------------
 * FP4 layers (the W-fp4/A-fp4 benchmark on Blackwell's fp4 tensor cores
 * that the "SpinQuant" review discussion, reviewer brBn W3/A3, names as
 * planned work, with no format given).  Read as the e2m1 element type with
 * a per-row fp32 scale, the analogue of the INT4 quantizer: per row,
 * s = alpha * absmax / 6 and the code of x is the e2m1 value nearest x / s
 * (ties to the even mantissa, saturating at +-6).  An e2m1 nibble is sign
 * (bit 3), exponent (bits 2-1, bias 1), mantissa (bit 0); -0 may appear and
 * decodes to 0.  Codes are packed two per byte, element 2j in the low
 * nibble: uint8 [rows x K_p / 2], 32-byte aligned.
 *
 * qr_rotate_quant_fp4 / qr_pack_weights_fp4: arguments and errors as
 * qr_rotate_quant / qr_pack_weights.  Supported rotations: HADAMARD or
 * GSR with blocks of 64, 128, 256 or 4096 (outlier columns allowed);
 * others, and KRON, are UNSUPPORTED.
 * qr_fp4_linear: as qr_w4a4_linear for packed e2m1 codes
 * (K_p % 128 == 0, K_p <= 65536, code pointers 32-byte aligned):
 *   acc[m, n] = sum_k e2m1(qa[m, k]) e2m1(qw[n, k])   (fp32; every product
 *               and partial sum is a multiple of 1/4 of magnitude at most
 *               36 K_p < 2^22, exactly representable)
 *   Y[m, n]   = fp16(acc * a_scales[m] * w_scales[n] + X_out[m] . W_out[n])
 * acc_debug (optional, float [M x N]) receives acc. */
QR_API qr_status qr_rotate_quant_fp4(const qr_rotation* rot, const uint16_t* X, int64_t M,
                                     int64_t K, int64_t ldx, const int32_t* outlier_idx,
                                     int32_t n_out, uint8_t* codes, float* scales,
                                     uint16_t* x_out, float* x_rot_debug, qr_stream stream);
QR_API qr_status qr_pack_weights_fp4(const qr_rotation* rot_w, const uint16_t* W, int64_t N,
                                     int64_t K, int64_t ldw, const int32_t* outlier_idx,
                                     int32_t n_out, uint8_t* w_codes, float* w_scales,
                                     uint16_t* w_out, float* w_rot_debug, qr_stream stream);
QR_API qr_status qr_fp4_linear(const uint8_t* a_codes, const float* a_scales,
                               const uint8_t* w_codes, const float* w_scales, int64_t M,
                               int64_t N, int64_t K_p, const uint16_t* x_out,
                               const uint16_t* w_out, int32_t n_out, uint16_t* Y, int64_t ldy,
                               float* acc_debug, qr_stream stream);

/* ----------------------------------------------------------------------
 * Asymmetric per-token activations ("QUIK：LLM上的一种4-bit推理方法",
 * QUIK量化 §1: activations are quantized asymmetrically per token and
 * dynamically, weights symmetrically).
 *
 * qr_rotate_quant_asym: as qr_rotate_quant, but each rotated row x is
 * quantized over [0, 15]: lo = alpha*min(x), hi = alpha*max(x),
 * s = (hi - lo)/15, z = round(-lo/s), q = clamp(round(x/s) + z, 0, 15)
 * (float32, half to even).  Codes are stored as the signed nibble q - 8
 * (same packing as qr_rotate_quant), scales[m] = s, zeros[m] = z - 8
 * (int32 [M], device), so x ~= s * (code - zero).  A zero row gets s = 0.
 * Not for QR_ROT_KRON (UNSUPPORTED).  Errors as qr_rotate_quant, plus
 * INVALID_ARG for a null zeros with M > 0. */
QR_API qr_status qr_rotate_quant_asym(const qr_rotation* rot, const uint16_t* X, int64_t M,
                                      int64_t K, int64_t ldx, const int32_t* outlier_idx,
                                      int32_t n_out, uint8_t* a_codes, float* a_scales,
                                      int32_t* a_zeros, uint16_t* x_out, float* x_rot_debug,
                                      qr_stream stream);

/* Per weight row, the sum of its packed signed codes: w_sums[n] =
 * sum_k q_w[n, k] (int32 [N], device), for the zero-point term of
 * qr_w4a4_linear_asym.  Offline, once per layer.  w_codes [N x K_p/2],
 * 16-byte aligned; K_p % 128 == 0.  Errors: INVALID_ARG, ALIGNMENT. */
QR_API qr_status qr_weight_code_sums(const uint8_t* w_codes, int64_t N, int64_t K_p,
                                     int32_t* w_sums, qr_stream stream);

/* qr_w4a4_linear for asymmetric activation codes:
 *   acc[m, n] = sum_k code_a[m, k] q_w[n, k]          (int32, exact)
 *   Y[m, n]   = fp16( (acc - zero_a[m] * w_sums[n]) * s_a[m] * s_w[n]
 *                     + X_out[m] . W_out[n] )
 * i.e. the product of the dequantized operands s_a (code - zero) and
 * s_w q_w.  a_zeros int32 [M], w_sums int32 [N] from qr_weight_code_sums;
 * acc_debug receives acc.  Other arguments and errors as qr_w4a4_linear,
 * plus INVALID_ARG for a null a_zeros or w_sums. */
QR_API qr_status qr_w4a4_linear_asym(const uint8_t* a_codes, const float* a_scales,
                                     const int32_t* a_zeros, const uint8_t* w_codes,
                                     const float* w_scales, const int32_t* w_sums, int64_t M,
                                     int64_t N, int64_t K_p, const uint16_t* x_out,
                                     const uint16_t* w_out, int32_t n_out, uint16_t* Y,
                                     int64_t ldy, int32_t* acc_debug, qr_stream stream);

/* QUIK calibration (QUIK §3: outliers are the columns with the largest
 * infinity-norm over a calibration batch).  Writes the k selected column
 * indices of X_calib [T x ldx] (fp16, ldx >= K) to idx_out[k] in ascending
 * order; ties in the norm go to the lower column index.
 * Limits: 1 <= K <= 16384, 0 <= k <= K.  One CTA; offline. */
QR_API qr_status qr_select_outliers(const uint16_t* X_calib, int64_t T, int64_t K,
                             int64_t ldx, int32_t k, int32_t* idx_out,
                             qr_stream stream);

/* Weight-side Kronecker factor (FlatQuant §2.3: W is multiplied by the
 * inverse of the affine transform): out = (P^{-1})^T for a row-major
 * n x n matrix P, by Gauss-Jordan elimination with partial pivoting in
 * fp64, rounded to fp32.  info (int32 [1]) receives 0, or j+1 if column j
 * had no usable pivot (P singular to working precision; out is then
 * undefined).  1 <= n <= 256.  One CTA; offline. */
QR_API qr_status qr_invert_transpose(const float* P, int32_t n, float* out,
                              int32_t* info, qr_stream stream);

/* ----------------------------------------------------------------------
 * KV cache ("SpinQuant: LLM Quantization with Learned Rotations" review,
 * reviewer brBn Q2/A2: the same R3 on the query and key rows after RoPE,
 * (q R3)(k R3)^T = q k^T; FlatQuant §3, quantization setting: the KV cache
 * quantized group-wise asymmetrically, groups of 128).  R3 is the
 * normalized Hadamard of the head dimension, H_d / sqrt(d), on every head.
 *
 * Q, K, V   fp16 [tokens x heads*head_dim], contiguous rows (the layout
 *           after the projections and RoPE), device
 * q_rot     fp16 [tokens x heads*head_dim]: Q with R3 on every head
 * k_codes   uint8 [tokens x heads*head_dim/2]: K with R3 on every head,
 *           then each run of `group` consecutive values of a row quantized
 *           as by qr_rotate_quant_asym (4-bit, asymmetric, codes q - 8 packed
 *           two per byte, element 2j in the low nibble); k_scales float32
 *           and k_zeros int32 [tokens x heads*head_dim/group]
 * v_codes, v_scales, v_zeros: the same for V without a rotation
 * Q/q_rot, the four K arrays and the four V arrays are each all given or
 * all NULL (a part that is NULL is skipped).  Caller-owned device memory;
 * Q, K, V, q_rot, k_codes and v_codes 16-byte aligned (ALIGNMENT otherwise).
 * head_dim in {32, 64, 128, 256}; group 128 or 256, a multiple of head_dim
 * that divides heads*head_dim (UNSUPPORTED otherwise).  Errors: INVALID_ARG
 * for negative sizes or a partly given side, ALIGNMENT, CUDA. */
QR_API qr_status qr_kv_quantize(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                int64_t tokens, int32_t heads, int32_t head_dim, int32_t group,
                                uint16_t* q_rot, uint8_t* k_codes, float* k_scales,
                                int32_t* k_zeros, uint8_t* v_codes, float* v_scales,
                                int32_t* v_zeros, qr_stream stream);

/* Codes a kernel records in the device status word when one of its bounded
 * waits runs out (the role that gave up); 0 = nothing recorded. */
#define QR_DEV_TIMEOUT_PRODUCER  0x101   /* a loader / producer role */
#define QR_DEV_TIMEOUT_WIDEN     0x102   /* an operand-conversion role */
#define QR_DEV_TIMEOUT_MMA       0x103   /* the MMA-issuing thread */
#define QR_DEV_TIMEOUT_EPILOGUE  0x104   /* an epilogue role */
#define QR_DEV_TIMEOUT_DRAIN     0x105   /* draining in-flight work on abort */
#define QR_DEV_TIMEOUT_GRID_SYNC 0x106   /* qr_w4a4_linear_fused's grid-wide barrier */
#define QR_DEV_TIMEOUT_SELFCHECK 0x1FF   /* qr_check_wait_timeout */

/* Reads, and clears, the current device's status word that kernels set when
 * a bounded wait ran out.  Synchronizes the device.  *code_out = 0 when no
 * kernel reported anything. */
QR_API qr_status qr_device_status(int32_t* code_out);

/* Failure-detection self-check.  The pages have no counterpart: this checks
 * the library's own guard against a wait that never ends.  Launches one
 * thread on `stream` that waits, for at most limit_ns nanoseconds, on an
 * mbarrier that nothing ever arrives on, through the same bounded-wait
 * routine every kernel of the library uses.  The wait runs out, records
 * QR_DEV_TIMEOUT_SELFCHECK in the device status word (unless a code is
 * already there) and the kernel returns normally: no fault, no trap, and the
 * CUDA context stays usable.  Read and clear the code with
 * qr_device_status().  limit_ns in [1000, 100000000] (1 us to 0.1 s).
 * Errors: INVALID_ARG for a limit outside that range, CUDA. */
QR_API qr_status qr_check_wait_timeout(int64_t limit_ns, qr_stream stream);

#ifdef __cplusplus
}
#endif

#endif  /* QR_H_ */
