/*
 * wush.h -- C ABI of the B200 WUSH transform-then-quantize linear layer.
 *
 * The layer (AI Radio episode "WUSH: Near-Optimal Adaptive Transforms for LLM
 * Quantization", "Problem Setup and Goal") computes
 *     y = q(T_W W)^T q(T_X X)
 * with per-block transforms T_X, T_W = T_X^{-T} built from second moments
 * (WUSH news article, paragraphs on the construction and the deployment
 * workflow), microscaled low-bit quantisation q (MXFP4, NVFP4, INT4; WUSH news
 * article, experiments paragraph) and a block-scaled FP4 GEMM (AI Radio
 * episode, "Conclusion").  An ITQ3_S-style 3-bit weight path with a 256-wide
 * Walsh-Hadamard rotation (ITQ3_S article, "核心技术：FWHT预旋转与TurboQuant的完美融合")
 * is a secondary variant.
 *
 * Storage conventions (PyTorch-native, K contiguous):
 *   activations X^T : [rows = tokens, d_in] row-major
 *   weights     W^T : [d_out, d_in]        row-major (the same row transform)
 *   output      y^T : [tokens, d_out]      row-major, fp32
 * A transform block is ``b`` consecutive d_in elements of one row; b is also the
 * quantisation group: 32 for MXFP4 and INT4, 16 for NVFP4.  Block j of a row,
 * x_j, is replaced by T[j] x_j with T stored as fp32 [d_in/b, b, b], T[j][i][k]
 * at ((j*b)+i)*b+k.
 *
 * General rules for every entry point:
 *   - The caller owns every buffer; no entry point allocates device memory and
 *     none synchronises the stream unless it says so.
 *   - "device" pointers are CUDA device (or managed) memory; "host" pointers are
 *     ordinary host memory.
 *   - Every argument is checked before any launch. A failed check returns
 *     WUSH_ERR_INVALID_ARG / WUSH_ERR_UNSUPPORTED and launches nothing.
 *   - A CUDA launch error returns WUSH_ERR_CUDA (cudaGetLastError after launch).
 *   - Device pointers must be 16-byte aligned.
 *   - ``stream`` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Work is enqueued in stream order.
 *   - Inputs must be finite.  The host calls (calibration, ITQ3 weight
 *     quantisation) check and return WUSH_ERR_INVALID_ARG for NaN or an
 *     infinity; the device kernels do not check, and give unspecified codes.
 *   - Waits inside kernels are bounded. A kernel that gives up sets a device
 *     error word which wush_check_device_status() reports as WUSH_ERR_TIMEOUT.
 */
#ifndef WUSH_H
#define WUSH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WUSH_OK = 0,
  WUSH_ERR_INVALID_ARG = -1,
  WUSH_ERR_UNSUPPORTED = -2,
  WUSH_ERR_NOT_SPD = -3,
  WUSH_ERR_CUDA = -4,
  WUSH_ERR_TIMEOUT = -5,
  WUSH_ERR_BUFFER_TOO_SMALL = -6,
  WUSH_ERR_IO = -7
} wush_status;

typedef enum { WUSH_FMT_MXFP4 = 0, WUSH_FMT_NVFP4 = 1, WUSH_FMT_INT4 = 2 } wush_format;

typedef enum {
  WUSH_T_IDENTITY = 0,
  WUSH_T_HADAMARD = 1,
  WUSH_T_WUS = 2,
  WUSH_T_WUSH = 3,
  WUSH_T_WUSH_DIAG = 4
} wush_transform;

typedef enum { WUSH_IN_BF16 = 0, WUSH_IN_FP32 = 1 } wush_input_dtype;

/* Human-readable name of a status code (static storage). */
const char* wush_status_string(int status);

/* Block size (quantisation group) of a format: 32, 16, 32. 0 for an unknown format. */
int wush_block_size(int fmt);

/* ---------------------------------------------------------------------------
 * Calibration (host, fp64 inside, not on the timed path)
 *
 * WUSH news article, paragraph 3 (W = Cholesky factor of the weights, U and S
 * from an SVD, H = Hadamard; second-order statistics of weights and
 * activations) and paragraph 6 (collect moments from calibration data, then
 * Cholesky and SVD per block, in parallel).  Per block j:
 *   Sigma_X = X_j X_j^T / n_calib,  Sigma_W = W_j W_j^T / d_out,
 *   W' = chol(Sigma_W) (lower),  W'^T Sigma_X W' = U diag(lambda) U^T,
 *   S = diag(sqrt(lambda)) (descending),  Hn = H_b / sqrt(b),
 *   T_X = Hn S^{-1/2} U^T W'^T,   T_W = T_X^{-T} = Hn S^{1/2} U^T W'^{-1}.
 * WUS drops Hn; HADAMARD gives T_X = T_W = Hn; IDENTITY gives I.
 * WUSH_DIAG (paragraphs 6 and 8: the data-aware component approximated by a
 * diagonal matrix) runs the same construction on the diagonals of the two
 * moments, which gives T_X = Hn D, T_W = Hn D^{-1} with
 * D = diag((Sigma_W[k][k] / Sigma_X[k][k])^{1/4}); each diagonal is floored at
 * 1e-12 of its largest entry (1 if all are zero).  It applies like WUSH (dense T).
 * Columns of U are signed so that their largest-magnitude entry is positive
 * (ties: lowest index); eigenvalues are floored at 1e-12 * max.  A Cholesky
 * failure is retried once with Sigma_W + 1e-8 * mean(diag) I; if that fails
 * too, WUSH_ERR_NOT_SPD.
 * ------------------------------------------------------------------------- */

/* x_calib: host fp32 [n_calib, d_in]; w: host fp32 [d_out, d_in] (W^T);
 * block in {16, 32} (any power of two 2..256 is accepted), d_in % block == 0;
 * t_x, t_w: host fp32 outputs [d_in/block, block, block].  Uses the host's cores. */
int wush_calibrate(const float* x_calib, int64_t n_calib, const float* w, int64_t d_out,
                   int64_t d_in, int block, int kind, float* t_x, float* t_w);

/* The same from precomputed per-block moments (host fp64 [d_in/block, block, block],
 * e.g. from existing Hessians); t_x, t_w as above. */
int wush_calibrate_from_moments(const double* sigma_x, const double* sigma_w, int64_t d_in,
                                int block, int kind, float* t_x, float* t_w);

/* Transform sharing (WUSH news article, paragraph 6: share transform matrices
 * between similar blocks; the pages give no algorithm).  The d_in/block blocks
 * are put in ``groups`` groups by k-means over their moments divided by their
 * traces (both moments, flattened): centres start at blocks
 * round(g * nb / groups) (halves to even), squared Euclidean distance, ties to
 * the lowest group, empty groups keep their centre, until no block moves (at most
 * 50 rounds).  Each group's transform (kind WUS, WUSH or WUSH_DIAG) comes from
 * its members' mean moments (a group left empty: from its starting block).
 * Outputs: t_x, t_w host fp32 [groups, block, block]; index host int32
 * [d_in/block], block j -> group.  1 <= groups <= d_in/block; apply with
 * wush_transform_quant_indexed.  groups = d_in/block reproduces the per-block
 * transforms. */
int wush_calibrate_shared(const float* x_calib, int64_t n_calib, const float* w, int64_t d_out,
                          int64_t d_in, int block, int kind, int groups, float* t_x, float* t_w,
                          int32_t* index);
int wush_calibrate_shared_from_moments(const double* sigma_x, const double* sigma_w, int64_t d_in,
                                       int block, int kind, int groups, float* t_x, float* t_w,
                                       int32_t* index);

/* Static NVFP4 per-tensor scale (host, no CUDA).  The pages name NVFP4 without
 * its scale rule (WUSH news article, experiments paragraph); the reading used
 * throughout is s_g = amax / 2688 with 2688 = 6 * 448 (the largest E2M1 magnitude
 * times the largest UE4M3 block scale), so the largest value of the tensor maps to
 * the top of both grids.  ``amax`` is the largest |T x| of the calibration tokens
 * (activations; e.g. from wush_transform_amax) or of the transformed weights.
 * *s_g receives fp32(amax / 2688) rounded once to nearest even, or 1 when that is
 * below 1e-30 (an all-zero tensor, whose codes are 0 whatever the scale): the
 * same rule the device applies in wush_transform_quant_nvfp4_dynamic.
 * WUSH_ERR_INVALID_ARG for a negative or non-finite amax or a NULL s_g. */
int wush_nvfp4_global_scale(float amax, float* s_g);

/* The NVFP4 GEMM's alpha for wush_qgemm: *alpha = fp32(s_gx * s_gw), the product
 * of the activations' and the weights' per-tensor scales rounded once (the device
 * forms the same product in wush_qgemm_nvfp4_dynamic).  WUSH_ERR_INVALID_ARG for
 * a non-positive or non-finite scale or a NULL alpha. */
int wush_nvfp4_alpha(float s_gx, float s_gw, float* alpha);

/* How the second moments behind a set of transforms were normalised (recorded in
 * the transforms file; see below). */
typedef enum { WUSH_NORM_UNKNOWN = 0, WUSH_NORM_MEAN = 1 } wush_sigma_norm;

/* ---------------------------------------------------------------------------
 * Checkpointing calibrated transforms (host, no CUDA)
 *
 * Calibration runs once, offline, and every block's matrices need storage
 * (WUSH news article, paragraph 6); these calls write and read its output.
 *
 * File layout, little-endian, 48 header bytes: the 8 bytes "WUSHTRF1", u32
 * version (1), u32 block size b, u32 kind (wush_transform), u32 dtype (0 = fp32,
 * the only one), u32 sigma_norm (wush_sigma_norm), u32 has_index, i64 n_t, i64
 * n_blocks; then fp32 T_X [n_t, b, b], fp32 T_W [n_t, b, b] (row-major per
 * block) and, when has_index is 1, int32 index [n_blocks] (block j of d_in uses
 * transform index[j]).  Without an index n_blocks = n_t.
 *
 * sigma_norm records how the second moments were normalised: the transforms
 * scale with that choice by a factor that is not a power of two, so the codes
 * depend on it.  wush_calibrate* use WUSH_NORM_MEAN (Sigma_X = X X^T / n_calib,
 * Sigma_W = W W^T / d_out); WUSH_NORM_UNKNOWN marks transforms from elsewhere.
 *
 * wush_save_transforms: t_x, t_w host fp32 [n_t, b, b]; index host int32
 * [n_blocks] or NULL (then n_blocks is ignored).  b a power of two in [2, 256],
 * kind a wush_transform value, sigma_norm a wush_sigma_norm value, every index
 * entry in [0, n_t): else WUSH_ERR_INVALID_ARG before the file is opened.
 * WUSH_ERR_IO when the file cannot be opened or fully written (a partial file
 * may remain).
 *
 * wush_transforms_file_info: reads the header and returns its fields, after
 * checking it as wush_load_transforms does, the file's length included (a file
 * longer or shorter than its header implies gives WUSH_ERR_INVALID_ARG), so that
 * buffers may be sized from what it returns.
 *
 * wush_load_transforms: reads the whole file into t_x and t_w (capacity_floats
 * floats each, at least n_t * b * b) and, when the file holds an index, into
 * index (index_capacity entries, at least n_blocks): WUSH_ERR_BUFFER_TOO_SMALL
 * otherwise, with nothing read.  WUSH_ERR_IO when the file cannot be opened or
 * its header is cut short; WUSH_ERR_INVALID_ARG for a wrong magic, version or
 * dtype, a header outside the limits above, a body cut short or followed by
 * extra bytes, or an index entry out of range (the buffers may then hold part
 * of the file).
 * ------------------------------------------------------------------------- */
int wush_save_transforms(const char* path, int block, int kind, int sigma_norm, int64_t n_t,
                         const float* t_x, const float* t_w, const int32_t* index, int64_t n_blocks);
int wush_transforms_file_info(const char* path, int* block, int* kind, int* sigma_norm,
                              int64_t* n_t, int64_t* n_blocks, int* has_index);
int wush_load_transforms(const char* path, float* t_x, float* t_w, int64_t capacity_floats,
                         int32_t* index, int64_t index_capacity);

/* ---------------------------------------------------------------------------
 * Output buffer sizes for wush_transform_quant (bytes)
 *
 * codes:  two 4-bit codes per byte, K contiguous, lower d_in index in the low
 *         nibble: rows * d_in / 2 bytes.
 * scales: MXFP4 (UE8M0, one byte per 32) and NVFP4 (UE4M3, one byte per 16) are
 *         written in the scale-factor tile layout of the block-scaled MMA: the
 *         rows x (d_in/b) scale matrix is cut into 128-row x 4-column atoms of
 *         512 contiguous bytes; scale (r, c) of an atom sits at byte
 *         (r % 32) * 16 + (r / 32) * 4 + c; atoms are ordered row-block-major
 *         (all column atoms of rows 0..127 first).  rows is padded up to 128 and
 *         d_in/b up to 4; padding bytes are written as zero.
 *         INT4 scales are fp16, plain row-major [rows, d_in/32].
 * ------------------------------------------------------------------------- */
size_t wush_codes_bytes(int64_t rows, int64_t d_in, int fmt);
size_t wush_scales_bytes(int64_t rows, int64_t d_in, int fmt);

/* ---------------------------------------------------------------------------
 * Fused block transform + microscaled quantisation (device, one launch)
 *
 * WUSH news article, paragraph 6: at inference only the input activations are
 * transformed (weights are transformed and quantised once, offline, with the
 * same call and T_W); AI Radio episode, "The gist": the transform admits a fused
 * GPU implementation.  Rules per format (the pages name the formats only):
 *   MXFP4: amax = max|y| over 32; e = clamp(floor(log2 amax) - 2, -127, 127)
 *          (e = -127 for amax 0); scale byte e + 127; code = E2M1 RNE-satfinite
 *          of y / 2^e.
 *   NVFP4: s_b = UE4M3 RNE-satfinite(amax / (6 global_scale));
 *          code = E2M1 RNE-satfinite(y / (s_b global_scale)); codes 0 when s_b = 0.
 *          global_scale is the per-tensor fp32 scale, in [1e-30, 1e30).
 *   INT4:  s = fp16 RNE(amax / 7) (saturating at 65504);
 *          q = clamp(RNE(y / s), -7, 7) (0 if s = 0);
 *          code = q & 0xF (two's complement nibble).
 *   y is the fp32 transformed value.  Every decision is the round-to-nearest-even
 *   (ties to even) of the exact quotient, as written, of that fp32 value: the
 *   kernels multiply by reciprocals nudged 2^-20 below and above the scale's, and
 *   settle the rare values whose two results differ with an exact comparison
 *   against the boundary.  E2M1 codes carry the sign of y even when the magnitude
 *   rounds to 0; an all-zero block gives +0.
 *
 * x:       device [rows, d_in], bf16 (x_dtype = WUSH_IN_BF16) or fp32.
 * t:       device fp32 [d_in/b, b, b] for WUS/WUSH/WUSH_DIAG; ignored (may be NULL) for
 *          IDENTITY and HADAMARD (computed with in-register butterflies, then
 *          scaled by the fp32 constant 1/sqrt(b)).
 * codes:   device, wush_codes_bytes(rows, d_in, fmt) bytes.
 * scales:  device, wush_scales_bytes(rows, d_in, fmt) bytes.
 * y_debug: optional device fp32 [rows, d_in] receiving the transformed values
 *          before rounding (NULL to skip; costs 4 bytes/element of traffic).
 * Requirements: rows >= 0 (0 is a no-op), d_in % b == 0, d_in > 0.
 * ------------------------------------------------------------------------- */
int wush_transform_quant(const void* x, int x_dtype, int64_t rows, int64_t d_in,
                         const float* t, int kind, int fmt, float global_scale,
                         uint8_t* codes, void* scales, float* y_debug, void* stream);

/* wush_transform_quant with shared transforms: block j of every row uses
 * t[t_index[j]].  t: device fp32 [n_t, b, b]; t_index: device int32 [d_in/b]
 * (4-byte aligned), each entry clamped to [0, n_t - 1] on use; kind WUS, WUSH or
 * WUSH_DIAG (WUSH_ERR_INVALID_ARG otherwise).  Other arguments as in
 * wush_transform_quant.  With t_index[j] = j it equals wush_transform_quant. */
int wush_transform_quant_indexed(const void* x, int x_dtype, int64_t rows, int64_t d_in,
                                 const float* t, const int32_t* t_index, int n_t, int kind, int fmt,
                                 float global_scale, uint8_t* codes, void* scales, float* y_debug,
                                 void* stream);

/* max |T x| over a whole [rows, d_in] tensor, written as one fp32 to device
 * *amax_out (the call zeroes it first, in stream order).  Used offline for the
 * per-tensor NVFP4 scale global_scale = amax / (6 * 448) of a transformed
 * weight or calibration tensor.  Arguments as in wush_transform_quant with the
 * block size b given explicitly (16 or 32). */
int wush_transform_amax(const void* x, int x_dtype, int64_t rows, int64_t d_in,
                        const float* t, int kind, int block, float* amax_out, void* stream);

/* Dynamic per-tensor NVFP4 scale: wush_transform_quant for NVFP4 whose
 * global_scale is derived on the device from ``amax`` (device fp32, e.g.
 * written by wush_transform_amax on the same x, t and kind with block 16,
 * earlier in the stream) as
 *   global_scale = fp32(amax / 2688)   (2688 = 6 * 448),
 *   or 1 if that is below 1e-30 (an all-zero tensor: every code is 0).
 * The scale is written to device *global_scale_out (if not NULL) for
 * wush_qgemm_nvfp4_dynamic; with rows = 0 nothing is launched or written.
 * The pages name NVFP4 only; the static calibrated scale of
 * wush_transform_quant is the default reading, this is the per-batch variant.
 * Other arguments and requirements as in wush_transform_quant; amax and
 * global_scale_out 4-byte aligned. */
int wush_transform_quant_nvfp4_dynamic(const void* x, int x_dtype, int64_t rows, int64_t d_in,
                                       const float* t, int kind, const float* amax,
                                       float* global_scale_out, uint8_t* codes, void* scales,
                                       float* y_debug, void* stream);

/* ---------------------------------------------------------------------------
 * Block-scaled FP4 GEMM on tcgen05 tensor cores (device)
 *
 * AI Radio episode, "Conclusion": the W4A4 layer runs an FP4 MatMul (up to
 * 5.8x per layer over BF16).  y[m, n] = alpha * sum_k dq(a)[m, k] dq(b)[n, k]
 * with dq the element code times its block scale, products exact and fp32
 * accumulation.
 *
 * a_codes/a_scales: activation codes and scales from wush_transform_quant
 *                   (rows = M, d_in = K).
 * b_codes/b_scales: weight codes and scales from wush_transform_quant
 *                   (rows = N, d_in = K).
 * fmt:    WUSH_FMT_MXFP4 (UE8M0 per 32) or WUSH_FMT_NVFP4 (UE4M3 per 16).
 * alpha:  fp32 epilogue scale (NVFP4: global_scale_x * global_scale_w; MXFP4: 1).
 * y:      device fp32 [M, N] row-major, overwritten.
 * Requirements: M % 128 == 0, N % 128 == 0, K % 256 == 0, all > 0.
 * ------------------------------------------------------------------------- */
int wush_qgemm(const uint8_t* a_codes, const void* a_scales, const uint8_t* b_codes,
               const void* b_scales, int64_t M, int64_t N, int64_t K, int fmt, float alpha,
               float* y, void* stream);

/* NVFP4 wush_qgemm whose alpha is formed on the device as
 *   alpha = fp32(*a_global_scale * b_global_scale),
 * a_global_scale a device fp32 (4-byte aligned), e.g. written by
 * wush_transform_quant_nvfp4_dynamic earlier in the stream; b_global_scale the
 * weights' static scale.  Other arguments as in wush_qgemm with fmt NVFP4. */
int wush_qgemm_nvfp4_dynamic(const uint8_t* a_codes, const void* a_scales, const uint8_t* b_codes,
                             const void* b_scales, int64_t M, int64_t N, int64_t K,
                             const float* a_global_scale, float b_global_scale, float* y, void* stream);

/* ---------------------------------------------------------------------------
 * INT4 GEMM with per-32-group fp16 scales (device)
 *
 * WUSH news article, experiments paragraph (INT4 is the format with the largest
 * loss reduction).  y[m, n] = sum_g s_a[m, g] s_b[n, g] sum_{k in g} q_a q_b.
 * B200 tensor cores have no 4-bit integer or per-group-scaled integer MMA, so each
 * element is dequantised to fp16(q * s) (one rounding, relative error <= 2^-11)
 * and multiplied with fp16 MMAs accumulating in fp32.
 *
 * a_codes/a_scales: INT4 codes and fp16 scales of the activations from
 *                   wush_transform_quant (rows = M, d_in = K).
 * b_codes/b_scales: the same for the weights (rows = N).
 * y:      device fp32 [M, N] row-major, overwritten.
 * Requirements: M % 128 == 0, N % 256 == 0, K % 64 == 0, all > 0; scales 4-byte
 * aligned.
 * ------------------------------------------------------------------------- */
int wush_qgemm_int4(const uint8_t* a_codes, const void* a_scales, const uint8_t* b_codes,
                    const void* b_scales, int64_t M, int64_t N, int64_t K, float* y, void* stream);

/* Bytes of device workspace wush_qgemm_int4_ws needs: (M + N) * K * 2 (the fp16
 * operands); 0 if any size is <= 0. */
size_t wush_qgemm_int4_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Two-pass form of wush_qgemm_int4 with the same definition of y: every INT4
 * element of A and B is dequantised once to fp16(q * s) into ``workspace``
 * (device, caller-owned, A's [M, K] then B's [N, K], row-major), then the fp16
 * operands are multiplied with CTA-pair fp16 MMAs accumulating in fp32.  Cheaper
 * than the fused form whenever the operands are reused by many output tiles (the
 * fused form converts an element once per tile that reads it).
 * Requirements: M % 256 == 0, N % 256 == 0, K % 64 == 0, all > 0; codes,
 * workspace and y 16-byte aligned, scales 2-byte aligned; workspace_bytes >=
 * wush_qgemm_int4_workspace_bytes(M, N, K), else WUSH_ERR_BUFFER_TOO_SMALL.  All
 * checks run before any launch; three kernels are launched on ``stream``. */
int wush_qgemm_int4_ws(const uint8_t* a_codes, const void* a_scales, const uint8_t* b_codes,
                       const void* b_scales, int64_t M, int64_t N, int64_t K, void* workspace,
                       size_t workspace_bytes, float* y, void* stream);

/* ---------------------------------------------------------------------------
 * ITQ3_S-style 3-bit weights with a 256-wide Walsh-Hadamard rotation
 *
 * ITQ3_S article, "核心技术：FWHT预旋转与TurboQuant的完美融合": each 256-element
 * weight vector (256 consecutive d_in weights of one output row) is rotated with
 * the FWHT before a uniform 3-bit quantiser, and the exact inverse transform is
 * applied when the weights are loaded for the matmul.
 *   r = H_256 w / 16;  s = fp16 RNE(max|r| / 3.5);
 *   c = clamp(rint(r / s + 3.5), 0, 7) (c = 0 when s = 0), all in fp64;
 *   dequantised w_hat = H_256 ((c - 3.5) s) / 16.
 * Packed code layout (our own; the article calls its layout "interleaved"
 * without detail): per row and 256-block, 96 bytes holding the 256 three-bit
 * codes packed little-endian, element e at bits 3e .. 3e + 2 (bit b of the block
 * is bit b % 8 of byte b / 8).  rows * d_in * 3 / 8 bytes in all.
 * ------------------------------------------------------------------------- */

/* Host: w_fp16 host fp16 bits [d_out, d_in]; d_in % 256 == 0;
 * codes: host, d_out * d_in * 3 / 8 bytes; scales_fp16: host fp16 bits [d_out, d_in/256]. */
int itq3_quantize_weights(const uint16_t* w_fp16, int64_t d_out, int64_t d_in, uint8_t* codes,
                          uint16_t* scales_fp16);

/* y[t, o] = sum_k w_hat[o, k] x[t, k] on the device.
 * codes, scales_fp16: device, as written by itq3_quantize_weights.
 * x_fp16: device fp16 [tokens, d_in]; y: device fp32 [tokens, d_out], overwritten.
 * mode 0: the inverse FWHT is applied to every weight block as it is loaded
 *         (the article's fused design);
 * mode 1: the algebraically identical activation-side form
 *         sum_k ((c - 3.5) s)[o, k] (H_256 x / 16)[t, k]: x is rotated once per
 *         call into ``workspace`` (device fp32 [tokens, d_in], caller-owned
 *         scratch), then each weight is used without a transform.  When
 *         tokens >= 3 and d_out % 128 == 0 the weights meet x on the tensor
 *         cores: the levels
 *         c - 3.5 are exact fp16 MMA operands and each block of rotated x is
 *         split exactly enough (hi + lo fp16 after a power-of-two scale) that
 *         only the fp32 accumulation rounds; otherwise CUDA cores run it.
 *         For one or two tokens with tokens * d_in <= 40960 the call is a
 *         single kernel in which every CTA rotates x into its own shared
 *         memory; the workspace is then not touched.
 * workspace may be NULL for mode 0.  Requirements: 1 <= tokens <= 16,
 * d_in % 256 == 0, d_out % 8 == 0, codes, scales, x_fp16 and workspace 16-byte
 * aligned; WUSH_ERR_INVALID_ARG otherwise, before any launch. */
int itq3_dequant_gemv(const uint8_t* codes, const void* scales_fp16, const void* x_fp16,
                      int64_t tokens, int64_t d_out, int64_t d_in, int mode, float* workspace,
                      float* y, void* stream);

/* Allocation-free form of itq3_dequant_gemv mode 1.  The pages have no
 * counterpart: it exists for callers that cannot call cudaMalloc where they run
 * the GEMV (an engine that reserves all device memory in its own pool at start-up
 * and allows no later allocation, a real-time loop that cannot take an
 * allocation's latency or failure, a plugin whose host owns device memory).
 * Instead of a caller workspace, the rotated activations go to one fixed array
 * inside the library, 262,144 fp32 values (1 MiB) per device, held by every GPU
 * that loads the library until the process exits.
 * Arguments as in itq3_dequant_gemv; tokens * d_in must be <= 262,144, else
 * WUSH_ERR_BUFFER_TOO_SMALL and nothing is launched.  Calls no allocating
 * routine.  The first call on a device looks up the array's device address (with
 * that device current); make that first call before any stream capture.  The
 * address is kept per device and CUDA context: after a device reset (which makes
 * a new context) the next call looks it up again, so it too is a first call.  All
 * calls on a device share the array: calls whose kernels overlap on the GPU
 * (different streams, no ordering between them) race on it.  Nothing needs to
 * start at zero: every call overwrites the part of the array it reads.  One or two
 * tokens with tokens * d_in <= 40960 do not use the array (the single-kernel form
 * above). */
int itq3_dequant_gemv_noalloc(const uint8_t* codes, const void* scales_fp16, const void* x_fp16,
                              int64_t tokens, int64_t d_out, int64_t d_in, float* y, void* stream);

/* ---------------------------------------------------------------------------
 * Diagnostics
 * ------------------------------------------------------------------------- */

/* Synchronises ``stream``, then reports (and clears) the device error word set by
 * a kernel whose bounded wait gave up: WUSH_ERR_TIMEOUT, else WUSH_OK, or
 * WUSH_ERR_CUDA if the stream itself reports an error. */
int wush_check_device_status(void* stream);

/* Test hook: makes the next wush_qgemm launches give up their first barrier wait
 * after ``max_polls`` polls (0 restores the default limit) so that the timeout
 * path can be exercised without hanging anything. */
int wush_debug_set_wait_limit(int64_t max_polls);

/* Test hook: 0 (default) lets wush_qgemm use CTA-pair (cta_group::2) 256 x 256
 * tiles when M % 256 == 0 and N % 256 == 0; 1 uses single-CTA 128 x 256 tiles
 * (when N % 256 == 0), 2 single-CTA 128 x 128 tiles, so that the forms can be
 * checked against each other. */
int wush_debug_set_gemm_variant(int variant);

/* Test hook: 0 (default) lets itq3_dequant_gemv mode 1 and
 * itq3_dequant_gemv_noalloc run the single-kernel form when tokens <= 2 and
 * tokens * d_in <= 40960, and the tensor-core kernel when tokens >= 3,
 * d_out % 128 == 0 and no CTA gets more than 64 of the 256-blocks (always so for
 * d_in <= 16384); 1 always uses the CUDA-core kernel from 3 tokens on; 2 uses the
 * rotation kernel followed by the CUDA-core kernel for every token count; 3 uses
 * the single-kernel form for up to 8 tokens whenever tokens * d_in <= 40960.  So
 * the forms can be checked against each other.  WUSH_ERR_INVALID_ARG for other
 * values. */
int wush_debug_set_itq3_variant(int variant);

#ifdef __cplusplus
}
#endif

#endif /* WUSH_H */
