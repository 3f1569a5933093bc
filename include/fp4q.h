/*
 * fp4q.h -- C ABI of the block-scaled FP4 weight quantizer (CUDA, sm_100a).
 *
 * The library quantizes a dense row-major weight matrix W[rows][cols]
 * (bf16 or fp32) to
 *   NVFP4: 16-element blocks along a row, E2M1 elements, one E4M3 block scale
 *          chosen by a ScaleSweep window search, one FP32 global scale S;
 *   MXFP4: 32-element blocks along a row, E2M1 elements, one E8M0 block scale
 *          chosen by an exponent sweep, optionally after a fused random-sign
 *          32-point block Hadamard rotation.
 * Sources: "Resumo Tecnico: ScaleSweep" (gist.science, arXiv 2606.07618),
 * "Metodologia: ScaleSweep" secs. 1-3; "Bridging the Gap Between Promise and
 * Performance for Microscaling FP4 Quantization" (gist.science, arXiv
 * 2509.23202), technical summary secs. 1-3; "Resumo Tecnico: TORQ"
 * (gist.science, arXiv 2605.19561) sec. 2.B.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every pointer argument is DEVICE memory owned by the caller
 *           (for example a torch tensor's data pointer) unless stated.  The
 *           library allocates nothing and keeps no state between calls; it
 *           may be called from several host threads at once.
 * Streams.  Work is enqueued on `stream` (NULL = the legacy default stream)
 *           and the call returns without waiting.  No call synchronizes,
 *           allocates or copies through the host, so a sequence of calls can
 *           be captured into a CUDA graph.
 * Layout.   W is dense row-major, no leading-dimension stride.  Blocks never
 *           cross a row (cols is a multiple of the block size), so block b of
 *           the flattened tensor covers elements [b*B, b*B + B).
 *           codes:  rows*cols/2 bytes; element 2j is the low nibble of byte j,
 *                   element 2j+1 the high nibble; a nibble is sign<<3 | m
 *                   with magnitude code m: 0:0 1:0.5 2:1 3:1.5 4:2 5:3 6:4 7:6.
 *           scales: one byte per block, row-major [rows][cols/B]: an E4M3
 *                   bit pattern 0x01..0x7E (NVFP4) or an E8M0 byte e+127
 *                   (MXFP4).
 *           deq:    the reconstruction q * d in the input dtype (RN to bf16).
 *           block_loss: one fp32 per block, the selected candidate's loss.
 * Errors.   Argument errors are returned at once and nothing is enqueued:
 *           NULL required pointer (FP4Q_ERR_NULL), negative sizes or cols not
 *           a multiple of the block size (FP4Q_ERR_SHAPE), unknown dtype or
 *           format (FP4Q_ERR_DTYPE), a data pointer not aligned as stated
 *           (FP4Q_ERR_ALIGN).  A failed launch returns FP4Q_ERR_CUDA (see
 *           fp4q_last_cuda_error).  An empty tensor (rows or cols == 0) is
 *           valid: after the dtype and shape checks the call returns FP4Q_OK,
 *           enqueues nothing (except where stated) and reads none of its data
 *           pointers, which may then be NULL.
 *           Data-dependent errors are found on the device and OR-ed into the
 *           caller's int32 status word *d_status as FP4Q_FLAG_* bits; the
 *           caller zeroes it before the calls and reads it after a
 *           synchronize.  When a flag is set the outputs are unspecified.
 * Numerics. All arithmetic is IEEE binary32 with round-to-nearest-even, no
 *           fused multiply-add (except the error updates that
 *           fp4q_nvfp4_gptq defines as fused) and no flush-to-zero.  Each block's loss is
 *           accumulated sequentially over its elements in column order:
 *             r = x*inv; q = E2M1(r); y = q*d; e = x - y;
 *             MSE: L = L + e*e        WMSE: L = L + w[col]*(e*e)
 *           and candidates are visited in ascending order, the first one kept
 *           and a later one taken only on a strictly smaller loss (ties go to
 *           the smaller bit pattern).  E2M1 rounding is to nearest, ties to
 *           the even code, saturating at 6; the sign of the input is kept,
 *           so a negative value that rounds to zero encodes as 0x8.
 */
#ifndef FP4Q_H
#define FP4Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* fp4q_stream_t;

typedef enum {
    FP4Q_OK = 0,
    FP4Q_ERR_NULL = 1,
    FP4Q_ERR_SHAPE = 2,
    FP4Q_ERR_DTYPE = 3,
    FP4Q_ERR_ALIGN = 4,
    FP4Q_ERR_NONFINITE = 5,
    FP4Q_ERR_CUDA = 6,
    FP4Q_ERR_RANGE = 7,
    FP4Q_ERR_ARG = 8
} fp4q_status;

typedef enum { FP4Q_F32 = 0, FP4Q_BF16 = 1 } fp4q_dtype;
typedef enum { FP4Q_NVFP4 = 0, FP4Q_MXFP4 = 1 } fp4q_format;

/* Bits OR-ed into *d_status by the device. */
#define FP4Q_FLAG_NONFINITE 1  /* a NaN or Inf reached the scale search     */
#define FP4Q_FLAG_RANGE     2  /* NVFP4: max|x| nonzero and outside [2^-64, 2^64] */
#define FP4Q_FLAG_TIMEOUT   4  /* batch: a tile gave up waiting for its weight's max */

#define FP4Q_NVFP4_BLOCK 16
#define FP4Q_MXFP4_BLOCK 32

/* Library version: major*10000 + minor*100 + patch. */
int fp4q_version(void);

/* Static description of a status code. */
const char* fp4q_status_string(fp4q_status status);

/* Text of the CUDA error behind the calling thread's last FP4Q_ERR_CUDA. */
const char* fp4q_last_cuda_error(void);

/*
 * fp4q_global_absmax -- gmax = max |x_i| over n elements.
 * ScaleSweep summary, "Metodologia" sec. 2: the FP32 global scale is
 * S = max|x| / (256*6), so the whole tensor's max magnitude is needed first.
 *   x       device, n elements of dtype `dt`, 16-byte aligned.
 *   d_amax  device, one float; overwritten (the call first zeroes it, then
 *           every thread block merges its maximum with an atomic max on the
 *           bit pattern).  A NaN anywhere makes *d_amax a NaN; an Inf makes it
 *           +Inf.  n == 0 leaves *d_amax = 0.
 *   d_status  device int32 or NULL.  When given, a one-warp kernel enqueued
 *           after the reduction reads the final *d_amax and ORs
 *           FP4Q_FLAG_NONFINITE into *d_status if it is a NaN or an Inf, or
 *           FP4Q_FLAG_RANGE if it is nonzero and outside [2^-64, 2^64] (the
 *           range inside which the NVFP4 sweep accepts a global max), so a
 *           caller of this call alone learns whether the global scale is
 *           usable.  NULL skips that check (the sweep performs it anyway).
 * Errors: FP4Q_ERR_NULL, FP4Q_ERR_SHAPE (n < 0), FP4Q_ERR_DTYPE,
 * FP4Q_ERR_ALIGN, FP4Q_ERR_CUDA.
 */
fp4q_status fp4q_global_absmax(const void* x, fp4q_dtype dt, int64_t n, float* d_amax,
                               int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_nvfp4_sweepmse -- NVFP4 ScaleSweep with the MSE objective.
 * ScaleSweep summary, "Metodologia" secs. 1-3: S = gmax / 1536 (S = 1 when
 * gmax == 0); per 16-element block s_base = E4M3_rne_sat(amax / (6*S)) (the
 * block maximum relative to S rounded to FP8, pattern p); the candidates are
 * the E4M3 patterns p-3 .. p+7 (Lemma 4.3 lower bound 4/5 s_base, Lemma 4.1
 * upper bound 12/7 s_base) clipped to 0x01..0x7E; candidate p' has step
 * d = E4M3(p')*S and reciprocal inv = 1/d; the block keeps the candidate with
 * the smallest loss (conventions above).
 *   w            device, rows*cols elements of `dt`, 16-byte aligned.
 *   rows, cols   cols % 16 == 0.
 *   d_amax       device, one float: max|w| from fp4q_global_absmax.
 *   codes        device, rows*cols/2 bytes, 8-byte aligned.
 *   scales_e4m3  device, rows*cols/16 bytes.
 *   d_global_scale  device, one float: receives S.
 *   deq          device or NULL, rows*cols elements of `dt`, 16-byte aligned.
 *   block_loss   device or NULL, rows*cols/16 floats, 4-byte aligned.
 *   d_status     device int32: FP4Q_FLAG_NONFINITE if gmax is NaN/Inf,
 *                FP4Q_FLAG_RANGE if gmax is nonzero and outside [2^-64, 2^64].
 */
fp4q_status fp4q_nvfp4_sweepmse(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                                const float* d_amax, uint8_t* codes, uint8_t* scales_e4m3,
                                float* d_global_scale, void* deq, float* block_loss,
                                int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_nvfp4_sweepwmse -- NVFP4 ScaleSweep with the importance-weighted MSE.
 * ScaleSweep summary, "Metodologia" sec. 1 (WMSE weights errors by importance
 * scores from activation norms or Gram-matrix diagonals) and sec. 2 (the lower
 * bound is set empirically to 1/2 s_base, offset -8): candidates p-8 .. p+7,
 * loss L = L + importance[col]*(e*e).  Arguments as fp4q_nvfp4_sweepmse plus
 *   importance   device, cols floats (one per input column), 16-byte aligned,
 *                used as given (diag(X^T X) or any non-negative weights).
 */
fp4q_status fp4q_nvfp4_sweepwmse(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                                 const float* d_amax, const float* importance, uint8_t* codes,
                                 uint8_t* scales_e4m3, float* d_global_scale, void* deq,
                                 float* block_loss, int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_mxfp4_quant -- MXFP4 with an E8M0 exponent sweep.
 * MR-GPTQ summary, technical sec. 1 (32-element groups, power-of-two E8M0
 * scales) and sec. 2 (scales chosen to minimise the MSE); TORQ summary sec.
 * 2.B (the block maximum maps onto the largest code).  Per 32-element block:
 * e0 = the smallest e with 6*2^e >= amax (e0 = -127 for a zero block), clamped
 * to [-127, 127]; the candidates e0-1, e0, e0+1 (clamped) use d = 2^e and
 * inv = 2^-e with the MSE loss; the scale byte is e*+127.
 *   w        device, rows*cols elements of `dt`, 16-byte aligned; cols % 32 == 0.
 *   codes    device, rows*cols/2 bytes, 16-byte aligned.
 *   scales_e8m0  device, rows*cols/32 bytes.
 *   deq      device or NULL, rows*cols elements of `dt`, 16-byte aligned.
 *   block_loss   device or NULL, rows*cols/32 floats.
 *   d_status device int32: FP4Q_FLAG_NONFINITE if a block holds a NaN/Inf.
 */
fp4q_status fp4q_mxfp4_quant(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                             uint8_t* codes, uint8_t* scales_e8m0, void* deq, float* block_loss,
                             int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_mxfp4_quant_hadamard -- MXFP4 after a fused random-sign block Hadamard.
 * MR-GPTQ summary, technical sec. 2 ("Rotacoes Online Fundidas": block
 * Hadamard micro-rotations fused into the GPU kernels) and sec. 3.  Each
 * 32-block is rotated in registers before the exponent sweep:
 * y = c * H32 * diag(sigma) * x, sigma_j = -1 where bit j of
 * sign_masks[col/32] is set, H32 the Sylvester (natural-order) Hadamard applied
 * as five butterfly stages h = 1,2,4,8,16 ((a,b) -> (a+b, a-b)), then every
 * element times c = RN(1/sqrt(32)).  The codes, scales, deq and loss are those
 * of the rotated block (deq is in the rotated domain).
 *   sign_masks  device, cols/32 uint32 (one mask per 32-column group, shared
 *               by all rows), 4-byte aligned.
 * Other arguments as fp4q_mxfp4_quant; FP4Q_FLAG_NONFINITE also covers a
 * rotation that overflows.
 */
fp4q_status fp4q_mxfp4_quant_hadamard(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                                      const uint32_t* sign_masks, uint8_t* codes,
                                      uint8_t* scales_e8m0, void* deq, float* block_loss,
                                      int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_mxfp4_quant_absmax -- fp4q_mxfp4_quant (sign_masks == NULL) or
 * fp4q_mxfp4_quant_hadamard (sign_masks != NULL) that also writes max|w| of
 * the unrotated weight to *d_amax, exactly as fp4q_global_absmax would (NaN
 * and Inf propagate), so that an NVFP4 sweep of the same weight needs no
 * separate read for its global scale ("Metodologia: ScaleSweep" sec. 2).
 *   d_amax  device float, overwritten (zeroed first, then atomic max).
 * Other arguments and errors as fp4q_mxfp4_quant; an empty tensor only
 * zeroes *d_amax.
 */
fp4q_status fp4q_mxfp4_quant_absmax(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                                    const uint32_t* sign_masks, uint8_t* codes, uint8_t* scales_e8m0,
                                    void* deq, float* block_loss, float* d_amax, int32_t* d_status,
                                    fp4q_stream_t stream);

/*
 * fp4q_quantize_dual -- NVFP4 ScaleSweep and MXFP4 of the same weight.
 * The same results as fp4q_global_absmax + fp4q_nvfp4_sweep{mse,wmse} +
 * fp4q_mxfp4_quant{,_hadamard}, in two launches instead of three:
 * fp4q_mxfp4_quant_absmax, then the NVFP4 sweep (MSE when importance is NULL,
 * WMSE otherwise) on its *d_amax, so W is read twice instead of three times.
 *   importance  device or NULL (cols floats, 16-byte aligned): WMSE weights.
 *   sign_masks  device or NULL (cols/32 uint32): rotate the MXFP4 blocks.
 *   d_amax, d_global_scale  device floats (written).
 *   nv_*        NVFP4 outputs as in fp4q_nvfp4_sweepmse (nv_deq, nv_loss
 *               may be NULL).
 *   mx_*        MXFP4 outputs as in fp4q_mxfp4_quant (mx_deq, mx_loss may be
 *               NULL).
 * cols % 32 == 0.  Errors as the separate calls; d_status collects both.
 */
fp4q_status fp4q_quantize_dual(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                               const float* importance, const uint32_t* sign_masks, float* d_amax,
                               uint8_t* nv_codes, uint8_t* nv_scales, float* d_global_scale,
                               void* nv_deq, float* nv_loss, uint8_t* mx_codes, uint8_t* mx_scales,
                               void* mx_deq, float* mx_loss, int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_focus_quant -- the FOCUS forward quantizer ("FOCUS" summary,
 * gist.science, arXiv 2608.01847, "Metodologia" 2-3): quantize with a
 * quantization scale decoupled from the stored one.  Each hardware block
 * keeps its dequantization scale S_dq (NVFP4: E4M3 pattern p times the global
 * scale S; MXFP4: E8M0 byte b, 2^(b-127)); sub-block k of sub_block elements
 * is quantized with S_q = S_dq * c_k (CRS: sub_block = the block size; DGS: a
 * smaller sub-block, e.g. 8), and the stored reconstruction uses S_dq:
 *   d = RN(E4M3(p) * S) or 2^(b-127);  dq = RN(d * c_k);  inv = RN(1 / dq)
 *   code = E2M1(RN(x * inv));  deq = RN(q * d);
 *   block_loss = sum over the block, in column order, of RN(x - deq)^2.
 * The codes with the given scales are a standard NVFP4/MXFP4 tensor (the
 * coefficients are not stored).
 *   fmt         FP4Q_NVFP4 (16-element blocks) or FP4Q_MXFP4 (32).
 *   w, dt, rows, cols   as the quantizers (cols a multiple of the block).
 *   scales      device, one byte per block (E4M3 patterns 0x01..0x7E or E8M0
 *               bytes 0..254), row-major [rows][cols/block].
 *   d_global_scale  device float S (NVFP4; ignored and may be NULL for MXFP4).
 *   coeffs_f16  device, IEEE binary16 coefficients c_k, [rows][cols/sub_block],
 *               2-byte aligned; must be positive and finite.
 *   sub_block   4, 8 or 16 (and 32 for MXFP4).
 *   codes, deq, block_loss  as the quantizers (deq, block_loss may be NULL).
 * Errors: as the quantizers, FP4Q_ERR_ARG for another sub_block; on the
 * device FP4Q_FLAG_RANGE for a scale byte or coefficient outside the allowed
 * values and FP4Q_FLAG_NONFINITE for a NaN/Inf input (outputs of such blocks
 * unspecified).
 */
fp4q_status fp4q_focus_quant(fp4q_format fmt, const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                             const uint8_t* scales, const float* d_global_scale, const void* coeffs_f16,
                             int32_t sub_block, uint8_t* codes, void* deq, float* block_loss, int32_t* d_status,
                             fp4q_stream_t stream);

/*
 * fp4q_mxfp4_unrotate -- map a rotated-domain MXFP4 reconstruction (the deq of
 * fp4q_mxfp4_quant_hadamard) back to the original domain (MR-GPTQ summary,
 * technical sec. 2).  Per 32-block: the five butterfly stages h = 1..16 of
 * the rotation, every element times c = RN(1/sqrt(32)), then the sign flips
 * of sign_masks; (c * H32)^2 = I, so this inverts the rotation up to rounding.
 *   y, out      device, rows x cols of dt, 16-byte aligned (may not overlap).
 *   sign_masks  device, cols/32 uint32 as for the rotation.
 * cols % 32 == 0.  Errors as fp4q_mxfp4_quant_hadamard.
 */
fp4q_status fp4q_mxfp4_unrotate(const void* y, fp4q_dtype dt, int64_t rows, int64_t cols,
                                const uint32_t* sign_masks, void* out, fp4q_stream_t stream);

/*
 * fp4q_gptq_workspace_bytes -- workspace of fp4q_nvfp4_gptq: the scaled errors
 * of two consecutive 128-column blocks, 2 * 128 * ceil4(rows) floats
 * (ceil4: rounded up to a multiple of 4); 0 for rows <= 0.
 */
size_t fp4q_gptq_workspace_bytes(int64_t rows);

/*
 * fp4q_nvfp4_gptq -- NVFP4 with the ScaleSweep inside GPTQ (ScaleSweep
 * summary, "Contribuicoes" 2: the sweep selects the block scales of GPTQ
 * pipelines too).  GPTQ in its Cholesky form: U is the upper Cholesky factor
 * of the inverse of the layer's dampened input Gram matrix (U^T U = H^-1;
 * the caller computes it).  Rows are independent; along a row, at the first
 * column of every 16-column group the ScaleSweep (MSE window -3..+7, global
 * scale S = max|w|/1536 of the ORIGINAL weight) picks the group's pattern from
 * the row's current, error-compensated values, and every column j is
 * quantized with its group's step d and spreads its error:
 *   y_j = RN(E2M1(RN(w_j * RN(1/d))) * d);   e_j = RN((w_j - y_j) / U[j][j])
 *   w_c = fma(-e_j, U[j][c], w_c) for every c > j (one rounding each).
 * The blocked GPU algorithm applies these updates to every element in the
 * same order, so its bytes are those of the sequential definition.
 *   w          device fp32 rows x cols (cols % 16 == 0), 16-byte aligned;
 *              used as scratch and OVERWRITTEN: each 128-column block is
 *              left holding its values after the updates of the blocks
 *              before it (the updates inside the block stay in registers),
 *              so keep a copy if the original weight is needed.
 *   U          device fp32 cols x cols, row-major; only the upper triangle
 *              (diagonal included) is read.
 *   d_amax     device float: max|w| of the original weight
 *              (fp4q_global_absmax before this call).
 *   codes, scales_e4m3, d_global_scale, deq (fp32, may be NULL) as
 *              fp4q_nvfp4_sweepmse.
 *   workspace  device, 16-byte aligned, fp4q_gptq_workspace_bytes(rows).
 * 2 * ceil(cols/128) - 1 launches: per block of 128 columns one launch runs
 * the block's in-block GPTQ beside the trailing update of the previous
 * block's errors, and a small one applies the block's errors to the next
 * block.  Errors as fp4q_nvfp4_sweepmse, plus
 * FP4Q_ERR_ARG for a small workspace and FP4Q_ERR_SHAPE for cols > 2^20.
 */
fp4q_status fp4q_nvfp4_gptq(float* w, int64_t rows, int64_t cols, const float* U, const float* d_amax,
                            uint8_t* codes, uint8_t* scales_e4m3, float* d_global_scale, float* deq,
                            void* workspace, size_t workspace_bytes, int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_mma_scale_bytes -- bytes of the tiled scale layout written by
 * fp4q_scales_to_mma_layout for a [rows][scale_cols] scale matrix:
 * ceil(rows/128) * ceil(scale_cols/4) * 512; -1 for a negative or
 * overflowing size.
 */
int64_t fp4q_mma_scale_bytes(int64_t rows, int64_t scale_cols);

/*
 * fp4q_scales_to_mma_layout -- block scales in the layout that Blackwell
 * block-scaled FP4 GEMMs read (the MR-GPTQ summary, technical sec. 3, runs the
 * quantized weights through such kernels; the pages do not describe the
 * layout, it is the hardware's).  The [rows][scale_cols] matrix of scale
 * bytes (E4M3 for NVFP4 with scale_cols = cols/16, E8M0 for MXFP4 with
 * scale_cols = cols/32, as written by the quantizers above) is cut into tiles
 * of 128 rows x 4 scale columns, zero-padded at the bottom and right edges;
 * tiles are stored one after the other, the column tiles of one row tile
 * together; inside a 512-byte tile the byte of (row r, column c) is at
 * (r % 32) * 16 + (r / 32) * 4 + c.  The packed codes need no change: their
 * row-major nibble order (element 2j in the low nibble of byte j) is the
 * K-major operand order of those GEMMs.
 *   scales  device, rows * scale_cols bytes, row-major.
 *   out     device, 16-byte aligned, fp4q_mma_scale_bytes(rows, scale_cols)
 *           bytes, fully written (padding zeroed).
 * Errors: FP4Q_ERR_SHAPE (negative sizes), FP4Q_ERR_NULL, FP4Q_ERR_ALIGN; an
 * empty matrix touches nothing.
 */
fp4q_status fp4q_scales_to_mma_layout(const uint8_t* scales, int64_t rows, int64_t scale_cols, uint8_t* out,
                                      fp4q_stream_t stream);

/*
 * fp4q_dynamic_workspace_bytes -- size of the workspace of
 * fp4q_nvfp4_sweep_dynamic (16 bytes).
 */
size_t fp4q_dynamic_workspace_bytes(void);

/*
 * fp4q_nvfp4_sweep_dynamic -- fp4q_global_absmax followed by
 * fp4q_nvfp4_sweepmse (importance == NULL) or fp4q_nvfp4_sweepwmse, in ONE
 * launch, for tensors quantized at every call (the activations of the
 * weights+activations configurations, ScaleSweep summary "Resultados
 * Experimentais"; S = max|x|/(256*6), "Metodologia: ScaleSweep" sec. 2).
 * The global max and the sweep are separated by a barrier inside the launch:
 * tensors of at most 16 x 256 16-element blocks run as one thread-block
 * cluster (hardware cluster barriers, maxima exchanged through distributed
 * shared memory; the workspace is not touched), larger ones as a cooperative
 * launch (every thread block resident at once) with a grid-wide barrier on
 * the workspace.  The bytes written are those of the two separate calls.
 *   x, dt, rows, cols        as fp4q_nvfp4_sweepmse (cols % 16 == 0).
 *   importance               device or NULL (cols floats, 16-byte aligned).
 *   d_amax, d_global_scale   device floats, written (max|x| and S).
 *   codes, scales_e4m3, deq, block_loss   as fp4q_nvfp4_sweepmse.
 *   workspace                device, 16-byte aligned, at least
 *                            fp4q_dynamic_workspace_bytes() bytes, ZEROED
 *                            before its first use.  Every call leaves it
 *                            zeroed again, except one that raised
 *                            FP4Q_FLAG_TIMEOUT (zero it again after that).
 *                            Calls that may run at the same time need
 *                            separate workspaces.
 * The barrier wait is bounded (about two seconds); on expiry
 * FP4Q_FLAG_TIMEOUT is raised and the sweep is skipped.  Errors otherwise as
 * the separate calls, plus FP4Q_ERR_ARG for a workspace that is too small
 * and FP4Q_ERR_CUDA if the device cannot run a cooperative launch.  An empty
 * tensor only zeroes *d_amax.  The paper has no counterpart of the workspace:
 * it is how one launch replaces two.
 */
fp4q_status fp4q_nvfp4_sweep_dynamic(const void* x, fp4q_dtype dt, int64_t rows, int64_t cols,
                                     const float* importance, float* d_amax, uint8_t* codes,
                                     uint8_t* scales_e4m3, float* d_global_scale, void* deq,
                                     float* block_loss, void* workspace, size_t workspace_bytes,
                                     int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_quantize_batch -- fp4q_quantize_dual for a list of weights, in one
 * persistent launch per FP4Q_BATCH_MAX weights.
 * Thread blocks take 16384-element tiles from a device queue ordered
 * MXFP4(0) MXFP4(1) NVFP4(0) MXFP4(2) NVFP4(1) ...: the MXFP4 tiles of a weight
 * also reduce its max|w|, and its NVFP4 tiles (ScaleSweep summary,
 * "Metodologia: ScaleSweep" secs. 2-3: S = max|x|/(256*6)) start once all of
 * them have finished, so memory-bound and arithmetic-bound tiles share the
 * SMs.  Results are identical to the single-weight calls.
 *   tensors   HOST array of n descriptors; it is read during the call only
 *             (the descriptors travel to the device as a kernel argument).
 *             Per weight: w (16-byte aligned, rows x cols, cols % 32 == 0);
 *             importance (NULL: NVFP4 MSE, else WMSE weights [cols]);
 *             sign_masks (NULL: plain MXFP4, else the block Hadamard masks
 *             [cols/32]); amax and global_scale (device floats, written);
 *             nv_codes, nv_scales, nv_deq, nv_loss and mx_codes, mx_scales,
 *             mx_deq, mx_loss as in fp4q_quantize_dual (deq/loss may be NULL).
 *   dt        dtype of every w (and of every deq).
 *   workspace device scratch of at least fp4q_batch_workspace_bytes()
 *             bytes, 16-byte aligned, owned by the caller; zeroed by the call
 *             (stream-ordered) before each launch.  Launches that overlap on
 *             the device must not share a workspace.
 *   d_status  FP4Q_FLAG_NONFINITE / FP4Q_FLAG_RANGE as the single calls, and
 *             FP4Q_FLAG_TIMEOUT if an NVFP4 tile waited about two seconds for
 *             its weight's MXFP4 tiles (the tile is then skipped; this does
 *             not happen when the tiles make progress).
 * An empty weight (rows or cols == 0) gets amax = 0 and global_scale = 1.
 * Errors: FP4Q_ERR_SHAPE (n < 0, a bad shape), FP4Q_ERR_NULL, FP4Q_ERR_ALIGN,
 * FP4Q_ERR_DTYPE, FP4Q_ERR_ARG (workspace too small), FP4Q_ERR_CUDA; the
 * descriptors are all checked before anything is enqueued.
 */
#define FP4Q_BATCH_MAX 128

typedef struct {
    const void* w;
    int64_t rows;
    int64_t cols;
    const float* importance;
    const uint32_t* sign_masks;
    float* amax;
    float* global_scale;
    uint8_t* nv_codes;
    uint8_t* nv_scales;
    void* nv_deq;
    float* nv_loss;
    uint8_t* mx_codes;
    uint8_t* mx_scales;
    void* mx_deq;
    float* mx_loss;
} fp4q_batch_tensor;

size_t fp4q_batch_workspace_bytes(void);

fp4q_status fp4q_quantize_batch(const fp4q_batch_tensor* tensors, int32_t n, fp4q_dtype dt,
                                void* workspace, size_t workspace_bytes, int32_t* d_status,
                                fp4q_stream_t stream);

/*
 * fp4q_quantize_batch_static -- fp4q_quantize_batch without a caller-provided
 * workspace, for callers that cannot allocate device memory when they
 * quantize: a process whose device memory is handed out entirely by another
 * allocator (so that an extra cudaMalloc could fail or fragment its pool), a
 * fixed device-memory budget set at start-up, or a latency-critical path that
 * must not call cudaMalloc (which can synchronize the device).  The pages have
 * no counterpart; this is a library convenience.
 * The scratch (the tile queue counter and the per-weight max and completion
 * counters, a little over 1 KB) is a static array inside the library, which
 * every GPU that loads the library holds until the process exits.  The call
 * allocates nothing and calls no allocating routine.
 *   n         at most FP4Q_BATCH_MAX weights per call (one launch); more
 *             returns FP4Q_ERR_ARG before anything is enqueued.
 * Other arguments, results and errors as fp4q_quantize_batch.
 * The first call on a device looks up the scratch's device address
 * (cudaGetSymbolAddress, with that device current) and keeps it for the rest
 * of the process; make that first call before any stream capture.  Under lazy
 * module loading that first call is also what loads the library's device code
 * on that device, which is when the runtime places the scratch (the one
 * allocation involved, done by the runtime, once).  The kept address belongs
 * to the device's current context: after cudaDeviceReset on that device it is
 * stale and this entry point must not be called again in the process.  The
 * scratch is zeroed, stream-ordered, at the
 * start of every call, but it is shared by all calls on a device: calls whose
 * launches overlap on the GPU (different streams without ordering between
 * them) race on it and give wrong results.
 */
fp4q_status fp4q_quantize_batch_static(const fp4q_batch_tensor* tensors, int32_t n, fp4q_dtype dt,
                                       int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_mxfp4_quant_group -- fp4q_mxfp4_quant_absmax for a list of weights,
 * one launch per FP4Q_GROUP_MAX weights of one kind (plain and rotated
 * weights go to separate launches, in list order).  The launch's thread
 * blocks are split among its weights in proportion to their sizes, each block
 * working on one weight exactly as the single call's kernel would, so a list
 * of small weights does not leave the GPU idle at the end of each one.
 * Results are identical to the single calls.
 *   tensors   HOST array of n fp4q_batch_tensor descriptors (read during the
 *             call only).  Read per weight: w, rows, cols (cols % 32 == 0),
 *             sign_masks (NULL: plain MXFP4, else the block Hadamard masks),
 *             amax (written: max|w| of the unrotated weight, 0 if empty),
 *             mx_codes, mx_scales, mx_deq and mx_loss (deq/loss may be NULL);
 *             the other fields are ignored.
 *   dt, d_status, stream   as fp4q_mxfp4_quant_absmax.
 * Errors as fp4q_mxfp4_quant_absmax; every descriptor is checked before
 * anything is enqueued.
 */
#define FP4Q_GROUP_MAX 32

fp4q_status fp4q_mxfp4_quant_group(const fp4q_batch_tensor* tensors, int32_t n, fp4q_dtype dt,
                                   int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_nvfp4_sweep_group -- fp4q_nvfp4_sweepmse / fp4q_nvfp4_sweepwmse for a
 * list of weights, one launch per FP4Q_GROUP_MAX weights of one kind (MSE and
 * WMSE weights go to separate launches), thread blocks split as in
 * fp4q_mxfp4_quant_group (ScaleSweep summary, "Metodologia: ScaleSweep"
 * secs. 2-3 per weight).  Results are identical to the single calls.
 *   tensors   HOST array of n descriptors.  Read per weight: w, rows, cols
 *             (cols % 16 == 0), importance (NULL: MSE window, else the WMSE
 *             weights [cols]), amax (read: max|w|, e.g. written by
 *             fp4q_mxfp4_quant_group earlier on the stream), global_scale
 *             (written), nv_codes, nv_scales, nv_deq, nv_loss (deq/loss may be
 *             NULL); the other fields are ignored.  An empty weight is skipped.
 *   dt, d_status, stream   as fp4q_nvfp4_sweepmse.
 * Errors as fp4q_nvfp4_sweepmse; every descriptor is checked first.
 */
fp4q_status fp4q_nvfp4_sweep_group(const fp4q_batch_tensor* tensors, int32_t n, fp4q_dtype dt,
                                   int32_t* d_status, fp4q_stream_t stream);

/*
 * fp4q_dequant -- decode codes and scales back to values.
 * NVFP4: out = RN(q * RN(E4M3(s) * S)), S = *d_global_scale; MXFP4:
 * out = q * 2^(b-127); then rounded to `out_dt`.  Reproduces the `deq` output
 * of the quantizers bit for bit.  A NaN scale pattern (E4M3 0x7F/0xFF, E8M0
 * 0xFF) decodes to NaN; E4M3 patterns with the sign bit decode as negative.
 *   codes   device, rows*cols/2 bytes, 8-byte aligned (16 for MXFP4).
 *   scales  device, rows*cols/16 (NVFP4) or rows*cols/32 (MXFP4) bytes.
 *   d_global_scale  device float (NVFP4 only; ignored and may be NULL for MXFP4).
 *   out     device, rows*cols elements of `out_dt`, 16-byte aligned.
 */
fp4q_status fp4q_dequant(fp4q_format format, const uint8_t* codes, const uint8_t* scales,
                         const float* d_global_scale, int64_t rows, int64_t cols, void* out,
                         fp4q_dtype out_dt, fp4q_stream_t stream);

/*
 * Diagnostic entry points: the device's element and scale rounding primitives
 * applied to n floats, so that they can be compared with a reference codec.
 *   fp4q_probe_e2m1: out[i] = E2M1 nibble of r[i] (sign<<3 | code).
 *   fp4q_probe_e4m3: out[i] = E4M3 pattern of v[i] >= 0 (RNE, saturating).
 * r/v device, 4-byte aligned; out device bytes.
 */
fp4q_status fp4q_probe_e2m1(const float* r, uint8_t* out, int64_t n, fp4q_stream_t stream);
fp4q_status fp4q_probe_e4m3(const float* v, uint8_t* out, int64_t n, fp4q_stream_t stream);

/*
 * fp4q_probe_copy -- diagnostic with no counterpart in the papers: a plain
 * streaming copy of `bytes` bytes (a multiple of 16, both pointers 16-byte
 * aligned, not overlapping) with the library's 16-byte loads and stores, so
 * that a benchmark can measure the copy bandwidth the library's own memory
 * instructions reach (its HBM roofline peak).
 */
fp4q_status fp4q_probe_copy(const void* src, void* dst, int64_t bytes, fp4q_stream_t stream);

/*
 * fp4q_probe_wait -- diagnostic with no counterpart in the papers: the
 * library's bounded spin-wait (the one the batch kernel and the one-launch
 * sweep use to wait for other thread blocks) run by one thread on its own.
 * It polls *flag until it is at least `target`, at most `limit` times about
 * 128 ns apart, and raises FP4Q_FLAG_TIMEOUT in *d_status if it gave up; so a
 * test can watch a wait run out and the context stay usable.
 *   flag      device uint32 (4-byte aligned), read only.
 *   limit     at most 2^24 (the library's own limit), else FP4Q_ERR_ARG.
 */
fp4q_status fp4q_probe_wait(const uint32_t* flag, uint32_t target, uint32_t limit, int32_t* d_status,
                            fp4q_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP4Q_H */
