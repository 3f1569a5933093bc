/*
 * fp4q_oracle.c -- plain, slow CPU oracle for block-scaled FP4 weight
 * quantization with a per-block scale search.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, table or constant generator with the
 * CUDA library; every routine here is written from the format definitions
 * and the method descriptions below, one IEEE-754 binary32 operation at a
 * time (compile with -ffp-contract=off and without -ffast-math).
 *
 * Sources (cited by page title and section):
 *  [SS]  "Resumo Tecnico: ScaleSweep" (gist.science, arXiv 2606.07618):
 *        "Declaracao do Problema" (NVFP4 = E2M1 elements, FP8 block scale,
 *        FP32 global scale), "Metodologia: ScaleSweep" sec. 1 (MSE / WMSE
 *        objectives), sec. 2 (126 finite positive FP8 values; S = max|x| /
 *        (256*6); s_base = block max rounded to FP8; Lemma 4.1 -> +7,
 *        Lemma 4.3 -> -3, WMSE empirical bound -> -8), sec. 3 (sweep the
 *        window and keep the candidate with the smallest objective).
 *  [MR]  "Bridging the Gap Between Promise and Performance for Microscaling
 *        FP4 Quantization" (gist.science, arXiv 2509.23202), technical
 *        summary sec. 1 (MXFP4 power-of-two E8M0 scales, 32-element groups),
 *        sec. 2 (MSE-optimised grid; fused block Hadamard micro-rotation).
 *  [TQ]  "Resumo Tecnico: TORQ" (gist.science, arXiv 2605.19561), sec. 2.B
 *        S-step: the block scale maps the block maximum onto the largest
 *        MXFP4 code.
 *  [FC]  "FOCUS" summary (gist.science, arXiv 2608.01847), "Declaracao do
 *        Problema": blocks of 32 (MXFP4) or 16 (NVFP4) values share one
 *        low-precision scale.
 *
 * Where the pages leave a step open the reading taken is stated at the
 * routine (E2M1 grid and ties-to-even, E4M3 rounding, window clamping, the
 * MXFP4 centre exponent, Hadamard order and normalisation, loss order).
 *
 * Parity pins: every function here is checked by tests/test_oracle_*.py
 * against values fixed by the format definitions and the pages (exhaustive
 * codec sweeps against nearest-value search, the 126-value count, the window
 * ratios of Lemmas 4.1/4.3, brute force over all 126 scales, closed forms,
 * fp64 recomputation of losses, the dense Sylvester Hadamard matrix).
 * orc_scales_to_mma_layout (a hardware layout the pages do not describe) is
 * pinned against CUTLASS's shape/stride definition of the same layout, and
 * by a library GEMM reading it on the GPU.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_NONFINITE 5
#define ORC_RANGE 7

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* E2M1 magnitudes indexed by the 3-bit magnitude code: exponent bits e (2),
 * mantissa bit m (1), bias 1; e == 0 is subnormal (m * 0.5), otherwise
 * 2^(e-1) * (1 + m/2).  [SS] "Declaracao do Problema" names E2M1. */
static float e2m1_mag(int code)
{
    int e = (code >> 1) & 3, m = code & 1;
    if (e == 0) return 0.5f * (float)m;
    return ldexpf(1.0f + 0.5f * (float)m, e - 1);
}

/* Round r to the nearest E2M1 value, ties to the even code (code LSB 0),
 * saturating to 6.  The sign bit is copied from r, so a negative value that
 * rounds to zero gives nibble 0x8 (-0).  Nibble = sign<<3 | magnitude code. */
int orc_e2m1_encode(float r)
{
    int sign = (int)(f2u(r) >> 31);
    float m = fabsf(r);
    int k, best = 7;                       /* beyond the last midpoint: 6 */
    if (isnan(r)) return (sign << 3) | 7;  /* never reached: inputs are checked finite */
    for (k = 0; k < 7; ++k) {
        float lo = e2m1_mag(k), hi = e2m1_mag(k + 1);
        float mid = 0.5f * (lo + hi);       /* exact: both have <= 2 significant bits */
        if (m < mid) { best = k; break; }
        if (m == mid) { best = (k % 2 == 0) ? k : k + 1; break; }
    }
    return (sign << 3) | best;
}

float orc_e2m1_decode(int nibble)
{
    float v = e2m1_mag(nibble & 7);
    return (nibble & 8) ? -v : v;
}

/* E4M3 (the FN variant: bias 7, subnormals, no infinity, 0x7F = NaN).
 * Pattern p in 0..126 of the non-negative finite values.  [SS] sec. 2 counts
 * 126 finite positive values: patterns 0x01..0x7E. */
float orc_e4m3_value(int p)
{
    int sign = (p >> 7) & 1, e = (p >> 3) & 15, m = p & 7;
    float v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexpf((float)m, -9);                   /* m/8 * 2^-6 */
    else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return sign ? -v : v;
}

/* Round v >= 0 to the nearest E4M3 value, ties to the even pattern, values
 * at or above 448 saturate to 0x7E.  Reading: the pages say "rounded to
 * FP8" without a mode; round-to-nearest-even with saturation is taken. */
int orc_e4m3_encode(float v)
{
    int p;
    if (!(v > 0.0f)) return 0;
    if (v >= 448.0f) return 0x7E;
    for (p = 0; p < 126; ++p) {
        float lo = orc_e4m3_value(p), hi = orc_e4m3_value(p + 1);
        if (v < hi) {
            float mid = 0.5f * (lo + hi);   /* exact: few significant bits */
            if (v < mid) return p;
            if (v > mid) return p + 1;
            return (p % 2 == 0) ? p : p + 1;
        }
    }
    return 0x7E;
}

/* E8M0: byte b encodes 2^(b-127); 0xFF is NaN.  [MR] sec. 1. */
float orc_e8m0_value(int b)
{
    if (b == 255) return NAN;
    return ldexpf(1.0f, b - 127);
}

/* binary32 -> bfloat16, round to nearest even on the dropped 16 bits. */
uint16_t orc_bf16_rne(float x)
{
    uint32_t u = f2u(x);
    if (isnan(x)) return (uint16_t)((u >> 16) | 0x40);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Array forms of the codecs, for exhaustive sweeps in the tests. */
void orc_e2m1_encode_array(const float* r, uint8_t* out, int64_t n)
{
    int64_t i;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (i = 0; i < n; ++i) out[i] = (uint8_t)orc_e2m1_encode(r[i]);
}

void orc_e4m3_encode_array(const float* v, uint8_t* out, int64_t n)
{
    int64_t i;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (i = 0; i < n; ++i) out[i] = (uint8_t)orc_e4m3_encode(v[i]);
}

void orc_round_bf16(const float* x, uint16_t* out, int64_t n)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = orc_bf16_rne(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Global absmax and global scale  ([SS] sec. 2: S = max|x| / (256*6))       */
/* ------------------------------------------------------------------------ */

/* max |x| over the tensor; NaN if any element is NaN. */
float orc_global_absmax(const float* x, int64_t n)
{
    float m = 0.0f;
    int64_t i;
    for (i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (isnan(a)) return NAN;
        if (a > m) m = a;
    }
    return m;
}

/* Supported magnitude of a non-zero max|x| for NVFP4: [2^-64, 2^64].  Inside
 * it every candidate scale and its reciprocal are finite normal numbers. */
int orc_gmax_status(float gmax)
{
    if (!isfinite(gmax)) return ORC_NONFINITE;
    if (gmax != 0.0f && (gmax < ldexpf(1.0f, -64) || gmax > ldexpf(1.0f, 64)))
        return ORC_RANGE;
    return ORC_OK;
}

/* S = max|x| / 1536, one IEEE division; S = 1 for an all-zero tensor. */
float orc_global_scale(float gmax)
{
    return (gmax > 0.0f) ? gmax / 1536.0f : 1.0f;
}

/* ------------------------------------------------------------------------ */
/* One block under one scale d: the objective of [SS] sec. 1                 */
/* ------------------------------------------------------------------------ */

/* Quantize the bs values of x with step d (reciprocal inv = 1/d) and return
 * the fp32 loss accumulated sequentially in column order:
 *   r = x_i * inv;  q = E2M1(r);  y = q * d;  e = x_i - y;
 *   MSE:  L = L + e*e            WMSE:  L = L + w_i * (e*e)
 * Every operation is a separately rounded binary32 operation (no fusion).
 * Optionally returns the nibbles and the reconstruction y. */
static float block_loss(const float* x, const float* w, int bs, float d, float inv,
                        uint8_t* nib, float* y_out)
{
    float L = 0.0f;
    int i;
    for (i = 0; i < bs; ++i) {
        float r = x[i] * inv;
        int c = orc_e2m1_encode(r);
        float q = orc_e2m1_decode(c);
        float y = q * d;
        float e = x[i] - y;
        float e2 = e * e;
        if (w) {
            float we2 = w[i] * e2;
            L = L + we2;
        } else {
            L = L + e2;
        }
        if (nib) nib[i] = (uint8_t)c;
        if (y_out) y_out[i] = y;
    }
    return L;
}

static void pack_nibbles(const uint8_t* nib, int bs, uint8_t* out)
{
    int j;
    for (j = 0; j < bs / 2; ++j)                   /* element 2j in the low nibble */
        out[j] = (uint8_t)((nib[2 * j] & 15) | ((nib[2 * j + 1] & 15) << 4));
}

/* ------------------------------------------------------------------------ */
/* NVFP4 ScaleSweep  ([SS] sec. 2 and 3)                                     */
/* ------------------------------------------------------------------------ */

/* Quantize a row-major rows x cols fp32 matrix (cols % 16 == 0) to NVFP4 with
 * the global scale S.  For every 16-element block along a row:
 *   amax = max|x_i|;  v = amax / (6*S);  p = E4M3_rne_sat(v)   (s_base)
 *   candidates p' = max(1, p+lo) .. min(126, p+hi), ascending
 *   d = E4M3(p') * S;  inv = 1/d;  L = block_loss(...)
 *   keep the first candidate, then any later one with L < best (strict):
 *   on equal losses the smaller bit pattern wins.
 * MSE uses (lo,hi) = (-3,+7) and importance == NULL; WMSE (-8,+7) with
 * importance[cols]; AbsMax is (0,0); the exhaustive search passes (-126,126).
 * Outputs (each may be NULL): codes[rows*cols/2], scales[rows*cols/16],
 * y[rows*cols] (reconstruction in fp32), loss[rows*cols/16], base[...] (s_base
 * pattern). */
/* The ScaleSweep selection for one 16-element block: s_base pattern p from
 * amax / (6*S), then the window p+lo .. p+hi clipped to 0x01..0x7E, first
 * minimum of block_loss.  Returns the chosen pattern; *best its loss, *base p. */
static int sweep_select(const float* xb, const float* wb, float S, int lo, int hi, float* best, int* base)
{
    const int bs = 16;
    float amax = 0.0f, t6, v;
    int i, p, pp, first, last, bp = 0;
    for (i = 0; i < bs; ++i) {
        float a = fabsf(xb[i]);
        if (a > amax) amax = a;
    }
    t6 = 6.0f * S;
    v = amax / t6;
    p = orc_e4m3_encode(v);
    first = p + lo < 1 ? 1 : p + lo;
    last = p + hi > 126 ? 126 : p + hi;
    *best = 0.0f;
    for (pp = first; pp <= last; ++pp) {
        float d = orc_e4m3_value(pp) * S;
        float inv = 1.0f / d;
        float L = block_loss(xb, wb, bs, d, inv, NULL, NULL);
        if (pp == first || L < *best) { *best = L; bp = pp; }
    }
    *base = p;
    return bp;
}

int orc_nvfp4_quant(const float* x, int64_t rows, int64_t cols, float S,
                    const float* importance, int lo, int hi,
                    uint8_t* codes, uint8_t* scales, float* y, float* loss,
                    uint8_t* base, int threads)
{
    const int bs = 16;
    int64_t nb = cols / bs, r;
    if (cols % bs) return 2;
#ifdef _OPENMP
    const int nt = threads > 0 ? threads : omp_get_max_threads();   /* this call only */
#pragma omp parallel for schedule(static) num_threads(nt)
#endif
    for (r = 0; r < rows; ++r) {
        int64_t b;
        for (b = 0; b < nb; ++b) {
            const float* xb = x + r * cols + b * bs;
            const float* wb = importance ? importance + b * bs : NULL;
            int64_t blk = r * nb + b;
            float best = 0.0f;
            int p, bp;
            uint8_t nib[16];
            bp = sweep_select(xb, wb, S, lo, hi, &best, &p);
            {
                float d = orc_e4m3_value(bp) * S;
                float inv = 1.0f / d;
                block_loss(xb, wb, bs, d, inv, nib, y ? y + r * cols + b * bs : NULL);
            }
            if (codes) pack_nibbles(nib, bs, codes + blk * (bs / 2));
            if (scales) scales[blk] = (uint8_t)bp;
            if (loss) loss[blk] = best;
            if (base) base[blk] = (uint8_t)p;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* ScaleSweep inside GPTQ  ([SS] "Contribuicoes" 2)                          */
/* ------------------------------------------------------------------------ */

/* [SS] presents ScaleSweep as the block-scale selection of both RTN and GPTQ
 * pipelines.  Reading (the page does not spell GPTQ out): GPTQ in its
 * Cholesky form, with U the upper Cholesky factor of the inverse of the
 * layer's dampened input Gram matrix (U^T U = H^-1), supplied by the caller.
 * Rows are independent; along a row the columns are taken in order.  At the
 * first column of every 16-column group the ScaleSweep (window lo..hi,
 * global scale S of the original weight) picks the group's E4M3 pattern from
 * the row's current, error-compensated values of the group; then every column
 * j is quantized with its group's step d (inv = RN(1/d)) and its scaled error
 * is spread over the later columns:
 *   y_j = RN(E2M1(RN(w_j * inv)) * d);   e_j = RN((w_j - y_j) / U[j][j])
 *   w_c = fma(-e_j, U[j][c], w_c)        for every c > j
 * (each update one fused multiply-add, one rounding).  Outputs: codes,
 * scales, the reconstruction y, and err[rows][cols] = e (may be NULL). */
int orc_nvfp4_gptq(const float* x, int64_t rows, int64_t cols, const float* U, float S, int lo, int hi,
                   uint8_t* codes, uint8_t* scales, float* y, float* err, int threads)
{
    const int bs = 16;
    int64_t nb = cols / bs, r;
    int status = ORC_OK;
    if (cols % bs) return 2;
#ifdef _OPENMP
    const int nt = threads > 0 ? threads : omp_get_max_threads();   /* this call only */
#pragma omp parallel for schedule(static) num_threads(nt)
#endif
    for (r = 0; r < rows; ++r) {
        float* w = (float*)malloc((size_t)cols * sizeof(float));
        int64_t j, c;
        float d = 1.0f, inv = 1.0f;
        uint8_t nib[16];
        if (!w) {
            status = 2;
            continue;
        }
        for (j = 0; j < cols; ++j) w[j] = x[r * cols + j];
        for (j = 0; j < cols; ++j) {
            float rr, q, yy, e;
            int code;
            if (j % bs == 0) {
                float best;
                int base, bp = sweep_select(w + j, NULL, S, lo, hi, &best, &base);
                d = orc_e4m3_value(bp) * S;
                inv = 1.0f / d;
                if (scales) scales[r * nb + j / bs] = (uint8_t)bp;
            }
            rr = w[j] * inv;
            code = orc_e2m1_encode(rr);
            q = orc_e2m1_decode(code);
            yy = q * d;
            e = (w[j] - yy) / U[j * cols + j];
            nib[j % bs] = (uint8_t)code;
            if (y) y[r * cols + j] = yy;
            if (err) err[r * cols + j] = e;
            for (c = j + 1; c < cols; ++c) w[c] = fmaf(-e, U[j * cols + c], w[c]);
            if (j % bs == bs - 1 && codes) pack_nibbles(nib, bs, codes + (r * nb + j / bs) * (bs / 2));
        }
        free(w);
    }
    return status;
}

/* Exhaustive search statistics per block over all 126 finite positive E4M3
 * scales ([SS] sec. 2, the naive sweep): the minimum loss, its first
 * (smallest) pattern and the number of patterns that reach it. */
int orc_nvfp4_bruteforce(const float* x, int64_t rows, int64_t cols, float S,
                         const float* importance, uint8_t* best_pattern,
                         float* best_loss, uint8_t* n_ties, int threads)
{
    const int bs = 16;
    int64_t nb = cols / bs, r;
    if (cols % bs) return 2;
#ifdef _OPENMP
    const int nt = threads > 0 ? threads : omp_get_max_threads();   /* this call only */
#pragma omp parallel for schedule(static) num_threads(nt)
#endif
    for (r = 0; r < rows; ++r) {
        int64_t b;
        for (b = 0; b < nb; ++b) {
            const float* xb = x + r * cols + b * bs;
            const float* wb = importance ? importance + b * bs : NULL;
            int64_t blk = r * nb + b;
            float best = 0.0f;
            int pp, bp = 1, ties = 0;
            for (pp = 1; pp <= 126; ++pp) {
                float d = orc_e4m3_value(pp) * S;
                float inv = 1.0f / d;
                float L = block_loss(xb, wb, bs, d, inv, NULL, NULL);
                if (pp == 1 || L < best) { best = L; bp = pp; ties = 1; }
                else if (L == best) ++ties;
            }
            best_pattern[blk] = (uint8_t)bp;
            best_loss[blk] = best;
            n_ties[blk] = (uint8_t)ties;
        }
    }
    return ORC_OK;
}

/* Dequantize NVFP4: y = q * (E4M3(s) * S), in fp32. */
void orc_nvfp4_dequant(const uint8_t* codes, const uint8_t* scales, float S,
                       int64_t rows, int64_t cols, float* y)
{
    int64_t i, n = rows * cols;
    for (i = 0; i < n; ++i) {
        int nib = (codes[i / 2] >> ((i % 2) * 4)) & 15;
        float d = orc_e4m3_value(scales[i / 16]) * S;
        y[i] = orc_e2m1_decode(nib) * d;
    }
}

/* ------------------------------------------------------------------------ */
/* MXFP4 with optional random-sign block Hadamard  ([MR] sec. 1-2, [TQ])      */
/* ------------------------------------------------------------------------ */

/* RN(1/sqrt(32)): the orthonormal scaling of the 32-point Hadamard. */
float orc_hadamard_scale(void)
{
    return (float)(1.0 / sqrt(32.0));
}

/* y = c * H32 * diag(sigma) * x for one 32-block: sign flips (bit j of mask
 * set negates element j), then the fast Walsh-Hadamard transform in natural
 * (Sylvester) order, stage by stage for h = 1, 2, 4, 8, 16, each butterfly
 * (a, b) -> (a + b, a - b), then every element multiplied by c. */
void orc_hadamard32(const float* x, uint32_t mask, float* y)
{
    int i, h;
    float c = orc_hadamard_scale();
    for (i = 0; i < 32; ++i) y[i] = ((mask >> i) & 1u) ? -x[i] : x[i];
    for (h = 1; h < 32; h *= 2) {
        for (i = 0; i < 32; ++i) {
            if (i & h) continue;
            {
                float a = y[i], b = y[i + h];
                y[i] = a + b;
                y[i + h] = a - b;
            }
        }
    }
    for (i = 0; i < 32; ++i) y[i] = y[i] * c;
}

/* Centre exponent: the smallest e with 6 * 2^e >= amax (the block maximum
 * maps onto the largest E2M1 magnitude, [TQ] S-step), clamped to
 * [-127, 127]; -127 for an all-zero block.  floor(log2 amax) comes from
 * frexp, which is exact. */
int orc_mx_centre_exponent(float amax)
{
    int ex, a, e0;
    if (amax == 0.0f) return -127;
    frexpf(amax, &ex);           /* amax = f * 2^ex, f in [0.5, 1) */
    a = ex - 1;                  /* floor(log2 amax) */
    e0 = a - 2;
    if (ldexpf(6.0f, e0) < amax) e0 = a - 1;
    if (e0 < -127) e0 = -127;
    if (e0 > 127) e0 = 127;
    return e0;
}

/* Quantize rows x cols (cols % 32 == 0) to MXFP4.  Per 32-block: optional
 * rotation (sign_masks[cols/32] != NULL), amax, centre exponent e0, then the
 * exponents e = max(-127, e0-1) .. min(127, e0+1) ascending with d = 2^e,
 * inv = 2^-e and the MSE block loss; first candidate kept, later ones only
 * on a strictly smaller loss.  Emits E8M0 byte e*+127, nibbles, the
 * reconstruction y (rotated domain when rotating), the loss, and optionally
 * the rotated input.  Returns ORC_NONFINITE if a block holds a NaN/Inf. */
int orc_mxfp4_quant(const float* x, int64_t rows, int64_t cols, const uint32_t* sign_masks,
                    uint8_t* codes, uint8_t* scales, float* y, float* loss,
                    float* rotated, int threads)
{
    const int bs = 32;
    int64_t nb = cols / bs, r;
    int status = ORC_OK;
    if (cols % bs) return 2;
#ifdef _OPENMP
    const int nt = threads > 0 ? threads : omp_get_max_threads();   /* this call only */
#pragma omp parallel for schedule(static) num_threads(nt)
#endif
    for (r = 0; r < rows; ++r) {
        int64_t b;
        for (b = 0; b < nb; ++b) {
            const float* xb = x + r * cols + b * bs;
            int64_t blk = r * nb + b;
            float v[32], amax = 0.0f, best = 0.0f;
            int i, e, e0, first, last, be = 0, bad = 0;
            uint8_t nib[32];
            if (sign_masks) orc_hadamard32(xb, sign_masks[b], v);
            else for (i = 0; i < bs; ++i) v[i] = xb[i];
            for (i = 0; i < bs; ++i) {
                float a = fabsf(v[i]);
                if (!isfinite(a)) bad = 1;
                else if (a > amax) amax = a;
            }
            if (bad) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                status = ORC_NONFINITE;
            }
            e0 = orc_mx_centre_exponent(amax);
            first = e0 - 1 < -127 ? -127 : e0 - 1;
            last = e0 + 1 > 127 ? 127 : e0 + 1;
            for (e = first; e <= last; ++e) {
                float d = ldexpf(1.0f, e), inv = ldexpf(1.0f, -e);
                float L = block_loss(v, NULL, bs, d, inv, NULL, NULL);
                if (e == first || L < best) { best = L; be = e; }
            }
            {
                float d = ldexpf(1.0f, be), inv = ldexpf(1.0f, -be);
                block_loss(v, NULL, bs, d, inv, nib, y ? y + r * cols + b * bs : NULL);
            }
            if (codes) pack_nibbles(nib, bs, codes + blk * (bs / 2));
            if (scales) scales[blk] = (uint8_t)(be + 127);
            if (loss) loss[blk] = best;
            if (rotated) for (i = 0; i < bs; ++i) rotated[r * cols + b * bs + i] = v[i];
        }
    }
    return status;
}

/* Dequantize MXFP4: y = q * 2^(b-127), in fp32. */
void orc_mxfp4_dequant(const uint8_t* codes, const uint8_t* scales,
                       int64_t rows, int64_t cols, float* y)
{
    int64_t i, n = rows * cols;
    for (i = 0; i < n; ++i) {
        int nib = (codes[i / 2] >> ((i % 2) * 4)) & 15;
        y[i] = orc_e2m1_decode(nib) * orc_e8m0_value(scales[i / 32]);
    }
}

/* Inverse of orc_hadamard32: x = sigma o (c * H32 * y).  (c*H32)^2 = I in
 * exact arithmetic (H32 symmetric, H32^2 = 32 I, c = 1/sqrt(32)) and
 * sigma o sigma = 1, so the same five butterfly stages h = 1,2,4,8,16, then
 * the multiply by c, then the sign flips, undo the rotation up to rounding
 * ([MR] sec. 2: the deployed weights live in the rotated domain; this maps a
 * reconstruction back to the original one). */
void orc_hadamard32_inverse(const float* y, uint32_t mask, float* x)
{
    int i, h;
    float c = orc_hadamard_scale();
    float v[32];
    for (i = 0; i < 32; ++i) v[i] = y[i];
    for (h = 1; h < 32; h *= 2) {
        for (i = 0; i < 32; ++i) {
            if (i & h) continue;
            {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
        }
    }
    for (i = 0; i < 32; ++i) {
        float t = v[i] * c;
        x[i] = ((mask >> i) & 1u) ? -t : t;
    }
}

/* Rows x cols (cols % 32 == 0) of rotated-domain values back to the original
 * domain, block by block (sign_masks[cols/32] as in orc_mxfp4_quant). */
void orc_mxfp4_unrotate(const float* y, int64_t rows, int64_t cols, const uint32_t* sign_masks, float* x)
{
    int64_t r, b, nb = cols / 32;
    for (r = 0; r < rows; ++r)
        for (b = 0; b < nb; ++b)
            orc_hadamard32_inverse(y + r * cols + b * 32, sign_masks[b], x + r * cols + b * 32);
}

/* ------------------------------------------------------------------------ */
/* FOCUS forward quantizer  ([FC] "Metodologia" 2-3)                          */
/* ------------------------------------------------------------------------ */

/* Quantize with a quantization scale decoupled from the stored one.  [FC]
 * keeps the hardware dequantization scale S_dq of every block (E4M3 x S for
 * NVFP4, E8M0 for MXFP4) and quantizes sub-block k of the block with
 * S_q = S_dq * c_k, c_k a full-precision coefficient (CRS: one per block;
 * DGS: one per sub-block, e.g. 8 elements); the codes are Q(W_k / S_q) and
 * the stored reconstruction is q * S_dq.  Reading taken (the page gives the
 * formula only): with d = S_dq computed as everywhere else (NVFP4
 * d = RN(E4M3(p) * S), MXFP4 d = 2^(b-127)),
 *   dq_k = RN(d * c_k);  inv_k = RN(1 / dq_k)
 *   r = x_i * inv_k;  q = E2M1(r);  y = RN(q * d);  e = x_i - y;  L = L + e*e
 * with L the block's loss in column order.  fmt 0 = NVFP4 (16-element blocks,
 * scales E4M3 patterns, S the global scale), 1 = MXFP4 (32, E8M0 bytes).
 * coeffs[rows * cols / sub] (sub divides the block).  Returns ORC_RANGE if a
 * scale byte is not a positive finite value (NVFP4 0x01..0x7E, MXFP4 not
 * 0xFF) or a coefficient is not positive and finite, ORC_NONFINITE if an
 * input is not finite; the outputs of such blocks are then unspecified. */
int orc_focus_quant(int fmt, const float* x, int64_t rows, int64_t cols, const uint8_t* scales, float S,
                    const float* coeffs, int sub, uint8_t* codes, float* y, float* loss)
{
    const int bs = fmt == 0 ? 16 : 32;
    int64_t nb = cols / bs, r;
    int status = ORC_OK;
    if (cols % bs || sub <= 0 || bs % sub) return 2;
    for (r = 0; r < rows; ++r) {
        int64_t b;
        for (b = 0; b < nb; ++b) {
            const float* xb = x + r * cols + b * bs;
            int64_t blk = r * nb + b;
            int i, sb = scales[blk];
            uint8_t nib[32];
            float d, L = 0.0f;
            if (fmt == 0) {
                if (sb < 1 || sb > 126) status = ORC_RANGE;
                d = orc_e4m3_value(sb) * S;
            } else {
                if (sb == 255) status = ORC_RANGE;
                d = orc_e8m0_value(sb);
            }
            for (i = 0; i < bs; ++i) {
                float c = coeffs[(r * cols + b * bs + i) / sub];
                float dq = d * c;
                float inv = 1.0f / dq;
                float rr = xb[i] * inv;
                int code = orc_e2m1_encode(rr);
                float q = orc_e2m1_decode(code);
                float yy = q * d;
                float e = xb[i] - yy;
                float e2 = e * e;
                if (!(c > 0.0f) || isinf(c)) status = ORC_RANGE;
                if (!isfinite(xb[i]) && status == ORC_OK) status = ORC_NONFINITE;
                L = L + e2;
                nib[i] = (uint8_t)code;
                if (y) y[r * cols + b * bs + i] = yy;
            }
            if (codes) pack_nibbles(nib, bs, codes + blk * (bs / 2));
            if (loss) loss[blk] = L;
        }
    }
    return status;
}

/* ------------------------------------------------------------------------ */
/* Block scales in the layout of Blackwell block-scaled FP4 GEMMs            */
/* ------------------------------------------------------------------------ */

/* [MR] sec. 3 runs the quantized weights through block-scaled FP4 GEMM
 * kernels on Blackwell.  Those read the block scales of an operand not row by
 * row but in tiles: the [rows][scols] scale matrix (scols = cols/16 for
 * NVFP4, cols/32 for MXFP4) is cut into tiles of 128 rows x 4 scale columns,
 * zero-padded at the bottom and right edges, and the tiles are stored one
 * after the other, the column tiles of one row tile together.  A tile is 512
 * bytes: 32 lines of 16 bytes, line j holding rows j, j+32, j+64, j+96 of the
 * tile, 4 scale bytes each.  This is a hardware interface, not part of the
 * method; the pages do not describe it.  Parity pinned on the CPU against
 * CUTLASS's shape/stride definition of the same layout (byte for byte, ragged
 * shapes; tests/test_oracle_mxfp4.py) and on the GPU by a library
 * block-scaled GEMM that reads it (tests/test_gpu_mma_layout.py). */
int64_t orc_mma_scale_bytes(int64_t rows, int64_t scols)
{
    return ((rows + 127) / 128) * ((scols + 3) / 4) * 512;
}

void orc_scales_to_mma_layout(const uint8_t* s, int64_t rows, int64_t scols, uint8_t* out)
{
    int64_t r, c;
    int64_t col_tiles = (scols + 3) / 4;
    memset(out, 0, (size_t)orc_mma_scale_bytes(rows, scols));
    for (r = 0; r < rows; ++r) {
        for (c = 0; c < scols; ++c) {
            int64_t tile = (r / 128) * col_tiles + c / 4;
            int64_t line = r % 32;
            int64_t slot = (r % 128) / 32;
            out[tile * 512 + line * 16 + slot * 4 + c % 4] = s[r * scols + c];
        }
    }
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
