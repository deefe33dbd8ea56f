/*
 * nvfp4_oracle.c -- plain CPU oracle for NVFP4 block quantization and the W4A4 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  The product library never links, loads or calls this
 * file; only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * do.  It shares no code, header, table or constant generator with the CUDA path.
 * It is deliberately slow: every rounding decision is a search over the grid of
 * representable values, written so that it can be checked against the pages by eye.
 *
 * Sources (web pages, cited by title and section):
 *   [G4] "Tu pipeline NVFP4: meter 62 GB de modelo en 24 GB de laptop",
 *        section 2 "Qué es realmente NVFP4":
 *          - box "Fundamento matemático: bitfield E2M1 y cuantización jerárquica":
 *            the E2M1 bitfield v(s,e,m) with bias B = 1, the grid G_E2M1, the
 *            equations q_ij = argmin_q |W_ij/(s_b s_g) - q| and W^_ij = q_ij s_b s_g,
 *            and the two-level scale (E4M3 per 16-block, one FP32 per tensor);
 *          - box "Derivación del objetivo de optimización MSE vs Absmax":
 *            s_absmax = max_k |W_k| / 6 and
 *            s_b* = argmin_{s_b} sum_k (W_k - s_b s_g Q(W_k/(s_b s_g)))^2;
 *          - cards "E2M1", "Bloques de 16", "Escala E4M3 por bloque".
 *   [DF] "NVFP4 en difusión: la misma cuantización, un motor completamente distinto",
 *        section 2 "NVFP4 sin vLLM: torch._scaled_mm a mano": codes (out, in/2) uint8
 *        with two FP4 values per byte, scales (out, in/16) E4M3 along the input
 *        dimension, out = (A s_a)(B s_b)^T with scales applied per block, BF16 out;
 *        section 8 "Para practicar": the scale search over factors of the absmax
 *        scale from 0.3 to 1.0 that keeps a candidate only on a strict improvement.
 *
 * Arithmetic: every float operation is IEEE binary32 round-to-nearest-even
 * (build with -O1 -ffp-contract=off, no fast-math; x86-64 SSE has no excess
 * precision).  fmaf appears only where the definition below says fused
 * multiply-add.  The GEMM reference is in binary64.
 *
 * Readings of points the pages leave open (each repeated where it is used):
 *   R1 global scale: s_g = RN32(amax_t / 2688), 2688 = 6 * 448, so that the
 *      block holding the tensor maximum gets the largest E4M3 scale; s_g = 1
 *      for an all-zero tensor.  (parity unpinned: a convention.)
 *   R2 operation order: v_b = RN32(amax_b / RN32(6 s_g)); per candidate
 *      u = RN32(f v_b), s = E4M3(u), eff = RN32(dec(s) s_g), r = RN32(1/eff),
 *      y = RN32(|x| r).  (parity unpinned: a convention.)
 *   R3 E2M1 rounding: nearest grid value, ties to the even mantissa bit,
 *      values above 6 go to 6; the sign bit of x is kept (-0 is code 0x8).
 *   R4 E4M3 rounding: nearest, ties to even mantissa, saturating at 448.
 *   R5 MSE candidates: f_i = RN32((3+i)/10), i = 0..7 (0.3 .. 1.0); block error
 *      e = sum_k d_k^2 with d_k = fmaf(-q_k, eff, x_k), e = fmaf(d, d, e) in k
 *      order; walk i = 7 down to 0 and keep a candidate only on a strict
 *      improvement, so ties keep the larger scale.  Absmax is candidate f = 1.
 *   R6 packing: element 2j in bits 3:0 of byte j, element 2j+1 in bits 7:4.
 *   R7 swizzled scale layout (the one the block-scaled tensor-core MMA reads):
 *      rows padded to 128, block columns padded to 4, zero fill; byte of
 *      (r, c) at ((r/128)*(Cp/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + c%4.
 *   R9 LoRA branch ([DF] section 3, "¿Cómo fine-tuneás algo que ya está en 4
 *      bits?": y = W_4bit x + B (A x), the low-rank term in 16 bits, added to the
 *      quantized matmul before the result is returned): x is the activation
 *      before quantization (BF16), A (r x K) and B (N x r) are BF16; the
 *      intermediate t = A x is rounded to BF16 (the 16-bit term), the sums are
 *      binary64 here; the W4A4 accumulator plus the low-rank term is rounded to
 *      BF16 once.  (parity unpinned: where the 16-bit rounding happens is a reading.)
 *   R8 four-over-six: two candidates per block, the absmax scale (maximum
 *      mapped to 6) first and s = E4M3(RN32(amax_b / RN32(4 s_g))) (maximum
 *      mapped to 4) second, errors as in R5, the second kept only on a strict
 *      improvement (ties keep the 6 mapping).  (parity unpinned: the order and
 *      the tie rule are conventions; the pages name the choice, not its steps.)
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* BF16 <-> binary32                                                          */
/* ------------------------------------------------------------------------- */

/* A BF16 value is the top half of a binary32 value, so widening is exact. */
float ora_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> BF16, round to nearest, ties to even (textbook bit form). */
uint16_t ora_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) /* NaN stays NaN (quiet) */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------- */
/* E2M1: [G4] box "Fundamento matemático: bitfield E2M1 ..."                  */
/* ------------------------------------------------------------------------- */

/* v(s,e,m) = (-1)^s * { 0                       if e = 0, m = 0
 *                       2^(1-B) (0 + m/2)       if e = 0, m = 1 (subnormal)
 *                       2^(e-B) (1 + m/2)       if e > 0 }          with B = 1.
 * Code layout: bit 3 = s, bits 2:1 = e, bit 0 = m. */
double ora_e2m1_decode(uint8_t code)
{
    const int B = 1;
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v;
    if (e == 0)
        v = ldexp(0.0 + m * 0.5, 1 - B);
    else
        v = ldexp(1.0 + m * 0.5, e - B);
    return s ? -v : v;
}

/* Magnitude code (0..7) of y >= 0: the argmin over the grid of |y - q| (the
 * q_ij equation).  R3: at an exact midpoint take the neighbour whose mantissa
 * bit is 0 (grid codes alternate m = 0, 1, 0, 1, ... so ties only occur between
 * neighbours of different parity).  Any y at or above 6 is nearest to 6
 * (saturation); it is returned before the search because for y beyond 2^53
 * the binary64 distances to 4 and to 6 round to the same number. */
uint8_t ora_e2m1_encode_mag(float y)
{
    if (y >= 6.0f)
        return 7;
    uint8_t best = 0;
    double best_d = INFINITY;
    for (uint8_t c = 0; c < 8; c++) {
        double d = fabs((double)y - ora_e2m1_decode(c));
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best_d = d;
            best = c;
        }
    }
    return best;
}

/* ------------------------------------------------------------------------- */
/* E4M3 block scale: [G4] card "Escala E4M3 por bloque" (4 exponent bits, 3    */
/* mantissa bits).  The "fn" variant: bias 7, subnormals m/8 * 2^-6, no        */
/* infinities, 0x7F = NaN, largest finite 0x7E = 448.                          */
/* ------------------------------------------------------------------------- */

double ora_e4m3_decode(uint8_t b)
{
    int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7)
        return NAN;
    double v = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

static double e4m3_table[128];
static int e4m3_table_ready = 0;

static void e4m3_table_init(void)
{
    if (e4m3_table_ready)
        return;
    for (int c = 0; c < 128; c++)
        e4m3_table[c] = ora_e4m3_decode((uint8_t)c);
    e4m3_table_ready = 1;
}

/* R4: nearest non-negative finite E4M3 value to u >= 0, ties to the even
 * mantissa bit (adjacent codes alternate parity), saturating at 448: any u at
 * or above 448 is nearest to 448 among the finite codes; it is returned before
 * the search because binary64 distances stop separating codes for huge u. */
uint8_t ora_e4m3_encode(float u)
{
    e4m3_table_init();
    if (u >= 448.0f)
        return 0x7E;
    uint8_t best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; c++) {
        double d = fabs((double)u - e4m3_table[c]);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best_d = d;
            best = (uint8_t)c;
        }
    }
    return best;
}

/* ------------------------------------------------------------------------- */
/* Global (per-tensor) FP32 scale: [G4] "Fundamento matemático", last         */
/* paragraph: one FP32 scale per tensor; the block scale only covers the       */
/* block's range relative to the tensor.                                       */
/* ------------------------------------------------------------------------- */

float ora_amax(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld)
{
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            float a = fabsf(ora_bf16_to_f32(x[r * ld + c]));
            if (a > amax)
                amax = a;
        }
    return amax;
}

/* R1: s_g = RN32(amax / 2688); an all-zero tensor gets s_g = 1. */
float ora_global_scale_from_amax(float amax)
{
    if (amax == 0.0f)
        return 1.0f;
    return amax / 2688.0f;
}

float ora_global_scale(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld)
{
    return ora_global_scale_from_amax(ora_amax(x, rows, cols, ld));
}

/* ------------------------------------------------------------------------- */
/* One block of 16: the q_ij / W^_ij equations of [G4] "Fundamento            */
/* matemático" for a given effective scale eff = s_b * s_g, and the block      */
/* error of [G4] "Derivación ... MSE vs Absmax".                               */
/* ------------------------------------------------------------------------- */

/* Encode 16 values with effective scale eff (R2, R3) and return the block's
 * squared error in the order of R5.  codes[k] gets the signed 4-bit code. */
static float encode_block_with_eff(const float x[16], float eff, uint8_t codes[16])
{
    float e = 0.0f;
    for (int k = 0; k < 16; k++) {
        uint8_t mag = 0;
        if (eff != 0.0f && x[k] != 0.0f) {
            float r = 1.0f / eff;      /* RN32 reciprocal of the effective scale */
            float y = fabsf(x[k]) * r; /* RN32 */
            mag = ora_e2m1_encode_mag(y);
        }
        codes[k] = (uint8_t)((signbit(x[k]) ? 8 : 0) | mag);
        float q = (float)ora_e2m1_decode(codes[k]); /* exact */
        float d = fmaf(-q, eff, x[k]);
        e = fmaf(d, d, e);
    }
    return e;
}

#define ORA_SCALE_ABSMAX 0
#define ORA_SCALE_MSE 1
#define ORA_SCALE_FOUR_OVER_SIX 2

/* Quantize one block of 16 (R2, R5).  Absmax: the single candidate f = 1, i.e.
 * s_b = E4M3(amax_b / (6 s_g)) -- s_absmax = max|W|/6 measured in units of s_g.
 * MSE: the candidates f = 0.3, 0.4, ..., 1.0 times the absmax scale, keeping
 * the least squared error (strict improvement while walking from f = 1 down).
 * Four-over-six ([G4] section 2, table of block-scale algorithms, row
 * "Four-over-six": each block picks the larger of two possible maxima, 4 or 6,
 * by least error): the absmax scale (block maximum mapped to 6), then
 * s_b = E4M3(amax_b / (4 s_g)) (block maximum mapped to 4), kept only on a
 * strictly smaller squared error (R8). */
static uint8_t quantize_block(const float x[16], float sg, int mode, uint8_t codes[16],
                              float *err)
{
    float amax_b = 0.0f;
    for (int k = 0; k < 16; k++) {
        float a = fabsf(x[k]);
        if (a > amax_b)
            amax_b = a;
    }
    float d6 = 6.0f * sg;     /* RN32 */
    float vb = amax_b / d6;   /* RN32 */
    int lowest = (mode == ORA_SCALE_MSE) ? 0 : 7;

    uint8_t best_s = 0, best_codes[16];
    float best_e = 0.0f;
    for (int i = 7; i >= lowest; i--) {
        float f = (float)(3 + i) / 10.0f; /* RN32((3+i)/10) */
        float u = f * vb;                 /* RN32 */
        uint8_t s = ora_e4m3_encode(u);
        float eff = (float)ora_e4m3_decode(s) * sg; /* RN32 */
        uint8_t c[16];
        float e = encode_block_with_eff(x, eff, c);
        if (i == 7 || e < best_e) {
            best_e = e;
            best_s = s;
            memcpy(best_codes, c, 16);
        }
    }
    if (mode == ORA_SCALE_FOUR_OVER_SIX) {
        float d4 = 4.0f * sg;   /* RN32 (exact: a power of two) */
        float v4 = amax_b / d4; /* RN32 */
        uint8_t s = ora_e4m3_encode(v4);
        float eff = (float)ora_e4m3_decode(s) * sg; /* RN32 */
        uint8_t c[16];
        float e = encode_block_with_eff(x, eff, c);
        if (e < best_e) {
            best_e = e;
            best_s = s;
            memcpy(best_codes, c, 16);
        }
    }
    memcpy(codes, best_codes, 16);
    if (err)
        *err = best_e;
    return best_s;
}

/* ------------------------------------------------------------------------- */
/* Tensor quantization: [DF] section 2 -- codes (rows, cols/2) uint8, two FP4  */
/* values per byte (R6); scales (rows, cols/16) E4M3 along the input dimension. */
/* ------------------------------------------------------------------------- */

/* x: rows x cols BF16 bit patterns with row stride ld (elements); cols % 16 == 0.
 * codes: rows * cols/2 bytes; scales: rows * cols/16 bytes (linear layout);
 * block_err: rows * cols/16 floats or NULL.  Returns 0, or -1 on a bad shape. */
int ora_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int mode,
                 float sg, uint8_t *codes, uint8_t *scales, float *block_err)
{
    if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols)
        return -1;
    int64_t nblk = cols / 16;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < nblk; b++) {
            float xb[16];
            for (int k = 0; k < 16; k++)
                xb[k] = ora_bf16_to_f32(x[r * ld + b * 16 + k]);
            uint8_t c[16];
            float e;
            scales[r * nblk + b] = quantize_block(xb, sg, mode, c, &e);
            if (block_err)
                block_err[r * nblk + b] = e;
            for (int j = 0; j < 8; j++)
                codes[r * (cols / 2) + b * 8 + j] = (uint8_t)((c[2 * j] & 0xF) | (c[2 * j + 1] << 4));
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Scale layouts (R7)                                                          */
/* ------------------------------------------------------------------------- */

int64_t ora_swizzled_scales_bytes(int64_t rows, int64_t nblk)
{
    int64_t rp = (rows + 127) / 128 * 128;
    int64_t cp = (nblk + 3) / 4 * 4;
    return rp * cp;
}

int64_t ora_swizzled_offset(int64_t r, int64_t c, int64_t nblk)
{
    int64_t cp = (nblk + 3) / 4 * 4;
    return ((r / 128) * (cp / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

void ora_swizzle_scales(const uint8_t *linear, int64_t rows, int64_t nblk, uint8_t *swz)
{
    memset(swz, 0, (size_t)ora_swizzled_scales_bytes(rows, nblk));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < nblk; c++)
            swz[ora_swizzled_offset(r, c, nblk)] = linear[r * nblk + c];
}

void ora_unswizzle_scales(const uint8_t *swz, int64_t rows, int64_t nblk, uint8_t *linear)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < nblk; c++)
            linear[r * nblk + c] = swz[ora_swizzled_offset(r, c, nblk)];
}

/* ------------------------------------------------------------------------- */
/* Reconstruction: W^_ij = q_ij * s_b * s_g ([G4] "Fundamento matemático"),    */
/* evaluated as RN32(q * RN32(dec(s_b) * s_g)) and rounded to BF16 (RNE).      */
/* ------------------------------------------------------------------------- */

void ora_dequantize(const uint8_t *codes, const uint8_t *scales, float sg, int64_t rows,
                    int64_t cols, uint16_t *out)
{
    int64_t nblk = cols / 16;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            float eff = (float)ora_e4m3_decode(scales[r * nblk + c / 16]) * sg;
            float v = (float)ora_e2m1_decode(code) * eff;
            out[r * cols + c] = ora_f32_to_bf16(v);
        }
}

/* ------------------------------------------------------------------------- */
/* GEMM reference: [DF] section 2, out = (A s_a)(B s_b)^T with the scales       */
/* applied per 16-block along K, both global scales applied, in binary64.      */
/* A is M x K (codes M x K/2, linear scales M x K/16), B is N x K likewise.    */
/* out[m,n] = sum_k a[m,k] b[n,k]; absum[m,n] = sum_k |a[m,k] b[n,k]|.          */
/* Every operand value q * dec(s) * s_g is exact in binary64; the products are */
/* summed in k order.                                                          */
/* ------------------------------------------------------------------------- */

/* Row `row` of an operand as float64 values q * dec(s_b) * s_g (each exact). */
static void decode_row(const uint8_t *codes, const uint8_t *scales, double sg, int64_t row, int64_t K,
                       double *out)
{
    double e2m1[16];
    for (int c = 0; c < 16; c++)
        e2m1[c] = ora_e2m1_decode((uint8_t)c);
    e4m3_table_init();
    for (int64_t k = 0; k < K; k++) {
        uint8_t byte = codes[row * (K / 2) + k / 2];
        uint8_t code = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        uint8_t s = scales[row * (K / 16) + k / 16];
        double dec_s = (s & 0x80) ? -e4m3_table[s & 0x7F] : e4m3_table[s];
        out[k] = e2m1[code] * dec_s * sg;
    }
}

/* out = sum_k a[k] b[k] in k order; absum = sum_k |a[k] b[k]|. */
static void dot_f64(const double *a, const double *b, int64_t K, double *out, double *absum)
{
    double acc = 0.0, mag = 0.0;
    for (int64_t k = 0; k < K; k++) {
        double p = a[k] * b[k];
        acc += p;
        mag += fabs(p);
    }
    *out = acc;
    if (absum)
        *absum = mag;
}

/* Returns 0, or -1 when a work buffer cannot be allocated. */
int ora_gemm_f64(const uint8_t *a_codes, const uint8_t *a_scales, float a_sg, int64_t M,
                 const uint8_t *b_codes, const uint8_t *b_scales, float b_sg, int64_t N, int64_t K,
                 double *out, double *absum)
{
    double *a = (double *)malloc(sizeof(double) * (size_t)(M * K + K));
    if (!a)
        return -1;
    double *b = a + M * K;
    for (int64_t m = 0; m < M; m++)
        decode_row(a_codes, a_scales, a_sg, m, K, a + m * K);
    for (int64_t n = 0; n < N; n++) {
        decode_row(b_codes, b_scales, b_sg, n, K, b);
        for (int64_t m = 0; m < M; m++)
            dot_f64(a + m * K, b, K, &out[m * N + n], absum ? &absum[m * N + n] : NULL);
    }
    free(a);
    return 0;
}

/* The same reference at `count` sampled positions (m_idx[i], n_idx[i]). */
int ora_gemm_f64_at(const uint8_t *a_codes, const uint8_t *a_scales, float a_sg,
                    const uint8_t *b_codes, const uint8_t *b_scales, float b_sg, int64_t K,
                    const int64_t *m_idx, const int64_t *n_idx, int64_t count, double *out,
                    double *absum)
{
    double *a = (double *)malloc(sizeof(double) * (size_t)(2 * K));
    if (!a)
        return -1;
    double *b = a + K;
    for (int64_t i = 0; i < count; i++) {
        decode_row(a_codes, a_scales, a_sg, m_idx[i], K, a);
        decode_row(b_codes, b_scales, b_sg, n_idx[i], K, b);
        dot_f64(a, b, K, &out[i], absum ? &absum[i] : NULL);
    }
    free(a);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Array forms of the scalar codecs (loops over the functions above), so the  */
/* tests can sweep many inputs per call.                                       */
/* ------------------------------------------------------------------------- */

void ora_e2m1_encode_mag_array(const float *y, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = ora_e2m1_encode_mag(y[i]);
}

void ora_e4m3_encode_array(const float *u, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = ora_e4m3_encode(u[i]);
}

void ora_f32_to_bf16_array(const float *f, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = ora_f32_to_bf16(f[i]);
}

/* ------------------------------------------------------------------------- */
/* LoRA branch (R9): the low-rank term of y = W_4bit x + B (A x).             */
/* ------------------------------------------------------------------------- */

/* x: M x K BF16 bits (row stride K); a: R x K; b: N x R (both BF16 bits).
 * t_out (M x R BF16 bits, optional): t = BF16_RNE(RN32(sum_k x[m][k] a[j][k])).
 * out (M x N): out[m][n] = sum_j t[m][j] b[n][j] in binary64; absum: the sum of
 * the terms' magnitudes.  Returns 0, or -1 on a bad size or allocation. */
int ora_lora_f64(const uint16_t *x, int64_t M, int64_t K, const uint16_t *a, int64_t R, const uint16_t *b,
                 int64_t N, double *out, double *absum, uint16_t *t_out)
{
    if (M < 0 || K < 0 || R < 0 || N < 0)
        return -1;
    double *t = (double *)malloc(sizeof(double) * (size_t)(M * R + 1));
    if (!t)
        return -1;
    for (int64_t m = 0; m < M; m++)
        for (int64_t j = 0; j < R; j++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += (double)ora_bf16_to_f32(x[m * K + k]) * (double)ora_bf16_to_f32(a[j * K + k]);
            /* the 16-bit intermediate: BF16_RNE(RN32(acc)), the rounding a binary32
             * accumulator followed by a BF16 store performs */
            uint16_t tb = ora_f32_to_bf16((float)acc);
            if (t_out)
                t_out[m * R + j] = tb;
            t[m * R + j] = (double)ora_bf16_to_f32(tb);
        }
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0, mag = 0.0;
            for (int64_t j = 0; j < R; j++) {
                double p = t[m * R + j] * (double)ora_bf16_to_f32(b[n * R + j]);
                acc += p;
                mag += fabs(p);
            }
            out[m * N + n] = acc;
            if (absum)
                absum[m * N + n] = mag;
        }
    free(t);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* MXFP4 (NEXT: the "MXFP4 / NVFP4: Blackwell agresivo" section of "Cuantización */
/* en Producción: AWQ, GPTQ, GGUF K-quants, FP8, MXFP4/NVFP4" names the format  */
/* but gives neither its block size nor its scale type).  Outside reading, the  */
/* public OCP Microscaling Formats (MX) specification v1.0: blocks of 32 values  */
/* along K, one E8M0 scale per block (a power of two 2^(e - 127), e = 0..254,    */
/* 0xFF = NaN), E2M1 elements, no per-tensor scale.  The block's scale is       */
/* 2^(floor(log2(amax)) - 2) -- 2 being the exponent of the largest E2M1 value   */
/* 6 = 1.5 * 2^2 -- clamped to the E8M0 range; each element is x / 2^e rounded  */
/* to the E2M1 grid (RNE, saturating at 6, the sign kept).  An all-zero block   */
/* takes the smallest scale (byte 0).                                          */
/* ------------------------------------------------------------------------- */

double ora_e8m0_decode(uint8_t b)
{
    if (b == 0xFF)
        return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* floor(log2(a)) of a positive finite float, exact (frexp: a = f 2^e, 0.5 <= f < 1). */
static int floor_log2f(float a)
{
    int e;
    frexpf(a, &e);
    return e - 1;
}

/* One block of 32: returns the E8M0 scale byte; codes[k] gets the signed 4-bit code. */
static uint8_t mx_quantize_block(const float x[32], uint8_t codes[32])
{
    float amax = 0.0f;
    for (int k = 0; k < 32; k++) {
        float a = fabsf(x[k]);
        if (a > amax)
            amax = a;
    }
    int shared = (amax == 0.0f) ? -127 : floor_log2f(amax) - 2;
    if (shared < -127)
        shared = -127;
    if (shared > 127)
        shared = 127;
    for (int k = 0; k < 32; k++) {
        /* |x| / 2^shared, exact in binary64 (8 significant bits); below binary32's range
           the value is far below the smallest E2M1 step and codes to 0 either way */
        float y = (float)ldexp((double)fabsf(x[k]), -shared);
        uint8_t mag = (x[k] == 0.0f) ? 0 : ora_e2m1_encode_mag(y);
        codes[k] = (uint8_t)((signbit(x[k]) ? 8 : 0) | mag);
    }
    return (uint8_t)(shared + 127);
}

/* x: rows x cols BF16 bits (row stride ld), cols % 32 == 0.  codes (rows, cols/2),
   scales (rows, cols/32) linear.  Returns 0, or -1 on a bad shape. */
int ora_quantize_mx(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, uint8_t *codes, uint8_t *scales)
{
    if (rows < 0 || cols < 0 || cols % 32 != 0 || ld < cols)
        return -1;
    int64_t nblk = cols / 32;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t b = 0; b < nblk; b++) {
            float xb[32];
            uint8_t c[32];
            for (int k = 0; k < 32; k++)
                xb[k] = ora_bf16_to_f32(x[r * ld + b * 32 + k]);
            scales[r * nblk + b] = mx_quantize_block(xb, c);
            for (int j = 0; j < 16; j++)
                codes[r * (cols / 2) + b * 16 + j] = (uint8_t)((c[2 * j] & 0xF) | (c[2 * j + 1] << 4));
        }
    return 0;
}

/* BF16 bits of q * 2^(s - 127) (exact in binary32, rounded to BF16 RNE). */
void ora_dequantize_mx(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols, uint16_t *out)
{
    int64_t nblk = cols / 32;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            double v = ora_e2m1_decode(code) * ora_e8m0_decode(scales[r * nblk + c / 32]);
            out[r * cols + c] = ora_f32_to_bf16((float)v);
        }
}

/* Row of an MXFP4 operand as binary64 values q * 2^(s - 127) (each exact). */
static void decode_row_mx(const uint8_t *codes, const uint8_t *scales, int64_t row, int64_t K, double *out)
{
    for (int64_t k = 0; k < K; k++) {
        uint8_t byte = codes[row * (K / 2) + k / 2];
        uint8_t code = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        out[k] = ora_e2m1_decode(code) * ora_e8m0_decode(scales[row * (K / 32) + k / 32]);
    }
}

/* C = A B^T of two MXFP4 operands (A M x K, B N x K, linear scales), binary64, with
   absum = sum |a b|; at `count` sampled positions (m_idx[i], n_idx[i]). */
int ora_gemm_mx_f64_at(const uint8_t *a_codes, const uint8_t *a_scales, const uint8_t *b_codes,
                       const uint8_t *b_scales, int64_t K, const int64_t *m_idx, const int64_t *n_idx, int64_t count,
                       double *out, double *absum)
{
    double *a = (double *)malloc(sizeof(double) * (size_t)(2 * K));
    if (!a)
        return -1;
    double *b = a + K;
    for (int64_t i = 0; i < count; i++) {
        decode_row_mx(a_codes, a_scales, m_idx[i], K, a);
        decode_row_mx(b_codes, b_scales, n_idx[i], K, b);
        dot_f64(a, b, K, &out[i], absum ? &absum[i] : NULL);
    }
    free(a);
    return 0;
}
