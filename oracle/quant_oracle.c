/*
 * oracle/quant_oracle.c -- TEST INFRASTRUCTURE, not product code.
 *
 * Block-scaled low-precision expert weights: the plain CPU definition of
 * the two formats the pages name for MoE expert weights on Blackwell-class
 * GPUs -- FP8 (the W8A8 reference and the "B200 FP8 x FP4" policy of
 * DeepGEMM fork PR #5 "big M opt: splitT1 + L2 scatter + 2 stream" and
 * DeepGEMM PR #381 "Add B200-Calibrated Sparse-Routing Adaptive Wave
 * Sizing") and NVFP4 (the megamoe_nvfp4 kernels of the same fork, and the
 * NVFP4 target of SpecForge PR #943).  The pages name the formats without
 * defining them; the definitions below are the published ones:
 *
 *  - E4M3 ("FP8 E4M3", the variant without infinities): sign bit 7,
 *    exponent bits 6..3 with bias 7, mantissa bits 2..0.  Normal values
 *    (-1)^s 2^(e-7) (1 + m/8), subnormals (e = 0) (-1)^s 2^-6 (m/8); the
 *    two codes with every exponent and mantissa bit set are NaN; the
 *    largest finite value is 448.
 *  - E2M1 (FP4): sign bit 3, exponent bits 2..1 with bias 1, mantissa bit 0;
 *    magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; no NaN or infinity.
 *  - UE8M0 (the MX block scale): an unsigned power of two 2^(c - 127);
 *    c = 255 is NaN.
 *  - MXFP8 (OCP Microscaling formats, version 1.0, "MXFP8 E4M3"): blocks
 *    of 32 consecutive elements along the reduction dimension share one
 *    UE8M0 scale X = 2^(floor(log2(amax)) - 8), 8 being the exponent of the
 *    largest E4M3 power of two; each element is x / X rounded to E4M3.
 *  - NVFP4: blocks of 16 consecutive elements share one E4M3 scale, and the
 *    whole matrix one fp32 scale s_t = amax / (6 * 448), so that a block
 *    scale never exceeds 448 and an element never exceeds 6:
 *    s_b = E4M3(amax_b / (6 * s_t)), element = E2M1(x / (s_b * s_t)).
 *
 * Readings where the definitions leave a step open:
 *  - rounding: to the nearest representable value, ties to the code whose
 *    lowest (mantissa) bit is clear; a magnitude beyond the largest finite
 *    value takes the largest finite value (saturation: it is the nearest);
 *  - the sign bit copies the input's sign bit, so -0.0 (and a negative
 *    value that rounds to zero) keeps it;
 *  - MXFP8: an all-zero block takes the smallest scale, 2^-127 (code 0);
 *    scale exponents are clamped to [-127, 127];
 *  - NVFP4: s_t, the block-scale argument and the element argument are
 *    computed with IEEE fp32 operations in the order written above
 *    (6.0f * s_t, then the division; s_b * s_t, then the division), the
 *    precision in which a GPU quantiser takes the same decisions; an
 *    all-zero matrix takes s_t = 1, a block whose scale rounds to zero
 *    stores zero elements;
 *  - NVFP4 packs two elements per byte, element 2i in the low nibble;
 *  - "the matrix" of the fp32 scale is one expert's gate, up or down
 *    projection (each has its own).
 *
 * Every encoder below searches the code table for the nearest value, the
 * plain definition of rounding; nothing here is tuned for speed.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)

static double bf16_value(uint16_t v)
{
    uint32_t u = ((uint32_t)v) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------ codecs -- */
static double e4m3_value(uint8_t c)
{
    const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

static double e2m1_value(uint8_t c)
{
    const int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    const double mag = e == 0 ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, e - 1);
    return s ? -mag : mag;
}

/* Nearest code among the non-negative finite codes 0..n_pos-1 (values
 * strictly increasing with the code), ties to the even code.  At or beyond
 * the largest value that value is the nearest (saturation); it is returned
 * directly, since far beyond it the distances to the top codes round to the
 * same double. */
static uint8_t nearest_code(double mag, double (*value)(uint8_t), int n_pos)
{
    if (mag >= value((uint8_t)(n_pos - 1))) return (uint8_t)(n_pos - 1);
    int best = 0;
    double best_d = fabs(mag - value(0));
    for (int c = 1; c < n_pos; ++c) {
        const double d = fabs(mag - value((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) != 0)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)best;
}

static uint8_t e4m3_code(double x)
{
    const uint8_t c = nearest_code(fabs(x), e4m3_value, 127); /* 0x00..0x7E; 0x7F is NaN */
    return signbit(x) ? (uint8_t)(c | 0x80) : c;
}

static uint8_t e2m1_code(double x)
{
    const uint8_t c = nearest_code(fabs(x), e2m1_value, 8);
    return signbit(x) ? (uint8_t)(c | 0x8) : c;
}

void oracle_e4m3_decode(int64_t n, const uint8_t *codes, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(codes[i]);
}

void oracle_e4m3_encode(int64_t n, const double *x, uint8_t *codes)
{
    for (int64_t i = 0; i < n; ++i) codes[i] = e4m3_code(x[i]);
}

void oracle_e2m1_decode(int64_t n, const uint8_t *codes, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = e2m1_value(codes[i] & 15);
}

void oracle_e2m1_encode(int64_t n, const double *x, uint8_t *codes)
{
    for (int64_t i = 0; i < n; ++i) codes[i] = e2m1_code(x[i]);
}

void oracle_ue8m0_decode(int64_t n, const uint8_t *codes, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = codes[i] == 255 ? NAN : ldexp(1.0, (int)codes[i] - 127);
}

/* ------------------------------------------------------------- MXFP8 -- */
/* w [rows, K] bf16 bit patterns, K a multiple of 32 -> codes [rows, K] E4M3,
 * scales [rows, K / 32] UE8M0. */
int oracle_mxfp8_quantize(int64_t rows, int64_t K, const uint16_t *w, uint8_t *codes, uint8_t *scales)
{
    if (rows < 0 || K < 32 || K % 32 != 0) return ORACLE_EINVAL;
    /* rows are independent: split over the host threads (no effect on any value) */
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < K / 32; ++b) {
            const uint16_t *x = w + r * K + b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs(bf16_value(x[i])));
            int se = -127;
            if (amax > 0.0) {
                int e2;
                frexp(amax, &e2); /* amax = f 2^e2, f in [0.5, 1): floor(log2 amax) = e2 - 1 */
                se = e2 - 1 - 8;
                if (se < -127) se = -127;
                if (se > 127) se = 127;
            }
            scales[r * (K / 32) + b] = (uint8_t)(se + 127);
            for (int i = 0; i < 32; ++i) codes[r * K + b * 32 + i] = e4m3_code(ldexp(bf16_value(x[i]), -se));
        }
    return ORACLE_OK;
}

/* codes [rows, K] E4M3 and scales [rows, K / 32] UE8M0 -> out [rows, K]:
 * element value times 2^(scale - 127), in fp64. */
int oracle_mxfp8_dequantize(int64_t rows, int64_t K, const uint8_t *codes, const uint8_t *scales, double *out)
{
    if (rows < 0 || K < 32 || K % 32 != 0) return ORACLE_EINVAL;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < K; ++i)
            out[r * K + i] = ldexp(e4m3_value(codes[r * K + i]), (int)scales[r * (K / 32) + i / 32] - 127);
    return ORACLE_OK;
}

/* ------------------------------------------------------------- NVFP4 -- */
/* w [rows, K] bf16 bit patterns, K a multiple of 16 -> codes [rows, K / 2]
 * (two E2M1 codes per byte, element 2i in the low nibble), scales
 * [rows, K / 16] E4M3, *tensor_scale the fp32 matrix scale. */
int oracle_nvfp4_quantize(int64_t rows, int64_t K, const uint16_t *w, uint8_t *codes, uint8_t *scales,
                          float *tensor_scale)
{
    if (rows < 0 || K < 16 || K % 16 != 0) return ORACLE_EINVAL;
    float amax = 0.0f;
    for (int64_t i = 0; i < rows * K; ++i) amax = fmaxf(amax, fabsf((float)bf16_value(w[i])));
    const float st = amax > 0.0f ? amax / 2688.0f : 1.0f; /* 2688 = 6 * 448 */
    *tensor_scale = st;
    memset(codes, 0, (size_t)(rows * K / 2));
    /* rows are independent (K is even, so no code byte spans two rows) */
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < K / 16; ++b) {
            const uint16_t *x = w + r * K + b * 16;
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf((float)bf16_value(x[i])));
            const float arg = amax_b / (6.0f * st);
            const uint8_t sc = e4m3_code((double)arg);
            scales[r * (K / 16) + b] = sc;
            const float sb = (float)e4m3_value(sc);
            for (int i = 0; i < 16; ++i) {
                uint8_t q = 0;
                if (sb > 0.0f) {
                    const float d = sb * st;
                    q = e2m1_code((double)((float)bf16_value(x[i]) / d));
                }
                const int64_t at = r * K + b * 16 + i;
                codes[at / 2] |= (uint8_t)(at % 2 == 0 ? q : q << 4);
            }
        }
    return ORACLE_OK;
}

/* The inverse: element value times its block scale times the matrix scale,
 * in fp64. */
int oracle_nvfp4_dequantize(int64_t rows, int64_t K, const uint8_t *codes, const uint8_t *scales,
                            float tensor_scale, double *out)
{
    if (rows < 0 || K < 16 || K % 16 != 0) return ORACLE_EINVAL;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < K; ++i) {
            const int64_t at = r * K + i;
            const uint8_t q = (uint8_t)(at % 2 == 0 ? codes[at / 2] & 15 : codes[at / 2] >> 4);
            out[at] = e2m1_value(q) * e4m3_value(scales[r * (K / 16) + i / 16]) * (double)tensor_scale;
        }
    return ORACLE_OK;
}
