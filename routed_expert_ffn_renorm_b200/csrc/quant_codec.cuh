// Block-scaled expert-weight codes: MXFP8 (E4M3 elements, one UE8M0 scale
// per 32 consecutive elements along the reduction axis) and NVFP4 (E2M1
// elements, one E4M3 scale per 16, one fp32 scale per matrix) -- the FP8
// and NVFP4 expert-weight formats of DeepGEMM fork PR #5 "big M opt:
// splitT1 + L2 scatter + 2 stream" (its megamoe_nvfp4 kernels and the B200
// FP8 x FP4 policy), with the published format definitions (OCP
// Microscaling Formats v1.0 for MXFP8; NVFP4's E4M3 block scale and fp32
// tensor scale, amax / (6 * 448)).
//
// Every function here uses integer and IEEE fp32 arithmetic only -- no
// conversion intrinsics -- so the same source compiled for the host takes
// exactly the decisions the kernels take.  Rounding is to nearest, ties to
// the even code, saturating at the largest finite value (448 for E4M3, 6
// for E2M1); the sign bit copies the input's (so -0.0 keeps it).
//
// One block's work is one function (mxfp8_block, nvfp4_block), called by
// the kernels in quant.cu for every block index and by the host unit test.
#pragma once

#include <stdint.h>
#include <string.h>

#ifdef __CUDACC__
#define MOE_HD __host__ __device__ __forceinline__
#else
#define MOE_HD inline
#endif

namespace moe {
namespace quant {

constexpr int kMxBlock = 32;  // MXFP8 elements per scale
constexpr int kNvBlock = 16;  // NVFP4 elements per scale

MOE_HD uint32_t f32_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return u;
}
MOE_HD float bits_f32(uint32_t u) {
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}
MOE_HD float bf16_f32(uint16_t v) { return bits_f32((uint32_t)v << 16); }

// |a| rounded to E4M3 (a >= 0): the 7-bit magnitude code, 0x7E (448) at most.
MOE_HD uint32_t e4m3_magnitude(float a) {
    if (!(a < 448.0f)) return 0x7Eu;
    const uint32_t b = f32_bits(a);
    const int e = (int)(b >> 23) - 127;  // floor(log2 a) for a normal a
    if (e < -6) {
        // E4M3 subnormals are the multiples of 2^-9 below 2^-6: round a * 2^9
        // (exact) to an integer; 8 is code 0x08 = 2^-6, the smallest normal
        const float s = a * 512.0f;
        uint32_t q = (uint32_t)s;
        const float frac = s - (float)q;
        if (frac > 0.5f || (frac == 0.5f && (q & 1u))) ++q;
        return q;
    }
    // normal: keep 3 of the 23 mantissa bits, round the other 20 to nearest
    // even; a carry out of the mantissa moves to the next exponent
    const uint32_t m = (b >> 20) & 7u, rest = b & 0xFFFFFu;
    uint32_t code = ((uint32_t)(e + 7) << 3) | m;
    if (rest > 0x80000u || (rest == 0x80000u && (m & 1u))) ++code;
    return code > 0x7Eu ? 0x7Eu : code;
}

MOE_HD uint8_t e4m3_encode(float v) {
    const uint32_t b = f32_bits(v);
    return (uint8_t)(((b >> 24) & 0x80u) | e4m3_magnitude(bits_f32(b & 0x7FFFFFFFu)));
}

// Value of a finite E4M3 code (the two NaN codes are never produced here).
MOE_HD float e4m3_decode(uint8_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    const float mag = e == 0 ? (float)m * (1.0f / 512.0f) : bits_f32(((e + 120u) << 23) | (m << 20));
    return (c & 0x80u) ? -mag : mag;
}

// |a| rounded to E2M1 (a >= 0): magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 are codes
// 0..7; the code is the number of midpoints below a, a midpoint itself
// counting only when the code above it is even.
MOE_HD uint32_t e2m1_magnitude(float a) {
    const float mid[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
    uint32_t c = 0;
    for (int i = 0; i < 7; ++i) c += (a > mid[i] || (a == mid[i] && (i & 1) == 1)) ? 1u : 0u;
    return c;
}

MOE_HD uint8_t e2m1_encode(float v) {
    const uint32_t b = f32_bits(v);
    return (uint8_t)(((b >> 28) & 0x8u) | e2m1_magnitude(bits_f32(b & 0x7FFFFFFFu)));
}

// Largest |x| of n bf16 values, as fp32 bits (an integer maximum: exact and
// independent of order).
MOE_HD uint32_t bf16_amax_bits(const uint16_t *x, int n) {
    uint32_t m = 0;
    for (int i = 0; i < n; ++i) {
        const uint32_t a = (uint32_t)(x[i] & 0x7FFFu) << 16;
        m = a > m ? a : m;
    }
    return m;
}

// One MXFP8 block: 32 bf16 values -> 32 E4M3 codes; returns the UE8M0 scale
// code.  The scale is 2^(floor(log2 amax) - 8), clamped to [2^-127, 2^127]
// (an all-zero block takes 2^-127); each element is x * 2^-se rounded to E4M3.
MOE_HD uint8_t mxfp8_block(const uint16_t *x, uint8_t *codes) {
    const uint32_t amax = bf16_amax_bits(x, kMxBlock);
    const int ea = (int)(amax >> 23);  // biased exponent; 0 for zero or a subnormal maximum
    int se = ea == 0 ? -127 : ea - 127 - 8;
    se = se < -127 ? -127 : (se > 127 ? 127 : se);
    const float inv = bits_f32((uint32_t)(127 - se) << 23);  // 2^-se, a normal fp32 for se in [-127, 119]
    for (int i = 0; i < kMxBlock; ++i) codes[i] = e4m3_encode(bf16_f32(x[i]) * inv);
    return (uint8_t)(se + 127);
}

// The fp32 scale of an NVFP4 matrix from its largest |x|: amax / (6 * 448),
// 1 for an all-zero matrix.
MOE_HD float nvfp4_tensor_scale(uint32_t amax_bits) {
    const float amax = bits_f32(amax_bits);
    return amax > 0.0f ? amax / 2688.0f : 1.0f;
}

// One NVFP4 block: 16 bf16 values and the matrix scale -> 8 bytes of E2M1
// codes (element 2i in the low nibble); returns the E4M3 block scale code,
// E4M3(amax_b / (6 * st)).  Each element is x / (s_b * st) rounded to E2M1;
// a block whose scale rounds to zero stores zeros.
MOE_HD uint8_t nvfp4_block(const uint16_t *x, float st, uint8_t *packed) {
    const float amax_b = bits_f32(bf16_amax_bits(x, kNvBlock));
    const float arg = amax_b / (6.0f * st);
    const uint8_t sc = e4m3_encode(arg);
    const float sb = e4m3_decode(sc);
    for (int j = 0; j < kNvBlock / 2; ++j) packed[j] = 0;
    if (sb > 0.0f) {
        const float d = sb * st;
        for (int i = 0; i < kNvBlock; ++i) {
            const uint8_t q = e2m1_encode(bf16_f32(x[i]) / d);
            packed[i / 2] = (uint8_t)(packed[i / 2] | ((i & 1) ? (q << 4) : q));
        }
    }
    return sc;
}

// ------------------------------------------------------------ decoders --
// The weight a block-scaled code stands for, as the bf16 value the tensor
// cores take (exact: these values have at most 6 significant bits).

// E4M3 code c times 2^se as bf16 bits, built from the code's bits.  Exact
// for every finite code while se lies in [-117, 119] (a normal bf16); an
// MXFP8 scale is outside that only for blocks whose largest |x| is below
// 2^-109.
MOE_HD uint16_t e4m3_scaled_bf16(uint8_t c, int se) {
    const uint32_t sign = (uint32_t)(c & 0x80u) << 8;
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    if (e == 0 && m == 0) return (uint16_t)sign;
    if (e != 0) return (uint16_t)(sign | ((uint32_t)((int)e + 120 + se) << 7) | (m << 4));
    // subnormal code: m 2^-9 = (1.f) 2^p 2^-9 with p = floor(log2 m); the
    // leading bit of m becomes the implicit one
    const uint32_t p = m >= 4u ? 2u : (m >= 2u ? 1u : 0u);
    return (uint16_t)(sign | ((uint32_t)((int)p + 118 + se) << 7) | ((m << (7u - p)) & 0x7Fu));
}

// Value of an E2M1 code (low nibble).
MOE_HD float e2m1_decode(uint8_t c) {
    const uint32_t e = (c >> 1) & 3u, m = c & 1u;
    const float mag = e == 0 ? 0.5f * (float)m : bits_f32(((e + 126u) << 23) | (m << 22));
    return (c & 0x8u) ? -mag : mag;
}

// E2M1 code q times the E4M3 block scale sc, as bf16 bits (the NVFP4 weight
// without its fp32 matrix scale, which multiplies the projection's output).
// The fp32 product is exact and its low 16 bits are zero.
MOE_HD uint16_t nvfp4_scaled_bf16(uint8_t q, uint8_t sc) {
    return (uint16_t)(f32_bits(e2m1_decode(q) * e4m3_decode(sc)) >> 16);
}

}  // namespace quant
}  // namespace moe
