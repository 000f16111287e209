// Host build of the CUDA library's block-scaled weight codes
// (routed_expert_ffn_renorm_b200/csrc/quant_codec.cuh), for the CPU test that
// compares them bit for bit with the oracle.  The per-block functions are the
// ones the quantiser kernels call; the loops below walk the blocks in the
// kernels' order.
#include <stdint.h>

#include "../../routed_expert_ffn_renorm_b200/csrc/quant_codec.cuh"

using namespace moe::quant;

extern "C" {

void host_e4m3_encode(int64_t n, const float *v, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(v[i]);
}

void host_e4m3_decode(int64_t n, const uint8_t *c, float *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_decode(c[i]);
}

void host_e2m1_encode(int64_t n, const float *v, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e2m1_encode(v[i]);
}

void host_mxfp8_quantize(int64_t rows, int32_t K, const uint16_t *w, uint8_t *codes, uint8_t *scales) {
    const int64_t nblocks = rows * (K / kMxBlock);
    for (int64_t b = 0; b < nblocks; ++b)
        scales[b] = mxfp8_block(w + b * kMxBlock, codes + b * kMxBlock);
}

void host_nvfp4_quantize(int32_t nmat, int64_t rows, int32_t K, const uint16_t *w, uint8_t *codes,
                         uint8_t *scales, float *tensor_scale) {
    const int64_t per_mat = rows * K;
    for (int32_t m = 0; m < nmat; ++m)
        tensor_scale[m] = nvfp4_tensor_scale(bf16_amax_bits(w + m * per_mat, (int)per_mat));
    const int64_t nblocks = (int64_t)nmat * per_mat / kNvBlock, per_mat_blocks = per_mat / kNvBlock;
    for (int64_t b = 0; b < nblocks; ++b)
        scales[b] = nvfp4_block(w + b * kNvBlock, tensor_scale[b / per_mat_blocks], codes + b * (kNvBlock / 2));
}

// out[r, i] = bf16 bits of codes[r, i] x 2^(scales[r, i / 32] - 127)
void host_mxfp8_to_bf16(int64_t rows, int32_t K, const uint8_t *codes, const uint8_t *scales, uint16_t *out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t i = 0; i < K; ++i)
            out[r * K + i] = e4m3_scaled_bf16(codes[r * K + i], (int)scales[r * (K / kMxBlock) + i / kMxBlock] - 127);
}

// out[r, i] = bf16 bits of the E2M1 element (packed, 2i low) x its E4M3 block scale
void host_nvfp4_to_bf16(int64_t rows, int32_t K, const uint8_t *codes, const uint8_t *scales, uint16_t *out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t i = 0; i < K; ++i) {
            const int64_t at = r * K + i;
            const uint8_t q = (uint8_t)((at & 1) ? codes[at / 2] >> 4 : codes[at / 2] & 15);
            out[at] = nvfp4_scaled_bf16(q, scales[r * (K / kNvBlock) + i / kNvBlock]);
        }
}

}  // extern "C"
