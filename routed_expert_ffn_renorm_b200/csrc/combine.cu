// Combine: out_t = sum_{j < keff[t]} ybuf[t, j] + [shared] ybuf[t, k].
// The expert FFN already wrote every kept slot's weighted output into the
// token-ordered buffer ybuf [T, k+1, H] (the gate weight is applied in its
// epilogue), so this is a fixed-order fp32 sum of a token's contiguous rows
// and one round to bf16.  HBM-bound: it reads (keff + shared) rows and
// writes one row per token, 8 bf16 per 16-byte access.
#include "moe_internal.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(128) combine_kernel(int T, int k, int H, int has_shared,
                                                      const uint4 *__restrict__ ybuf,
                                                      const int32_t *__restrict__ keff, uint4 *__restrict__ out) {
    const int t = blockIdx.x;
    const int vec = H / 8;
    const int ke = keff ? keff[t] : k;
    const uint4 *rows = ybuf + (size_t)t * (k + 1) * vec;
    for (int c = threadIdx.x; c < vec; c += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int j = 0; j <= k; ++j) {
            if (j < k ? j >= ke : !has_shared) continue;
            const uint4 v = __ldg(rows + (size_t)j * vec + c);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[2 * q] += bf16_bits_to_f32((uint16_t)(u[q] & 0xffffu));
                acc[2 * q + 1] += bf16_bits_to_f32((uint16_t)(u[q] >> 16));
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = (uint32_t)f32_to_bf16_bits(acc[2 * q]) | ((uint32_t)f32_to_bf16_bits(acc[2 * q + 1]) << 16);
        out[(size_t)t * vec + c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace

cudaError_t launch_combine(int T, int k, int H, int has_shared, const uint16_t *ybuf, const int32_t *keff,
                           uint16_t *out, cudaStream_t st) {
    combine_kernel<<<T, 128, 0, st>>>(T, k, H, has_shared, reinterpret_cast<const uint4 *>(ybuf), keff,
                                      reinterpret_cast<uint4 *>(out));
    return cudaGetLastError();
}

}  // namespace moe
