// Combine: out_t = sum_{j < keff[t]} ybuf[t, j] + [shared] ybuf[t, k].
// The expert FFN already wrote every kept slot's weighted output into the
// token-ordered buffer ybuf [T, k+1, H] (the gate weight is applied in its
// epilogue), so this is a fixed-order fp32 sum of a token's contiguous rows
// and one round to bf16.  HBM-bound: it reads (keff + shared) rows and
// writes one row per token, 8 bf16 per 16-byte access.
#include "moe_internal.cuh"

namespace moe {

namespace {

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        acc[2 * q] += bf16_bits_to_f32((uint16_t)(u[q] & 0xffffu));
        acc[2 * q + 1] += bf16_bits_to_f32((uint16_t)(u[q] >> 16));
    }
}

// One thread per (token, 16-byte column vector); the rows of a token are
// added in slot order.  The first four slot rows and the shared row are
// loaded together with keff (every row of ybuf is in bounds; rows past keff
// are loaded but not added), so the common case takes one memory round trip.
__global__ void __launch_bounds__(256) combine_kernel(int T, int k, int vec, int has_shared,
                                                      const uint4 *__restrict__ ybuf,
                                                      const int32_t *__restrict__ keff, uint4 *__restrict__ out) {
    pdl_launch_dependents();
    pdl_wait();
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int t = (int)(gid / vec), c = (int)(gid % vec);
    if (t >= T) return;
    const uint4 *rows = ybuf + (size_t)t * (k + 1) * vec + c;
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = u < k ? __ldg(rows + (size_t)u * vec) : make_uint4(0, 0, 0, 0);
    const uint4 vs = has_shared ? __ldg(rows + (size_t)k * vec) : make_uint4(0, 0, 0, 0);
    const int ke = keff ? min(max(__ldg(keff + t), 0), k) : k;  // a token's rows only, whatever keff holds
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u)
        if (u < ke) add_bf16x8(acc, v[u]);
    for (int j0 = 4; j0 < ke; j0 += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = (j0 + u < ke) ? __ldg(rows + (size_t)(j0 + u) * vec) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (j0 + u < ke) add_bf16x8(acc, v[u]);
    }
    if (has_shared) add_bf16x8(acc, vs);
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
        o[q] = (uint32_t)f32_to_bf16_bits(acc[2 * q]) | ((uint32_t)f32_to_bf16_bits(acc[2 * q + 1]) << 16);
    out[(size_t)t * vec + c] = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace

cudaError_t launch_combine(int T, int k, int H, int has_shared, const uint16_t *ybuf, const int32_t *keff,
                           uint16_t *out, cudaStream_t st) {
    const int vec = H / 8;
    const long long threads = (long long)T * vec;
    return launch_pdl(combine_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, st, T, k, vec, has_shared,
                      reinterpret_cast<const uint4 *>(ybuf), keff, reinterpret_cast<uint4 *>(out));
}

}  // namespace moe
