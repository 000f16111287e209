// Weight quantisers for block-scaled expert weights (MXFP8, NVFP4): the
// pack step that turns bf16 expert matrices into the FP8 / NVFP4 formats of
// DeepGEMM fork PR #5 "big M opt: splitT1 + L2 scatter + 2 stream" (see
// quant_codec.cuh for the formats and their rounding).  Run once when the
// weights are loaded, not per layer call; every block goes through the one
// per-block function of quant_codec.cuh, which the host test builds too.
//
// MXFP8: one thread per 32-element block (its 64 bytes of bf16 in, 32 code
// bytes and one scale byte out), blocks strided over the grid.
// NVFP4: (1) the largest |x| of each matrix, an integer max of the fp32
// bits (order-independent), accumulated with atomicMax into tensor_scale
// reused as uint32; (2) one thread per matrix turns it into the fp32 matrix
// scale in place; (3) one thread per 16-element block.
#include <algorithm>

#include "moe_internal.cuh"
#include "quant_codec.cuh"

namespace moe {

namespace {

constexpr int kQuantThreads = 256;

__global__ void __launch_bounds__(kQuantThreads) mxfp8_quantize_kernel(long long nblocks, const uint16_t *__restrict__ w,
                                                                        uint8_t *__restrict__ codes,
                                                                        uint8_t *__restrict__ scales) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
        uint16_t x[quant::kMxBlock];
        const uint4 *src = reinterpret_cast<const uint4 *>(w + b * quant::kMxBlock);
#pragma unroll
        for (int v = 0; v < quant::kMxBlock / 8; ++v) {
            const uint4 q = __ldg(src + v);
            memcpy(x + 8 * v, &q, sizeof q);
        }
        uint8_t c[quant::kMxBlock];
        scales[b] = quant::mxfp8_block(x, c);
        uint4 *dst = reinterpret_cast<uint4 *>(codes + b * quant::kMxBlock);
#pragma unroll
        for (int v = 0; v < quant::kMxBlock / 16; ++v) {
            uint4 q;
            memcpy(&q, c + 16 * v, sizeof q);
            dst[v] = q;
        }
    }
}

// amax_bits[m] = max over matrix m of |x| as fp32 bits; per_mat_vec 16-byte
// vectors per matrix, blockIdx.y = matrix.
__global__ void __launch_bounds__(kQuantThreads) nvfp4_amax_kernel(long long per_mat_vec, const uint16_t *__restrict__ w,
                                                                    uint32_t *__restrict__ amax_bits) {
    const int m = blockIdx.y;
    const uint4 *src = reinterpret_cast<const uint4 *>(w) + (long long)m * per_mat_vec;
    uint32_t mx = 0;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < per_mat_vec; i += stride) {
        uint16_t x[8];
        const uint4 q = __ldg(src + i);
        memcpy(x, &q, sizeof q);
        const uint32_t a = quant::bf16_amax_bits(x, 8);
        mx = a > mx ? a : mx;
    }
    mx = __reduce_max_sync(0xffffffffu, mx);
    if ((threadIdx.x & 31) == 0 && mx != 0) atomicMax(amax_bits + m, mx);
}

__global__ void nvfp4_scale_kernel(int nmat, float *__restrict__ tensor_scale) {
    const int m = blockIdx.x * blockDim.x + threadIdx.x;
    if (m < nmat) tensor_scale[m] = quant::nvfp4_tensor_scale(__float_as_uint(tensor_scale[m]));
}

__global__ void __launch_bounds__(kQuantThreads) nvfp4_quantize_kernel(long long nblocks, long long per_mat_blocks,
                                                                        const uint16_t *__restrict__ w,
                                                                        const float *__restrict__ tensor_scale,
                                                                        uint8_t *__restrict__ codes,
                                                                        uint8_t *__restrict__ scales) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
        uint16_t x[quant::kNvBlock];
        const uint4 *src = reinterpret_cast<const uint4 *>(w + b * quant::kNvBlock);
#pragma unroll
        for (int v = 0; v < quant::kNvBlock / 8; ++v) {
            const uint4 q = __ldg(src + v);
            memcpy(x + 8 * v, &q, sizeof q);
        }
        uint8_t c[quant::kNvBlock / 2];
        scales[b] = quant::nvfp4_block(x, __ldg(tensor_scale + b / per_mat_blocks), c);
        uint2 q;
        memcpy(&q, c, sizeof q);
        reinterpret_cast<uint2 *>(codes)[b] = q;
    }
}

int grid_for(long long work) {
    const long long g = (work + kQuantThreads - 1) / kQuantThreads;
    const long long cap = 8LL * device_sm_count();
    return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

// MXFP8 scales [rows, K / 32] -> [rows / 64][K / 128][64][4]: for every
// 64-row group and 128-wide K step, the 4 block scales of each of its 64
// rows in one contiguous 256-byte run, which the expert FFN's producer loads
// with one bulk copy per ring step.  One thread per 4-byte run.
__global__ void __launch_bounds__(kQuantThreads) mxfp8_pack_scales_kernel(long long rows, int K,
                                                                           const uint8_t *__restrict__ in,
                                                                           uint32_t *__restrict__ out) {
    const int kb = K / 32, ksteps = K / 128;
    const long long n = rows * ksteps;  // 4-byte runs
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x; o < n; o += stride) {
        const long long rgks = o >> 6;  // (row group, K step)
        const int r = (int)(o & 63);
        const long long rg = rgks / ksteps;
        const int ks = (int)(rgks - rg * ksteps);
        const uint8_t *src = in + (rg * 64 + r) * kb + ks * 4;
        out[o] = (uint32_t)src[0] | ((uint32_t)src[1] << 8) | ((uint32_t)src[2] << 16) | ((uint32_t)src[3] << 24);
    }
}

// NVFP4 block scales [rows, K / 16] -> [rows / 64][K / 128][64][8]: for each
// 64-row group and 128-wide K step, the 8 block scales of each of its 64 rows
// in one contiguous 512-byte run.  One thread per 8-byte run.
__global__ void __launch_bounds__(kQuantThreads) nvfp4_pack_scales_kernel(long long rows, int K,
                                                                          const uint8_t *__restrict__ in,
                                                                          uint2 *__restrict__ out) {
    const int kb = K / 16, ksteps = K / 128;
    const long long n = rows * ksteps;  // 8-byte runs
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x; o < n; o += stride) {
        const long long rgks = o >> 6;  // (row group, K step)
        const int r = (int)(o & 63);
        const long long rg = rgks / ksteps;
        const int ks = (int)(rgks - rg * ksteps);
        const uint8_t *src = in + (rg * 64 + r) * kb + ks * 8;
        uint2 v;
        v.x = (uint32_t)src[0] | ((uint32_t)src[1] << 8) | ((uint32_t)src[2] << 16) | ((uint32_t)src[3] << 24);
        v.y = (uint32_t)src[4] | ((uint32_t)src[5] << 8) | ((uint32_t)src[6] << 16) | ((uint32_t)src[7] << 24);
        out[o] = v;
    }
}

}  // namespace

cudaError_t launch_nvfp4_pack_scales(long long rows, int K, const uint8_t *scales, uint8_t *packed, cudaStream_t st) {
    const long long n = rows * (K / 128);
    nvfp4_pack_scales_kernel<<<grid_for(n), kQuantThreads, 0, st>>>(rows, K, scales, reinterpret_cast<uint2 *>(packed));
    return cudaGetLastError();
}

cudaError_t launch_mxfp8_pack_scales(long long rows, int K, const uint8_t *scales, uint8_t *packed, cudaStream_t st) {
    const long long n = rows * (K / 128);
    mxfp8_pack_scales_kernel<<<grid_for(n), kQuantThreads, 0, st>>>(rows, K, scales,
                                                                     reinterpret_cast<uint32_t *>(packed));
    return cudaGetLastError();
}

cudaError_t launch_quantize_mxfp8(long long rows, int K, const uint16_t *w, uint8_t *codes, uint8_t *scales,
                                  cudaStream_t st) {
    const long long nblocks = rows * (K / quant::kMxBlock);
    mxfp8_quantize_kernel<<<grid_for(nblocks), kQuantThreads, 0, st>>>(nblocks, w, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_quantize_nvfp4(int nmat, long long rows, int K, const uint16_t *w, uint8_t *codes,
                                  uint8_t *scales, float *tensor_scale, cudaStream_t st) {
    const long long per_mat = rows * K;
    cudaError_t e = cudaMemsetAsync(tensor_scale, 0, sizeof(float) * (size_t)nmat, st);
    if (e != cudaSuccess) return e;
    const long long per_mat_vec = per_mat / 8;
    const int gx = std::min(grid_for(per_mat_vec), 1024);
    nvfp4_amax_kernel<<<dim3(gx, nmat), kQuantThreads, 0, st>>>(per_mat_vec, w,
                                                                 reinterpret_cast<uint32_t *>(tensor_scale));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    nvfp4_scale_kernel<<<(nmat + 127) / 128, 128, 0, st>>>(nmat, tensor_scale);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long per_mat_blocks = per_mat / quant::kNvBlock, nblocks = (long long)nmat * per_mat_blocks;
    nvfp4_quantize_kernel<<<grid_for(nblocks), kQuantThreads, 0, st>>>(nblocks, per_mat_blocks, w, tensor_scale,
                                                                        codes, scales);
    return cudaGetLastError();
}

}  // namespace moe
