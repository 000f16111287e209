// Internal declarations shared by the CUDA translation units of libmoe.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;

// ---------------------------------------------------------------- helpers --
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t v) {
    return __uint_as_float(((uint32_t)v) << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t *>(&b);
}

// ------------------------------------------------------- launch wrappers --
// Every wrapper enqueues on `st` and returns cudaGetLastError().

// Route (one warp per token).
cudaError_t launch_route(int T, int E, int k, int norm_topk, const float *logits, int32_t *idx,
                         float *w, int32_t *keff, const uint16_t *x, const uint16_t *gvec, int H,
                         float *sgate, cudaStream_t st);

// Budget: per-chunk partial aggregates, then selection and compaction.
int budget_chunks(int T);
cudaError_t launch_budget(int T, int E, int k, int N, int norm_topk, int32_t *idx, float *w,
                          int32_t *keff, uint8_t *kept, int32_t *n_dropped, float *part_agg,
                          int32_t *part_cnt, cudaStream_t st);

// Dispatch: histogram, scan, stable scatter, row gather.
int dispatch_chunks(int T);
cudaError_t launch_dispatch(int T, int E, int k, const int32_t *idx, const int32_t *keff,
                            int32_t *hist, int32_t *counts, int32_t *offsets, int32_t *perm,
                            int32_t *slot_pos, cudaStream_t st);
cudaError_t launch_gather_rows(int T, int k, int H, const int32_t *offsets, int E,
                               const int32_t *perm, const uint16_t *x, uint16_t *x_perm,
                               cudaStream_t st);

// Combine.
cudaError_t launch_combine(int T, int k, int H, int has_shared, const uint16_t *ybuf,
                           const int32_t *keff, uint16_t *out, cudaStream_t st);

// Grouped expert FFN (tcgen05).
struct FfnArgs {
    int T, H, E, I, k, Is;
    const uint16_t *x, *x_perm;
    const int32_t *offsets, *perm;
    const float *topk_w, *sgate;
    const uint16_t *w_gate, *w_up, *w_down, *ws_gate, *ws_up, *ws_down;
    uint16_t *h_perm, *h_shared, *ybuf;
    int32_t *status;
};
// Each returns MOE_OK / MOE_ERR_*.  gate_up writes h_perm / h_shared; down
// reads them and writes ybuf.
int ffn_launch_gate_up(const FfnArgs &a, cudaStream_t st);
int ffn_launch_down(const FfnArgs &a, cudaStream_t st);

}  // namespace moe
