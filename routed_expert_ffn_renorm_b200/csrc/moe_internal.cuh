// Internal declarations shared by the CUDA translation units of libmoe.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

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

// Bounds-checked build (-DMOE_DEBUG_BOUNDS, libmoe_checked.so): index inputs
// that come from the caller are range-checked where they are used; a bad one
// sets MOE_STATUS_BOUNDS in the status word and the access is skipped (no
// trap).  kDebugBounds is false in the release build, so the checks compile
// away there.
#ifdef MOE_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif

// Programmatic dependent launch: every kernel of the layer lets the next one
// launch as soon as all of its CTAs are running, and waits for its own
// predecessor (grid completion and memory flush) before it reads anything
// the predecessor wrote.  Set-up that touches no such data (barrier init,
// TMEM allocation, tensor-map prefetch) runs before the wait.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------- launch wrappers --
// Every wrapper enqueues on `st` and returns cudaGetLastError().

// Route (one warp per token).
// Checked library: sets MOE_STATUS_NONFINITE in *status when any of the n
// logits is a NaN or an infinity.
cudaError_t launch_check_logits(long long n, const float *logits, int32_t *status, cudaStream_t st);
cudaError_t launch_route(int T, int E, int k, int norm_topk, float topp, const float *logits, int32_t *idx,
                         float *w, int32_t *keff, const uint16_t *x, const uint16_t *gvec, int H,
                         float *sgate, cudaStream_t st);

// Budget: per-chunk partial aggregates, then selection and compaction.
int budget_chunks(int T);
cudaError_t launch_budget(int T, int E, int k, int N, int norm_topk, int32_t *idx, float *w,
                          int32_t *keff, uint8_t *kept, int32_t *n_dropped, float *part_agg,
                          int32_t *part_cnt, cudaStream_t st);

// Dispatch: histogram, scan, stable scatter, row gather.
int dispatch_chunks(int T);
// `status_block`, `hdone` (may be null): the dispatch kernels also zero the
// grouped FFN's work-item counters and gate/up completion counters [E + 2].
// x_perm (may be null): also gather x_perm[p] = x[perm[p] / k].
cudaError_t launch_dispatch(int T, int E, int k, const int32_t *idx, const int32_t *keff,
                            int32_t *hist, int32_t *counts, int32_t *offsets, int32_t *perm,
                            int32_t *slot_pos, int32_t *status_block, int32_t *hdone, const uint16_t *x,
                            uint16_t *x_perm, int H, cudaStream_t st);
int device_sm_count();  // SMs of the current device (cached)
cudaError_t launch_gather_rows(int T, int k, int H, const int32_t *offsets, int E,
                               const int32_t *perm, const uint16_t *x, uint16_t *x_perm,
                               cudaStream_t st);

// Fused small-batch front end: route -> budget (N > 0) -> dispatch -> row
// gather + shared gate in one launch, for T*k <= kFrontMaxSlots and
// T*E <= kFrontMaxLogits.  Same outputs, bit for bit, as launch_route,
// launch_budget and launch_dispatch in sequence.
constexpr int kFrontMaxSlots = 8192;
constexpr int kFrontMaxLogits = 16384;
bool front_fits(int T, int E, int k);
cudaError_t launch_front(int T, int E, int k, int N, int norm_topk, float topp, int H, const float *logits,
                         const uint16_t *x,
                         const uint16_t *gvec, int32_t *idx, float *w, float *sgate, int32_t *keff, uint8_t *kept,
                         int32_t *n_dropped, int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *slot_pos,
                         uint16_t *x_perm, int32_t *status_block, int32_t *hdone, cudaStream_t st);

// Router projection logits = x . W_r^T on the tensor cores (router_proj.cu).
// `part` holds rp_partial_bytes(T, E, H) bytes of K-split partials.
size_t rp_partial_bytes(int T, int E, int H);
cudaError_t launch_router_proj(int T, int E, int H, const uint16_t *x, const uint16_t *w_router, float *logits,
                               float *part, int32_t *status, cudaStream_t st);

// Weight quantisers (quant.cu): MXFP8 over rows x K (K % 32 == 0), NVFP4 over
// nmat matrices of rows x K (K % 16 == 0); all pointers 16-byte aligned.
cudaError_t launch_quantize_mxfp8(long long rows, int K, const uint16_t *w, uint8_t *codes, uint8_t *scales,
                                  cudaStream_t st);
cudaError_t launch_quantize_nvfp4(int nmat, long long rows, int K, const uint16_t *w, uint8_t *codes,
                                  uint8_t *scales, float *tensor_scale, cudaStream_t st);
// MXFP8 scales [rows, K / 32] -> the FFN's layout [rows / 64][K / 128][64][4]
// (rows % 64 == 0, K % 128 == 0).
cudaError_t launch_mxfp8_pack_scales(long long rows, int K, const uint8_t *scales, uint8_t *packed, cudaStream_t st);
cudaError_t launch_nvfp4_pack_scales(long long rows, int K, const uint8_t *scales, uint8_t *packed, cudaStream_t st);

// Expert parallelism (ep.cu): destination ranks of slots, the send metadata
// in send order, and the returned rows back to token order.  n_dev: the
// number of sent (returned) rows, on the device (the dispatch's offsets[W]).
cudaError_t launch_ep_rank_ids(int n, int epr, const int32_t *idx, int32_t *rank_idx, cudaStream_t st);
cudaError_t launch_ep_pack(int n_max, const int32_t *n_dev, int epr, const int32_t *perm, const int32_t *idx,
                           const float *w, int32_t *local_idx, float *local_w, cudaStream_t st);
cudaError_t launch_ep_unpack(int n_max, const int32_t *n_dev, int k, int H, const int32_t *perm, const uint16_t *rows,
                             uint16_t *ybuf, cudaStream_t st);

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
    // fmt 1 (MXFP8 weights): the w_* / ws_* pointers above hold E4M3 codes (one
    // byte per weight, same shapes) and sf_* the packed UE8M0 scales; fmt 2
    // (NVFP4): they hold E2M1 codes (two per byte), sf_* the packed E4M3 block
    // scales, ts_* the fp32 matrix scales ([E] each) and tss the shared
    // expert's {gate, up, down}
    int fmt;
    const uint8_t *sf_gate, *sf_up, *sf_down, *sfs_gate, *sfs_up, *sfs_down;
    const float *ts_gate, *ts_up, *ts_down, *tss;
    uint16_t *h_perm, *h_shared, *ybuf;
    int32_t *status;  // the workspace's status block: [0] status word,
                      // [4..5] gate/up (or fused) and [8..9] down work-item counters
    int32_t *hdone;   // [E + 2] per-group finished gate/up tiles, then all of them (fused launches)
};
// One launch of the grouped FFN kernel.  phases: 1 = gate/up (writes
// h_perm / h_shared), 2 = down (reads them, writes ybuf), 3 = both in one
// launch.  Returns MOE_OK / MOE_ERR_*.
int ffn_launch(const FfnArgs &a, int phases, cudaStream_t st);
// Both FFN phases of a layer: one fused launch while the groups are small
// (weight streaming; the fused launch hides the tail of the gate/up phase),
// two launches once the mean group fills a 128-token tile (tensor-bound).
int ffn_launch_both(const FfnArgs &a, cudaStream_t st);

}  // namespace moe
