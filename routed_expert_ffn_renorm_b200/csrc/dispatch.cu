// Dispatch: group the kept (token, slot) pairs by expert for the grouped
// GEMMs (SpecForge PR #943, "Modifications": grouped_mm dispatch), as a
// deterministic counting sort -- bit-exact, no atomics on the ordering.
//
//   hist     one block per chunk of kTokChunk tokens: per-expert counts of
//            the chunk's kept slots in shared memory -> hist[chunk][e];
//   scan     one block: counts[e] = sum over chunks, offsets = exclusive
//            scan over experts, and hist[chunk][e] rewritten in place to the
//            first position the chunk's slots of expert e take;
//   scatter  one warp per chunk walks the chunk's slots in ascending slot
//            id, 32 at a time; __match_any_sync groups lanes with the same
//            expert, the rank inside the group is the count of lower lanes,
//            so positions follow slot order exactly;
//   gather   x_perm[p] = x[perm[p] / k], four 16-byte vectors per thread.
// Batches of up to kSmallSlots slots run all of it as one launch
// (dispatch_small_kernel).
#include <algorithm>
#include <atomic>

#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kTokChunk = 64;
constexpr int kSmallSlots = 8192;  // T*k up to this: the whole sort in one CTA

// Exclusive prefix sum of one value per thread over a 1024-thread block.
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_sums) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int ws = warp_sums[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, ws, off);
            if (lane >= off) ws += o;
        }
        warp_sums[lane] = ws;  // inclusive over warps
    }
    __syncthreads();
    return incl - v + (wid ? warp_sums[wid - 1] : 0);
}

__global__ void __launch_bounds__(256) hist_kernel(int T, int E, int k, const int32_t *__restrict__ idx,
                                                   const int32_t *__restrict__ keff, int32_t *__restrict__ hist,
                                                   int32_t *__restrict__ status) {
    __shared__ int h[kMaxExperts];
    pdl_launch_dependents();
    pdl_wait();
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kTokChunk, t1 = min(T, t0 + kTokChunk);
    for (int s = t0 * k + threadIdx.x; s < t1 * k; s += blockDim.x) {
        const int t = s / k, j = s - t * k;
        const int ke = keff ? keff[t] : k;
        if (j < ke) {
            const int e = idx[s];
            if (e >= 0 && e < E) atomicAdd(&h[e], 1);
            else if (kDebugBounds && e != -1 && status) atomicOr(status, MOE_STATUS_BOUNDS);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = h[e];
}

__global__ void __launch_bounds__(1024) scan_kernel(int E, int nchunks, int32_t *__restrict__ hist,
                                                    int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                                                    int32_t *__restrict__ sched, int32_t *__restrict__ hdone) {
    __shared__ int warp_sums[32];
    pdl_launch_dependents();
    pdl_wait();
    const int e = threadIdx.x;  // blockDim.x == 1024 >= E
    if (sched != nullptr && e < 2) {  // fresh work-item counters for the grouped FFN launches
        sched[4 + e] = 0;
        sched[8 + e] = 0;
    }
    if (hdone != nullptr)
        for (int g = e; g <= E + 1; g += blockDim.x) hdone[g] = 0;
    int c = 0;
    if (e < E)
        for (int b = 0; b < nchunks; ++b) c += hist[(size_t)b * E + e];
    const int excl = block_exclusive_scan(c, warp_sums);
    if (e < E) {
        counts[e] = c;
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + c;
        int run = excl;
        for (int b = 0; b < nchunks; ++b) {
            const int hb = hist[(size_t)b * E + e];
            hist[(size_t)b * E + e] = run;
            run += hb;
        }
    }
}

__global__ void __launch_bounds__(32) scatter_kernel(int T, int E, int k, const int32_t *__restrict__ idx,
                                                     const int32_t *__restrict__ keff,
                                                     const int32_t *__restrict__ hist, int32_t *__restrict__ perm,
                                                     int32_t *__restrict__ slot_pos) {
    __shared__ int base[kMaxExperts];
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x;
    for (int e = lane; e < E; e += 32) base[e] = hist[(size_t)blockIdx.x * E + e];
    __syncwarp();
    const int t0 = blockIdx.x * kTokChunk, t1 = min(T, t0 + kTokChunk);
    for (int s0 = t0 * k; s0 < t1 * k; s0 += 32) {
        const int s = s0 + lane;
        int e = -1;
        bool valid = false;
        if (s < t1 * k) {
            const int t = s / k, j = s - t * k;
            const int ke = keff ? keff[t] : k;
            e = idx[s];
            valid = j < ke && e >= 0 && e < E;
            if (!valid) slot_pos[s] = -1;
        }
        const int key = valid ? e : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        int pos = 0;
        if (valid) {
            pos = base[e] + rank;
            perm[pos] = s;
            slot_pos[s] = pos;
        }
        __syncwarp();
        if (valid && lane == 31 - __clz(peers)) base[e] += __popc(peers);
        __syncwarp();
    }
}

// Small batches: the whole counting sort, redundantly in every CTA of the
// grid (it costs a few microseconds of the CTA's own time), then each CTA
// gathers its share of x_perm rows from its own copy of perm -- one launch
// for hist + scan + scatter + gather.  In each 1024-thread CTA, warps
// 0..W-1 own contiguous runs of slots: per-warp counts in shared memory, one
// exclusive scan over experts, per-warp bases, then each warp places its run
// in slot order with __match_any_sync ranks.  CTA 0 writes counts, offsets,
// perm and slot_pos and zeroes the FFN's scheduling counters.
__global__ void __launch_bounds__(1024) dispatch_small_kernel(int T, int E, int k, int W, int vec,
                                                              const int32_t *__restrict__ idx,
                                                              const int32_t *__restrict__ keff,
                                                              const uint4 *__restrict__ x, uint4 *__restrict__ x_perm,
                                                              int32_t *__restrict__ counts,
                                                              int32_t *__restrict__ offsets,
                                                              int32_t *__restrict__ perm,
                                                              int32_t *__restrict__ slot_pos, int32_t *__restrict__ sched,
                                                              int32_t *__restrict__ hdone) {
    extern __shared__ int smem_i[];
    int *hist = smem_i;               // [W][E]
    int *perm_s = smem_i + W * E;     // [T*k]
    __shared__ int warp_sums[32];
    __shared__ int total_s;
    pdl_launch_dependents();
    pdl_wait();
    const bool writer = blockIdx.x == 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Tk = T * k, chunk = (Tk + W - 1) / W;
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) hist[i] = 0;
    if (writer && sched != nullptr && threadIdx.x < 2) {
        sched[4 + threadIdx.x] = 0;
        sched[8 + threadIdx.x] = 0;
    }
    if (writer && hdone != nullptr)
        for (int g = threadIdx.x; g <= E + 1; g += blockDim.x) hdone[g] = 0;
    __syncthreads();
    const int s_begin = warp * chunk, s_end = min(Tk, s_begin + chunk);
    if (warp < W) {
        for (int s0 = s_begin; s0 < s_end; s0 += 32) {
            const int s = s0 + lane;
            int key = -1;
            if (s < s_end) {
                const int t = s / k, j = s - t * k;
                const int e = __ldg(idx + s);
                const bool kept = j < (keff ? __ldg(keff + t) : k);
                if (kept && e >= 0 && e < E) key = e;
                else if (kDebugBounds && kept && e != -1 && writer && sched) atomicOr(sched, MOE_STATUS_BOUNDS);
            }
            const unsigned peers = __match_any_sync(0xffffffffu, key);
            if (key >= 0 && lane == __ffs(peers) - 1) hist[warp * E + key] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();
    const int e = threadIdx.x;
    int c = 0;
    if (e < E)
        for (int w = 0; w < W; ++w) c += hist[w * E + e];
    const int excl = block_exclusive_scan(c, warp_sums);
    if (e < E) {
        if (writer) {
            counts[e] = c;
            offsets[e] = excl;
            if (e == E - 1) offsets[E] = excl + c;
        }
        if (e == E - 1) total_s = excl + c;
        int run = excl;
        for (int w = 0; w < W; ++w) {
            const int hw = hist[w * E + e];
            hist[w * E + e] = run;
            run += hw;
        }
    }
    __syncthreads();
    if (warp < W) {
        int *base = hist + warp * E;
        for (int s0 = s_begin; s0 < s_end; s0 += 32) {
            const int s = s0 + lane;
            int key = -1;
            if (s < s_end) {
                const int t = s / k, j = s - t * k;
                const int ee = __ldg(idx + s);
                if (j < (keff ? __ldg(keff + t) : k) && ee >= 0 && ee < E) key = ee;
                else if (writer) slot_pos[s] = -1;
            }
            const unsigned peers = __match_any_sync(0xffffffffu, key);
            if (key >= 0) {
                const int pos = base[key] + __popc(peers & ((1u << lane) - 1u));
                perm_s[pos] = s;
                if (writer) {
                    perm[pos] = s;
                    slot_pos[s] = pos;
                }
            }
            __syncwarp();
            if (key >= 0 && lane == 31 - __clz(peers)) base[key] += __popc(peers);
            __syncwarp();
        }
    }
    if (x_perm == nullptr) return;
    __syncthreads();
    const int total = total_s;
    for (int pr = blockIdx.x; pr < total; pr += gridDim.x) {
        const uint4 *src = x + (size_t)(perm_s[pr] / k) * vec;
        uint4 *dst = x_perm + (size_t)pr * vec;
        for (int cc = threadIdx.x; cc < vec; cc += blockDim.x) dst[cc] = __ldg(src + cc);
    }
}

__global__ void __launch_bounds__(256) gather_kernel(int k, int vec4, const int32_t *__restrict__ offsets, int E,
                                                     const int32_t *__restrict__ perm, const uint4 *__restrict__ x,
                                                     uint4 *__restrict__ x_perm) {
    pdl_launch_dependents();
    pdl_wait();
    // one thread copies 4 consecutive 16-byte vectors (64 B) of one row
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int p = (int)(gid / vec4), c = (int)(gid % vec4) * 4;
    if (p >= __ldg(offsets + E)) return;
    const int t = __ldg(perm + p) / k;
    const uint4 *src = x + (size_t)t * vec4 * 4 + c;
    uint4 *dst = x_perm + (size_t)p * vec4 * 4 + c;
    const uint4 a = __ldg(src), b = __ldg(src + 1), d = __ldg(src + 2), e = __ldg(src + 3);
    dst[0] = a;
    dst[1] = b;
    dst[2] = d;
    dst[3] = e;
}

}  // namespace

int dispatch_chunks(int T) { return (T + kTokChunk - 1) / kTokChunk; }

bool dispatch_is_small(int T, int k) { return (long long)T * k <= kSmallSlots; }

cudaError_t launch_dispatch(int T, int E, int k, const int32_t *idx, const int32_t *keff, int32_t *hist,
                            int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *slot_pos,
                            int32_t *status_block, int32_t *hdone, const uint16_t *x, uint16_t *x_perm, int H,
                            cudaStream_t st) {
    if (dispatch_is_small(T, k)) {
        // per-warp counts fit in 32 KB; no more warps than 32-slot passes (fewer columns to scan)
        const int W = std::min(E <= 256 ? 32 : (E <= 512 ? 16 : 8), std::max(1, (T * k + 31) / 32));
        const size_t smem = ((size_t)W * E + (size_t)T * k) * 4;  // <= 64 KB
        static std::atomic<int> attr_set[64];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        if (!attr_set[dev].load(std::memory_order_acquire)) {
            const cudaError_t e = cudaFuncSetAttribute(dispatch_small_kernel,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, 65536);
            if (e != cudaSuccess) return e;
            attr_set[dev].store(1, std::memory_order_release);
        }
        const int grid = x_perm ? std::max(1, std::min(device_sm_count(), T * k)) : 1;
        return launch_pdl(dispatch_small_kernel, dim3(grid), dim3(1024), smem, st, T, E, k, W, H / 8, idx, keff,
                          reinterpret_cast<const uint4 *>(x), reinterpret_cast<uint4 *>(x_perm), counts, offsets,
                          perm, slot_pos, status_block, hdone);
    }
    const int nchunks = dispatch_chunks(T);
    cudaError_t e = launch_pdl(hist_kernel, dim3(nchunks), dim3(256), 0, st, T, E, k, idx, keff, hist, status_block);
    if (e != cudaSuccess) return e;
    e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, st, E, nchunks, hist, counts, offsets, status_block, hdone);
    if (e != cudaSuccess) return e;
    e = launch_pdl(scatter_kernel, dim3(nchunks), dim3(32), 0, st, T, E, k, idx, keff, hist, perm, slot_pos);
    if (e != cudaSuccess || x_perm == nullptr) return e;
    return launch_gather_rows(T, k, H, offsets, E, perm, x, x_perm, st);
}

cudaError_t launch_gather_rows(int T, int k, int H, const int32_t *offsets, int E, const int32_t *perm,
                               const uint16_t *x, uint16_t *x_perm, cudaStream_t st) {
    const int vec4 = H / 32;  // groups of four 16-byte vectors per row (H % 128 == 0)
    const long long threads = (long long)T * k * vec4;
    return launch_pdl(gather_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, st, k, vec4, offsets, E,
                      perm, reinterpret_cast<const uint4 *>(x), reinterpret_cast<uint4 *>(x_perm));
}

}  // namespace moe
