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
//   gather   x_perm[p] = x[perm[p] / k], one 16-byte vector per thread.
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kTokChunk = 64;

__global__ void __launch_bounds__(256) hist_kernel(int T, int E, int k, const int32_t *__restrict__ idx,
                                                   const int32_t *__restrict__ keff, int32_t *__restrict__ hist) {
    __shared__ int h[kMaxExperts];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kTokChunk, t1 = min(T, t0 + kTokChunk);
    for (int s = t0 * k + threadIdx.x; s < t1 * k; s += blockDim.x) {
        const int t = s / k, j = s - t * k;
        const int ke = keff ? keff[t] : k;
        if (j < ke) {
            const int e = idx[s];
            if (e >= 0 && e < E) atomicAdd(&h[e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = h[e];
}

__global__ void __launch_bounds__(1024) scan_kernel(int E, int nchunks, int32_t *__restrict__ hist,
                                                    int32_t *__restrict__ counts, int32_t *__restrict__ offsets) {
    __shared__ int warp_sums[32];
    const int e = threadIdx.x;  // blockDim.x == 1024 >= E
    int c = 0;
    if (e < E)
        for (int b = 0; b < nchunks; ++b) c += hist[(size_t)b * E + e];
    // block-wide exclusive scan of c over e
    const int lane = e & 31, wid = e >> 5;
    int incl = c;
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
        warp_sums[lane] = ws;  // inclusive
    }
    __syncthreads();
    const int excl = incl - c + (wid ? warp_sums[wid - 1] : 0);
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

__global__ void __launch_bounds__(256) gather_kernel(int k, int H, const int32_t *__restrict__ offsets, int E,
                                                     const int32_t *__restrict__ perm, const uint4 *__restrict__ x,
                                                     uint4 *__restrict__ x_perm, int rows_per_block) {
    const int total = offsets[E];
    const int vec = H / 8;  // 16-byte vectors per row
    const int p0 = blockIdx.x * rows_per_block;
    for (int r = 0; r < rows_per_block; ++r) {
        const int p = p0 + r;
        if (p >= total) return;
        const int t = perm[p] / k;
        const uint4 *src = x + (size_t)t * vec;
        uint4 *dst = x_perm + (size_t)p * vec;
        for (int c = threadIdx.x; c < vec; c += blockDim.x) dst[c] = __ldg(src + c);
    }
}

}  // namespace

int dispatch_chunks(int T) { return (T + kTokChunk - 1) / kTokChunk; }

cudaError_t launch_dispatch(int T, int E, int k, const int32_t *idx, const int32_t *keff, int32_t *hist,
                            int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *slot_pos, cudaStream_t st) {
    const int nchunks = dispatch_chunks(T);
    hist_kernel<<<nchunks, 256, 0, st>>>(T, E, k, idx, keff, hist);
    scan_kernel<<<1, 1024, 0, st>>>(E, nchunks, hist, counts, offsets);
    scatter_kernel<<<nchunks, 32, 0, st>>>(T, E, k, idx, keff, hist, perm, slot_pos);
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(int T, int k, int H, const int32_t *offsets, int E, const int32_t *perm,
                               const uint16_t *x, uint16_t *x_perm, cudaStream_t st) {
    const int rows_per_block = 4;
    const long long max_rows = (long long)T * k;
    const int blocks = (int)((max_rows + rows_per_block - 1) / rows_per_block);
    gather_kernel<<<blocks, 256, 0, st>>>(k, H, offsets, E, perm, reinterpret_cast<const uint4 *>(x),
                                          reinterpret_cast<uint4 *>(x_perm), rows_per_block);
    return cudaGetLastError();
}

}  // namespace moe
