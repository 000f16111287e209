// Fused front end of a small batch: route -> (budget) -> dispatch -> row
// gather and shared-expert gate in one launch, for batches whose logits
// (T x E) and slots (T x k) fit one block's shared memory.
//
// Every CTA copies the T x E logits to shared memory in one coalesced pass and
// routes all T tokens itself from there (route_token_lane, one token per
// thread, for 32 < E <= 64; route_token, one warp per token, otherwise),
// applies the budget (budget_block) and sorts the kept slots by expert
// (block_sort_by_expert, or regroup_kept from the budget's own sort) -- the
// same device code, or the same order, as the stand-alone route / budget /
// dispatch kernels, so the results are the same bits.  CTA 0 writes the routing, budget and dispatch outputs; all CTAs
// then share the rest: x_perm rows in CTA-strided order and the shared
// gate sigmoid(g . x_t) for tokens in CTA-strided order (a 128-thread group
// per token, as in the route kernel).  Redundant routing costs each CTA one
// read of the T x E logits from L2 and saves two to four launches and their
// global round trips.
#include <algorithm>
#include <atomic>

#include "front.cuh"

namespace moe {

namespace {

constexpr int kFrontThreads = 1024;
constexpr int kFrontGroups = kFrontThreads / kGateThreads;  // shared-gate groups per CTA

struct FrontArgs {
    int T, E, k, N, norm_topk, H;
    float topp;
    const float *logits;
    const uint16_t *x, *gvec;
    int32_t *idx;
    float *w;
    float *sgate;  // null: no shared expert
    int32_t *keff;
    uint8_t *kept;  // with N > 0
    int32_t *n_dropped;
    int32_t *counts, *offsets, *perm, *slot_pos;
    uint16_t *x_perm;
    int32_t *sched;  // the FFN's work-item counters [4..5], [8..9]: zeroed here
    int32_t *hdone;  // the FFN's gate/up completion counters [E + 2]: zeroed here
};

size_t front_smem(int T, int E, int k) {
    const size_t Tk = (size_t)T * k;
    return (size_t)T * (E + 1) * 4 + Tk * 12 + (size_t)T * 4 + (size_t)sort_warps(E) * E * 4 +
           (size_t)(E + 1) * 4 + (size_t)E * 6 + 16;
}

// Upper bound of front_smem over T*k <= kFrontMaxSlots, T*E <= kFrontMaxLogits
// (largest at T = 8192, E = 2, k = 1: 229,672 bytes with the padded logit rows).
constexpr int kFrontSmemMax = 225 * 1024;

constexpr int kGatherInFlight = 4;  // 16-byte row vectors each thread loads before it stores

template <int V>  // logits per lane: V * 32 >= E
__global__ void __launch_bounds__(kFrontThreads, 1) front_small_kernel(const FrontArgs a) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int T = a.T, E = a.E, k = a.k, Tk = T * k, W = sort_warps(E);
    // logit rows: stride E for warp routing, an odd stride for lane routing (a
    // warp then reads 32 rows at once without bank conflicts)
    const bool lane_route = lane_routed(E);
    const int ls = lane_route ? (E | 1) : E;
    float *logit_s = reinterpret_cast<float *>(sm);  // [T * ls]
    int32_t *idx_s = reinterpret_cast<int32_t *>(logit_s + (size_t)T * (E + 1));
    float *w_s = reinterpret_cast<float *>(idx_s + Tk);
    int *sorted = reinterpret_cast<int *>(w_s + Tk);
    int32_t *keff_s = sorted + Tk;
    int *hist = keff_s + T;
    int *off = hist + W * E;
    float *agg = reinterpret_cast<float *>(off + E + 1);
    uint8_t *pres = reinterpret_cast<uint8_t *>(agg + E);
    uint8_t *keep = pres + E;
    __shared__ int warp_sums[32];
    __shared__ int nd_s;
    __shared__ float part[kFrontGroups][kGateThreads / 32];
    pdl_launch_dependents();
    pdl_wait();
    const bool writer = blockIdx.x == 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // the logits to shared memory (16-byte loads; T * E * 4 is a multiple of 16
    // whenever T * E % 4 == 0, else a scalar copy), then route every token
    const int TE = T * E;
    if (ls == E && (TE & 3) == 0) {
        const float4 *src = reinterpret_cast<const float4 *>(a.logits);
        float4 *dst = reinterpret_cast<float4 *>(logit_s);
        for (int i = threadIdx.x; i < TE / 4; i += kFrontThreads) dst[i] = __ldg(src + i);
    } else {
        for (int i = threadIdx.x; i < TE; i += kFrontThreads) {
            const int t = i / E;
            logit_s[(size_t)t * ls + (i - t * E)] = __ldg(a.logits + i);
        }
    }
    __syncthreads();
    if (lane_route) {
        for (int t = threadIdx.x; t < T; t += kFrontThreads)
            keff_s[t] = route_token_lane<false>(t, E, k, a.norm_topk, a.topp, logit_s + (size_t)t * ls, idx_s, w_s);
    } else {
        for (int t = warp; t < T; t += kFrontThreads / 32) {
            const int c = route_token<V, false>(t, E, k, a.norm_topk, a.topp, logit_s, idx_s, w_s, nullptr, lane);
            if (lane == 0) keff_s[t] = c;
        }
    }
    __syncthreads();
    // budget (a union of at most N experts, or N == 0, leaves everything as it is)
    // and dispatch: kept slots by expert, slot order inside one
    if (a.N > 0) {
        budget_block(T, E, k, a.N, a.norm_topk, idx_s, w_s, keff_s, keep, &nd_s, hist, off, sorted, agg, pres,
                     warp_sums);
        regroup_kept(E, k, idx_s, keff_s, keep, off, sorted, hist, warp_sums);
    } else {
        block_sort_by_expert(
            Tk, E, sort_warps_for(Tk, E),
            [=](int s) {
                const int e = idx_s[s];
                return (e >= 0 && e < E) ? e : -1;
            },
            hist, off, sorted, warp_sums);
    }
    const int total = off[E];
    if (writer) {
        for (int s = threadIdx.x; s < Tk; s += kFrontThreads) {
            a.idx[s] = idx_s[s];
            a.w[s] = w_s[s];
            a.slot_pos[s] = -1;
        }
        for (int t = threadIdx.x; t < T; t += kFrontThreads) a.keff[t] = keff_s[t];
        for (int e = threadIdx.x; e < E; e += kFrontThreads) {
            a.counts[e] = off[e + 1] - off[e];
            a.offsets[e] = off[e];
            if (a.N > 0) a.kept[e] = keep[e];
        }
        if (threadIdx.x == 0) {
            a.offsets[E] = total;
            if (a.N > 0) *a.n_dropped = nd_s;
        }
        if (threadIdx.x < 2) {
            a.sched[4 + threadIdx.x] = 0;
            a.sched[8 + threadIdx.x] = 0;
        }
        for (int g = threadIdx.x; g <= E + 1; g += kFrontThreads) a.hdone[g] = 0;
        __syncthreads();  // slot_pos = -1 first, then the kept slots' positions
        for (int p = threadIdx.x; p < total; p += kFrontThreads) {
            a.perm[p] = sorted[p];
            a.slot_pos[sorted[p]] = p;
        }
    }
    // shared gate: one 128-thread group per token, tokens CTA-strided
    if (a.sgate != nullptr) {
        const int grp = threadIdx.x / kGateThreads, tid = threadIdx.x % kGateThreads;
        for (int t = blockIdx.x * kFrontGroups + grp; t < T; t += gridDim.x * kFrontGroups) {
            const float g = shared_gate_group(t, a.x, a.gvec, a.H, part[grp], 1 + grp, tid);
            if (tid == 0) a.sgate[t] = g;
        }
    }
    // x_perm[p] = x[perm[p] / k]: the total * vec 16-byte vectors spread over all
    // threads of the grid, kGatherInFlight loads in flight per thread
    const int vec = a.H / 8;
    const uint4 *x4 = reinterpret_cast<const uint4 *>(a.x);
    uint4 *xp4 = reinterpret_cast<uint4 *>(a.x_perm);
    const long long nvec = (long long)total * vec, stride = (long long)gridDim.x * kFrontThreads;
    for (long long i0 = (long long)blockIdx.x * kFrontThreads + threadIdx.x; i0 < nvec;
         i0 += stride * kGatherInFlight) {
        uint4 v[kGatherInFlight];
#pragma unroll
        for (int u = 0; u < kGatherInFlight; ++u) {
            const long long i = i0 + u * stride;
            if (i < nvec) {
                const int pr = (int)(i / vec), c = (int)(i - (long long)pr * vec);
                v[u] = __ldg(x4 + (size_t)(sorted[pr] / k) * vec + c);
            }
        }
#pragma unroll
        for (int u = 0; u < kGatherInFlight; ++u) {
            const long long i = i0 + u * stride;
            if (i < nvec) xp4[i] = v[u];
        }
    }
}

template <int V>
cudaError_t launch_v(const FrontArgs &a, cudaStream_t st) {
    static std::atomic<int> attr_set[64];  // per device: opted in to the largest front_smem
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        const cudaError_t e = cudaFuncSetAttribute(front_small_kernel<V>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   kFrontSmemMax);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(1, std::memory_order_release);
    }
    const int grid = std::max(1, std::min(device_sm_count(), a.T * a.k));
    return launch_pdl(front_small_kernel<V>, dim3(grid), dim3(kFrontThreads), front_smem(a.T, a.E, a.k), st, a);
}

}  // namespace

bool front_fits(int T, int E, int k) {
    return (long long)T * k <= kFrontMaxSlots && (long long)T * E <= kFrontMaxLogits &&
           front_smem(T, E, k) <= (size_t)kFrontSmemMax;
}

cudaError_t launch_front(int T, int E, int k, int N, int norm_topk, float topp, int H, const float *logits,
                         const uint16_t *x,
                         const uint16_t *gvec, int32_t *idx, float *w, float *sgate, int32_t *keff, uint8_t *kept,
                         int32_t *n_dropped, int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *slot_pos,
                         uint16_t *x_perm, int32_t *status_block, int32_t *hdone, cudaStream_t st) {
    FrontArgs a{T, E, k, N, norm_topk, H, topp, logits, x, gvec, idx, w, sgate, keff, kept, n_dropped,
                counts, offsets, perm, slot_pos, x_perm, status_block, hdone};
    if (E <= 128) return launch_v<4>(a, st);  // E <= 64 routes lane by lane
    if (E <= 256) return launch_v<8>(a, st);
    if (E <= 512) return launch_v<16>(a, st);
    return launch_v<32>(a, st);
}

}  // namespace moe
