// Router: softmax over the E logits of a token, top-k by logit with the
// kept probabilities renormalised (SpecForge PR #943, "Modifications":
// softmax router with renormalised top-k), the optional per-token top-p trim
// (colibri issue_budget.md, "Relationship to existing features"), plus the
// sigmoid gate of the shared expert.
//
// route_kernel<V>: one block per token; its first warp routes (route_token,
// front.cuh) while the next four compute the shared-expert gate
// (shared_gate_group), side by side.  route_lane_kernel (32 < E <= 64):
// separate blocks route 32 tokens lane by lane and compute the gates.  Both read the logits (and
// x) once; they are latency-bound and small next to the expert FFN.
#include <algorithm>

#include "front.cuh"

namespace moe {

namespace {

constexpr int kRouteThreads = 32 + kGateThreads;  // one token per block: warp 0 routes, warps 1.. dot

// V >= 16 wants more registers than the default occupancy target leaves
// (that build spilled); the narrower routers keep a high block occupancy.
template <int V>  // logits per lane: V * 32 >= E
__global__ void __launch_bounds__(kRouteThreads, V >= 16 ? 1 : 8) route_kernel(int T, int E, int k, int norm_topk, float topp,
                                                              const float *__restrict__ logits,
                                                              int32_t *__restrict__ idx, float *__restrict__ w,
                                                              int32_t *__restrict__ keff,
                                                              const uint16_t *__restrict__ x,
                                                              const uint16_t *__restrict__ gvec, int H,
                                                              float *__restrict__ sgate) {
    __shared__ float part[kGateThreads / 32];
    pdl_launch_dependents();
    pdl_wait();
    const int t = blockIdx.x;  // one token per block
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (wid == 0) {
        route_token<V>(t, E, k, norm_topk, topp, logits, idx, w, keff, lane);
        return;
    }
    if (sgate == nullptr) return;
    const int tid = threadIdx.x - 32;
    const float g = shared_gate_group(t, x, gvec, H, part, 1, tid);
    if (tid == 0) sgate[t] = g;
}

// 32 < E <= kLaneRouteMaxE: the first ceil(T / 32) blocks route 32 tokens each, one
// token per lane of their first warp (route_token_lane), from the tokens'
// logits staged in shared memory; the remaining T blocks (with a shared
// expert) compute one token's shared gate each.  Routing and gate blocks run
// side by side instead of one after the other.
__global__ void __launch_bounds__(kGateThreads) route_lane_kernel(int T, int E, int k, int norm_topk, float topp,
                                                                   const float *__restrict__ logits,
                                                                   int32_t *__restrict__ idx, float *__restrict__ w,
                                                                   int32_t *__restrict__ keff,
                                                                   const uint16_t *__restrict__ x,
                                                                   const uint16_t *__restrict__ gvec, int H,
                                                                   float *__restrict__ sgate) {
    __shared__ float part[kGateThreads / 32];
    __shared__ float lg[32 * (kLaneRouteMaxE + 1)];  // 32 rows of logits, odd stride: no bank conflicts
    pdl_launch_dependents();
    pdl_wait();
    const int nrt = (T + 31) / 32;  // routing blocks
    if ((int)blockIdx.x < nrt) {
        if (threadIdx.x >= 32) return;
        const int lane = threadIdx.x, t0 = blockIdx.x * 32, n = min(32, T - t0), ls = E | 1;
        for (int i = lane; i < n * E; i += 32) {  // coalesced copy of the 32 tokens' rows
            const int r = i / E;
            lg[r * ls + (i - r * E)] = __ldg(logits + (size_t)t0 * E + i);
        }
        __syncwarp();
        if (lane < n) {
            const int c = route_token_lane<false>(t0 + lane, E, k, norm_topk, topp, lg + lane * ls, idx, w);
            if (keff != nullptr) keff[t0 + lane] = c;
        }
        return;
    }
    const int t = blockIdx.x - nrt;
    const float g = shared_gate_group(t, x, gvec, H, part, 1, threadIdx.x);
    if (threadIdx.x == 0) sgate[t] = g;
}

template <int V>
cudaError_t launch_v(int T, int E, int k, int norm_topk, float topp, const float *logits, int32_t *idx, float *w,
                     int32_t *keff, const uint16_t *x, const uint16_t *gvec, int H, float *sgate,
                     cudaStream_t st) {
    return launch_pdl(route_kernel<V>, dim3(T), dim3(kRouteThreads), 0, st, T, E, k, norm_topk, topp, logits, idx, w,
                      keff, x, gvec, H, sgate);
}

}  // namespace

namespace {
// One pass over the logits (checked library only): a block that sees a NaN or
// an infinity sets the status bit once.
__global__ void __launch_bounds__(256) check_logits_kernel(long long n, const float *__restrict__ logits,
                                                         int32_t *__restrict__ status) {
    pdl_wait();
    bool bad = false;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        bad |= !isfinite(__ldg(logits + i));
    pdl_launch_dependents();
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(status, MOE_STATUS_NONFINITE);
}
}  // namespace

cudaError_t launch_check_logits(long long n, const float *logits, int32_t *status, cudaStream_t st) {
    const long long blocks = std::min<long long>((n + 255) / 256, 1184);
    return launch_pdl(check_logits_kernel, dim3((unsigned)std::max<long long>(blocks, 1)), dim3(256), 0, st, n,
                      logits, status);
}

cudaError_t launch_route(int T, int E, int k, int norm_topk, float topp, const float *logits, int32_t *idx, float *w,
                         int32_t *keff, const uint16_t *x, const uint16_t *gvec, int H, float *sgate,
                         cudaStream_t st) {
    if (lane_routed(E))
        return launch_pdl(route_lane_kernel, dim3((T + 31) / 32 + (sgate != nullptr ? T : 0)), dim3(kGateThreads), 0,
                          st, T, E, k, norm_topk, topp, logits, idx, w, keff, x, gvec, H, sgate);
    if (E <= 128) return launch_v<4>(T, E, k, norm_topk, topp, logits, idx, w, keff, x, gvec, H, sgate, st);
    if (E <= 256) return launch_v<8>(T, E, k, norm_topk, topp, logits, idx, w, keff, x, gvec, H, sgate, st);
    if (E <= 512) return launch_v<16>(T, E, k, norm_topk, topp, logits, idx, w, keff, x, gvec, H, sgate, st);
    return launch_v<32>(T, E, k, norm_topk, topp, logits, idx, w, keff, x, gvec, H, sgate, st);
}

}  // namespace moe
