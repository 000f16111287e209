// Router: softmax over the E logits of a token, top-k by logit with the
// kept probabilities renormalised (SpecForge PR #943, "Modifications":
// softmax router with renormalised top-k), plus the sigmoid gate of the
// shared expert.
//
// One block per token: its four warps compute the shared-expert gate
// (shared_gate_group, front.cuh) and the routing is done by its first warp
// (route_token), or, for E <= 64, by the first warp of every 32nd block, one
// token per lane (route_token_lane).  The kernel reads the logits (and x)
// once; it is latency-bound and small next to the expert FFN.
#include "front.cuh"

namespace moe {

namespace {

constexpr int kRouteThreads = kGateThreads;  // one token per block: warp 0 routes, all warps dot

template <int V>  // logits per lane: V * 32 >= E
__global__ void __launch_bounds__(kRouteThreads) route_kernel(int T, int E, int k, int norm_topk,
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
    if (wid == 0) route_token<V>(t, E, k, norm_topk, logits, idx, w, keff, lane);
    if (sgate == nullptr) return;
    const float g = shared_gate_group(t, x, gvec, H, part, 1, threadIdx.x);
    if (threadIdx.x == 0) sgate[t] = g;
}

// E <= kLaneRouteMaxE: block b routes tokens b .. b+31 lane by lane when b is a
// multiple of 32 (route_token_lane), and every block computes its token's
// shared gate.
__global__ void __launch_bounds__(kRouteThreads) route_lane_kernel(int T, int E, int k, int norm_topk,
                                                                   const float *__restrict__ logits,
                                                                   int32_t *__restrict__ idx, float *__restrict__ w,
                                                                   int32_t *__restrict__ keff,
                                                                   const uint16_t *__restrict__ x,
                                                                   const uint16_t *__restrict__ gvec, int H,
                                                                   float *__restrict__ sgate) {
    __shared__ float part[kGateThreads / 32];
    pdl_launch_dependents();
    pdl_wait();
    if ((blockIdx.x & 31) == 0 && threadIdx.x < 32) {
        const int t = blockIdx.x + threadIdx.x;
        if (t < T) {
            route_token_lane<true>(t, E, k, norm_topk, logits + (size_t)t * E, idx, w);
            if (keff != nullptr) keff[t] = k;
        }
    }
    if (sgate == nullptr) return;
    const int t = blockIdx.x;
    const float g = shared_gate_group(t, x, gvec, H, part, 1, threadIdx.x);
    if (threadIdx.x == 0) sgate[t] = g;
}

template <int V>
cudaError_t launch_v(int T, int E, int k, int norm_topk, const float *logits, int32_t *idx, float *w,
                     int32_t *keff, const uint16_t *x, const uint16_t *gvec, int H, float *sgate,
                     cudaStream_t st) {
    return launch_pdl(route_kernel<V>, dim3(T), dim3(kRouteThreads), 0, st, T, E, k, norm_topk, logits, idx, w, keff,
                      x, gvec, H, sgate);
}

}  // namespace

cudaError_t launch_route(int T, int E, int k, int norm_topk, const float *logits, int32_t *idx, float *w,
                         int32_t *keff, const uint16_t *x, const uint16_t *gvec, int H, float *sgate,
                         cudaStream_t st) {
    if (E <= kLaneRouteMaxE)
        return launch_pdl(route_lane_kernel, dim3(T), dim3(kRouteThreads), 0, st, T, E, k, norm_topk, logits, idx, w,
                          keff, x, gvec, H, sgate);
    if (E <= 128) return launch_v<4>(T, E, k, norm_topk, logits, idx, w, keff, x, gvec, H, sgate, st);
    if (E <= 256) return launch_v<8>(T, E, k, norm_topk, logits, idx, w, keff, x, gvec, H, sgate, st);
    if (E <= 512) return launch_v<16>(T, E, k, norm_topk, logits, idx, w, keff, x, gvec, H, sgate, st);
    return launch_v<32>(T, E, k, norm_topk, logits, idx, w, keff, x, gvec, H, sgate, st);
}

}  // namespace moe
