// Router: softmax over the E logits of a token, top-k by logit with the
// kept probabilities renormalised (SpecForge PR #943, "Modifications":
// softmax router with renormalised top-k), plus the sigmoid gate of the
// shared expert.
//
// One block per token; its first warp routes.  Lane l holds the logits of experts l, l+32, ...
// (coalesced 128-byte loads).  Each of the k selection rounds takes a
// lane-local best and a 5-step shuffle argmax ordered by (logit descending,
// expert id ascending), so equal logits keep the lower id, and the winner's
// owner lane masks it out.  The shared-expert gate is a block-wide dot
// product with every load in flight at once.  The kernel
// reads the logits (and x) once; it is latency-bound and small next to the
// expert FFN.
#include <math.h>

#include "moe_internal.cuh"

namespace moe {

namespace {

__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

constexpr int kRouteThreads = 128;  // one token per block: warp 0 routes, all warps dot
constexpr int kGVec = 8;             // 16-byte slices of x and g per thread per pass

template <int V>  // logits per lane: V * 32 >= E
__device__ __forceinline__ void route_token(int t, int E, int k, int norm_topk, const float *__restrict__ logits,
                                            int32_t *__restrict__ idx, float *__restrict__ w,
                                            int32_t *__restrict__ keff, int lane) {
    const float *l = logits + (size_t)t * E;
    float v[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < E) ? __ldg(l + e) : -INFINITY;
    }
    // softmax denominator: max, then sum of exp(l - max) over all E
    float m = v[0];
#pragma unroll
    for (int i = 1; i < V; ++i) m = fmaxf(m, v[i]);
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < V; ++i)
        if (lane + 32 * i < E) s += expf(v[i] - m);
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);

    // k selection rounds; lane j keeps the j-th winner
    uint32_t taken = 0;
    int my_idx = -1;
    float my_logit = -INFINITY;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && better(v[i], e, bv, bi)) {
                bv = v[i];
                bi = e;
            }
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (better(ov, oi, bv, bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == j) {
            my_idx = bi;
            my_logit = bv;
        }
    }
    // probabilities of the kept experts; renormalise with the sum taken in
    // slot order
    float p = (lane < k) ? expf(my_logit - m) / s : 0.f;
    if (norm_topk) {
        float ps = 0.f;
        for (int j = 0; j < k; ++j) ps += __shfl_sync(0xffffffffu, p, j);
        p = p / ps;
    }
    if (lane < k) {
        idx[(size_t)t * k + lane] = my_idx;
        w[(size_t)t * k + lane] = p;
    }
    if (keff != nullptr && lane == 0) keff[t] = k;
}

template <int V>  // logits per lane: V * 32 >= E
__global__ void __launch_bounds__(kRouteThreads) route_kernel(int T, int E, int k, int norm_topk,
                                                              const float *__restrict__ logits,
                                                              int32_t *__restrict__ idx, float *__restrict__ w,
                                                              int32_t *__restrict__ keff,
                                                              const uint16_t *__restrict__ x,
                                                              const uint16_t *__restrict__ gvec, int H,
                                                              float *__restrict__ sgate) {
    pdl_launch_dependents();
    pdl_wait();
    const int t = blockIdx.x;  // one token per block
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (wid == 0) route_token<V>(t, E, k, norm_topk, logits, idx, w, keff, lane);
    if (sgate == nullptr) return;
    // sigmoid(g . x_t): each thread loads up to kGVec 16-byte slices of x_t and
    // of g, all in flight at once, then a block reduction.
    __shared__ float part[kRouteThreads / 32];
    const int nv = H / 8;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
    const uint4 *gr = reinterpret_cast<const uint4 *>(gvec);
    float z = 0.f;
    for (int c0 = threadIdx.x; c0 < nv; c0 += kRouteThreads * kGVec) {
        uint4 a[kGVec], g[kGVec];
#pragma unroll
        for (int q = 0; q < kGVec; ++q) {
            const int c = c0 + q * kRouteThreads;
            a[q] = c < nv ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
            g[q] = c < nv ? __ldg(gr + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int q = 0; q < kGVec; ++q) {
            const uint32_t av[4] = {a[q].x, a[q].y, a[q].z, a[q].w}, bv[4] = {g[q].x, g[q].y, g[q].z, g[q].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                z = fmaf(bf16_bits_to_f32((uint16_t)(av[h] & 0xffffu)), bf16_bits_to_f32((uint16_t)(bv[h] & 0xffffu)),
                         z);
                z = fmaf(bf16_bits_to_f32((uint16_t)(av[h] >> 16)), bf16_bits_to_f32((uint16_t)(bv[h] >> 16)), z);
            }
        }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane == 0) part[wid] = z;
    __syncthreads();
    if (threadIdx.x == 0) {
        float zz = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kRouteThreads / 32; ++w2) zz += part[w2];
        sgate[t] = 1.f / (1.f + expf(-zz));
    }
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
    if (E <= 32) return launch_v<1>(T, E, k, norm_topk, logits, idx, w, keff, x, gvec, H, sgate, st);
    if (E <= 64) return launch_v<2>(T, E, k, norm_topk, logits, idx, w, keff, x, gvec, H, sgate, st);
    if (E <= 128) return launch_v<4>(T, E, k, norm_topk, logits, idx, w, keff, x, gvec, H, sgate, st);
    if (E <= 256) return launch_v<8>(T, E, k, norm_topk, logits, idx, w, keff, x, gvec, H, sgate, st);
    if (E <= 512) return launch_v<16>(T, E, k, norm_topk, logits, idx, w, keff, x, gvec, H, sgate, st);
    return launch_v<32>(T, E, k, norm_topk, logits, idx, w, keff, x, gvec, H, sgate, st);
}

}  // namespace moe
