// Device building blocks of the layer's front end -- routing, the shared
// expert's gate, the stable sort of slots by expert and the expert budget --
// shared by the stand-alone stage kernels (router.cu, budget.cu) and the
// fused small-batch front-end kernel (front.cu), so that every path
// computes the same bits.
#pragma once

#include <math.h>

#include "moe_internal.cuh"

namespace moe {

// ---------------------------------------------------------------- routing --
// Softmax over the E logits of a token, top-k by logit with the kept
// probabilities renormalised (SpecForge PR #943, "Modifications": softmax
// router with renormalised top-k).  One warp per token; each lane holds V
// logits as order-preserving integer keys (-0 and +0 share one; a taken or
// absent expert holds 0, below every logit's key).  For E > 128 a multiple
// of 4, with 16-byte aligned rows (kVec), lane l holds experts 128c + 4l + q
// (one 16-byte load per c), else experts l + 32i; either way a lane's slots
// run in ascending expert order.  Each of the k selection rounds takes the lane's
// best key (a tree over its V keys; equal keys keep the lower slot, so the
// lower expert), then two warp reductions: the largest key, and the lowest
// expert id among the lanes holding it -- so equal logits keep the lower id.
// The winner's lane clears its key; lane j keeps the j-th winner and its key.
// The logits come from global memory (kGlobal, read-only path) or from
// shared memory; idx / w may point to global or shared memory; keff (may be
// null) receives the kept slot count, which the function also returns.
//
// Top-p trim (colibri issue_budget.md, "Relationship to existing features":
// TOPP trims a position's top-K to its top-p mass, before the budget), for
// 0 < topp < 1: slot 0 stays; slot j > 0 stays while the weights of slots
// 0..j-1 (after the norm_topk renormalisation), added in slot order, are
// below topp.  The dropped tail becomes (idx -1, w 0), and with norm_topk
// the kept weights are divided by their sum in slot order.
__device__ __forceinline__ uint32_t float_order_key(float v) {
    const uint32_t b = v == 0.f ? 0u : __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float order_key_float(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

template <int V, bool kGlobal, bool kVec>
__device__ __forceinline__ int route_token_impl(int t, int E, int k, int norm_topk, float topp,
                                                const float *__restrict__ logits, int32_t *idx, float *w,
                                                int32_t *keff, int lane) {
    const float *l = logits + (size_t)t * E;
    // expert of slot i of this lane
    auto expert = [&](int i) { return kVec ? 128 * (i >> 2) + 4 * lane + (i & 3) : lane + 32 * i; };
    // only the keys stay live: a logit comes back from its key exactly (up to
    // the sign of a zero, which neither the max nor exp sees), so the V
    // logits need no registers of their own
    uint32_t key[V];
    if constexpr (kVec) {
#pragma unroll
        for (int c = 0; c < V / 4; ++c) {
            const int e0 = 128 * c + 4 * lane;  // E % 4 == 0: all four present or none
            float4 q = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            if (e0 < E) q = kGlobal ? __ldg(reinterpret_cast<const float4 *>(l + e0)) : *reinterpret_cast<const float4 *>(l + e0);
            const bool in = e0 < E;
            key[4 * c] = in ? float_order_key(q.x) : 0u;
            key[4 * c + 1] = in ? float_order_key(q.y) : 0u;
            key[4 * c + 2] = in ? float_order_key(q.z) : 0u;
            key[4 * c + 3] = in ? float_order_key(q.w) : 0u;
        }
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int e = expert(i);
            key[i] = e < E ? float_order_key(kGlobal ? __ldg(l + e) : l[e]) : 0u;
        }
    }
    // softmax denominator: the largest logit, then sum of exp(l - max) over all E
    uint32_t km = key[0];
#pragma unroll
    for (int i = 1; i < V; ++i) km = max(km, key[i]);
    const float m = order_key_float(__reduce_max_sync(0xffffffffu, km));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < V; ++i)
        if (expert(i) < E) s += expf(order_key_float(key[i]) - m);
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);

    // k selection rounds; lane j keeps the j-th winner
    int my_idx = -1;
    uint32_t my_key = 0u;
    for (int j = 0; j < k; ++j) {
        uint32_t tk[V];
        int ti[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            tk[i] = key[i];
            ti[i] = i;
        }
#pragma unroll
        for (int d = 1; d < V; d *= 2)
#pragma unroll
            for (int i = 0; i + d < V; i += 2 * d)
                if (tk[i + d] > tk[i]) {  // strict: the lower slot keeps a tie
                    tk[i] = tk[i + d];
                    ti[i] = ti[i + d];
                }
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, tk[0]);
        const int win = (int)__reduce_min_sync(0xffffffffu, tk[0] == kmax ? (uint32_t)expert(ti[0]) : 0xffffffffu);
        const int owner = kVec ? (win & 127) >> 2 : win & 31;
        const int wslot = kVec ? 4 * (win >> 7) + (win & 3) : win >> 5;
        if (owner == lane) {
#pragma unroll
            for (int i = 0; i < V; ++i)
                if (i == wslot) key[i] = 0u;
        }
        if (lane == j) {
            my_idx = win;
            my_key = kmax;
        }
    }
    // probabilities of the kept experts (the logit back from its key: exact up
    // to the sign of a zero, which exp does not see); renormalise with the sum
    // taken in slot order
    float p = (lane < k) ? expf(order_key_float(my_key) - m) / s : 0.f;
    if (norm_topk) {
        float ps = 0.f;
        for (int j = 0; j < k; ++j) ps += __shfl_sync(0xffffffffu, p, j);
        p = p / ps;
    }
    int c = k;  // kept slots
    if (topp > 0.f && topp < 1.f) {
        float mass = 0.f;  // the same in every lane
        for (int j = 0; j < k; ++j) {
            const float pj = __shfl_sync(0xffffffffu, p, j);
            if (j > 0 && mass >= topp) {
                c = j;
                break;
            }
            mass += pj;
        }
        if (norm_topk && c < k) {
            float s2 = 0.f;
            for (int j = 0; j < c; ++j) s2 += __shfl_sync(0xffffffffu, p, j);
            p = p / s2;
        }
    }
    if (lane < k) {
        idx[(size_t)t * k + lane] = lane < c ? my_idx : -1;
        w[(size_t)t * k + lane] = lane < c ? p : 0.f;
    }
    if (keff != nullptr && lane == 0) keff[t] = c;
    return c;
}

template <int V, bool kGlobal = true>  // logits per lane: V * 32 >= E, V a power of two >= 4
__device__ __forceinline__ int route_token(int t, int E, int k, int norm_topk, float topp,
                                           const float *__restrict__ logits, int32_t *idx, float *w, int32_t *keff,
                                           int lane) {
    static_assert(V >= 4 && (V & (V - 1)) == 0, "V: a power of two >= 4");
    if (V >= 8 && (E & 3) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15u) == 0)  // measured: no gain at V = 4
        return route_token_impl<V, kGlobal, true>(t, E, k, norm_topk, topp, logits, idx, w, keff, lane);
    return route_token_impl<V, kGlobal, false>(t, E, k, norm_topk, topp, logits, idx, w, keff, lane);
}

// One token per thread, for 32 < E <= kLaneRouteMaxE: the same decisions as
// route_token, with every sum taken in expert order (max, then
// sum_e exp(l_e - max), then k rounds of first-maximum selection over the
// untaken experts, then the renormalising sum in slot order, then the top-p
// trim).  A warp routes 32 tokens at once with no shuffles.  `l` is the
// token's row of logits (global memory when kGlobal, else shared memory).
// Returns the kept slot count.  Used for 32 < E <= 64: at most 32 experts one
// logit per lane of the warp router is faster (measured, the 16-expert drafter
// layer), above 64 the warp router is.
constexpr int kLaneRouteMinE = 33;
constexpr int kLaneRouteMaxE = 64;
__host__ __device__ inline bool lane_routed(int E) { return E >= kLaneRouteMinE && E <= kLaneRouteMaxE; }

template <bool kGlobal>
__device__ __forceinline__ int route_token_lane(int t, int E, int k, int norm_topk, float topp, const float *l,
                                                int32_t *idx, float *w) {
    auto L = [&](int e) { return kGlobal ? __ldg(l + e) : l[e]; };
    float m = L(0);
    for (int e = 1; e < E; ++e) {
        const float v = L(e);
        if (v > m) m = v;
    }
    float s = 0.f;
    for (int e = 0; e < E; ++e) s += expf(L(e) - m);
    uint64_t taken = 0;
    float ps = 0.f;
    for (int j = 0; j < k; ++j) {
        int best = -1;
        float bv = 0.f;
        for (int e = 0; e < E; ++e) {
            if ((taken >> e) & 1ull) continue;
            const float v = L(e);
            if (best < 0 || v > bv) {  // strict: equal logits keep the lower id
                best = e;
                bv = v;
            }
        }
        taken |= 1ull << best;
        const float p = expf(bv - m) / s;
        idx[(size_t)t * k + j] = best;
        w[(size_t)t * k + j] = p;
        ps += p;
    }
    if (norm_topk)
        for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = w[(size_t)t * k + j] / ps;
    int c = k;  // kept slots
    if (topp > 0.f && topp < 1.f) {
        float *tw = w + (size_t)t * k;
        float mass = 0.f;
        for (int j = 0; j < k; ++j) {
            if (j > 0 && mass >= topp) {
                c = j;
                break;
            }
            mass += tw[j];
        }
        if (norm_topk && c < k) {
            float s2 = 0.f;
            for (int j = 0; j < c; ++j) s2 += tw[j];
            for (int j = 0; j < c; ++j) tw[j] = tw[j] / s2;
        }
        for (int j = c; j < k; ++j) {
            idx[(size_t)t * k + j] = -1;
            tw[j] = 0.f;
        }
    }
    return c;
}

// ------------------------------------------------------------ shared gate --
// sigmoid(g . x_t) (SpecForge PR #943, "Modifications": sigmoid-gated
// shared expert), computed by a group of kGateThreads threads: each loads up
// to kGateVec 16-byte slices of x_t and of g, all in flight at once, then a
// warp reduction and the kGateThreads / 32 warp partials in order.  `tid`
// is the thread's index in the group, `part` the group's kGateThreads / 32
// floats of shared memory, `bar` a named barrier id the group owns.  The
// result is valid in group thread 0.
constexpr int kGateThreads = 128;
constexpr int kGateVec = 8;

__device__ __forceinline__ float shared_gate_group(int t, const uint16_t *__restrict__ x,
                                                   const uint16_t *__restrict__ gvec, int H, float *part, int bar,
                                                   int tid) {
    const int lane = tid & 31, wid = tid >> 5;
    const int nv = H / 8;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
    const uint4 *gr = reinterpret_cast<const uint4 *>(gvec);
    float z = 0.f;
    for (int c0 = tid; c0 < nv; c0 += kGateThreads * kGateVec) {
        uint4 a[kGateVec], g[kGateVec];
#pragma unroll
        for (int q = 0; q < kGateVec; ++q) {
            const int c = c0 + q * kGateThreads;
            a[q] = c < nv ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
            g[q] = c < nv ? __ldg(gr + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int q = 0; q < kGateVec; ++q) {
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
    asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(kGateThreads) : "memory");
    float r = 0.f;
    if (tid == 0) {
        float zz = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kGateThreads / 32; ++w2) zz += part[w2];
        r = 1.f / (1.f + expf(-zz));
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(kGateThreads) : "memory");  // part reusable afterwards
    return r;
}

// ------------------------------------------------- block sort by expert --
// Exclusive prefix sum of one value per thread over a 1024-thread block.
__device__ __forceinline__ int block_exclusive_scan_1024(int v, int *warp_sums) {
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
    const int r = incl - v + (wid ? warp_sums[wid - 1] : 0);
    __syncthreads();  // warp_sums reusable afterwards
    return r;
}

// Per-warp count columns for a block sort over E experts: [W][E] ints fit in 32 KB.
__host__ __device__ inline int sort_warps(int E) { return E <= 256 ? 32 : (E <= 512 ? 16 : 8); }
// Warps a sort of n slots uses: one 32-slot pass each where sort_warps allows
// (fewer count columns to zero and scan for small n).
__device__ __forceinline__ int sort_warps_for(int n, int E) { return max(1, min(sort_warps(E), (n + 31) >> 5)); }

// Stable counting sort of the slots 0..n-1 by expert inside one 1024-thread
// block: key(s) is the slot's expert in [0, E), or -1 to leave it out.  W
// warps each take a contiguous chunk of slots; __match_any_sync groups the
// lanes with the same expert, and a lane's position inside its group is the
// number of lower lanes, so the order inside an expert is ascending slot id.
// Out (shared memory): sorted[pos] = slot, off[e] = first position of expert
// e, off[E] = number of sorted slots.  hist: W * E ints; warp_sums: 32 ints.
// The result does not depend on W.
template <class Key>
__device__ __forceinline__ void block_sort_by_expert(int n, int E, int W, Key key, int *hist, int *off, int *sorted,
                                                     int *warp_sums) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunk = (n + W - 1) / W;
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int s_begin = warp * chunk, s_end = min(n, s_begin + chunk);
    if (warp < W) {
        for (int s0 = s_begin; s0 < s_end; s0 += 32) {
            const int s = s0 + lane;
            const int kk = s < s_end ? key(s) : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, kk);
            if (kk >= 0 && lane == __ffs(peers) - 1) hist[warp * E + kk] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();
    const int e = threadIdx.x;  // blockDim.x == 1024 >= E
    int c = 0;
    if (e < E)
#pragma unroll 8
        for (int w = 0; w < W; ++w) c += hist[w * E + e];
    const int excl = block_exclusive_scan_1024(c, warp_sums);
    if (e < E) {
        off[e] = excl;
        if (e == E - 1) off[E] = excl + c;
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
            const int kk = s < s_end ? key(s) : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, kk);
            if (kk >= 0) sorted[base[kk] + __popc(peers & ((1u << lane) - 1u))] = s;
            __syncwarp();
            if (kk >= 0 && lane == 31 - __clz(peers)) base[kk] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------- budget --
// Expert budget (colibri issue_budget.md, "EXPERT_BUDGET", section "How it
// works", steps 1-5) inside one 1024-thread block, on a routing held in
// shared memory (idx_s, w_s: T * k slots; a token's valid slots first, then
// idx -1 where a top-p trim dropped them).
//   step 1: agg[e] = the weights routed to e summed in token-then-slot order
//           (the slots are sorted by expert first, so each expert's thread
//           sums exactly that sequence);
//   step 2-3: the union is every expert with a slot; each union expert's
//           rank is the number of union experts ahead of it in (agg
//           descending, id ascending); the first N are kept;
//   step 4: each token's kept slots move to the front in order, the others
//           become (-1, 0); a token that lost some but not all of its valid
//           slots renormalises;
//   step 5: n_dropped = union size - N.
// A budget of 0, or a union of at most N experts, changes nothing (keff =
// the token's valid slots, kept = the union).  Out (shared memory): idx_s / w_s compacted, keff_s[T],
// keep[E], *nd_s; off / sorted keep the sort of all slots by expert.
// Scratch: hist (sort_warps(E) * E), off (E + 1), sorted (T * k), agg (E),
// pres (E), warp_sums (32).  The ranks are counted by up to blockDim / E
// threads per expert, each over a range of the others (integer sums: the
// result does not depend on the split).
__device__ __forceinline__ void budget_block(int T, int E, int k, int N, int norm_topk, int32_t *idx_s, float *w_s,
                                             int32_t *keff_s, uint8_t *keep, int *nd_s, int *hist, int *off,
                                             int *sorted, float *agg, uint8_t *pres, int *warp_sums) {
    const int Tk = T * k;
    block_sort_by_expert(
        Tk, E, sort_warps_for(Tk, E),
        [=](int s) {
            const int x = idx_s[s];
            return (x >= 0 && x < E) ? x : -1;
        },
        hist, off, sorted, warp_sums);
    const int e = threadIdx.x;
    int *rank = hist;  // free once the sort is done
    int my_present = 0;
    if (e < E) {
        float a = 0.f;
        for (int p = off[e]; p < off[e + 1]; ++p) a += w_s[sorted[p]];
        agg[e] = a;
        my_present = off[e + 1] > off[e];
        pres[e] = (uint8_t)my_present;
        rank[e] = 0;
    }
    const int nu = __syncthreads_count(my_present);
    const bool active = N > 0 && nu > N;  // the same in every thread
    if (active) {
        const int parts = max(1, min(E, (int)blockDim.x / E));
        if ((int)threadIdx.x < parts * E) {
            const int re = threadIdx.x % E, part = threadIdx.x / E;
            if (pres[re]) {
                const float a = agg[re];
                int r = 0;
                const int o1 = (part + 1) * E / parts;
                for (int o = part * E / parts; o < o1; ++o) r += pres[o] && (agg[o] > a || (agg[o] == a && o < re));
                if (r) atomicAdd(rank + re, r);
            }
        }
        __syncthreads();
    }
    if (e < E) keep[e] = pres[e] && (!active || rank[e] < N);
    __syncthreads();
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
        int32_t *ti = idx_s + (size_t)t * k;
        float *tw = w_s + (size_t)t * k;
        int valid = 0;
        for (int j = 0; j < k; ++j) valid += ti[j] >= 0;
        int c = valid;
        if (active) {
            c = 0;
            for (int j = 0; j < k; ++j) {
                const int ej = ti[j];
                if (ej >= 0 && ej < E && keep[ej]) {
                    const float wj = tw[j];
                    ti[c] = ej;
                    tw[c] = wj;
                    ++c;
                }
            }
            for (int j = c; j < k; ++j) {
                ti[j] = -1;
                tw[j] = 0.f;
            }
            if (norm_topk && c > 0 && c < valid) {
                float s = 0.f;
                for (int j = 0; j < c; ++j) s += tw[j];
                for (int j = 0; j < c; ++j) tw[j] = tw[j] / s;
            }
        }
        keff_s[t] = c;
    }
    if (threadIdx.x == 0) *nd_s = active ? nu - N : 0;
    __syncthreads();
}

// The dispatch order from the budget's own sort.  budget_block leaves off /
// sorted holding every slot by expert, ascending slot id inside an expert --
// that is, ascending token, as a token holds an expert at most once.  A kept
// expert keeps its slots in that token order, each renamed to the slot the
// expert now holds in its token's compacted list; a dropped expert's slots
// go.  That is the order block_sort_by_expert gives the kept slots, here
// without a second sort.  Positions only move down, and each pass reads its
// 1024 positions before any is written.  Scratch: hist (E + 1 ints),
// warp_sums (32).
__device__ __forceinline__ void regroup_kept(int E, int k, const int32_t *idx_s, const int32_t *keff_s,
                                             const uint8_t *keep, int *off, int *sorted, int *hist, int *warp_sums) {
    const int e = threadIdx.x;
    const int cnt = (e < E && keep[e]) ? off[e + 1] - off[e] : 0;
    const int nofs = block_exclusive_scan_1024(cnt, warp_sums);
    if (e < E) {
        hist[e] = nofs;
        if (e == E - 1) hist[E] = nofs + cnt;
    }
    __syncthreads();
    const int total = off[E];
    for (int p0 = 0; p0 < total; p0 += blockDim.x) {
        const int p = p0 + threadIdx.x;
        int np = -1, ns = 0;
        if (p < total) {
            int lo = 0, hi = E - 1;  // the expert whose range holds p
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (off[mid] <= p)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            if (keep[lo]) {
                const int t = sorted[p] / k;
                const int32_t *ti = idx_s + (size_t)t * k;
                int j = 0;
                while (j < keff_s[t] - 1 && ti[j] != lo) ++j;
                np = hist[lo] + (p - off[lo]);
                ns = t * k + j;
            }
        }
        __syncthreads();
        if (np >= 0) sorted[np] = ns;
        __syncthreads();
    }
    for (int i = threadIdx.x; i <= E; i += blockDim.x) off[i] = hist[i];
    __syncthreads();
}

}  // namespace moe
