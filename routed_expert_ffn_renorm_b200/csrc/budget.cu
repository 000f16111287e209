// Expert budget (colibri issue_budget.md, "EXPERT_BUDGET", section "How it
// works", steps 1-5): cap the number of distinct experts the batch uses at
// N, keeping the experts with the highest aggregate gate weight, dropping
// the rest from every token and renormalising what survives.
//
// Batches of up to kSmallSlots slots: one block does all of it in shared
// memory (budget_block, front.cuh), the aggregates summed in exactly
// token-then-slot order.  Larger batches take two kernels:
// kernel 1 (one block per chunk of kChunk tokens): thread e sums, in token
// then slot order, the weights routed to expert e inside the chunk, and
// counts the slots; chunk partials go to the workspace.
// Kernel 2 (one block): agg[e] = chunk partials summed in chunk order, the
// union is every expert with a routed slot, each union expert's rank is the
// number of union experts ahead of it in (agg descending, id ascending),
// the first N are kept; then one thread per token compacts its slots in
// order and renormalises when it lost one.  Slots with idx -1 (dropped by a
// top-p trim) take no part; keff counts a token's valid slots.
// Every sum has a fixed order, so the result is deterministic; the
// two-kernel path rounds the aggregates chunk by chunk.
#include <atomic>

#include "front.cuh"

namespace moe {

namespace {

constexpr int kChunk = 256;        // tokens per partial-sum chunk
constexpr int kSmallSlots = 8192;  // T*k up to this: one block in shared memory

// Shared memory of budget_small_kernel.
size_t budget_small_smem(int T, int E, int k) {
    const size_t Tk = (size_t)T * k;
    return Tk * 12 + (size_t)T * 4 + (size_t)sort_warps(E) * E * 4 + (size_t)(E + 1) * 4 + (size_t)E * 6 + 16;
}

__global__ void __launch_bounds__(1024) budget_small_kernel(int T, int E, int k, int N, int norm_topk,
                                                            int32_t *__restrict__ idx, float *__restrict__ w,
                                                            int32_t *__restrict__ keff, uint8_t *__restrict__ kept,
                                                            int32_t *__restrict__ n_dropped) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int Tk = T * k, W = sort_warps(E);
    int32_t *idx_s = reinterpret_cast<int32_t *>(sm);
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
    pdl_launch_dependents();
    pdl_wait();
    for (int s = threadIdx.x; s < Tk; s += blockDim.x) {
        idx_s[s] = idx[s];
        w_s[s] = w[s];
    }
    __syncthreads();
    budget_block(T, E, k, N, norm_topk, idx_s, w_s, keff_s, keep, &nd_s, hist, off, sorted, agg, pres, warp_sums);
    for (int s = threadIdx.x; s < Tk; s += blockDim.x) {
        idx[s] = idx_s[s];
        w[s] = w_s[s];
    }
    for (int t = threadIdx.x; t < T; t += blockDim.x) keff[t] = keff_s[t];
    for (int e = threadIdx.x; e < E; e += blockDim.x) kept[e] = keep[e];
    if (threadIdx.x == 0) *n_dropped = nd_s;
}

__global__ void __launch_bounds__(256) budget_partial_kernel(int T, int E, int k, const int32_t *__restrict__ idx,
                                                             const float *__restrict__ w,
                                                             float *__restrict__ part_agg,
                                                             int32_t *__restrict__ part_cnt) {
    pdl_launch_dependents();
    pdl_wait();
    const int c = blockIdx.x;
    const int t0 = c * kChunk, t1 = min(T, t0 + kChunk);
    const size_t s0 = (size_t)t0 * k, s1 = (size_t)t1 * k;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float a = 0.f;
        int n = 0;
        for (size_t s = s0; s < s1; ++s) {  // every thread reads the same slot: broadcast
            if (__ldg(idx + s) == e) {
                a += __ldg(w + s);
                ++n;
            }
        }
        part_agg[(size_t)c * E + e] = a;
        part_cnt[(size_t)c * E + e] = n;
    }
}

__global__ void __launch_bounds__(1024) budget_select_kernel(int T, int E, int k, int N, int norm_topk,
                                                             int nchunks, int32_t *__restrict__ idx,
                                                             float *__restrict__ w, int32_t *__restrict__ keff,
                                                             uint8_t *__restrict__ kept,
                                                             int32_t *__restrict__ n_dropped,
                                                             const float *__restrict__ part_agg,
                                                             const int32_t *__restrict__ part_cnt) {
    __shared__ float agg[kMaxExperts];
    __shared__ uint8_t present[kMaxExperts];
    __shared__ uint8_t keep[kMaxExperts];
    __shared__ int nu_s;
    pdl_launch_dependents();
    pdl_wait();
    if (threadIdx.x == 0) nu_s = 0;
    __syncthreads();
    int my_present = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float a = 0.f;
        int n = 0;
        for (int c = 0; c < nchunks; ++c) {
            a += part_agg[(size_t)c * E + e];
            n += part_cnt[(size_t)c * E + e];
        }
        agg[e] = a;
        present[e] = n > 0;
        my_present += n > 0;
    }
    atomicAdd(&nu_s, my_present);  // integer: order-independent
    __syncthreads();
    const int nu = nu_s;
    const bool active = N > 0 && nu > N;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        uint8_t kp = present[e];
        if (active && kp) {
            const float a = agg[e];
            int rank = 0;
            for (int o = 0; o < E; ++o)
                rank += present[o] && (agg[o] > a || (agg[o] == a && o < e));
            kp = rank < N;
        }
        keep[e] = kp;
        kept[e] = kp;
    }
    __syncthreads();
    if (threadIdx.x == 0) *n_dropped = active ? nu - N : 0;
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
        int32_t *ti = idx + (size_t)t * k;
        float *tw = w + (size_t)t * k;
        int valid = 0;  // slots a top-p trim left (all k without one)
        for (int j = 0; j < k; ++j) valid += ti[j] >= 0;
        int c = valid;
        if (active) {
            c = 0;
            for (int j = 0; j < k; ++j) {
                const int e = ti[j];
                if (e >= 0 && e < E && keep[e]) {
                    const float wj = tw[j];
                    ti[c] = e;
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
        keff[t] = c;
    }
}

}  // namespace

int budget_chunks(int T) { return (T + kChunk - 1) / kChunk; }

cudaError_t launch_budget(int T, int E, int k, int N, int norm_topk, int32_t *idx, float *w, int32_t *keff,
                          uint8_t *kept, int32_t *n_dropped, float *part_agg, int32_t *part_cnt,
                          cudaStream_t st) {
    if ((long long)T * k <= kSmallSlots) {
        static std::atomic<int> attr_set[64];  // per device: opted in to more than 48 KB
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        if (!attr_set[dev].load(std::memory_order_acquire)) {
            const cudaError_t e = cudaFuncSetAttribute(budget_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)budget_small_smem(kSmallSlots, kMaxExperts, 1));
            if (e != cudaSuccess) return e;
            attr_set[dev].store(1, std::memory_order_release);
        }
        return launch_pdl(budget_small_kernel, dim3(1), dim3(1024), budget_small_smem(T, E, k), st, T, E, k, N,
                          norm_topk, idx, w, keff, kept, n_dropped);
    }
    const int nchunks = budget_chunks(T);
    cudaError_t e = launch_pdl(budget_partial_kernel, dim3(nchunks), dim3(256), 0, st, T, E, k, idx, w, part_agg,
                               part_cnt);
    if (e != cudaSuccess) return e;
    return launch_pdl(budget_select_kernel, dim3(1), dim3(1024), 0, st, T, E, k, N, norm_topk, nchunks, idx, w, keff,
                      kept, n_dropped, part_agg, part_cnt);
}

}  // namespace moe
