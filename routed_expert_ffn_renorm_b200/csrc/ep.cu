// Expert parallelism: the experts of a layer split over W ranks (GPUs), rank
// r holding experts [r * epr, (r + 1) * epr).  The MegaMoE designs of
// DeepGEMM PR #381 and DeepGEMM fork PR #5 send each token's routed rows to
// the ranks that hold its experts and bring the weighted expert outputs
// back (dispatch and combine over NVLink).  Here the exchange itself is the
// caller's collective (NCCL all-to-all through torch.distributed); these
// kernels are the per-rank steps around it:
//   ep_rank_ids: the destination rank of every kept slot (its expert's owner),
//     which moe_dispatch then groups the slots by, gathering the rows to send;
//   ep_pack: for the rows in that send order, the expert id at the destination
//     (local to its owner) and the routing weight;
//   ep_unpack: the returned weighted rows, in the same order, to their
//     token-ordered ybuf rows (t * (k + 1) + j), which moe_combine adds.
#include "moe_internal.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(256) ep_rank_ids_kernel(int n, int epr, const int32_t *__restrict__ idx,
                                                          int32_t *__restrict__ rank_idx) {
    pdl_launch_dependents();
    pdl_wait();
    for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < n; s += gridDim.x * blockDim.x) {
        const int e = idx[s];
        rank_idx[s] = e < 0 ? -1 : e / epr;
    }
}

__global__ void __launch_bounds__(256) ep_pack_kernel(const int32_t *__restrict__ n_dev, int epr,
                                                      const int32_t *__restrict__ perm, const int32_t *__restrict__ idx,
                                                      const float *__restrict__ w, int32_t *__restrict__ local_idx,
                                                      float *__restrict__ local_w) {
    pdl_launch_dependents();
    pdl_wait();
    const int n = *n_dev;
    for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < n; p += gridDim.x * blockDim.x) {
        const int s = perm[p];
        local_idx[p] = idx[s] % epr;
        local_w[p] = w[s];
    }
}

// One thread per 16-byte vector of a returned row.
__global__ void __launch_bounds__(256) ep_unpack_kernel(const int32_t *__restrict__ n_dev, int k, int vec,
                                                        const int32_t *__restrict__ perm, const uint4 *__restrict__ rows,
                                                        uint4 *__restrict__ ybuf) {
    pdl_launch_dependents();
    pdl_wait();
    const long long total = (long long)(*n_dev) * vec;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int p = (int)(i / vec), c = (int)(i - (long long)p * vec);
        const int s = perm[p];
        ybuf[(size_t)(s + s / k) * vec + c] = rows[i];
    }
}

int grid_of(long long work) {
    const long long g = (work + 255) / 256;
    return (int)std::min<long long>(std::max<long long>(g, 1), 4 * (long long)std::max(device_sm_count(), 1));
}

}  // namespace

cudaError_t launch_ep_rank_ids(int n, int epr, const int32_t *idx, int32_t *rank_idx, cudaStream_t st) {
    return launch_pdl(ep_rank_ids_kernel, dim3(grid_of(n)), dim3(256), 0, st, n, epr, idx, rank_idx);
}

cudaError_t launch_ep_pack(int n_max, const int32_t *n_dev, int epr, const int32_t *perm, const int32_t *idx,
                           const float *w, int32_t *local_idx, float *local_w, cudaStream_t st) {
    return launch_pdl(ep_pack_kernel, dim3(grid_of(n_max)), dim3(256), 0, st, n_dev, epr, perm, idx, w, local_idx,
                      local_w);
}

cudaError_t launch_ep_unpack(int n_max, const int32_t *n_dev, int k, int H, const int32_t *perm, const uint16_t *rows,
                             uint16_t *ybuf, cudaStream_t st) {
    const int vec = H / 8;
    return launch_pdl(ep_unpack_kernel, dim3(grid_of((long long)n_max * vec)), dim3(256), 0, st, n_dev, k, vec, perm,
                      reinterpret_cast<const uint4 *>(rows), reinterpret_cast<uint4 *>(ybuf));
}

}  // namespace moe
