// Router projection on the 5th-generation tensor cores:
//
//   logits[t, e] = sum_h x[t, h] * W_r[e, h]        (bf16 in, fp32 out)
//
// the router of the softmax MoE (SpecForge PR #943, "Modifications": the
// router whose logits the softmax top-k takes; a bias-free linear map of the
// hidden state).  One persistent, warp-specialised kernel over work items
// (token tile j, expert tile r, K split s): A = 128 rows of W_r (experts
// r*128 ..), B = BN rows of x (tokens j*BN ..), both K-major in 128-byte-
// swizzled shared memory, loaded by TMA in 64-wide K slices; the fp32
// accumulator (M = 128, N = BN) lives in TMEM, double buffered.  Rows past E
// or T are zero-filled by TMA and never stored.
//
// Small batches have few tiles and a long K (H / 64 slices), so a tile's K
// range is split over several CTAs: each split stores its fp32 partial in
// the workspace, and a second, element-parallel kernel adds the partials in
// split order -- a fixed order, so the logits are the same bits on every
// run.
//
// Roles (192 threads): warp 0 -- TMA producer (one lane); warp 1 -- TMEM
// allocation and MMA issue (one lane); warps 2..5 -- epilogue, one TMEM lane
// quarter (32 experts) each.  Every wait is bounded as in the expert FFN:
// past the limit the kernel sets MOE_STATUS_TIMEOUT and every role stops.
#include <algorithm>
#include <atomic>

#include "tc_common.cuh"

namespace moe {

namespace {
using namespace tc;

constexpr int kRpThreads = 192;
constexpr int kRpStages = 3;                      // ring stages of up to two K slices each
constexpr int kRpSlices = 2;                      // K slices per stage: one barrier round trip per two
constexpr int kRpBN = 128;                        // widest token tile (MMA N)
constexpr int kRpABytes = 128 * 64 * 2;           // 16 KB: 128 rows of W_r x 64 K
constexpr int kRpSubBytes = kRpABytes + kRpBN * 128;    // one slice: + BN token rows x 64 K
constexpr int kRpStageBytes = kRpSlices * kRpSubBytes;  // 64 KB
constexpr int kRpMinSlices = 4;                   // K slices per split at least
constexpr int kRpMaxSplits = 16;                  // K splits at most
constexpr int kRpMaxSms = 160;                    // no device has more SMs (workspace sizing)

struct __align__(64) RpMaps {
    CUtensorMap a;  // W_r [E, H], box 64 x 128
    CUtensorMap b;  // x [T, H], box 64 x BN
};

struct RpParams {
    int T, E, BN, nk;     // tokens, experts, token tile, K slices (H / 64)
    int S, kper;          // K splits per tile, K slices per split
    int wt, items;        // expert tiles, work items (token tiles x expert tiles x splits)
    float *logits;        // [T, E]
    float *part;          // [S, T, E] partials (S > 1)
    int32_t *status;
};

size_t rp_smem() { return 1024 + (size_t)kRpStages * kRpStageBytes + (2 * kRpStages + 5) * 8 + 16; }

__global__ void __launch_bounds__(kRpThreads, 1) router_proj_kernel(const __grid_constant__ RpMaps maps,
                                                                   const RpParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + (size_t)kRpStages * kRpStageBytes);
    uint64_t *empty = full + kRpStages;
    uint64_t *tfull = empty + kRpStages;   // [2]
    uint64_t *tempty = tfull + 2;          // [2]
    uint64_t *mma_done = tempty + 2;       // every MMA of the CTA has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_flag = reinterpret_cast<volatile int *>(tmem_slot + 2);  // elected -> epilogue: 0 go, -1 stop
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem_cols = 2 * kRpBN;  // two accumulators of up to 128 columns
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRpStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 1);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&maps.a);
        prefetch_tmap(&maps.b);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // x (and the previous user of the workspace) are ready past this point

    // item -> (token tile j, expert tile r, split s): splits innermost
    auto decode = [&](int item, int &j, int &r, int &s) {
        s = item % p.S;
        const int q = item / p.S;
        r = q % p.wt;
        j = q / p.wt;
    };

    if (warp == 0) {
        // ================= TMA producer =================
        if (lane == 0) {
            const uint32_t sub_bytes = kRpABytes + (uint32_t)p.BN * 128;
            int st = 0;
            uint32_t ph = 0;
            uint32_t issued = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < p.items; item += gridDim.x) {
                int j, r, s;
                decode(item, j, r, s);
                const int k0 = s * p.kper, k1 = min(p.nk, k0 + p.kper);
                for (int k = k0; k < k1; k += kRpSlices) {
                    const int n = min(kRpSlices, k1 - k);
                    if (issued >= (uint32_t)kRpStages &&
                        !mbar_wait_fast(&empty[st], ph ^ 1u, abort_flag, p.status, true)) {
                        ok = false;
                        break;
                    }
                    uint8_t *dst = ring + (size_t)st * kRpStageBytes;
                    mbar_arrive_expect_tx(&full[st], (uint32_t)n * sub_bytes);
                    for (int u = 0; u < n; ++u) {
                        tma_load_2d(&maps.a, &full[st], dst + u * kRpSubBytes, (k + u) * 64, r * 128);
                        tma_load_2d(&maps.b, &full[st], dst + u * kRpSubBytes + kRpABytes, (k + u) * 64, j * p.BN);
                    }
                    ++issued;
                    if (++st == kRpStages) {
                        st = 0;
                        ph ^= 1u;
                    }
                }
            }
            // wait for the copies still in flight before the CTA may exit
            for (uint32_t n = issued > (uint32_t)kRpStages ? issued - kRpStages : 0; n < issued; ++n)
                mbar_wait(&full[n % kRpStages], (n / kRpStages) & 1u, abort_flag, p.status, false);
        }
    } else if (warp == 1) {
        // ================= MMA issuer =================
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(p.BN);
            const uint64_t desc0 = sw128_desc(smem_u32(ring));
            int st = 0;
            uint32_t ph = 0;
            int li = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < p.items; item += gridDim.x, ++li) {
                int j, r, s;
                decode(item, j, r, s);
                const int k0 = s * p.kper, k1 = min(p.nk, k0 + p.kper);
                const int acc = li & 1;
                const uint32_t use = (uint32_t)(li >> 1);
                if (!mbar_wait_fast(&tempty[acc], (use & 1u) ^ 1u, abort_flag, p.status, true)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(acc * kRpBN);
                for (int k = k0; k < k1; k += kRpSlices) {
                    const int n = min(kRpSlices, k1 - k);
                    if (!mbar_wait_fast(&full[st], ph, abort_flag, p.status, true)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int u = 0; u < n; ++u) {
                        const uint64_t da = desc0 + (uint64_t)(st * kRpStageBytes + u * kRpSubBytes) / 16;
                        const uint64_t db = da + kRpABytes / 16;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)  // K16 steps: +32 bytes each
                            umma_bf16(d, da + 2 * kk, db + 2 * kk, idesc, (k + u > k0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[st]);
                    if (++st == kRpStages) {
                        st = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
            }
            umma_commit(mma_done);  // completes once every MMA above has (TMEM is freed after)
            mbar_wait(mma_done, 0, abort_flag, p.status, false);
        }
    } else {
        // ================= epilogue (warps 2..5) =================
        const int q = warp & 3;  // TMEM lane quarter of this warp: experts r*128 + 32q ..
        const bool elected = (warp == 2 && lane == 0);
        int li = 0;
        for (int item = blockIdx.x; item < p.items; item += gridDim.x, ++li) {
            int j, r, s;
            decode(item, j, r, s);
            const int acc = li & 1;
            const uint32_t use = (uint32_t)(li >> 1);
            if (elected) *epi_flag = mbar_wait(&tfull[acc], use & 1u, abort_flag, p.status, true) ? 0 : -1;
            named_bar_sync(1, 128);
            if (*epi_flag) break;
            tc_fence_after();
            float *dst = p.S > 1 ? p.part + (size_t)s * p.T * p.E : p.logits;
            const int e = r * 128 + q * 32 + lane;
            const uint32_t tbase = tmem_base + (uint32_t)(acc * kRpBN) + ((uint32_t)(q * 32) << 16);
            for (int c0 = 0; c0 < p.BN; c0 += 32) {
                float v[32];
                tmem_ld32(tbase + (uint32_t)c0, v);
                const int t0 = j * p.BN + c0;
                if (e < p.E) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (t0 + i < p.T) dst[(size_t)(t0 + i) * p.E + e] = v[i];
                }
            }
            tc_fence_before();
            named_bar_sync(1, 128);
            if (elected) mbar_arrive(&tempty[acc]);
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols)
                     : "memory");
    }
}

// logits = the S split partials of every element added in split order.
__global__ void __launch_bounds__(256) router_proj_reduce_kernel(long long n, int S, const float *__restrict__ part,
                                                                 float *__restrict__ logits) {
    pdl_launch_dependents();
    pdl_wait();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float v[kRpMaxSplits];  // every partial in flight at once
#pragma unroll
    for (int s = 0; s < kRpMaxSplits; ++s) v[s] = s < S ? __ldg(part + s * n + i) : 0.f;
    float a = v[0];
#pragma unroll
    for (int s = 1; s < kRpMaxSplits; ++s)
        if (s < S) a += v[s];
    logits[i] = a;
}

}  // namespace

// Token tile and K splits of a projection of T tokens over E experts with H
// hidden units on `sms` SMs: BN = the tokens rounded up to 16, at most 128;
// a tile's K range is split (into at most kRpMaxSplits) while there are fewer
// tiles than SMs, each split keeping at least kRpMinSlices slices.
void rp_shape(int T, int E, int H, int sms, int *BN, int *S, int *kper) {
    *BN = std::min(kRpBN, std::max(16, (T + 15) / 16 * 16));
    const int tt = (T + *BN - 1) / *BN, wt = (E + 127) / 128, nk = H / 64;
    const int tiles = tt * wt;
    int s = 1;
    if (tiles < sms) s = std::max(1, std::min(std::min(nk / kRpMinSlices, sms / tiles), kRpMaxSplits));
    *kper = (nk + s - 1) / s;
    *S = (nk + *kper - 1) / *kper;  // no empty split
}

size_t rp_partial_bytes(int T, int E, int H) {
    int BN, S, kper;
    rp_shape(T, E, H, kRpMaxSms, &BN, &S, &kper);  // the most splits any device takes
    return S > 1 ? (size_t)S * T * E * 4 : 0;
}

cudaError_t launch_router_proj(int T, int E, int H, const uint16_t *x, const uint16_t *w_router, float *logits,
                               float *part, int32_t *status, cudaStream_t st) {
    const int sms = device_sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    int BN, S, kper;
    rp_shape(T, E, H, std::min(sms, kRpMaxSms), &BN, &S, &kper);
    RpMaps m;
    if (!encode_2d(&m.a, w_router, (uint64_t)E, (uint64_t)H, 128) || !encode_2d(&m.b, x, (uint64_t)T, (uint64_t)H, BN))
        return cudaErrorInvalidValue;
    RpParams p;
    p.T = T;
    p.E = E;
    p.BN = BN;
    p.nk = H / 64;
    p.S = S;
    p.kper = kper;
    p.wt = (E + 127) / 128;
    p.items = ((T + BN - 1) / BN) * p.wt * S;
    p.logits = logits;
    p.part = part;
    p.status = status;
    static std::atomic<int> attr_set[64];  // per device: opted in to the ring's shared memory
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        const cudaError_t e =
            cudaFuncSetAttribute(router_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rp_smem());
        if (e != cudaSuccess) return e;
        attr_set[dev].store(1, std::memory_order_release);
    }
    const int grid = std::max(1, std::min(sms, p.items));
    cudaError_t e = launch_pdl(router_proj_kernel, dim3(grid), dim3(kRpThreads), rp_smem(), st, m, p);
    if (e != cudaSuccess || S == 1) return e;
    const long long n = (long long)T * E;
    return launch_pdl(router_proj_reduce_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, n, S,
                      static_cast<const float *>(part), logits);
}

}  // namespace moe
