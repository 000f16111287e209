// C ABI of libmoe: argument checks, workspace layout and the launch
// sequence.  No entry point allocates, frees or synchronises (except
// moe_status_read, which waits for its own copy); every launch goes on the
// caller's stream.
#include <cstring>
#include <mutex>

#include "moe_internal.cuh"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;
// Head of the workspace: [0, 256) status word and work-item counters,
// [256, 256 + 4 * (E + 2)) gate/up completion counters of the fused FFN.
constexpr size_t kHeadBytes = 8192;
constexpr size_t kHdoneOffset = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct WsLayout {
    size_t status, idx, w, sgate, keff, kept, ndrop, counts, offsets, perm, slot_pos, hist, bagg, bcnt;
    size_t x_perm, h_perm, h_shared, ybuf, logits, rpart, total;
};

WsLayout ws_layout(const moe_config_t &c, int T) {
    WsLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes);
        return o;
    };
    const size_t Tk = (size_t)T * c.num_experts_per_tok;
    const size_t E = (size_t)c.n_routed_experts;
    L.status = take(kHeadBytes);
    L.idx = take(Tk * 4);
    L.w = take(Tk * 4);
    L.sgate = take((size_t)T * 4);
    L.keff = take((size_t)T * 4);
    L.kept = take(E);
    L.ndrop = take(4);
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 4);
    L.perm = take(Tk * 4);
    L.slot_pos = take(Tk * 4);
    L.hist = take((size_t)dispatch_chunks(T) * E * 4);
    L.bagg = take((size_t)budget_chunks(T) * E * 4);
    L.bcnt = take((size_t)budget_chunks(T) * E * 4);
    L.x_perm = take(Tk * c.hidden * 2);
    L.h_perm = take(Tk * c.moe_intermediate_size * 2);
    L.h_shared = take((size_t)T * c.shared_intermediate_size * 2);
    L.ybuf = take((size_t)T * (c.num_experts_per_tok + 1) * c.hidden * 2);
    L.logits = take((size_t)T * E * 4);
    L.rpart = take(rp_partial_bytes(T, (int)E, c.hidden));
    L.total = off;
    return L;
}

// The top-p trim is on for 0 < topp < 1 (0, the default, and 1 or more leave the routing as it is).
bool topp_on(const moe_config_t *c) { return c->topp > 0.f && c->topp < 1.f; }

int check_config(const moe_config_t *c, int32_t T) {
    if (!c || T < 0) return MOE_ERR_INVALID_ARG;
    const int E = c->n_routed_experts, k = c->num_experts_per_tok;
    if (E < 1 || k < 1 || k > E || c->budget < 0 || c->shared_intermediate_size < 0 || c->hidden < 1 ||
        c->moe_intermediate_size < 1 || (c->norm_topk != 0 && c->norm_topk != 1) || !(c->topp >= 0.f) ||
        c->topp > 3.4e38f)  // NaN, negative or infinite top-p
        return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts || k > kMaxTopK || c->hidden % 128 != 0 || c->moe_intermediate_size % 64 != 0 ||
        c->shared_intermediate_size % 64 != 0)
        return MOE_ERR_UNSUPPORTED;
    if ((long long)T * (k + 1) * c->hidden >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

bool aligned(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_or_null(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <class T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace

extern "C" {

size_t moe_workspace_bytes(const moe_config_t *cfg, int32_t T) {
    if (check_config(cfg, T) != MOE_OK) return 0;
    return ws_layout(*cfg, T).total;
}

const char *moe_error_string(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or device";
        case MOE_ERR_WORKSPACE: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA launch or driver call failed";
        case MOE_ERR_DEVICE: return "device-side error reported in the status word";
        default: return "unknown error";
    }
}

int moe_route(const moe_config_t *cfg, int32_t T, const float *logits, const moe_bf16_t *x,
              const moe_bf16_t *ws_gate_vec, int32_t *topk_idx, float *topk_w, float *sgate, int32_t *keff,
              void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned(logits) || !aligned(topk_idx) || !aligned(topk_w) || !aligned_or_null(keff))
        return MOE_ERR_INVALID_ARG;
    if (topp_on(cfg) && keff == nullptr) return MOE_ERR_INVALID_ARG;  // the trimmed counts must go somewhere
    if (sgate && (cfg->shared_intermediate_size == 0 || !aligned(x) || !aligned(ws_gate_vec) || !aligned(sgate)))
        return MOE_ERR_INVALID_ARG;
    return cuda_rc(launch_route(T, cfg->n_routed_experts, cfg->num_experts_per_tok, cfg->norm_topk, cfg->topp,
                                logits, topk_idx, topk_w, keff, x, ws_gate_vec, cfg->hidden, sgate,
                                as_stream(stream)));
}

int moe_budget(const moe_config_t *cfg, int32_t T, int32_t *topk_idx, float *topk_w, int32_t *keff,
               uint8_t *expert_kept, int32_t *n_dropped, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned(topk_idx) || !aligned(topk_w) || !aligned(keff) || !expert_kept || !n_dropped || !aligned(ws))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    return cuda_rc(launch_budget(T, cfg->n_routed_experts, cfg->num_experts_per_tok, cfg->budget, cfg->norm_topk,
                                 topk_idx, topk_w, keff, expert_kept, n_dropped, at<float>(ws, L.bagg),
                                 at<int32_t>(ws, L.bcnt), as_stream(stream)));
}

int moe_dispatch(const moe_config_t *cfg, int32_t T, const int32_t *topk_idx, const int32_t *keff,
                 const moe_bf16_t *x, int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *slot_pos,
                 moe_bf16_t *x_perm, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned(topk_idx) || !aligned_or_null(keff) || !aligned(counts) || !aligned(offsets) || !aligned(perm) ||
        !aligned(slot_pos) || !aligned(ws) || !aligned_or_null(x_perm) || (x_perm && !aligned(x)))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    const int E = cfg->n_routed_experts, k = cfg->num_experts_per_tok;
    cudaStream_t st = as_stream(stream);
    return cuda_rc(launch_dispatch(T, E, k, topk_idx, keff, at<int32_t>(ws, L.hist), counts, offsets, perm, slot_pos,
                                   at<int32_t>(ws, L.status), at<int32_t>(ws, L.status + kHdoneOffset), x, x_perm,
                                   cfg->hidden, st));
}

}  // extern "C"

namespace {

// Common checks and argument block of the two FFN phases; `gate_up`
// selects which phase's inputs are checked.
int ffn_args(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
             const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
             const moe_weights_t *w, moe_bf16_t *ybuf, void *ws, size_t ws_bytes, bool gate_up, FfnArgs *a) {
    const bool sh = cfg->shared_intermediate_size > 0;
    if (!w || !aligned(offsets) || !aligned(ws)) return MOE_ERR_INVALID_ARG;
    if (gate_up && (!aligned(x_perm) || !aligned(w->w_gate) || !aligned(w->w_up) ||
                    (sh && (!aligned(x) || !aligned(w->ws_gate) || !aligned(w->ws_up)))))
        return MOE_ERR_INVALID_ARG;
    if (!gate_up && (!aligned(perm) || !aligned(topk_w) || !aligned(ybuf) || !aligned(w->w_down) ||
                     (sh && (!aligned(sgate) || !aligned(w->ws_down)))))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    *a = FfnArgs{};
    a->T = T;
    a->H = cfg->hidden;
    a->E = cfg->n_routed_experts;
    a->I = cfg->moe_intermediate_size;
    a->k = cfg->num_experts_per_tok;
    a->Is = cfg->shared_intermediate_size;
    a->x = x;
    a->x_perm = x_perm;
    a->offsets = offsets;
    a->perm = perm;
    a->topk_w = topk_w;
    a->sgate = sgate;
    a->w_gate = w->w_gate;
    a->w_up = w->w_up;
    a->w_down = w->w_down;
    a->ws_gate = w->ws_gate;
    a->ws_up = w->ws_up;
    a->ws_down = w->ws_down;
    a->h_perm = at<uint16_t>(ws, L.h_perm);
    a->h_shared = sh ? at<uint16_t>(ws, L.h_shared) : nullptr;
    a->ybuf = ybuf;
    a->status = at<int32_t>(ws, L.status);
    a->hdone = at<int32_t>(ws, L.status + kHdoneOffset);
    return MOE_OK;
}

// A block-scaled expert FFN's argument block: the bf16 block with the weight
// pointers replaced by the codes and the packed block scales added.  codes /
// scales: gate, up, down, shared gate, shared up, shared down.
int ffn_args_scaled(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                    const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                    const uint8_t *const (&codes)[6], const uint8_t *const (&scales)[6], int fmt, moe_bf16_t *ybuf,
                    void *ws, size_t ws_bytes, FfnArgs *a) {
    const bool sh = cfg->shared_intermediate_size > 0;
    for (int i = 0; i < (sh ? 6 : 3); ++i)
        if (!aligned(codes[i]) || !aligned(scales[i])) return MOE_ERR_INVALID_ARG;
    if (cfg->hidden % 128 != 0 || cfg->moe_intermediate_size % 128 != 0 || cfg->shared_intermediate_size % 128 != 0)
        return MOE_ERR_UNSUPPORTED;
    // the bf16 block's checks and fields, with the code pointers standing in for the weights
    moe_weights_t wb{};
    wb.w_gate = reinterpret_cast<const moe_bf16_t *>(codes[0]);
    wb.w_up = reinterpret_cast<const moe_bf16_t *>(codes[1]);
    wb.w_down = reinterpret_cast<const moe_bf16_t *>(codes[2]);
    wb.ws_gate = reinterpret_cast<const moe_bf16_t *>(codes[3]);
    wb.ws_up = reinterpret_cast<const moe_bf16_t *>(codes[4]);
    wb.ws_down = reinterpret_cast<const moe_bf16_t *>(codes[5]);
    FfnArgs b;
    int rc = ffn_args(cfg, T, x, x_perm, offsets, perm, topk_w, sgate, &wb, ybuf, ws, ws_bytes, true, a);
    if (rc) return rc;
    rc = ffn_args(cfg, T, x, x_perm, offsets, perm, topk_w, sgate, &wb, ybuf, ws, ws_bytes, false, &b);
    if (rc) return rc;
    a->fmt = fmt;
    a->sf_gate = scales[0];
    a->sf_up = scales[1];
    a->sf_down = scales[2];
    a->sfs_gate = sh ? scales[3] : nullptr;
    a->sfs_up = sh ? scales[4] : nullptr;
    a->sfs_down = sh ? scales[5] : nullptr;
    return MOE_OK;
}

int ffn_args_mxfp8(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                   const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                   const moe_weights_mxfp8_t *w, moe_bf16_t *ybuf, void *ws, size_t ws_bytes, FfnArgs *a) {
    if (!w) return MOE_ERR_INVALID_ARG;
    const uint8_t *const codes[6] = {w->w_gate, w->w_up, w->w_down, w->ws_gate, w->ws_up, w->ws_down};
    const uint8_t *const scales[6] = {w->w_gate_scale,  w->w_up_scale,  w->w_down_scale,
                                      w->ws_gate_scale, w->ws_up_scale, w->ws_down_scale};
    return ffn_args_scaled(cfg, T, x, x_perm, offsets, perm, topk_w, sgate, codes, scales, 1, ybuf, ws, ws_bytes, a);
}

bool f32_aligned(const float *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int ffn_args_nvfp4(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                   const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                   const moe_weights_nvfp4_t *w, moe_bf16_t *ybuf, void *ws, size_t ws_bytes, FfnArgs *a) {
    if (!w) return MOE_ERR_INVALID_ARG;
    const bool sh = cfg->shared_intermediate_size > 0;
    if (!f32_aligned(w->w_gate_tscale) || !f32_aligned(w->w_up_tscale) || !f32_aligned(w->w_down_tscale) ||
        (sh && !f32_aligned(w->ws_tscale)))
        return MOE_ERR_INVALID_ARG;
    const uint8_t *const codes[6] = {w->w_gate, w->w_up, w->w_down, w->ws_gate, w->ws_up, w->ws_down};
    const uint8_t *const scales[6] = {w->w_gate_scale,  w->w_up_scale,  w->w_down_scale,
                                      w->ws_gate_scale, w->ws_up_scale, w->ws_down_scale};
    const int rc =
        ffn_args_scaled(cfg, T, x, x_perm, offsets, perm, topk_w, sgate, codes, scales, 2, ybuf, ws, ws_bytes, a);
    if (rc) return rc;
    a->ts_gate = w->w_gate_tscale;
    a->ts_up = w->w_up_tscale;
    a->ts_down = w->w_down_tscale;
    a->tss = sh ? w->ws_tscale : nullptr;
    return MOE_OK;
}

}  // namespace

extern "C" {

int moe_expert_gate_up(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                       const int32_t *offsets, const moe_weights_t *w, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    FfnArgs a;
    rc = ffn_args(cfg, T, x, x_perm, offsets, nullptr, nullptr, nullptr, w, nullptr, ws, ws_bytes, true, &a);
    if (rc) return rc;
    return ffn_launch(a, 1, as_stream(stream));
}

int moe_expert_down(const moe_config_t *cfg, int32_t T, const int32_t *offsets, const int32_t *perm,
                    const float *topk_w, const float *sgate, const moe_weights_t *w, moe_bf16_t *ybuf, void *ws,
                    size_t ws_bytes, void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    FfnArgs a;
    rc = ffn_args(cfg, T, nullptr, nullptr, offsets, perm, topk_w, sgate, w, ybuf, ws, ws_bytes, false, &a);
    if (rc) return rc;
    return ffn_launch(a, 2, as_stream(stream));
}

int moe_expert_ffn(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                   const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                   const moe_weights_t *w, moe_bf16_t *ybuf, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    FfnArgs a, b;
    rc = ffn_args(cfg, T, x, x_perm, offsets, perm, topk_w, sgate, w, ybuf, ws, ws_bytes, true, &a);
    if (rc) return rc;
    rc = ffn_args(cfg, T, x, x_perm, offsets, perm, topk_w, sgate, w, ybuf, ws, ws_bytes, false, &b);
    if (rc) return rc;
    return ffn_launch_both(a, as_stream(stream));
}

}  // extern "C"

namespace {

// ---------------------------------------------------------------------------
// Expert FFN without any device allocation by the caller.
//
// Some callers cannot allocate device memory: a plugin that a host framework
// hands only its input and output buffers (no allocator, no way to keep a
// workspace of its own), or a serving loop that must not allocate once it
// is running (an allocation can synchronise the device and stall every
// stream).  For them the FFN's scratch -- the gate/up activations h and the
// scheduling counters -- lives in this file-scope device array instead of a
// caller workspace.  It is sized for decode-sized batches: the routed and
// shared h rows, 2 * (T*k*I + T*Is) bytes, must fit in kNoallocScratchBytes
// (8 MiB), plus an 8 KiB block of counters.  Every GPU that loads the library
// holds the array until the process exits.
constexpr size_t kNoallocScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kHeadBytes + kNoallocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device (with that
// device current) on the first call there.
void *noalloc_scratch_ptr(int dev) {
    static void *ptrs[64] = {};
    static std::mutex mu;
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        ptrs[dev] = p;
    }
    return ptrs[dev];
}

}  // namespace

extern "C" {

int moe_expert_ffn_noalloc(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                           const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                           const moe_weights_t *w, moe_bf16_t *ybuf, int32_t *device_status, void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    const bool sh = cfg->shared_intermediate_size > 0;
    if (!w || !aligned(offsets) || !aligned(x_perm) || !aligned(w->w_gate) || !aligned(w->w_up) || !aligned(perm) ||
        !aligned(topk_w) || !aligned(ybuf) || !aligned(w->w_down) || !aligned_or_null(device_status))
        return MOE_ERR_INVALID_ARG;
    if (sh && (!aligned(x) || !aligned(w->ws_gate) || !aligned(w->ws_up) || !aligned(sgate) || !aligned(w->ws_down)))
        return MOE_ERR_INVALID_ARG;
    // scratch layout after the counter block: h_perm [T*k, I], then h_shared [T, Is]
    const size_t h_perm_bytes = align_up((size_t)T * cfg->num_experts_per_tok * cfg->moe_intermediate_size * 2);
    const size_t h_shared_bytes = align_up((size_t)T * cfg->shared_intermediate_size * 2);
    if (h_perm_bytes + h_shared_bytes > kNoallocScratchBytes) return MOE_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    uint8_t *scratch = static_cast<uint8_t *>(noalloc_scratch_ptr(dev));
    if (!scratch) return MOE_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    // the counters must start at zero; the array keeps whatever the last call left
    if (cudaMemsetAsync(scratch, 0, kHeadBytes, st) != cudaSuccess) return MOE_ERR_CUDA;
    FfnArgs a{};
    a.T = T;
    a.H = cfg->hidden;
    a.E = cfg->n_routed_experts;
    a.I = cfg->moe_intermediate_size;
    a.k = cfg->num_experts_per_tok;
    a.Is = cfg->shared_intermediate_size;
    a.x = x;
    a.x_perm = x_perm;
    a.offsets = offsets;
    a.perm = perm;
    a.topk_w = topk_w;
    a.sgate = sgate;
    a.w_gate = w->w_gate;
    a.w_up = w->w_up;
    a.w_down = w->w_down;
    a.ws_gate = w->ws_gate;
    a.ws_up = w->ws_up;
    a.ws_down = w->ws_down;
    a.status = reinterpret_cast<int32_t *>(scratch);
    a.hdone = reinterpret_cast<int32_t *>(scratch + kHdoneOffset);
    a.h_perm = reinterpret_cast<uint16_t *>(scratch + kHeadBytes);
    a.h_shared = sh ? reinterpret_cast<uint16_t *>(scratch + kHeadBytes + h_perm_bytes) : nullptr;
    a.ybuf = ybuf;
    rc = ffn_launch_both(a, st);
    if (rc) return rc;
    if (device_status)  // hand the kernel's status word to the caller
        if (cudaMemcpyAsync(device_status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_ep_rank_ids(int32_t T, int32_t k, int32_t experts_per_rank, const int32_t *topk_idx, int32_t *rank_idx,
                    void *stream) {
    if (T < 0 || k < 1 || experts_per_rank < 1) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!aligned(topk_idx) || !aligned(rank_idx)) return MOE_ERR_INVALID_ARG;
    return cuda_rc(launch_ep_rank_ids(T * k, experts_per_rank, topk_idx, rank_idx, as_stream(stream)));
}

int moe_ep_pack(int32_t n_max, const int32_t *n_sent, int32_t experts_per_rank, const int32_t *perm,
                const int32_t *topk_idx, const float *topk_w, int32_t *local_idx, float *local_w, void *stream) {
    if (n_max < 0 || experts_per_rank < 1) return MOE_ERR_INVALID_ARG;
    if (n_max == 0) return MOE_OK;
    if (!n_sent || !aligned(perm) || !aligned(topk_idx) || !aligned(topk_w) || !aligned(local_idx) ||
        !aligned(local_w))
        return MOE_ERR_INVALID_ARG;
    return cuda_rc(launch_ep_pack(n_max, n_sent, experts_per_rank, perm, topk_idx, topk_w, local_idx, local_w,
                                  as_stream(stream)));
}

int moe_ep_unpack(const moe_config_t *cfg, int32_t T, int32_t n_max, const int32_t *n_returned, const int32_t *perm,
                  const moe_bf16_t *rows, moe_bf16_t *ybuf, void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (n_max < 0 || n_max > T * cfg->num_experts_per_tok) return MOE_ERR_INVALID_ARG;
    if (T == 0 || n_max == 0) return MOE_OK;
    if (!n_returned || !aligned(perm) || !aligned(rows) || !aligned(ybuf)) return MOE_ERR_INVALID_ARG;
    return cuda_rc(launch_ep_unpack(n_max, n_returned, cfg->num_experts_per_tok, cfg->hidden, perm, rows, ybuf,
                                    as_stream(stream)));
}

int moe_mxfp8_pack_scales(int64_t rows, int32_t K, const uint8_t *scales, uint8_t *packed, void *stream) {
    if (rows < 0 || rows % 64 != 0 || K < 128 || K % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!aligned(scales) || !aligned(packed)) return MOE_ERR_INVALID_ARG;
    return cuda_rc(launch_mxfp8_pack_scales(rows, K, scales, packed, as_stream(stream)));
}

int moe_nvfp4_pack_scales(int64_t rows, int32_t K, const uint8_t *scales, uint8_t *packed, void *stream) {
    if (rows < 0 || rows % 64 != 0 || K < 128 || K % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!aligned(scales) || !aligned(packed)) return MOE_ERR_INVALID_ARG;
    return cuda_rc(launch_nvfp4_pack_scales(rows, K, scales, packed, as_stream(stream)));
}

int moe_expert_ffn_nvfp4(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                         const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                         const moe_weights_nvfp4_t *w, moe_bf16_t *ybuf, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    FfnArgs a;
    rc = ffn_args_nvfp4(cfg, T, x, x_perm, offsets, perm, topk_w, sgate, w, ybuf, ws, ws_bytes, &a);
    if (rc) return rc;
    return ffn_launch_both(a, as_stream(stream));
}

int moe_expert_ffn_mxfp8(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *x_perm,
                         const int32_t *offsets, const int32_t *perm, const float *topk_w, const float *sgate,
                         const moe_weights_mxfp8_t *w, moe_bf16_t *ybuf, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    FfnArgs a;
    rc = ffn_args_mxfp8(cfg, T, x, x_perm, offsets, perm, topk_w, sgate, w, ybuf, ws, ws_bytes, &a);
    if (rc) return rc;
    return ffn_launch_both(a, as_stream(stream));
}

int moe_combine(const moe_config_t *cfg, int32_t T, const moe_bf16_t *ybuf, const int32_t *keff, moe_bf16_t *out,
                void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned(ybuf) || !aligned_or_null(keff) || !aligned(out)) return MOE_ERR_INVALID_ARG;
    return cuda_rc(launch_combine(T, cfg->num_experts_per_tok, cfg->hidden, cfg->shared_intermediate_size > 0, ybuf,
                                  keff, out, as_stream(stream)));
}

int moe_quantize_mxfp8(int64_t rows, int32_t K, const moe_bf16_t *w, uint8_t *codes, uint8_t *scales,
                       void *stream) {
    if (rows < 0 || K < 32 || K % 32 != 0) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!aligned(w) || !aligned(codes) || !scales) return MOE_ERR_INVALID_ARG;
    return cuda_rc(launch_quantize_mxfp8(rows, K, w, codes, scales, as_stream(stream)));
}

int moe_quantize_nvfp4(int32_t nmat, int64_t rows, int32_t K, const moe_bf16_t *w, uint8_t *codes, uint8_t *scales,
                       float *tensor_scale, void *stream) {
    if (nmat < 1 || nmat > 65535 || rows < 0 || K < 16 || K % 16 != 0) return MOE_ERR_INVALID_ARG;
    if (!tensor_scale || (reinterpret_cast<uintptr_t>(tensor_scale) & 3u) != 0) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!aligned(w) || !aligned(codes) || !scales) return MOE_ERR_INVALID_ARG;
    return cuda_rc(launch_quantize_nvfp4(nmat, rows, K, w, codes, scales, tensor_scale, as_stream(stream)));
}

int moe_router_logits(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const moe_bf16_t *w_router,
                      float *logits, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned(x) || !aligned(w_router) || !aligned(logits) || !aligned(ws)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    return cuda_rc(launch_router_proj(T, cfg->n_routed_experts, cfg->hidden, x, w_router, logits,
                                      at<float>(ws, L.rpart), at<int32_t>(ws, L.status), as_stream(stream)));
}

}  // extern "C"

namespace {

// The layer around an expert FFN: [router projection] -> route -> [budget]
// -> dispatch -> ffn(...) -> combine.  `ffn` enqueues the expert FFN of the
// dispatched batch (bf16, MXFP8 or NVFP4 weights).
template <class Ffn>
int forward_impl(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const float *logits,
                 const moe_bf16_t *w_router, const moe_bf16_t *ws_gate_vec, moe_bf16_t *out, const moe_aux_t *aux,
                 void *ws, size_t ws_bytes, void *stream, Ffn ffn) {
    int rc = check_config(cfg, T);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    const bool sh = cfg->shared_intermediate_size > 0;
    if (!aligned(x) || !aligned_or_null(logits) || !aligned(out) || !aligned(ws)) return MOE_ERR_INVALID_ARG;
    if (!logits && !aligned(w_router)) return MOE_ERR_INVALID_ARG;  // no logits: the projection makes them
    if (sh && !aligned(ws_gate_vec)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    moe_aux_t a{};
    if (aux) a = *aux;
    if (a.logits && !aligned(a.logits)) return MOE_ERR_INVALID_ARG;
    if (!logits) {  // router projection first
        float *lg = a.logits ? a.logits : at<float>(ws, L.logits);
        rc = moe_router_logits(cfg, T, x, w_router, lg, ws, ws_bytes, stream);
        if (rc) return rc;
        logits = lg;
    }
    int32_t *idx = a.topk_idx ? a.topk_idx : at<int32_t>(ws, L.idx);
    float *tw = a.topk_w ? a.topk_w : at<float>(ws, L.w);
    float *sgate = sh ? (a.sgate ? a.sgate : at<float>(ws, L.sgate)) : nullptr;
    int32_t *keff = a.keff ? a.keff : at<int32_t>(ws, L.keff);
    uint8_t *kept = a.expert_kept ? a.expert_kept : at<uint8_t>(ws, L.kept);
    int32_t *ndrop = a.n_dropped ? a.n_dropped : at<int32_t>(ws, L.ndrop);
    int32_t *counts = a.counts ? a.counts : at<int32_t>(ws, L.counts);
    int32_t *offsets = a.offsets ? a.offsets : at<int32_t>(ws, L.offsets);
    int32_t *perm = a.perm ? a.perm : at<int32_t>(ws, L.perm);
    int32_t *slot_pos = a.slot_pos ? a.slot_pos : at<int32_t>(ws, L.slot_pos);
    moe_bf16_t *x_perm = at<moe_bf16_t>(ws, L.x_perm);
    moe_bf16_t *ybuf = at<moe_bf16_t>(ws, L.ybuf);

    const int E = cfg->n_routed_experts, k = cfg->num_experts_per_tok;
    if constexpr (kDebugBounds) {  // checked library: non-finite logits are reported, not routed silently
        rc = cuda_rc(launch_check_logits((long long)T * E, logits, at<int32_t>(ws, L.status), as_stream(stream)));
        if (rc) return rc;
    }
    // A small batch with an expert budget: route, budget and dispatch in one launch
    // instead of four.  (Without a budget the separate route and dispatch
    // launches measured faster for the drafter layers.)
    if (cfg->budget > 0 && front_fits(T, E, k)) {
        rc = cuda_rc(launch_front(T, E, k, cfg->budget, cfg->norm_topk, cfg->topp, cfg->hidden, logits, x,
                                  sh ? ws_gate_vec : nullptr, idx, tw, sgate, keff, kept, ndrop, counts, offsets,
                                  perm, slot_pos, x_perm, at<int32_t>(ws, L.status),
                                  at<int32_t>(ws, L.status + kHdoneOffset), as_stream(stream)));
        if (rc) return rc;
    } else {
        rc = moe_route(cfg, T, logits, x, sh ? ws_gate_vec : nullptr, idx, tw, sgate, keff, stream);
        if (rc) return rc;
        if (cfg->budget > 0) {
            rc = moe_budget(cfg, T, idx, tw, keff, kept, ndrop, ws, ws_bytes, stream);
            if (rc) return rc;
        }
        rc = moe_dispatch(cfg, T, idx, keff, x, counts, offsets, perm, slot_pos, x_perm, ws, ws_bytes, stream);
        if (rc) return rc;
    }
    rc = ffn(x_perm, offsets, perm, tw, sgate, ybuf);
    if (rc) return rc;
    return moe_combine(cfg, T, ybuf, keff, out, stream);
}

}  // namespace

extern "C" {

int moe_forward(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const float *logits, const moe_weights_t *w,
                moe_bf16_t *out, const moe_aux_t *aux, void *ws, size_t ws_bytes, void *stream) {
    const int rc = check_config(cfg, T);
    if (rc || T == 0) return rc;
    if (!w) return MOE_ERR_INVALID_ARG;
    return forward_impl(cfg, T, x, logits, w->w_router, w->ws_gate_vec, out, aux, ws, ws_bytes, stream,
                        [&](const moe_bf16_t *x_perm, const int32_t *offsets, const int32_t *perm, const float *tw,
                            const float *sgate, moe_bf16_t *ybuf) {
                            return moe_expert_ffn(cfg, T, x, x_perm, offsets, perm, tw, sgate, w, ybuf, ws, ws_bytes,
                                                  stream);
                        });
}

int moe_forward_mxfp8(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const float *logits,
                      const moe_weights_mxfp8_t *w, moe_bf16_t *out, const moe_aux_t *aux, void *ws,
                      size_t ws_bytes, void *stream) {
    const int rc = check_config(cfg, T);
    if (rc || T == 0) return rc;
    if (!w) return MOE_ERR_INVALID_ARG;
    if (cfg->hidden % 128 != 0 || cfg->moe_intermediate_size % 128 != 0 || cfg->shared_intermediate_size % 128 != 0)
        return MOE_ERR_UNSUPPORTED;  // before anything is launched
    return forward_impl(cfg, T, x, logits, w->w_router, w->ws_gate_vec, out, aux, ws, ws_bytes, stream,
                        [&](const moe_bf16_t *x_perm, const int32_t *offsets, const int32_t *perm, const float *tw,
                            const float *sgate, moe_bf16_t *ybuf) {
                            return moe_expert_ffn_mxfp8(cfg, T, x, x_perm, offsets, perm, tw, sgate, w, ybuf, ws,
                                                        ws_bytes, stream);
                        });
}

int moe_forward_nvfp4(const moe_config_t *cfg, int32_t T, const moe_bf16_t *x, const float *logits,
                      const moe_weights_nvfp4_t *w, moe_bf16_t *out, const moe_aux_t *aux, void *ws,
                      size_t ws_bytes, void *stream) {
    const int rc = check_config(cfg, T);
    if (rc || T == 0) return rc;
    if (!w) return MOE_ERR_INVALID_ARG;
    if (cfg->hidden % 128 != 0 || cfg->moe_intermediate_size % 128 != 0 || cfg->shared_intermediate_size % 128 != 0)
        return MOE_ERR_UNSUPPORTED;  // before anything is launched
    return forward_impl(cfg, T, x, logits, w->w_router, w->ws_gate_vec, out, aux, ws, ws_bytes, stream,
                        [&](const moe_bf16_t *x_perm, const int32_t *offsets, const int32_t *perm, const float *tw,
                            const float *sgate, moe_bf16_t *ybuf) {
                            return moe_expert_ffn_nvfp4(cfg, T, x, x_perm, offsets, perm, tw, sgate, w, ybuf, ws,
                                                        ws_bytes, stream);
                        });
}

int moe_status_read(const void *ws, int32_t *status_out, void *stream) {
    if (!aligned(ws) || !status_out) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    if (cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cuda_rc(cudaStreamSynchronize(st));
}

int moe_status_clear(void *ws, void *stream) {
    if (!aligned(ws)) return MOE_ERR_INVALID_ARG;
    return cuda_rc(cudaMemsetAsync(ws, 0, kHeadBytes, as_stream(stream)));
}

}  // extern "C"
