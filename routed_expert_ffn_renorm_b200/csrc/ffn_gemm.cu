// Grouped expert FFN on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA: one persistent, warp-specialised kernel whose work items are
// tiles of two GEMM phases,
//
//   gate/up (phase 0):  h[p, i] = silu(W_gate[e] x_p)_i * (W_up[e] x_p)_i
//   down    (phase 1):  ybuf[row(p), :] = w_p * (W_down[e] h_p)
//
// for every dispatched row p of expert e (SpecForge PR #943,
// "Modifications": gated expert FFN, grouped dispatch; its parameter table
// fixes gate/up/down of H x I each), and the same for the shared expert,
// whose rows are all T tokens in token order and whose weight is the
// sigmoid gate.  A launch runs phase 0, phase 1 or both; with both, a
// down item of a group waits (bounded) until every gate/up item of that
// group has stored its h rows, so the tail of one phase overlaps the start
// of the other and the layer's FFN is one launch.
//
// Orientation ("swap AB").  The weights sit in the MMA M slot (128 weight
// rows per tile) and the tokens of one group in the N slot (16..256 per
// tile), so a group of 3 tokens costs an N=16 MMA, not a 128-row padded
// tile: decode-sized batches stream weights and barely touch the tensor
// pipe, large batches fill N = 256.
//   gate/up tile: A = [64 gate rows ; 64 up rows] of the same intermediate
//                 indices, so gate and up of index i land in TMEM lanes i and
//                 64 + i and the epilogue pairs them through shared memory;
//   down tile:    A = 128 rows of W_down (128 output columns); when the
//                 down phase has many items, a group of at most BN/2 tokens
//                 takes two such tiles per item, into two accumulators side
//                 by side, so the token box is read once for both and there
//                 are half as many short items.
// Both operands are K-major bf16 in 128-byte-swizzled shared memory, loaded
// by TMA boxes of 64 K-elements; the accumulator is fp32 in TMEM, double
// buffered (2 x BN columns) so the epilogue of one tile overlaps the
// mainloop of the next.
//
// Shared-memory ring.  One K step needs 16 KB of weights and 128 B per
// token row, and the token count of a tile ranges from 1 to 256, so the
// ring is cut into 2 KB pages and each K step takes 8 + 2^b consecutive
// pages, its token rows being one TMA box of 16 << b rows, the smallest that
// holds the tile (a step that would straddle the end of the ring starts
// over at page 0).  A 28-token step then holds 20 KB instead of a fixed
// 16 KB + 32 KB slot: narrow routed tiles keep ~10 steps of weights in
// flight, and the shared expert still gets whole 256-token tiles.  Producer
// and MMA lane walk the same page sequence; each K step has its own barrier
// pair ("ticket", 32 of them), and the producer reuses pages only after the
// MMAs of the steps that held them have committed.  Both lanes are on the
// critical path of every step, so a step carries two 64-wide K slices when
// they fit 24 pages, or 32 pages with room for two such steps in the ring
// (32 KB of weights per barrier round trip), and their loops avoid divisions
// and out-of-line calls on the common path.
//
// Roles (224 threads, one CTA per SM, persistent): warp 0 -- TMA producer
// (one lane; the weight boxes, and all copies of a CTA pair); warp 1 -- TMEM
// allocation and MMA issue (one lane); warps 2..5 -- epilogue, one TMEM lane
// quarter each; warp 6 -- the token loader of single CTAs (one lane).
// Block-scaled weights add eight converter warps (480 threads).
//
// Work items are handed out dynamically (a global counter, claimed one item
// ahead) in the order phase 0 [shared expert, routed experts ascending],
// phase 1 [shared expert, routed experts ascending] -- the shared expert's
// items are the longest, so they start first; inside a group, weight tile
// outer and token tile inner, so token tiles that reuse a weight tile run
// side by side (one HBM read, L2 hits).  The item table is derived in-kernel from the
// dispatch offsets -- no host sync.  The token box height (16..256 rows) is
// picked per tile and the MMA N is the valid token count rounded up to 16.
//
// Every wait is bounded: past the limit the kernel sets MOE_STATUS_TIMEOUT
// in the status word, the other roles see an abort flag and stop, the
// producer waits (bounded) for its copies in flight, the MMA lane for its
// MMAs, and TMEM is freed before exit.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "tc_common.cuh"

namespace moe {

namespace {
using namespace tc;

constexpr int kBlockK = 64;                    // K elements per step (128 B rows)
constexpr int kTileM = 128;                    // weight rows per tile (MMA M)
constexpr int kABytes = kTileM * kBlockK * 2;  // 16 KB
constexpr int kNumBox = 5;                     // token box heights 16 << i
// Warps: 0 producer (weights), 1 MMA issuer, 2..5 epilogue, 6 token loader
// (single CTAs), then the converters of block-scaled weights.
constexpr int kThreads = 224;
constexpr int kLoadWarp = 6;
// Block-scaled weights (kFmt 1: MXFP8, 2: NVFP4): converter warps after the
// epilogue warps turn each ring step's codes into the bf16 A operand in
// tensor memory.  A ring step covers 128 K of a 128-row weight tile: its
// codes (MXFP8: 128 B a row, 8 pages; NVFP4: 64 B a row, 4 pages), its
// block scales (one page: two runs of 64 rows, MXFP8 4 UE8M0 bytes a row,
// NVFP4 8 E4M3 bytes a row) and two token boxes.
constexpr int kConvWarps = 8;  // two groups of four, one warp of each per SM sub-partition
constexpr int kThreadsQ = kThreads + 32 * kConvWarps;
template <int kFmt> constexpr int qcode_pages() { return kFmt == 2 ? 4 : 8; }
template <int kFmt> constexpr int qscale_run() { return kFmt == 2 ? 512 : 256; }  // bytes per 64 rows
// A step's converted A operand (two bf16 K slices of 64: 64 TMEM columns) goes
// to one of kConvBufs buffers after the accumulators (from column kConvCol0
// on; the token tile is at most 128 wide then).
constexpr int kConvBufs = 4;
constexpr int kConvCols = 64;
constexpr int kConvCol0 = 256;
constexpr int kPageBytes = 2048;               // ring unit: 16 token rows of 128 B
constexpr int kAPages = kABytes / kPageBytes;  // 8 pages of weights per K step
constexpr int kMaxStepPages = kAPages + 256 * 128 / kPageBytes;  // 24: weights + 256 token rows
constexpr int kTwoSlicePages = 32;  // two K slices per ring step up to here, when the ring holds 4 slices
constexpr int kMaxPages = 112;
constexpr int kQMaxStepPages = 8 + 1 + 2 * (256 * 128 / 2048);  // 41: codes, scales, 2 token boxes (at most)
constexpr int kTickets = 32;                   // K steps in flight at most (barrier pairs)
constexpr int kSmemLimit = 232448;             // 227 KB opt-in per CTA
constexpr int kXchgStride = 33;                // fp32 exchange row stride (bank-conflict free)
constexpr int kQueue = 4;                      // work-item queue depth (producer -> MMA, epilogue)
constexpr int kReadyWords = (kMaxExperts + 1 + 31) / 32;  // one bit per group: its h rows are complete

struct PhaseMaps {
    CUtensorMap a0, a1;       // routed A: gate/up W_gate, W_up as [E*I, H]; down W_down as [E*H, I] (a1 unused)
    CUtensorMap s0, s1;       // shared A: gate/up ws_gate, ws_up [Is, H]; down ws_down [H, Is] (s1 unused)
    CUtensorMap b[kNumBox];   // routed activations [T*k, K], box heights 16 << i
    CUtensorMap bs[kNumBox];  // shared activations [T, K]
};

// The token copies of one ring step, which the producer hands the loader warp
// (single CTAs): n slices of `map` at (x + 64 j, y) into dst + j * dst_step;
// with block-scaled weights also the step's two runs of block scales,
// sc_bytes each from sc_src[i] to sc_dst + i * sc_bytes.
struct LoadDesc {
    const CUtensorMap *map;
    const uint8_t *sc_src[2];
    uint32_t dst, dst_step;
    int x, y;
    int n;
    int fence;  // 1: the slices are h rows other CTAs wrote (a proxy fence first)
    uint32_t sc_dst, sc_bytes;  // sc_bytes 0: no scale runs
};

struct __align__(64) FfnMaps {
    PhaseMaps ph[2];  // [0] gate/up, [1] down
};

struct FfnParams {
    int T, H, E, I, k, Is;
    int BN;             // token tile of the routed experts (power of two, 32..256)
    int BNs;            // token tile of the shared expert (power of two, 32..BN)
    int pages;          // shared-memory ring size in kPageBytes pages (>= kMaxStepPages)
    int phases;         // bit 0: gate/up items, bit 1: down items
    int R[2], Rs[2];    // weight tiles per routed / shared expert, per phase
    int nk[2], nks[2];  // K steps routed / shared, per phase
    // block-scaled weights only: the packed block scales of each matrix, [phase][0:
    // gate or down, 1: up], routed and shared; one run (qscale_run bytes) per
    // (64-row group, 128-wide K step), row-group major (moe_mxfp8_pack_scales,
    // moe_nvfp4_pack_scales)
    const uint8_t *sf[2][2];
    const uint8_t *sfs[2][2];
    // NVFP4 only: the fp32 matrix scales, [phase][0: gate or down, 1: up] with
    // one per expert, and the shared expert's {gate, up, down}
    const float *ts[2][2];
    const float *tss;
    // the group-readiness wait's limit (kWaitLimitNs), and a group whose
    // readiness target is one past what its gate/up items can reach (-1: none)
    // -- both only changed by the test hooks MOE_TEST_WAIT_LIMIT_US and
    // MOE_TEST_STALL_GROUP, to make a wait run out on purpose
    unsigned long long wait_limit_ns;
    int stall_group;
    const int32_t *offsets;
    const int32_t *perm;
    const float *topk_w;
    const float *sgate;
    uint16_t *h_perm;    // [T*k, I]
    uint16_t *h_shared;  // [T, Is]
    uint16_t *ybuf;      // [T, k+1, H]
    int32_t *status;     // status word
    int32_t *sched;      // [0] items claimed, [1] CTAs done; zero between launches
    int32_t *hdone;      // [E+2] finished gate/up items per group (E = shared), [E+1] in all; zero between launches
};

// ------------------------------------------------------------ scheduling --
struct Item {
    int ph;      // 0 gate/up, 1 down
    int shared;  // 1: shared expert
    int e;       // routed expert
    int r;       // weight tile
    int row0;    // first activation row of the token tile
    int nvalid;  // valid tokens in the tile (1..BN)
    int ntt;     // token tiles of the group
    int m;       // weight tiles r .. r+m-1 in this item (2: a down item of a group of <= BN/2 tokens)
};

struct ItemSlot {  // one work-item queue entry: the item number and its decoded form
    int item;        // -1: no more items
    Item it;
};

struct Schedule {
    int n[2];              // items per phase (0 when the phase is not run)
    int sh0, sh1;          // of which the shared expert's, per phase (they come first)
    int shared_ntt;        // token tiles of the shared expert (0 if none)
    int merge;             // down items of small groups take two weight tiles
    int shared_merge;      // the shared expert's down items take two weight tiles
    const int *tile_base;  // [E+1] prefix of token tiles over routed experts (shared memory)
    const int *dbase;      // [E+1] prefix of down items over routed experts when merging (shared memory)
    const int *offs;       // [E+1] dispatch offsets (shared memory)
};

// Down items of a group with `cnt` tokens.  When the down phase has plenty of
// items (`merge`: at least kMergePerCta per CTA), a group that fits half a
// token tile takes two weight tiles per item (two accumulators side by side
// in TMEM, one token box read for both): half the items, each twice as long.
// With few items the shorter ones balance the launch better.  Without
// merging a group has ntt * R1 down items (token tiles x weight tiles).
constexpr int kMergePerCta = 8;
__device__ __forceinline__ bool down_merged(int cnt, int BN, bool merge) {
    return merge && cnt > 0 && cnt <= (BN >> 1);
}
__device__ __forceinline__ int merged_down_items(int cnt, int BN, int R1) {
    return down_merged(cnt, BN, true) ? (R1 + 1) >> 1 : ((cnt + BN - 1) / BN) * R1;
}

// Work item -> (phase, group, weight tile(s), token tile).  Phase 0 items of a
// group: weight tile outer, token tile inner; phase 1 the same, or pairs of
// weight tiles for a merged group.
__device__ __forceinline__ Item decode_item(int item, const Schedule &sc, const FfnParams &p) {
    Item it;
    it.m = 1;
    it.ph = item < sc.n[0] ? 0 : 1;
    if (it.ph) item -= sc.n[0];
    const int sh_items = it.ph ? sc.sh1 : sc.sh0;
    if (item < sh_items) {  // the shared expert's items first (they are the longest)
        it.shared = 1;
        it.e = p.E;
        it.ntt = sc.shared_ntt;
        if (it.ph == 1 && sc.shared_merge) {
            it.r = 2 * item;
            it.m = min(2, p.Rs[1] - it.r);
            it.row0 = 0;
            it.nvalid = p.T;
        } else {
            const int j = item % sc.shared_ntt;
            it.r = item / sc.shared_ntt;
            it.row0 = j * p.BNs;
            it.nvalid = min(p.BNs, p.T - j * p.BNs);
        }
        return it;
    }
    item -= sh_items;
    // largest e whose first item is <= item: tile_base[e] * R (phase 0, or phase 1
    // unmerged), dbase[e] (phase 1 merged)
    const bool by_dbase = it.ph == 1 && sc.merge;
    const int R = p.R[it.ph];
    const int *base = by_dbase ? sc.dbase : sc.tile_base;
    const int scale = by_dbase ? 1 : R;
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (base[mid] * scale <= item) lo = mid;
        else hi = mid - 1;
    }
    const int cnt = sc.offs[lo + 1] - sc.offs[lo];
    const int ntt = (cnt + p.BN - 1) / p.BN;
    const int local = item - base[lo] * scale;
    it.shared = 0;
    it.e = lo;
    it.ntt = ntt;
    if (it.ph == 1 && down_merged(cnt, p.BN, sc.merge)) {
        it.r = 2 * local;
        it.m = min(2, p.R[1] - it.r);
        it.row0 = sc.offs[lo];
        it.nvalid = cnt;
    } else {
        const int j = local % ntt;
        it.r = local / ntt;
        it.row0 = sc.offs[lo] + j * p.BN;
        it.nvalid = min(p.BN, cnt - j * p.BN);
    }
    return it;
}

// Exclusive block scan over the experts of two counts at once:
// a[e] = sum_{e' < e} f(e').x, b[e] likewise with .y; a[E], b[E] = the totals.
// Every thread of the block calls it.
template <int NT, class F>
__device__ __forceinline__ void expert_scan2(int E, int *a, int *b, int2 *scan_tmp, F f) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per = (E + NT - 1) / NT;
    const int e0 = threadIdx.x * per, e1 = min(E, e0 + per);
    int2 local = make_int2(0, 0);
    for (int e = e0; e < e1; ++e) {
        const int2 v = f(e);
        local.x += v.x;
        local.y += v.y;
    }
    scan_tmp[threadIdx.x] = local;
    __syncthreads();
    if (warp == 0) {  // NT partials, NT / 32 per lane
        int2 v[NT / 32];
        int2 sum = make_int2(0, 0);
#pragma unroll
        for (int q = 0; q < NT / 32; ++q) {
            v[q] = scan_tmp[lane * (NT / 32) + q];
            sum.x += v[q].x;
            sum.y += v[q].y;
        }
        int2 incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, incl.x, o), y = __shfl_up_sync(0xffffffffu, incl.y, o);
            if (lane >= o) {
                incl.x += x;
                incl.y += y;
            }
        }
        int2 run = make_int2(incl.x - sum.x, incl.y - sum.y);
#pragma unroll
        for (int q = 0; q < NT / 32; ++q) {
            scan_tmp[lane * (NT / 32) + q] = run;
            run.x += v[q].x;
            run.y += v[q].y;
        }
    }
    __syncthreads();
    int2 run = scan_tmp[threadIdx.x];
    for (int e = e0; e < e1; ++e) {
        a[e] = run.x;
        b[e] = run.y;
        const int2 v = f(e);
        run.x += v.x;
        run.y += v.y;
    }
    if (e1 == E && e0 < e1) {
        a[E] = run.x;
        b[E] = run.y;
    }
    __syncthreads();
}

// Next K step of `need` pages.  `vhead` counts pages without wrapping,
// `off` is its position in the ring (vhead mod P, kept without a division).
// A step never straddles the ring end: the pages left before the end are
// skipped and belong to this step.  Returns the step's first ring page.  The
// producer and the MMA lane call this on the same sequence of steps.
__device__ __forceinline__ uint32_t ring_alloc(uint32_t &vhead, uint32_t &off, uint32_t need, uint32_t P) {
    if (off + need > P) {
        vhead += P - off;
        off = 0;
    }
    const uint32_t first = off;
    vhead += need;
    off += need;
    return first;
}

__device__ __forceinline__ int box_index(int nvalid) {  // smallest box of 16 << b rows holding the tile
    int b = 0;
    while ((16 << b) < nvalid) ++b;
    return b;
}

// Ring steps of an item.  A sub-step is one 64-wide K slice: 16 KB of
// weights per weight tile of the item (m of them) followed by one token box
// of 16 << bi rows (sub_pages pages).  A ring step carries ns sub-steps --
// two while they take at most kMaxStepPages pages, or at most kTwoSlicePages
// with room for two such steps in the ring -- so the per-step work of the
// producer and MMA lanes (a barrier round trip each, some hundreds of cycles)
// is spent once per 32 KB of weights.  Measured: wide tiles (a 256-token
// tile of a CTA pair, 16 pages a slice) ran their K loop 15% faster with two
// slices per step.
// A CTA pair splits a tile's MMA N (the valid tokens rounded up to 16) in two
// halves, one per CTA.
__device__ __forceinline__ int pair_half(int nvalid) { return ((nvalid + 15) & ~15) >> 1; }

struct StepShape {
    int bi;              // token box index
    uint32_t sub_pages;  // pages per sub-step
    int ns;              // sub-steps per ring step (the item's last step may hold fewer)
    int nk;              // 64-wide K slices of the item
};
template <bool kPair = false>
__device__ __forceinline__ StepShape step_shape(const Item &it, const FfnParams &p) {
    StepShape sh;
    sh.bi = box_index(kPair ? pair_half(it.nvalid) : it.nvalid);
    sh.sub_pages = (uint32_t)it.m * kAPages + (1u << sh.bi);
    const uint32_t two = 2 * sh.sub_pages;
    sh.ns = (two <= (uint32_t)kMaxStepPages || (two <= (uint32_t)kTwoSlicePages && 2 * two <= (uint32_t)p.pages)) ? 2 : 1;
    sh.nk = it.shared ? p.nks[it.ph] : p.nk[it.ph];
    return sh;
}

// Block-scaled ring step: 128 K elements -- the codes of one weight tile
// (MXFP8 8 pages, NVFP4 4), their scales (one page: 512 or 1024 bytes used)
// and the token rows as two bf16 boxes of 64 K (sub_pages = 2^bi pages
// each).  ns = 2 slices, nk counts 64-wide slices (even: K is a multiple of
// 128).
__device__ __forceinline__ StepShape qstep_shape(const Item &it, const FfnParams &p) {
    StepShape sh;
    sh.bi = box_index(it.nvalid);
    sh.sub_pages = 1u << sh.bi;
    sh.ns = 2;
    sh.nk = it.shared ? p.nks[it.ph] : p.nk[it.ph];
    return sh;
}
template <int kFmt>
__device__ __forceinline__ uint32_t qstep_pages(const StepShape &sh) {
    return qcode_pages<kFmt>() + 1 + 2 * sh.sub_pages;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + __expf(-g)); }

// ------------------------------------------------- MXFP8 weight conversion --
// An MXFP8 weight is an E4M3 code times its block's power of two 2^se (one
// UE8M0 scale per 32 consecutive K elements).  Every such value with se in
// [-117, 119] is a bf16 value, so the conversion below is exact and the MMA
// then runs on exactly the weights the format stands for.
//
// Two codes at once, bf16x2: the code's sign goes to bit 15 of its 16-bit
// lane and its 7 magnitude bits (eeee mmm) to bits 10..4, i.e. the low four
// exponent bits and the top three mantissa bits of a bf16.  As a bf16 that
// lane is 2^(e - 127) * 1.mmm for e > 0 and the subnormal 0.mmm * 2^-126 for
// e = 0; one multiply by 2^(120 + se) makes both the code's value
// (2^(e - 7) * 1.mmm, or 0.mmm * 2^-6) times 2^se.  The byte permute with
// sign replication puts each code's sign in the high byte of its lane, the
// shift and mask keep bit 15 and bits 10..4.
__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t e4m3x2_lanes(uint32_t w, uint32_t sel) {
    return (prmt_b32(w, 0u, sel) << 4) & 0x87F087F0u;
}

// 16 codes (one 16-byte chunk) -> 16 bf16 (two chunks): each pair of codes
// as two bf16 lanes, times the bf16x2 multiplier m.
__device__ __forceinline__ void e4m3x16_times(const uint4 &q, uint32_t m, uint32_t (&r)[8]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        r[2 * i] = bf16x2_mul(e4m3x2_lanes(w[i], 0x9180u), m);      // codes 4i, 4i + 1
        r[2 * i + 1] = bf16x2_mul(e4m3x2_lanes(w[i], 0xB3A2u), m);  // codes 4i + 2, 4i + 3
    }
}
// bf16x2 of 2^(120 + se) from the UE8M0 code sc = se + 127, sc <= 134: the
// exponent field sc + 120 in both halves, one multiply-add.
__device__ __forceinline__ uint32_t mx_mult(uint32_t sc) { return sc * 0x00800080u + 120u * 0x00800080u; }

// One converter thread's share of a ring step.  The step's weight tile is 128
// rows x 128 E4M3 codes as TMA left them (row r at r * 128 bytes, 16-byte chunk
// c at (c ^ (r & 7)) * 16: the 128-byte swizzle) with row r's four UE8M0 scales
// at byte 4r.  The thread turns row r into 128 bf16, two consecutive K per
// 32-bit column (the lower K in the low half), and stores them to 64 columns of
// TMEM lane r: the MMA's A operand.  The 8 lanes of a shared-memory phase read
// one chunk index of 8 consecutive rows, which the swizzle puts in 8 distinct
// 16-byte bank groups.  A block scale above 2^7 needs two multiplies; a warp
// takes that path only when one of its blocks needs it.
__device__ __forceinline__ void convert_mxfp8_row(uint32_t codes, uint32_t scales, int r, uint32_t taddr) {
    uint4 q[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(q[j].x), "=r"(q[j].y), "=r"(q[j].z), "=r"(q[j].w)
                     : "r"(codes + (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4))));
    uint32_t s4;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(s4) : "r"(scales + (uint32_t)(r * 4)));
    uint32_t sc[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) sc[b] = (s4 >> (8 * b)) & 0xffu;
    const bool fast = __all_sync(0xffffffffu, sc[0] <= 134u && sc[1] <= 134u && sc[2] <= 134u && sc[3] <= 134u);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t o[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t c = sc[2 * h + (j >> 1)];
            uint32_t t[8];
            if (fast) {
                e4m3x16_times(q[4 * h + j], mx_mult(c), t);
            } else {  // 2^(120 + se) as 2^127 (or 2^(120 + se) itself) times 2^(se - 7) (or 1)
                const bool one = c <= 134u;
                const uint32_t m1 = one ? (c + 120u) << 7 : 254u << 7, m2 = one ? 127u << 7 : (c - 7u) << 7;
                e4m3x16_times(q[4 * h + j], m1 | (m1 << 16), t);
#pragma unroll
                for (int i = 0; i < 8; ++i) t[i] = bf16x2_mul(t[i], m2 | (m2 << 16));
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) o[8 * j + i] = t[i];
        }
        tmem_st32(taddr + (uint32_t)(32 * h), o);
    }
}

// ------------------------------------------------- NVFP4 weight conversion --
// An NVFP4 weight is an E2M1 code c (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6)
// times its block's E4M3 scale s (one per 16 consecutive K elements), times
// the matrix's fp32 scale, which the epilogue applies.  c * s has at most 6
// significant bits and lies in [2^-10, 2688]: a bf16 value, so the
// conversion is exact.
//
// The hardware unpacks two codes into f16x2 exactly.  The f16 of a nonzero c
// is normal with its 9 low mantissa bits zero, so shifting the pair right by
// 3 and clearing the bits the signs leave behind gives, read as bf16x2, the
// magnitudes c * 2^-112 (exponent rebiased from 15 to 127).  One multiply by
// the block's 2^112 * s (at most 2^121: no overflow) makes c * s; the signs
// are put back last.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}
__device__ __forceinline__ uint32_t e2m1_f16x2_times(uint32_t x, uint32_t m) {
    return bf16x2_mul((x >> 3) & 0x0FFF0FFFu, m) | (x & 0x80008000u);
}
// bf16x2 of 2^112 * s for the two E4M3 scales in bytes 0 and 2 of `two`:
// each byte's 7 magnitude bits placed at bits 10..4 of its lane read as
// s * 2^-120 (the subnormal scales as bf16 subnormals), and two exact
// multiplies by 2^116 follow.  Block scales are never negative.
__device__ __forceinline__ uint32_t nv_mult2(uint32_t two) {
    constexpr uint32_t c116 = ((127u + 116u) << 7) * 0x00010001u;
    return bf16x2_mul(bf16x2_mul(two << 4, c116), c116);
}

// One converter thread's share of an NVFP4 ring step.  The step's weight tile
// is 128 rows x 64 bytes of codes (128 K, two codes a byte, the lower K in the
// low nibble) as TMA left them with the 64-byte swizzle (row r at r * 64,
// 16-byte chunk c at (c ^ ((r >> 1) & 3)) * 16), and row r's eight E4M3 block
// scales at byte 8r.  The thread turns row r into 128 bf16 and stores them to
// 64 columns of TMEM lane r, as convert_mxfp8_row does.  The 8 lanes of a
// shared-memory phase read one chunk index of 8 consecutive rows, which the
// swizzle puts in 8 distinct 16-byte bank groups.
__device__ __forceinline__ void convert_nvfp4_row(uint32_t codes, uint32_t scales, int r, uint32_t taddr) {
    uint4 q[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(q[j].x), "=r"(q[j].y), "=r"(q[j].z), "=r"(q[j].w)
                     : "r"(codes + (uint32_t)(r * 64 + ((j ^ ((r >> 1) & 3)) << 4))));
    uint32_t s0, s1;  // block scales 0..3, 4..7
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(s0), "=r"(s1) : "r"(scales + (uint32_t)(r * 8)));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t o[32];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int j = 2 * h + jj;  // chunk j: K 32 j .. 32 j + 31, blocks 2 j and 2 j + 1
            const uint32_t m2 = nv_mult2(prmt_b32(j < 2 ? s0 : s1, 0u, (j & 1) ? 0x4342u : 0x4140u));
            const uint32_t ma = prmt_b32(m2, 0u, 0x1010u), mb = prmt_b32(m2, 0u, 0x3232u);
            const uint32_t w[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // word i: K 32 j + 8 i .. + 7
                uint32_t x[4];
                e2m1x8_to_f16x2(w[i], x);
#pragma unroll
                for (int t = 0; t < 4; ++t) o[16 * jj + 4 * i + t] = e2m1_f16x2_times(x[t], i < 2 ? ma : mb);
            }
        }
        tmem_st32(taddr + (uint32_t)(32 * h), o);
    }
}

// Down item, token n of the tile: its ybuf row (t*(k+1) + j, or t*(k+1) + k for
// the shared expert) and the weight applied to it.
__device__ __forceinline__ void down_dest(const Item &it, int n, const FfnParams &p, int &mrow, float &mw) {
    mrow = 0;
    mw = 0.f;
    if (n >= it.nvalid) return;
    if (it.shared) {
        const int t = it.row0 + n;
        mrow = t * (p.k + 1) + p.k;
        mw = __ldg(p.sgate + t);
    } else {
        const int slot = __ldg(p.perm + it.row0 + n);
        if (kDebugBounds && (slot < 0 || slot >= p.T * p.k)) {  // skip the token's store
            atomicOr(p.status, MOE_STATUS_BOUNDS);
            mrow = -1;
            return;
        }
        mrow = slot + slot / p.k;  // t*(k+1) + j
        mw = __ldg(p.topk_w + slot);
    }
}

// --------------------------------------------------------------- kernel --
// kFmt: 0 bf16 weights; 1 MXFP8 weights (E4M3 codes + UE8M0 block scales);
// 2 NVFP4 weights (E2M1 codes + E4M3 block scales + an fp32 scale per
// matrix).  Block-scaled weights are converted to bf16 in tensor memory by
// kConvWarps converter warps (single CTAs only).
template <bool kPair, int kFmt>
__global__ void __launch_bounds__(kFmt ? kThreadsQ : kThreads, 1)
    ffn_kernel(const __grid_constant__ FfnMaps maps, const FfnParams p) {
    constexpr int NT = kFmt ? kThreadsQ : kThreads;
    static_assert(!(kPair && kFmt), "block-scaled weights run on single CTAs");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t P = (uint32_t)p.pages;
    uint8_t *ring = smem;
    float *xchg = reinterpret_cast<float *>(ring + (size_t)P * kPageBytes);
    int *tile_base = reinterpret_cast<int *>(xchg + 64 * kXchgStride);  // [E + 1]
    int *dbase = tile_base + (p.E + 1);                                 // [E + 1]
    int *offs = dbase + (p.E + 1);                                      // [E + 1]
    uint64_t *bars = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(offs + (p.E + 1)) + 7) & ~uintptr_t(7));
    uint64_t *full = bars, *empty = bars + kTickets, *tfull = bars + 2 * kTickets, *tempty = tfull + 2;
    uint64_t *mma_done = tfull + 4;
    uint64_t *qfull = tfull + 5, *qempty = qfull + kQueue;
    // block-scaled weights: conversion buffer (in TMEM) converted / free
    // block-scaled weights: TMEM conversion buffer converted (a buffer is free again
    // once the MMAs of the last step that used it are done: that step's empty barrier)
    uint64_t *cfull = qempty + kQueue;
    uint64_t *armed = cfull + kConvBufs;  // [kTickets] single CTAs: a step's token copies handed to the loader
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(armed + kTickets);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_flag = reinterpret_cast<volatile int *>(tmem_slot + 2);  // elected -> epilogue: 0 go, -1 stop
    ItemSlot *qdesc = reinterpret_cast<ItemSlot *>(tmem_slot + 4);  // [kQueue], written by the producer
    ItemSlot *epi_desc = qdesc + kQueue;                             // the epilogue's current item
    ItemSlot *conv_desc = epi_desc + 1;                              // [2] each converter group's current item
    int *scan_tmp = reinterpret_cast<int *>(                          // [2 * NT] (int2 partials)
        (reinterpret_cast<uintptr_t>(conv_desc + 2) + 7) & ~uintptr_t(7));
    uint32_t *ready_bits = reinterpret_cast<uint32_t *>(scan_tmp + 2 * NT);  // [kReadyWords], producer-private
    uint32_t *ticket_start = ready_bits + kReadyWords;  // [kTickets] first ring page (virtual) of each step; producer-private
    LoadDesc *ldesc = reinterpret_cast<LoadDesc *>(                    // [kTickets] producer -> loader
        (reinterpret_cast<uintptr_t>(ticket_start + kTickets) + 7) & ~uintptr_t(7));
    volatile int *stop_at = reinterpret_cast<volatile int *>(ldesc + kTickets);  // steps the producer armed, at its exit
    volatile int *loader_done = stop_at + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tmem_cols = kFmt ? 512 : 2 * p.BN;  // block-scaled weights: accumulators, then the conversion buffers
    const uint32_t rank = kPair ? cluster_ctarank() : 0u;  // 0: the pair's MMA issuer
    pdl_launch_dependents();

    // ---- setup: barriers, TMEM, tile schedule
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTickets; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&armed[s], 1);
        }
        *stop_at = 0x7fffffff;
        *loader_done = 0;
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], kPair ? 2 : 1);  // pair: both CTAs' epilogues
        }
        mbar_init(mma_done, 1);
        for (int q = 0; q < kQueue; ++q) {
            mbar_init(&qfull[q], 1);
            // the MMA lane and the elected epilogue thread (pair: and the other CTA's
            // producer and epilogue; block-scaled weights: and the two converter groups'
            // elected threads)
            mbar_init(&qempty[q], kPair ? 4 : (kFmt ? 4 : 2));
        }
        for (int b = 0; b < kConvBufs; ++b) mbar_init(&cfull[b], kConvWarps / 2);  // one arrival per warp of the converting group
        *abort_flag = 0;
        for (int w = 0; w < kReadyWords; ++w) ready_bits[w] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        for (int ph = 0; ph < 2; ++ph)
            if ((p.phases >> ph) & 1) {
                prefetch_tmap(&maps.ph[ph].a0);
                prefetch_tmap(&maps.ph[ph].s0);
            }
        if (p.phases & 1) {
            prefetch_tmap(&maps.ph[0].a1);
            prefetch_tmap(&maps.ph[0].s1);
        }
    }
    if (warp == 1) {
        if constexpr (kPair) {  // both CTAs' warp 1, same address: one allocation mirrored in the pair
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_slot)),
                         "r"(tmem_cols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_slot)),
                         "r"(tmem_cols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
        tc_fence_before();
    }
    if constexpr (kPair) cluster_sync();  // both CTAs' barriers initialised before any cross-CTA arrive
    pdl_wait();  // the dispatch outputs and activations are ready past this point
    // the producer's first claim, issued now so that its round trip overlaps the
    // schedule set-up below (the counter is zero here: the previous launch's last
    // CTA, or the dispatch kernel, left it so)
    int first_claim = 0;
    if (warp == 0 && lane == 0 && (!kPair || rank == 0)) first_claim = atomicAdd(p.sched, 1);
    // dispatch offsets to shared memory, then the per-expert prefix sums of token
    // tiles and of down items
    for (int e = threadIdx.x; e <= p.E; e += NT) offs[e] = __ldg(p.offsets + e);
    __syncthreads();
    if constexpr (kDebugBounds) {
        // the offsets must be a prefix sum from 0 to at most T*k; otherwise no
        // routed item runs (every CTA reads the same offsets and decides alike)
        bool bad = false;
        for (int e = threadIdx.x; e <= p.E; e += NT)
            bad |= (e == 0 && offs[0] != 0) || (e < p.E && offs[e] > offs[e + 1]) ||
                   (e == p.E && offs[e] > p.T * p.k);
        if (__syncthreads_or(bad)) {
            if (threadIdx.x == 0) atomicOr(p.status, MOE_STATUS_BOUNDS);
            for (int e = threadIdx.x; e <= p.E; e += NT) offs[e] = 0;
            __syncthreads();
        }
    }
    Schedule sc;
    sc.shared_ntt = p.Is > 0 ? (p.T + p.BNs - 1) / p.BNs : 0;
    {
        const int BN = p.BN, R1 = p.R[1];
        const int *o = offs;
        expert_scan2<NT>(p.E, tile_base, dbase, reinterpret_cast<int2 *>(scan_tmp), [=](int e) {
            const int cnt = o[e + 1] - o[e];
            return make_int2((cnt + BN - 1) / BN, merged_down_items(cnt, BN, R1));
        });
        // every CTA takes the same decision from the same offsets
        sc.merge = !kPair && kFmt == 0 &&
                   (tile_base[p.E] * R1 + p.Rs[1] * sc.shared_ntt) >= kMergePerCta * (int)gridDim.x;
    }
    tc_fence_after();
    sc.shared_merge = p.Is > 0 && sc.shared_ntt == 1 && down_merged(p.T, p.BN, sc.merge);
    sc.tile_base = tile_base;
    sc.dbase = dbase;
    sc.offs = offs;
    sc.sh0 = p.Rs[0] * sc.shared_ntt;
    sc.sh1 = sc.shared_merge ? (p.Rs[1] + 1) >> 1 : p.Rs[1] * sc.shared_ntt;
    sc.n[0] = (p.phases & 1) ? sc.sh0 + tile_base[p.E] * p.R[0] : 0;
    sc.n[1] = (p.phases & 2) ? sc.sh1 + (sc.merge ? dbase[p.E] : tile_base[p.E] * p.R[1]) : 0;
    const int total_items = sc.n[0] + sc.n[1];
    const bool fused = p.phases == 3;
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ================= TMA producer =================
        if (lane == 0) {
            uint32_t vhead = 0, off = 0;       // ring pages handed out (virtual: never wraps) / its ring position
            uint32_t issued = 0, retired = 0;  // K steps issued / whose MMAs have released their pages
            uint32_t oldest = 0;               // first page (virtual) of step `retired` while one is in flight
            // expert weights: evict-first where a weight tile is read once (a group of
            // one token tile).  A routed group of several token tiles reads each weight
            // tile once per token tile, so its loads keep the normal policy and the
            // repeats hit L2 (a 32-expert, 512-tokens-per-expert gate/up read 2.4
            // instead of 3.7 GB from DRAM).
            const uint64_t wpol = policy_evict_first();
            const uint64_t bpol = policy_evict_normal();  // token rows (pair loads take a policy)
            // Items are claimed from the counter, one ahead: the next claim's atomic
            // is issued when an item is taken, so its round trip overlaps that item's
            // loads.  Every item, the first included, comes from the counter, so the
            // items claimed so far are exactly those of CTAs that are running: a down
            // item waits only on gate/up items that running CTAs hold, even when not
            // every CTA of the grid is resident at once.
            int pending = first_claim;  // counter value of the claim in flight
            bool all_ready = false;     // every gate/up item of the launch is done
            for (int li = 0;; ++li) {
                const int slot = li % kQueue;
                const uint32_t qph = (uint32_t)(li / kQueue) & 1u;
                int item;
                Item it{};
                if (!kPair || rank == 0) {
                    if (!mbar_wait<kPair>(&qempty[slot], qph ^ 1u, abort_flag, p.status, true)) break;
                    item = pending;
                    if (item >= total_items) item = -1;
                    if (item >= 0) pending = atomicAdd(p.sched, 1);  // latency overlaps this item's loads
                    if (item >= 0) it = decode_item(item, sc, p);  // decoded once, for all roles
                    qdesc[slot].item = item;
                    qdesc[slot].it = it;
                    if constexpr (kPair) {  // the same entry in the other CTA's queue, then its qfull
                        const uint32_t *src = reinterpret_cast<const uint32_t *>(&qdesc[slot]);
                        const uint32_t dst = mapa(smem_u32(&qdesc[slot]), 1);
#pragma unroll
                        for (int w = 0; w < (int)(sizeof(ItemSlot) / 4); ++w) st_cluster_u32(dst + 4 * w, src[w]);
                        mbar_arrive_cluster(mapa(smem_u32(&qfull[slot]), 1));
                    }
                    mbar_arrive(&qfull[slot]);
                } else {  // the other CTA of a pair takes the item CTA 0 published
                    if (!mbar_wait<true>(&qfull[slot], qph, abort_flag, p.status, true)) break;
                    item = qdesc[slot].item;
                    it = qdesc[slot].it;
                    mbar_arrive_cluster(mapa(smem_u32(&qempty[slot]), 0));
                }
                if (item < 0) break;
                const int grp = it.shared ? p.E : it.e;
                const bool stalled = grp == p.stall_group;
                if (fused && it.ph == 1 && (!all_ready || stalled) && !((ready_bits[grp >> 5] >> (grp & 31)) & 1u)) {
                    // wait until every gate/up tile of the group has stored its h rows
                    // (or every gate/up item of the launch is done)
                    const int32_t *flag = p.hdone + grp;
                    const int target = (it.shared ? p.Rs[0] : p.R[0]) * it.ntt + (stalled ? 1 : 0);
                    auto check = [&]() {
                        const int all = ld_acquire(p.hdone + p.E + 1), mine = ld_acquire(flag);
                        if (!stalled && all >= sc.n[0]) all_ready = true;
                        return (all_ready && !stalled) || mine >= target;
                    };
                    bool ready = check();
                    const unsigned long long t0 = ready ? 0ull : globaltimer();
                    for (uint32_t spin = 1; !ready; ++spin) {
                        ready = check();
                        if (!ready && (spin & 63u) == 0) {
                            if (*abort_flag) break;
                            if (globaltimer() - t0 > p.wait_limit_ns) {
                                *abort_flag = 1;
                                atomicOr(p.status, MOE_STATUS_TIMEOUT);
                                break;
                            }
                        }
                    }
                    if (!ready) break;
                    ready_bits[grp >> 5] |= 1u << (grp & 31);  // counts only grow within a launch
                    fence_proxy_async_global();  // the TMA loads below read h written by other CTAs
                }
                const PhaseMaps &pm = maps.ph[it.ph];
                const CUtensorMap *ma0 = it.shared ? &pm.s0 : &pm.a0;
                const CUtensorMap *ma1 = it.shared ? &pm.s1 : &pm.a1;
                const StepShape sh = kFmt ? qstep_shape(it, p) : step_shape<kPair>(it, p);
                constexpr int kCP = qcode_pages<kFmt>(), kRun = qscale_run<kFmt>();
                const CUtensorMap *mb = it.shared ? &pm.bs[sh.bi] : &pm.b[sh.bi];
                // pair: this CTA's weight tile of the two, and its half of the token rows
                const int rt = kPair ? 2 * it.r + (int)rank : it.r;
                const int a_row = it.ph == 0 ? (it.shared ? 0 : it.e * p.I) + rt * 64
                                             : (it.shared ? 0 : it.e * p.H) + rt * kTileM;
                const int b_row = it.row0 + (kPair ? (int)rank * pair_half(it.nvalid) : 0);
                const uint64_t apol = (it.ntt > 1 && !it.shared) ? bpol : wpol;
                bool ok = true;
                for (int k0 = 0; k0 < sh.nk; k0 += sh.ns) {
                    const int nsub = min(sh.ns, sh.nk - k0);
                    const uint32_t need = kFmt ? qstep_pages<kFmt>(sh) : (uint32_t)nsub * sh.sub_pages;
                    const uint32_t first = ring_alloc(vhead, off, need, P);
                    // Free a ticket and the pages of this step: retire the oldest steps
                    // until the steps in flight and this one lie within P consecutive
                    // (virtual) pages -- then no two of them share a physical page.
                    while (issued != retired && (vhead - oldest > P || issued - retired >= (uint32_t)kTickets)) {
                        if (!mbar_wait_fast<kPair>(&empty[retired % kTickets], (retired / kTickets) & 1u, abort_flag,
                                            p.status, true)) {
                            ok = false;
                            break;
                        }
                        ++retired;
                        oldest = ticket_start[retired % kTickets];  // read only while retired != issued
                    }
                    if (!ok) break;
                    const uint32_t tk = issued % kTickets;
                    if (issued == retired) oldest = vhead - need;
                    ticket_start[tk] = vhead - need;
                    if constexpr (kFmt != 0) {
                        // codes of the weight tile, their scales, two token boxes
                        mbar_arrive_expect_tx(&full[tk], (kCP + 2 * sh.sub_pages) * kPageBytes + 2 * kRun);
                        uint8_t *sA = ring + (size_t)first * kPageBytes;
                        const int kx = k0 * kBlockK;  // = 128 * (K step)
                        const int kc = kFmt == 2 ? kx / 2 : kx;  // the codes' byte column
                        const int ks = k0 >> 1;
                        tma_load_2d_hint(ma0, &full[tk], sA, kc, a_row, apol);  // gate: 64 rows; down: 128 rows
                        if (it.ph == 0) tma_load_2d_hint(ma1, &full[tk], sA + kCP * kPageBytes / 2, kc, a_row, apol);
                        uint8_t *sS = sA + kCP * kPageBytes;
                        const size_t ksteps = (size_t)(sh.nk >> 1);
                        const size_t rg = (size_t)(a_row >> 6);  // 64-row group of the tile's first row
                        const uint8_t *const *sfp = it.shared ? p.sfs[it.ph] : p.sf[it.ph];
                        // the two runs of block scales (gate/up: the gate and the up rows;
                        // down: the tile's two 64-row groups) and the two token slices:
                        // the loader's
                        ldesc[tk] = LoadDesc{mb,
                                             {sfp[0] + (rg * ksteps + ks) * kRun,
                                              it.ph == 0 ? sfp[1] + (rg * ksteps + ks) * kRun
                                                         : sfp[0] + ((rg + 1) * ksteps + ks) * kRun},
                                             smem_u32(sS + kPageBytes),
                                             sh.sub_pages * kPageBytes,
                                             kx,
                                             it.row0,
                                             2,
                                             it.ph == 1,
                                             smem_u32(sS),
                                             (uint32_t)kRun};
                    } else if constexpr (kPair) {
                        // both CTAs' loads complete on CTA 0's barrier, armed there with both halves
                        if (rank == 0) mbar_arrive_expect_tx(&full[tk], 2 * need * kPageBytes);
                        const uint32_t bar0 = mapa(smem_u32(&full[tk]), 0);
                        for (int j = 0; j < nsub; ++j) {
                            uint8_t *sA = ring + (size_t)(first + j * sh.sub_pages) * kPageBytes;
                            const int kx = (k0 + j) * kBlockK;
                            if (it.ph == 0) {
                                tma_load_2d_pair(ma0, bar0, sA, kx, a_row, apol);
                                tma_load_2d_pair(ma1, bar0, sA + kABytes / 2, kx, a_row, apol);
                            } else {
                                tma_load_2d_pair(ma0, bar0, sA, kx, a_row, apol);
                            }
                            tma_load_2d_pair(mb, bar0, sA + kABytes, kx, b_row, bpol);
                        }
                    } else {
                        mbar_arrive_expect_tx(&full[tk], need * kPageBytes);
                        for (int j = 0; j < nsub; ++j) {
                            uint8_t *sA = ring + (size_t)(first + j * sh.sub_pages) * kPageBytes;
                            const int kx = (k0 + j) * kBlockK;
                            if (it.ph == 0) {
                                tma_load_2d_hint(ma0, &full[tk], sA, kx, a_row, apol);
                                tma_load_2d_hint(ma1, &full[tk], sA + kABytes / 2, kx, a_row, apol);
                            } else {
                                tma_load_2d_hint(ma0, &full[tk], sA, kx, a_row, apol);
                                if (it.m == 2)
                                    tma_load_2d_hint(ma0, &full[tk], sA + kABytes, kx, a_row + kTileM, apol);
                            }
                        }
                        // the token slice of every sub-step: the loader's
                        ldesc[tk] = LoadDesc{mb,
                                             {nullptr, nullptr},
                                             smem_u32(ring + (size_t)first * kPageBytes + it.m * kABytes),
                                             sh.sub_pages * kPageBytes,
                                             k0 * kBlockK,
                                             it.row0,
                                             nsub,
                                             it.ph == 1,
                                             0u,
                                             0u};
                    }
                    if constexpr (!kPair) mbar_arrive(&armed[tk]);  // after the full barrier is armed
                    ++issued;
                }
                if (!ok) break;
            }
            if constexpr (!kPair) {
                // the loader stops at the first step never armed; its copies of the
                // armed ones are issued once it says so (bounded wait)
                *stop_at = (int)issued;
                const unsigned long long t0 = globaltimer();
                while (!*loader_done)
                    if (globaltimer() - t0 > kWaitLimitNs) {
                        *abort_flag = 1;
                        atomicOr(p.status, MOE_STATUS_TIMEOUT);
                        break;
                    }
            }
            // wait for every copy still in flight before the CTA may exit (pair: the
            // copies complete on CTA 0's barrier; the MMAs that consumed them release
            // this CTA's pages)
            for (uint32_t j = retired; j < issued; ++j) {
                if constexpr (kPair)
                    mbar_wait<true>(&empty[j % kTickets], (j / kTickets) & 1u, abort_flag, p.status, false);
                else
                    mbar_wait(&full[j % kTickets], (j / kTickets) & 1u, abort_flag, p.status, false);
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer =================
        if (lane == 0 && (!kPair || rank == 0)) {  // a pair's MMAs are issued by CTA 0
            uint32_t vhead = 0, off = 0, step = 0;  // the producer's page sequence, replayed
            const uint64_t desc0 = sw128_desc(smem_u32(ring));  // ring page 0; other pages by addition
            for (int li = 0;; ++li) {
                const int slot = li % kQueue;
                if (!mbar_wait(&qfull[slot], (uint32_t)(li / kQueue) & 1u, abort_flag, p.status, true)) break;
                const int item = qdesc[slot].item;
                const Item it = qdesc[slot].it;
                mbar_arrive(&qempty[slot]);
                if (item < 0) break;
                const StepShape sh = kFmt ? qstep_shape(it, p) : step_shape<kPair>(it, p);
                const uint32_t idesc = idesc_bf16((it.nvalid + 15) & ~15, kPair ? 2 * kTileM : kTileM);
                const int acc = li & 1;
                const uint32_t use = (uint32_t)(li >> 1);
                if (!mbar_wait<kPair>(&tempty[acc], (use & 1u) ^ 1u, abort_flag, p.status, true)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(acc * p.BN), d1 = d + (uint32_t)(p.BN >> 1);
                bool ok = true;
                for (int k0 = 0; k0 < sh.nk; k0 += sh.ns) {
                    const int nsub = min(sh.ns, sh.nk - k0);
                    const uint32_t first =
                        ring_alloc(vhead, off, kFmt ? qstep_pages<kFmt>(sh) : (uint32_t)nsub * sh.sub_pages, P);
                    const uint32_t tk = step % kTickets;
                    // block-scaled weights: the converters arrive only after this step's full
                    // barrier (codes, scales and tokens), so their barrier stands for both
                    if (kFmt == 0 &&
                        !mbar_wait_fast<kPair>(&full[tk], (step / kTickets) & 1u, abort_flag, p.status, true)) {
                        ok = false;
                        break;
                    }
                    if constexpr (kFmt != 0) {
                        // the converted weights of this step (TMEM buffer step % kConvBufs, A read
                        // from tensor memory: 8 columns per K 16), and the token boxes in the ring
                        const uint32_t cb = step % kConvBufs;
                        if (!mbar_wait_fast(&cfull[cb], (step / kConvBufs) & 1u, abort_flag, p.status, true)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t db = desc0 + (first + qcode_pages<kFmt>() + 1) * (kPageBytes / 16);
                        const uint32_t ta = tmem_base + (uint32_t)(kConvCol0 + cb * kConvCols);
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const uint64_t dbj = db + j * sh.sub_pages * (kPageBytes / 16);
#pragma unroll
                            for (int kk = 0; kk < kBlockK / 16; ++kk)
                                umma_bf16_ts(d, ta + (uint32_t)(j * 32 + kk * 8), dbj + 2 * kk, idesc,
                                             (k0 | j | kk) != 0);
                        }
                        umma_commit(&empty[tk]);  // the ring pages (codes, scales, tokens) and the TMEM buffer
                        ++step;
                        continue;
                    }
                    tc_fence_after();
                    for (int j = 0; j < nsub; ++j) {
                        // descriptor start addresses count 16-byte units
                        const uint64_t da = desc0 + (first + j * sh.sub_pages) * (kPageBytes / 16);
                        if constexpr (kPair) {  // M = 256: each CTA's 128 weight rows, N split over the two
                            const uint64_t db = da + kABytes / 16;
#pragma unroll
                            for (int kk = 0; kk < kBlockK / 16; ++kk)
                                umma_bf16_pair(d, da + 2 * kk, db + 2 * kk, idesc, (k0 | j | kk) != 0);
                        } else if (it.m == 1) {
                            const uint64_t db = da + kABytes / 16;
#pragma unroll
                            for (int kk = 0; kk < kBlockK / 16; ++kk)  // +32 bytes per K16 step
                                umma_bf16(d, da + 2 * kk, db + 2 * kk, idesc, (k0 | j | kk) != 0);
                        } else {  // weight tile 1 -> accumulator columns BN/2 ..
                            const uint64_t db = da + 2 * kABytes / 16;
#pragma unroll
                            for (int kk = 0; kk < kBlockK / 16; ++kk) {
                                umma_bf16(d, da + 2 * kk, db + 2 * kk, idesc, (k0 | j | kk) != 0);
                                umma_bf16(d1, da + kABytes / 16 + 2 * kk, db + 2 * kk, idesc, (k0 | j | kk) != 0);
                            }
                        }
                    }
                    if constexpr (kPair) umma_commit_pair(&empty[tk]);  // frees the pages in both CTAs
                    else umma_commit(&empty[tk]);
                    ++step;
                }
                if (!ok) break;
                if constexpr (kPair) umma_commit_pair(&tfull[acc]);  // both CTAs' epilogues
                else umma_commit(&tfull[acc]);
            }
            if constexpr (kPair) umma_commit_pair_local(mma_done);  // completes once every MMA above has
            else umma_commit(mma_done);
            mbar_wait(mma_done, 0, abort_flag, p.status, false);
        }
    } else if (warp == kLoadWarp) {
        // ================= token loader (single CTAs) =================
        // Issues the token copies of every ring step, in step order, once the
        // producer has armed the step's full barrier and described them: one
        // thread issuing a TMA copy costs it ~40-50 ns, so at decode sizes the
        // copies of a step, not HBM, would set the pace of a single producer.
        // It stops at the first step the producer never armed (stop_at, set
        // when the producer leaves), so that every armed step's copies are
        // issued and the producer's final drain sees them all land.
        if (!kPair && lane == 0) {
            for (uint32_t step = 0;; ++step) {
                const uint32_t tk = step % kTickets, par = (step / kTickets) & 1u;
                bool go = false;
                const unsigned long long t0 = globaltimer();
                for (uint32_t spin = 0;; ++spin) {
                    if (mbar_try_wait(&armed[tk], par)) {
                        go = true;
                        break;
                    }
                    if ((int)step >= *stop_at) break;
                    if ((spin & 63u) == 63u && globaltimer() - t0 > kWaitLimitNs) {
                        *abort_flag = 1;
                        atomicOr(p.status, MOE_STATUS_TIMEOUT);
                        break;
                    }
                }
                if (!go) break;
                const LoadDesc d = ldesc[tk];
                if (d.fence) fence_proxy_async_global();  // h written by other CTAs (the producer saw it ready)
                for (int j = 0; j < d.n; ++j)
                    tma_load_2d_s(d.map, &full[tk], d.dst + (uint32_t)j * d.dst_step, d.x + j * kBlockK, d.y);
                for (int i = 0; i < 2 && d.sc_bytes; ++i)
                    bulk_load_s(d.sc_dst + (uint32_t)i * d.sc_bytes, d.sc_src[i], d.sc_bytes, &full[tk]);
            }
            *loader_done = 1;
        }
    } else if (kFmt != 0 && warp > kLoadWarp) {
        // ================= block-scaled weight converters (warps 7 ..) =================
        // Two groups of kConvWarps / 2 warps take alternate steps, so that one
        // group's conversion overlaps the other's loads and TMEM stores.  Each
        // group walks the producer's step sequence: once one of its steps' codes
        // and scales have landed and the MMAs of the step kConvBufs back have
        // released TMEM buffer step % kConvBufs, it writes that step's bf16
        // weights there and hands it to the MMA lane.  Thread lane of warp w
        // converts row 32 (w % 4) + lane: a warp reaches only its own quarter of
        // the TMEM lanes, and a group's warps cover the four quarters.
        // Every thread of a group takes the same waits and a warp leaves a step
        // loop only as a whole (a vote after the waits); a failed wait sets the
        // abort flag, and the group's elected thread then publishes "stop" at the
        // next queue read, so every thread of the group reaches the same named
        // barriers.
        const int ct = threadIdx.x - kThreads;  // 0 .. 32 * kConvWarps - 1
        const uint32_t g = (uint32_t)(ct / (16 * kConvWarps));  // group: steps with step % 2 == g
        const bool elected = ct % (16 * kConvWarps) == 0;
        ItemSlot *desc = conv_desc + g;
        const int cq = warp & 3, crow = 32 * cq + lane;
        const uint32_t tlane = tmem_base + ((uint32_t)(32 * cq) << 16) + (uint32_t)kConvCol0;
        uint32_t vhead = 0, off = 0, step = 0;
        for (int li = 0;; ++li) {
            const int slot = li % kQueue;
            if (elected) {
                if (!*abort_flag && mbar_wait(&qfull[slot], (uint32_t)(li / kQueue) & 1u, abort_flag, p.status, true)) {
                    *desc = qdesc[slot];
                    mbar_arrive(&qempty[slot]);
                } else {
                    desc->item = -2;
                }
            }
            named_bar_sync(2 + g, 16 * kConvWarps);
            const int item = desc->item;
            const Item it = desc->it;
            named_bar_sync(2 + g, 16 * kConvWarps);  // read by all before the elected thread's next write
            if (item < 0) break;
            const StepShape sh = qstep_shape(it, p);
            const uint32_t need = qstep_pages<kFmt>(sh);
            bool ok = true;
            for (int k0 = 0; k0 < sh.nk; k0 += sh.ns, ++step) {
                const uint32_t first = ring_alloc(vhead, off, need, P);
                if ((step & 1u) != g) continue;  // the other group's step
                const uint32_t tk = step % kTickets, cb = step % kConvBufs;
                // TMEM buffer cb is free once the MMAs of step - kConvBufs, its last user, are
                // done: that step's empty barrier.  It cannot have completed another phase
                // since: that takes the MMAs of step - kConvBufs + kTickets, which this group
                // converts after this one.
                const uint32_t prev = step - kConvBufs;
                ok = mbar_wait_fast(&full[tk], (step / kTickets) & 1u, abort_flag, p.status, true) &&
                     (step < kConvBufs ||
                      mbar_wait_fast(&empty[prev % kTickets], (prev / kTickets) & 1u, abort_flag, p.status, true));
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
                const uint32_t codes = smem_u32(ring + (size_t)first * kPageBytes);
                if constexpr (kFmt == 2)
                    convert_nvfp4_row(codes, codes + qcode_pages<kFmt>() * kPageBytes, crow, tlane + cb * kConvCols);
                else
                    convert_mxfp8_row(codes, codes + qcode_pages<kFmt>() * kPageBytes, crow, tlane + cb * kConvCols);
                tmem_wait_st();  // this thread's stores done, before the arrival
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&cfull[cb]);
            }
        }
    } else {
        // ================= epilogue (warps 2..5) =================
        const int q = warp & 3;  // TMEM lane quarter of this warp
        const bool elected = (warp == 2 && lane == 0);
        for (int li = 0;; ++li) {
            const int acc = li & 1;
            const uint32_t use = (uint32_t)(li >> 1);
            if (elected) {  // one thread takes the item; its accumulator is awaited below
                const int slot = li % kQueue;
                if (mbar_wait<kPair>(&qfull[slot], (uint32_t)(li / kQueue) & 1u, abort_flag, p.status, true)) {
                    *epi_desc = qdesc[slot];
                    if (kPair && rank != 0) mbar_arrive_cluster(mapa(smem_u32(&qempty[slot]), 0));
                    else mbar_arrive(&qempty[slot]);
                } else {
                    epi_desc->item = -2;
                }
            }
            named_bar_sync(1, 128);
            if (epi_desc->item < 0) break;
            const Item it = epi_desc->it;
            // down items: destination row and weight of token `lane`, loaded while the
            // item's MMAs still run
            int mrow0 = 0;
            float mw0 = 0.f;
            if (it.ph == 1) down_dest(it, lane, p, mrow0, mw0);
            // NVFP4: the matrix scales of this item's projections (gate or down, up)
            float ts0 = 1.f, ts1 = 1.f;
            if constexpr (kFmt == 2) {
                ts0 = it.shared ? p.tss[2 * it.ph] : __ldg(p.ts[it.ph][0] + it.e);
                if (it.ph == 0) ts1 = it.shared ? p.tss[1] : __ldg(p.ts[0][1] + it.e);
            }
            if (elected) *epi_flag = mbar_wait<kPair>(&tfull[acc], use & 1u, abort_flag, p.status, true) ? 0 : -1;
            named_bar_sync(1, 128);
            if (*epi_flag) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + (uint32_t)(acc * p.BN) + ((uint32_t)(q * 32) << 16);
            const int rt = kPair ? 2 * it.r + (int)rank : it.r;  // pair: this CTA's weight tile
            for (int c0 = 0; c0 < it.nvalid; c0 += 32) {
                if (it.ph == 0) {
                    float v[32];
                    tmem_ld32(tbase + (uint32_t)c0, v);
                    if constexpr (kFmt == 2) {
                        const float ts = q < 2 ? ts0 : ts1;
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= ts;
                    }
                    if (q < 2) {  // gate rows 0..63: silu(g) to the exchange buffer
                        float *xr = xchg + (q * 32 + lane) * kXchgStride;
#pragma unroll
                        for (int i = 0; i < 32; ++i) xr[i] = silu(v[i]);
                    }
                    named_bar_sync(1, 128);
                    if (q >= 2) {  // up rows 64..127: h = silu(g) * u
                        const int row = (q - 2) * 32 + lane;
                        const float *xr = xchg + row * kXchgStride;
                        uint16_t *out = it.shared ? p.h_shared : p.h_perm;
                        const int ld = it.shared ? p.Is : p.I;
                        uint16_t *dst = out + (size_t)(it.row0 + c0) * ld + rt * 64 + row;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (c0 + i < it.nvalid) dst[(size_t)i * ld] = f32_to_bf16_bits(xr[i] * v[i]);
                    }
                    named_bar_sync(1, 128);
                } else {
                    // per-token destination row of ybuf and weight, token c0 + lane
                    int mrow = mrow0;
                    float mw = mw0;
                    if (c0 > 0) down_dest(it, c0 + lane, p, mrow, mw);
                    if constexpr (kFmt == 2) mw *= ts0;
                    for (int t = 0; t < it.m; ++t) {  // weight tile r + t: accumulator columns t * BN/2
                        float v[32];
                        tmem_ld32(tbase + (uint32_t)(t * (p.BN >> 1) + c0), v);
                        uint16_t *out = p.ybuf + (rt + t) * kTileM + q * 32 + lane;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int rr = __shfl_sync(0xffffffffu, mrow, i);
                            const float ww = __shfl_sync(0xffffffffu, mw, i);
                            if (c0 + i < it.nvalid && (!kDebugBounds || rr >= 0))
                                out[(size_t)rr * p.H] = f32_to_bf16_bits(v[i] * ww);
                        }
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(1, 128);
            if (elected) {
                if (kPair && rank != 0) mbar_arrive_cluster(mapa(smem_u32(&tempty[acc]), 0));
                else mbar_arrive(&tempty[acc]);
                if (fused && it.ph == 0) {
                    // the CTA's h rows (ordered before this by the barrier) become visible
                    // device-wide before the group counter moves
                    __threadfence();
                    atomicAdd(p.hdone + (it.shared ? p.E : it.e), 1);
                    atomicAdd(p.hdone + p.E + 1, 1);
                }
            }
        }
    }

    __syncthreads();
    if constexpr (kPair) cluster_sync();  // the other CTA is done with the shared TMEM allocation and our barriers
    if (warp == 1) {
        tc_fence_after();
        if constexpr (kPair)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols)
                         : "memory");
    }
    // The last CTA out resets the counters for the next launch, all its threads
    // sharing the group counters (a serial loop of E + 2 atomics would hold the
    // grid open for microseconds).
    if (threadIdx.x == 0) {
        __threadfence();
        *epi_flag = atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (*epi_flag) {
        if (threadIdx.x == 0) {
            atomicExch(p.sched, 0);
            atomicExch(p.sched + 1, 0);
        }
        if (fused)
            for (int g = threadIdx.x; g <= p.E + 1; g += NT) atomicExch(p.hdone + g, 0);
        __threadfence();
    }
}

// ------------------------------------------------------------- host side --
// Token tile of the routed experts: the largest MMA N.  A tile's
// shared-memory cost follows its real token count (the paged ring), so a
// wide tile costs nothing for small groups and saves re-reading a weight
// tile for every 128 tokens of large ones.
// Block-scaled weights: 128, so that the two accumulators end where the
// conversion buffers start in tensor memory (column 256).
int pick_bn(int fmt) { return fmt ? 128 : 256; }

// Token tile of the shared expert, which sees all T tokens.  One 256-token
// tile streams each weight tile once, but its items then run about twice as
// long as the routed ones; when the gate/up phase has few items per SM that
// unbalances the launch, and two 128-token tiles (the second one's weights
// from L2) finish sooner.  The item estimate counts every expert as active.
int pick_bns(const FfnArgs &a, int bn, int sms) {
    if (a.Is == 0 || a.T <= 128) return bn;
    const long long est = std::min<long long>(a.E, (long long)a.T * a.k) * (a.I / 64);
    return est >= 4LL * sms ? bn : std::min(bn, 128);
}

size_t smem_bytes_for(int E, int pages, int fmt) {
    const int nt = fmt ? kThreadsQ : kThreads;
    return 1024 + (size_t)pages * kPageBytes + 64 * kXchgStride * 4 +
           3 * (size_t)(E + 1) * 4 + 8 + (size_t)(3 * kTickets + 5 + 2 * kQueue + kConvBufs) * 8 + 16 +
           (kQueue + 3) * sizeof(ItemSlot) + 8 + 2 * (size_t)nt * 4 + kReadyWords * 4 + kTickets * 4 + 8 +
           kTickets * sizeof(LoadDesc) + 8;
}

int min_pages(int fmt) { return fmt == 2 ? 4 + 1 + 2 * (256 * 128 / 2048) : fmt ? kQMaxStepPages : kMaxStepPages; }

int pick_pages(int E, int fmt) {
    const size_t fixed = smem_bytes_for(E, 0, fmt);
    if (fixed >= (size_t)kSmemLimit) return 0;
    return (int)std::min<size_t>(kMaxPages, ((size_t)kSmemLimit - fixed) / kPageBytes);
}

struct DeviceInfo {
    int sms = 0;
    int cc_major = 0;
};

DeviceInfo device_info() {
    static DeviceInfo cache[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DeviceInfo{};
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev].sms == 0) {
        cudaDeviceGetAttribute(&cache[dev].sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&cache[dev].cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    }
    return cache[dev];
}

// Benchmark/test overrides: MOE_FORCE_BN and MOE_FORCE_BNS in {32, 64, 128,
// 256} (routed / shared token tile, BNS <= BN) and MOE_FORCE_PAGES in
// [24, 112] (ring size in 2 KB pages, capped by shared memory; 24 holds one
// widest K step; 41 with block-scaled weights); any other value is rejected.
int parse_tile(const char *f, int *out) {
    char *end = nullptr;
    const long v = strtol(f, &end, 10);
    if (*f == 0 || *end != 0 || (v != 32 && v != 64 && v != 128 && v != 256)) return MOE_ERR_INVALID_ARG;
    *out = (int)v;
    return MOE_OK;
}

int choose_tiles(const FfnArgs &a, int sms, int *bn, int *bns, int *pages) {
    *bn = pick_bn(a.fmt);
    if (const char *f = getenv("MOE_FORCE_BN"))
        if (int rc = parse_tile(f, bn)) return rc;
    *bns = pick_bns(a, *bn, sms);
    if (const char *f = getenv("MOE_FORCE_BNS"))
        if (int rc = parse_tile(f, bns)) return rc;
    if (*bns > *bn) return MOE_ERR_INVALID_ARG;
    *pages = pick_pages(a.E, a.fmt);
    if (const char *f = getenv("MOE_FORCE_PAGES")) {
        char *end = nullptr;
        const long v = strtol(f, &end, 10);
        if (*f == 0 || *end != 0 || v < min_pages(a.fmt) || v > kMaxPages) return MOE_ERR_INVALID_ARG;
        *pages = std::min<int>((int)v, *pages);
    }
    return *pages >= min_pages(a.fmt) ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

// Test hooks (failure-path tests only): MOE_TEST_WAIT_LIMIT_US in [1, 4e6]
// shortens the fused launch's group-readiness wait, MOE_TEST_STALL_GROUP in
// [0, E] (E: the shared expert) gives that group's down items a readiness
// target its gate/up items never reach, so their wait runs out and the
// launch ends with MOE_STATUS_TIMEOUT after the limit.  Unset: 4 s, none.
int test_hooks(const FfnArgs &a, unsigned long long *limit_ns, int *stall) {
    *limit_ns = kWaitLimitNs;
    *stall = -1;
    if (const char *f = getenv("MOE_TEST_WAIT_LIMIT_US")) {
        char *end = nullptr;
        const long long v = strtoll(f, &end, 10);
        if (*f == 0 || *end != 0 || v < 1 || v > 4000000) return MOE_ERR_INVALID_ARG;
        *limit_ns = (unsigned long long)v * 1000ull;
    }
    if (const char *f = getenv("MOE_TEST_STALL_GROUP")) {
        char *end = nullptr;
        const long v = strtol(f, &end, 10);
        if (*f == 0 || *end != 0 || v < 0 || v > a.E) return MOE_ERR_INVALID_ARG;
        *stall = (int)v;
    }
    return MOE_OK;
}

}  // namespace

// CTA pairs (cta_group::2) for a single-phase launch whose groups fill wide
// token tiles: the mean group has at least 128 tokens (the regime where a
// 256-token tile's operand bytes, not the weight stream, limit the tensor
// pipe), and every weight-tile count of the phase is even.  MOE_FORCE_PAIR
// = 0 / 1 overrides the first condition (tests and benchmarking only).
int choose_pair(const FfnArgs &a, int phases, int sms, bool *pair) {
    *pair = false;
    bool want = phases != 3 && ((long long)a.T * a.k + a.E - 1) / a.E >= 128;
    if (const char *f = getenv("MOE_FORCE_PAIR")) {
        if (f[0] != '0' && f[0] != '1') return MOE_ERR_INVALID_ARG;
        if (f[1] != 0) return MOE_ERR_INVALID_ARG;
        want = f[0] == '1' && phases != 3;
    }
    const bool even = ((phases & 1) == 0 || ((a.I / 64) % 2 == 0 && (a.Is / 64) % 2 == 0)) &&
                      ((phases & 2) == 0 || (a.H / kTileM) % 2 == 0);
    *pair = want && even && sms >= 2 && a.fmt == 0;  // block-scaled weights: single CTAs
    return MOE_OK;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pair(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

int ffn_launch(const FfnArgs &a, int phases, cudaStream_t st) {
    const DeviceInfo di = device_info();
    if (di.cc_major != 10) return MOE_ERR_UNSUPPORTED;
    if (phases < 1 || phases > 3 || a.fmt < 0 || a.fmt > 2) return MOE_ERR_INVALID_ARG;
    // block-scaled weights: 128-wide K steps and 64-row scale groups
    if (a.fmt && (a.H % 128 != 0 || a.I % 128 != 0 || a.Is % 128 != 0)) return MOE_ERR_UNSUPPORTED;
    FfnParams p{};
    if (int rc = choose_tiles(a, di.sms, &p.BN, &p.BNs, &p.pages)) return rc;
    if (a.fmt && 2 * p.BN > kConvCol0) return MOE_ERR_UNSUPPORTED;  // accumulators end where the A buffers start
    if (int rc = test_hooks(a, &p.wait_limit_ns, &p.stall_group)) return rc;
    bool pair = false;
    if (int rc = choose_pair(a, phases, di.sms, &pair)) return rc;
    const int BN = p.BN;
    p.T = a.T;
    p.H = a.H;
    p.E = a.E;
    p.I = a.I;
    p.k = a.k;
    p.Is = a.Is;
    p.phases = phases;
    p.offsets = a.offsets;
    p.perm = a.perm;
    p.topk_w = a.topk_w;
    p.sgate = a.sgate;
    p.h_perm = a.h_perm;
    p.h_shared = a.h_shared;
    p.ybuf = a.ybuf;
    p.status = a.status;
    p.sched = a.status + (phases == 2 ? 8 : 4);
    p.hdone = a.hdone;
    const int per = pair ? 2 : 1;  // weight tiles per item (a pair covers two)
    p.R[0] = a.I / 64 / per;
    p.Rs[0] = a.Is / 64 / per;
    p.nk[0] = a.H / kBlockK;
    p.nks[0] = a.H / kBlockK;
    p.R[1] = a.H / kTileM / per;
    p.Rs[1] = a.H / kTileM / per;
    p.nk[1] = a.I / kBlockK;
    p.nks[1] = a.Is / kBlockK;
    p.sf[0][0] = a.sf_gate;
    p.sf[0][1] = a.sf_up;
    p.sf[1][0] = a.sf_down;
    p.sfs[0][0] = a.sfs_gate;
    p.sfs[0][1] = a.sfs_up;
    p.sfs[1][0] = a.sfs_down;
    p.ts[0][0] = a.ts_gate;
    p.ts[0][1] = a.ts_up;
    p.ts[1][0] = a.ts_down;
    p.tss = a.tss;

    static FfnMaps zero_maps;  // unused maps stay zero
    FfnMaps m = zero_maps;
    const uint64_t Tk = (uint64_t)a.T * a.k;
    bool ok = true;
    // weight maps: bf16 boxes of 64 K, or code boxes of 128 K (MXFP8: 128 bytes
    // a row, 128-byte swizzle; NVFP4: 64 bytes a row, 64-byte swizzle)
    auto wmap = [&](CUtensorMap *mp, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
        if (a.fmt == 2) return encode_2d_u8(mp, base, rows, cols / 2, box_rows, 64);
        return a.fmt ? encode_2d_u8(mp, base, rows, cols, box_rows, 128) : encode_2d(mp, base, rows, cols, box_rows);
    };
    if (phases & 1) {
        PhaseMaps &g = m.ph[0];
        ok = ok && wmap(&g.a0, a.w_gate, (uint64_t)a.E * a.I, a.H, 64) &&
             wmap(&g.a1, a.w_up, (uint64_t)a.E * a.I, a.H, 64);
        for (int b = 0; b < kNumBox && (16 << b) <= BN; ++b) ok = ok && encode_2d(&g.b[b], a.x_perm, Tk, a.H, 16 << b);
        if (a.Is > 0) {
            ok = ok && wmap(&g.s0, a.ws_gate, a.Is, a.H, 64) && wmap(&g.s1, a.ws_up, a.Is, a.H, 64);
            for (int b = 0; b < kNumBox && (16 << b) <= BN; ++b) ok = ok && encode_2d(&g.bs[b], a.x, a.T, a.H, 16 << b);
        }
    }
    if (phases & 2) {
        PhaseMaps &d = m.ph[1];
        ok = ok && wmap(&d.a0, a.w_down, (uint64_t)a.E * a.H, a.I, kTileM);
        for (int b = 0; b < kNumBox && (16 << b) <= BN; ++b) ok = ok && encode_2d(&d.b[b], a.h_perm, Tk, a.I, 16 << b);
        if (a.Is > 0) {
            ok = ok && wmap(&d.s0, a.ws_down, a.H, a.Is, kTileM);
            for (int b = 0; b < kNumBox && (16 << b) <= BN; ++b)
                ok = ok && encode_2d(&d.bs[b], a.h_shared, a.T, a.Is, 16 << b);
        }
    }
    if (!ok) return MOE_ERR_CUDA;

    const size_t smem = smem_bytes_for(a.E, p.pages, a.fmt);
    if (smem > (size_t)kSmemLimit) return MOE_ERR_UNSUPPORTED;
    static std::atomic<int> attr_set[64];  // per device: opted in to the full shared memory
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(ffn_kernel<false, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
                cudaSuccess ||
            cudaFuncSetAttribute(ffn_kernel<true, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
                cudaSuccess ||
            cudaFuncSetAttribute(ffn_kernel<false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
                cudaSuccess ||
            cudaFuncSetAttribute(ffn_kernel<false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
                cudaSuccess)
            return MOE_ERR_CUDA;
        attr_set[dev].store(1, std::memory_order_release);
    }
    // upper bound on work items (the real count is known only on the device)
    const long long slots = (long long)a.T * a.k;
    const long long tiles = std::min<long long>(a.E, slots) + (slots + BN - 1) / BN;
    const long long st_tiles = a.Is > 0 ? (a.T + p.BNs - 1) / p.BNs : 0;
    long long items = 0;
    for (int ph = 0; ph < 2; ++ph)
        if ((phases >> ph) & 1) items += tiles * p.R[ph] + st_tiles * p.Rs[ph];
    if (pair) {  // clusters of two CTAs: an even grid
        const int grid = 2 * (int)std::max<long long>(1, std::min<long long>(di.sms / 2, items));
        return launch_pair(ffn_kernel<true, 0>, dim3(grid), dim3(kThreads), smem, st, m, p) == cudaSuccess
                   ? MOE_OK
                   : MOE_ERR_CUDA;
    }
    const int grid = (int)std::max<long long>(1, std::min<long long>(di.sms, items));
    if (a.fmt == 1)
        return launch_pdl(ffn_kernel<false, 1>, dim3(grid), dim3(kThreadsQ), smem, st, m, p) == cudaSuccess
                   ? MOE_OK
                   : MOE_ERR_CUDA;
    if (a.fmt == 2)
        return launch_pdl(ffn_kernel<false, 2>, dim3(grid), dim3(kThreadsQ), smem, st, m, p) == cudaSuccess
                   ? MOE_OK
                   : MOE_ERR_CUDA;
    return launch_pdl(ffn_kernel<false, 0>, dim3(grid), dim3(kThreads), smem, st, m, p) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

int device_sm_count() { return device_info().sms; }

int ffn_launch_both(const FfnArgs &a, cudaStream_t st) {
    const long long avg = ((long long)a.T * a.k + a.E - 1) / a.E;
    if (avg < 128) return ffn_launch(a, 3, st);
    if (int rc = ffn_launch(a, 1, st)) return rc;
    return ffn_launch(a, 2, st);
}

}  // namespace moe
