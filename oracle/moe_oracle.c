/*
 * oracle/moe_oracle.c -- TEST INFRASTRUCTURE, not product code.
 *
 * A plain, slow, obviously-correct CPU definition of the routed
 * Mixture-of-Experts FFN forward.  Only tests/, the smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library; the CUDA
 * library never calls it and shares no source with it.
 *
 * Sources (web pages; cited by title and section):
 *  [SF943]  SpecForge PR #943 "Qwen3.8-27B DSpark MoE drafter with 16 x 1024
 *           top-2 experts", section "Modifications" (softmax router with
 *           renormalised top-k, "qwen3_5_moe preset"; shared expert of width
 *           2048, sigmoid-gated; grouped_mm dispatch) and the FFN parameter
 *           table of "End-to-end serving speed" (3*H*I parameters per expert:
 *           gate, up and down projections).
 *  [BUDGET] colibri issue_budget.md "EXPERT_BUDGET", section "How it works"
 *           (steps 1-5 of the batch-union cap) and section "Safety"
 *           (dropped experts omitted, the rest renormalised; off by default);
 *           section "Relationship to existing features" (TOPP trims each
 *           position to its top-p mass within its top-K, before the budget
 *           caps the union; the trimmed state is keff < K, as the budget's).
 *
 * Precision.  Routing weights, the budget's aggregate weights and every
 * quantity that decides an integer (which expert is kept) are computed in
 * fp32, the precision the CUDA path decides them in.  The expert FFN, the
 * shared expert and the combine accumulate in fp64 (no rounding at all of
 * the intermediate activation), which is at least as accurate as fp32.
 * Activations and weights arrive as bf16 bit patterns and are widened
 * exactly.
 *
 * Readings where the pages are silent or leave a step open:
 *  - top-k ties: equal logits -> the lower expert id ranks first;
 *  - slot order inside a token: descending logit;
 *  - budget ties: equal aggregate weight -> the lower expert id is kept;
 *  - budget aggregate: summed over tokens ascending, then slots ascending;
 *  - only tokens that lost a slot are renormalised;
 *  - top-p: the shortest prefix of a token's slots whose weights (after the
 *    norm_topk renormalisation, summed in slot order) reach topp; topp <= 0
 *    or >= 1 is off;
 *  - dispatch order inside an expert: slot id t*k+j ascending;
 *  - the shared-expert gate is a per-token scalar sigmoid(g . x_t).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ENOMEM (-2)

static double bf16_to_f64(uint16_t v)
{
    uint32_t u = ((uint32_t)v) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Number of parameters of one gated (SwiGLU) expert FFN of hidden size H and
 * intermediate size I: a gate and an up projection H->I and a down projection
 * I->H, no biases ([SF943] FFN parameter table). */
int64_t oracle_ffn_params(int64_t H, int64_t I) { return 3 * H * I; }

/* ---------------------------------------------------------------------- */
/* Router projection ([SF943] "Modifications": the softmax router whose     */
/* logits the route step takes; a bias-free linear map of the hidden state, */
/* the plain reading of a router over n_routed_experts).                   */
/* ---------------------------------------------------------------------- */
/* logits[t, e] = sum_h x[t, h] * W_r[e, h], accumulated in fp64 and rounded
 * once to fp32.  x [T, H] and W_r [E, H] are bf16 bit patterns. */
int oracle_router_logits(int32_t T, int32_t H, int32_t E, const uint16_t *x, const uint16_t *wr, float *logits)
{
    if (T < 0 || H < 1 || E < 1) return ORACLE_EINVAL;
    for (int32_t t = 0; t < T; ++t)
        for (int32_t e = 0; e < E; ++e) {
            double a = 0.0;
            for (int32_t h = 0; h < H; ++h)
                a += bf16_to_f64(x[(size_t)t * H + h]) * bf16_to_f64(wr[(size_t)e * H + h]);
            logits[(size_t)t * E + e] = (float)a;
        }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Route ([SF943] "Modifications": softmax router, renormalised top-k).    */
/* ---------------------------------------------------------------------- */
/* For each token t:
 *   1. rank the E experts by (logit descending, expert id ascending) and keep
 *      the first k, in that order, as idx[t, 0..k);
 *   2. p = softmax over all E logits (fp32, max subtracted, sum over experts
 *      in ascending id order);
 *   3. w[t, j] = p[idx[t, j]];
 *   4. if norm_topk: w[t, j] /= sum_j w[t, j] (summed j ascending). */
int oracle_route(int32_t T, int32_t E, int32_t k, int32_t norm_topk,
                 const float *logits, int32_t *idx, float *w)
{
    if (T < 0 || E < 1 || k < 1 || k > E) return ORACLE_EINVAL;
    char *taken = (char *)malloc((size_t)E);
    float *p = (float *)malloc(sizeof(float) * (size_t)E);
    if (!taken || !p) { free(taken); free(p); return ORACLE_ENOMEM; }
    for (int32_t t = 0; t < T; ++t) {
        const float *l = logits + (size_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int32_t j = 0; j < k; ++j) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict '>' keeps the lower id on ties */
            }
            taken[best] = 1;
            idx[(size_t)t * k + j] = best;
        }
        float m = l[0];
        for (int32_t e = 1; e < E; ++e) if (l[e] > m) m = l[e];
        float s = 0.0f;
        for (int32_t e = 0; e < E; ++e) { p[e] = expf(l[e] - m); s += p[e]; }
        for (int32_t e = 0; e < E; ++e) p[e] = p[e] / s;
        float ws = 0.0f;
        for (int32_t j = 0; j < k; ++j) {
            w[(size_t)t * k + j] = p[idx[(size_t)t * k + j]];
            ws += w[(size_t)t * k + j];
        }
        if (norm_topk)
            for (int32_t j = 0; j < k; ++j) w[(size_t)t * k + j] = w[(size_t)t * k + j] / ws;
    }
    free(taken);
    free(p);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Top-p trim ([BUDGET] "Relationship to existing features": TOPP trims     */
/* within one position's top-K; the two compose, TOPP first).              */
/* ---------------------------------------------------------------------- */
/* For each token t of the router output (slots in descending-logit order,
 * weights after the norm_topk renormalisation):
 *   1. slot 0 is kept; slot j > 0 is kept while the weights of slots
 *      0..j-1, added in slot order in fp32, are still below topp -- the
 *      shortest prefix whose mass reaches topp;
 *   2. the dropped tail becomes (idx -1, w 0) and keff[t] = kept slots;
 *   3. if norm_topk and a slot was dropped, the kept weights are divided by
 *      their sum (slot order, fp32), as the budget renormalises.
 * topp <= 0 (the default) or topp >= 1: no change, keff[t] = k. */
int oracle_topp(int32_t T, int32_t k, int32_t norm_topk, float topp, int32_t *idx, float *w, int32_t *keff)
{
    if (T < 0 || k < 1 || topp != topp) return ORACLE_EINVAL;
    for (int32_t t = 0; t < T; ++t) {
        int32_t *ti = idx + (size_t)t * k;
        float *tw = w + (size_t)t * k;
        int32_t c = k;
        if (topp > 0.0f && topp < 1.0f) {
            float mass = 0.0f; /* weights of the slots before j */
            for (int32_t j = 0; j < k; ++j) {
                if (j > 0 && mass >= topp) { c = j; break; }
                mass += tw[j];
            }
            for (int32_t j = c; j < k; ++j) { ti[j] = -1; tw[j] = 0.0f; }
            if (norm_topk && c < k) {
                float s = 0.0f;
                for (int32_t j = 0; j < c; ++j) s += tw[j];
                for (int32_t j = 0; j < c; ++j) tw[j] = tw[j] / s;
            }
        }
        keff[t] = c;
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Budget ([BUDGET] "How it works", steps 1-5; "Safety").                  */
/* ---------------------------------------------------------------------- */
/* Input: the router output idx/w [T, k], possibly trimmed by top-p (a
 * token's valid slots first, then idx = -1).
 * Output, in place: idx/w with each token's surviving slots first (original
 * order kept), the tail filled with idx = -1, w = 0; keff[t] = surviving
 * slots; kept[e] = 1 for experts of the (possibly capped) batch union;
 * *n_dropped = number of distinct experts dropped.
 * N <= 0, or a union no larger than N, changes nothing ("default off";
 * the cap applies only when the union exceeds the budget): keff[t] = the
 * token's valid slots. */
typedef struct { float agg; int32_t id; } agg_entry;

static int agg_cmp(const void *a, const void *b)
{
    const agg_entry *x = (const agg_entry *)a, *y = (const agg_entry *)b;
    if (x->agg > y->agg) return -1;   /* descending aggregate weight */
    if (x->agg < y->agg) return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id); /* equal -> lower id first */
}

/* Step 4 of the budget on its own, for a given kept set: every token's
 * slots whose expert is kept move to the front in their original order, the
 * tail becomes (idx -1, w 0), and a token that lost a valid slot has its
 * kept weights divided by their sum (slot order, fp32) when norm_topk.
 * keff[t] holds the token's valid slots on entry and its kept slots on exit.
 * oracle_budget calls this with the kept set of steps 1-3; a test may call
 * it with another kept set (a near-tie that the GPU decided the other way). */
int oracle_budget_apply(int32_t T, int32_t k, int32_t norm_topk, const uint8_t *kept,
                        int32_t *idx, float *w, int32_t *keff)
{
    if (T < 0 || k < 1) return ORACLE_EINVAL;
    for (int32_t t = 0; t < T; ++t) {
        int32_t *ti = idx + (size_t)t * k;
        float *tw = w + (size_t)t * k;
        int32_t c = 0;
        for (int32_t j = 0; j < k; ++j)
            if (ti[j] >= 0 && kept[ti[j]]) { ti[c] = ti[j]; tw[c] = tw[j]; ++c; }
        for (int32_t j = c; j < k; ++j) { ti[j] = -1; tw[j] = 0.0f; }
        if (norm_topk && c > 0 && c < keff[t]) {
            float s = 0.0f;
            for (int32_t j = 0; j < c; ++j) s += tw[j];
            for (int32_t j = 0; j < c; ++j) tw[j] = tw[j] / s;
        }
        keff[t] = c;
    }
    return ORACLE_OK;
}

int oracle_budget(int32_t T, int32_t E, int32_t k, int32_t N, int32_t norm_topk,
                  int32_t *idx, float *w, int32_t *keff, uint8_t *kept, int32_t *n_dropped)
{
    if (T < 0 || E < 1 || k < 1 || k > E || N < 0) return ORACLE_EINVAL;
    /* the batch union uniq[0..nu) over the valid slots */
    memset(kept, 0, (size_t)E);
    for (size_t s = 0; s < (size_t)T * k; ++s)
        if (idx[s] >= 0) kept[idx[s]] = 1;
    int32_t nu = 0;
    for (int32_t e = 0; e < E; ++e) nu += kept[e];
    for (int32_t t = 0; t < T; ++t) {
        int32_t v = 0;
        for (int32_t j = 0; j < k; ++j) v += idx[(size_t)t * k + j] >= 0;
        keff[t] = v;
    }
    *n_dropped = 0;
    if (N == 0 || nu <= N) return ORACLE_OK;

    /* step 1: aggregate gate weight per union expert, tokens then slots ascending */
    float *agg = (float *)calloc((size_t)E, sizeof(float));
    agg_entry *order = (agg_entry *)malloc(sizeof(agg_entry) * (size_t)nu);
    if (!agg || !order) { free(agg); free(order); return ORACLE_ENOMEM; }
    for (int32_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j)
            if (idx[(size_t)t * k + j] >= 0) agg[idx[(size_t)t * k + j]] += w[(size_t)t * k + j];
    /* step 2: sort the union by aggregate weight, descending */
    int32_t n = 0;
    for (int32_t e = 0; e < E; ++e)
        if (kept[e]) { order[n].agg = agg[e]; order[n].id = e; ++n; }
    qsort(order, (size_t)nu, sizeof(agg_entry), agg_cmp);
    /* step 3: keep the first N, mark the rest dropped */
    memset(kept, 0, (size_t)E);
    for (int32_t r = 0; r < N; ++r) kept[order[r].id] = 1;
    /* step 4: remove dropped experts from each token's list, renormalise the
     * tokens that lost a slot (keff[t] holds the valid slots before) */
    oracle_budget_apply(T, k, norm_topk, kept, idx, w, keff);
    /* step 5: the union is now the kept experts */
    *n_dropped = nu - N;
    free(agg);
    free(order);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Dispatch ([SF943] "Modifications": grouped_mm dispatch).                */
/* ---------------------------------------------------------------------- */
/* Groups the kept slots s = t*k + j (j < keff[t]) by expert:
 *   counts[e]  = number of kept slots routed to e;
 *   offsets    = exclusive prefix sum of counts, offsets[E] = total;
 *   perm[pos]  = slot ids, expert ascending, slot id ascending inside one;
 *   slot_pos[s] = pos of slot s, -1 for a slot that was dropped. */
int oracle_dispatch(int32_t T, int32_t E, int32_t k, const int32_t *idx, const int32_t *keff,
                    int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *slot_pos)
{
    if (T < 0 || E < 1 || k < 1) return ORACLE_EINVAL;
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (size_t s = 0; s < (size_t)T * k; ++s) slot_pos[s] = -1;
    for (int32_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < keff[t]; ++j) counts[idx[(size_t)t * k + j]] += 1;
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t pos = 0;
    for (int32_t e = 0; e < E; ++e)
        for (int32_t t = 0; t < T; ++t)
            for (int32_t j = 0; j < keff[t]; ++j)
                if (idx[(size_t)t * k + j] == e) {
                    perm[pos] = t * k + j;
                    slot_pos[(size_t)t * k + j] = pos;
                    ++pos;
                }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Expert FFN ([SF943] "Modifications" and FFN parameter table).           */
/* ---------------------------------------------------------------------- */
/* y = W_down . ( silu(W_gate . x) * (W_up . x) ),  silu(g) = g / (1 + e^-g).
 * W_gate, W_up: [I, H] row-major; W_down: [H, I] row-major; x: [H].
 * Everything accumulates in fp64.  `scale` (NULL: none) holds one factor per
 * projection {gate, up, down} that multiplies its output: the fp32 matrix
 * scale of weights stored in a block-scaled format (quant_oracle.c), whose
 * element-times-block-scale values are what W holds.  A factor of 1 leaves
 * every value bit-identical. */
static void swiglu_ffn(int32_t H, int32_t I, const uint16_t *wg, const uint16_t *wu,
                       const uint16_t *wd, const double *scale, const uint16_t *x, double *hbuf, double *y)
{
    const double sg = scale ? scale[0] : 1.0, su = scale ? scale[1] : 1.0, sd = scale ? scale[2] : 1.0;
    for (int32_t i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        const uint16_t *rg = wg + (size_t)i * H, *ru = wu + (size_t)i * H;
        for (int32_t c = 0; c < H; ++c) {
            double xc = bf16_to_f64(x[c]);
            g += bf16_to_f64(rg[c]) * xc;
            u += bf16_to_f64(ru[c]) * xc;
        }
        g *= sg;
        u *= su;
        hbuf[i] = g / (1.0 + exp(-g)) * u;
    }
    for (int32_t o = 0; o < H; ++o) {
        double a = 0.0;
        const uint16_t *rd = wd + (size_t)o * I;
        for (int32_t i = 0; i < I; ++i) a += bf16_to_f64(rd[i]) * hbuf[i];
        y[o] = sd * a;
    }
}

/* Expert FFN applied to n rows: y[r, :] = FFN(x[r, :]) for r < n. */
int oracle_expert_rows(int32_t H, int32_t I, const uint16_t *wg, const uint16_t *wu,
                       const uint16_t *wd, int32_t n, const uint16_t *x, double *y,
                       int32_t nthreads)
{
    if (H < 1 || I < 1 || n < 0) return ORACLE_EINVAL;
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *hbuf = (double *)malloc(sizeof(double) * (size_t)I);
        if (!hbuf) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int32_t r = 0; r < n; ++r)
                swiglu_ffn(H, I, wg, wu, wd, NULL, x + (size_t)r * H, hbuf, y + (size_t)r * H);
        }
        free(hbuf);
    }
    return err ? ORACLE_ENOMEM : ORACLE_OK;
}

/* Shared-expert gate ([SF943] "Modifications": sigmoid-gated shared expert):
 * s_t = 1 / (1 + e^-(g . x_t)), g: [H]. */
double oracle_shared_gate_row(int32_t H, const uint16_t *g, const uint16_t *x)
{
    double z = 0.0;
    for (int32_t c = 0; c < H; ++c) z += bf16_to_f64(g[c]) * bf16_to_f64(x[c]);
    return 1.0 / (1.0 + exp(-z));
}

/* ---------------------------------------------------------------------- */
/* Expert FFN + combine for given routing, for a chosen set of rows.       */
/* ---------------------------------------------------------------------- */
/* For each listed token t = rows[r]:
 *   out[r, :] = sum_{j < keff[t]} w[t, j] * FFN_{idx[t, j]}(x_t)
 *             + [Is > 0] * sigmoid(g . x_t) * FFN_shared(x_t)
 * (slots summed in order, the shared expert last, all in fp64).
 * Weights: w_gate[e], w_up[e] point to expert e's [I, H] projections and
 * w_down[e] to its [H, I] projection (an entry may be NULL when no listed
 * row routes to e); ws_gate, ws_up [Is, H]; ws_down [H, Is]; ws_gvec [H]
 * (all bf16 bit patterns, row-major).  scales [E][3] and shared_scales [3]
 * (NULL: none) are the per-projection output factors of swiglu_ffn. */
int oracle_combine_rows(int32_t T, int32_t H, int32_t I, int32_t k, int32_t Is,
                        const uint16_t *x, const int32_t *idx, const float *w, const int32_t *keff,
                        const uint16_t *const *w_gate, const uint16_t *const *w_up,
                        const uint16_t *const *w_down,
                        const uint16_t *ws_gate, const uint16_t *ws_up, const uint16_t *ws_down,
                        const uint16_t *ws_gvec, const double *scales, const double *shared_scales,
                        int32_t n_rows, const int32_t *rows, double *out, int32_t nthreads)
{
    if (T < 0 || H < 1 || I < 1 || k < 1 || Is < 0 || n_rows < 0) return ORACLE_EINVAL;
    for (int32_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= T) return ORACLE_EINVAL;
    const int32_t per_tok = k + (Is > 0 ? 1 : 0);
    const int32_t n_jobs = n_rows * per_tok;
    double *ys = (double *)malloc(sizeof(double) * (size_t)(n_jobs > 0 ? n_jobs : 1) * H);
    if (!ys) return ORACLE_ENOMEM;
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        int32_t hmax = I > Is ? I : Is;
        double *hbuf = (double *)malloc(sizeof(double) * (size_t)hmax);
        if (!hbuf) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int32_t job = 0; job < n_jobs; ++job) {
                int32_t r = job / per_tok, j = job % per_tok, t = rows[r];
                const uint16_t *xt = x + (size_t)t * H;
                double *y = ys + (size_t)job * H;
                if (j < k) {
                    if (j >= keff[t]) continue;
                    int32_t e = idx[(size_t)t * k + j];
                    if (e < 0 || !w_gate[e] || !w_up[e] || !w_down[e]) {
#pragma omp atomic write
                        err = 2;
                        continue;
                    }
                    swiglu_ffn(H, I, w_gate[e], w_up[e], w_down[e], scales ? scales + (size_t)e * 3 : NULL, xt,
                               hbuf, y);
                } else {
                    swiglu_ffn(H, Is, ws_gate, ws_up, ws_down, shared_scales, xt, hbuf, y);
                }
            }
        }
        free(hbuf);
    }
    if (err) { free(ys); return err == 2 ? ORACLE_EINVAL : ORACLE_ENOMEM; }
    /* combine: weighted sum in slot order, then the gated shared expert */
    for (int32_t r = 0; r < n_rows; ++r) {
        int32_t t = rows[r];
        double *o = out + (size_t)r * H;
        for (int32_t c = 0; c < H; ++c) o[c] = 0.0;
        for (int32_t j = 0; j < keff[t]; ++j) {
            double wj = (double)w[(size_t)t * k + j];
            const double *y = ys + ((size_t)r * per_tok + j) * H;
            for (int32_t c = 0; c < H; ++c) o[c] += wj * y[c];
        }
        if (Is > 0) {
            double s = oracle_shared_gate_row(H, ws_gvec, x + (size_t)t * H);
            const double *y = ys + ((size_t)r * per_tok + k) * H;
            for (int32_t c = 0; c < H; ++c) o[c] += s * y[c];
        }
    }
    free(ys);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Whole layer: route -> top-p -> budget -> dispatch over all T tokens    */
/* (the budget couples tokens), then FFN + combine for the listed rows.    */
/* ---------------------------------------------------------------------- */
int oracle_forward(int32_t T, int32_t H, int32_t E, int32_t I, int32_t k, int32_t Is,
                   int32_t norm_topk, int32_t budget, float topp,
                   const uint16_t *x, const float *logits,
                   const uint16_t *const *w_gate, const uint16_t *const *w_up,
                   const uint16_t *const *w_down,
                   const uint16_t *ws_gate, const uint16_t *ws_up, const uint16_t *ws_down,
                   const uint16_t *ws_gvec, const double *scales, const double *shared_scales,
                   int32_t n_rows, const int32_t *rows, double *out,
                   int32_t *idx, float *w, int32_t *keff, uint8_t *kept, int32_t *n_dropped,
                   int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *slot_pos,
                   int32_t nthreads)
{
    if (T < 0 || H < 1 || E < 1 || I < 1 || k < 1 || k > E || Is < 0 || budget < 0 || n_rows < 0)
        return ORACLE_EINVAL;
    int rc = oracle_route(T, E, k, norm_topk, logits, idx, w);
    if (rc) return rc;
    rc = oracle_topp(T, k, norm_topk, topp, idx, w, keff);
    if (rc) return rc;
    rc = oracle_budget(T, E, k, budget, norm_topk, idx, w, keff, kept, n_dropped);
    if (rc) return rc;
    rc = oracle_dispatch(T, E, k, idx, keff, counts, offsets, perm, slot_pos);
    if (rc) return rc;
    return oracle_combine_rows(T, H, I, k, Is, x, idx, w, keff, w_gate, w_up, w_down,
                               ws_gate, ws_up, ws_down, ws_gvec, scales, shared_scales, n_rows, rows, out,
                               nthreads);
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
