/*
 * uno_ref.c -- the ORACLE for UNO's per-cycle sampling and verification step.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, single-threaded CPU
 * restatement, in double precision, of what the CUDA library computes.  Only
 * the test suite, the package smoke check and the benchmark's CPU-baseline leg
 * may build, load or call it.  It shares no source, header, constant table or
 * helper with the CUDA library, and the library never calls it.
 *
 * Sources.  The method is described on two web pages:
 *   [UNO PR]        "sgl-project/sglang pull request 37667: UNO" -- sections
 *                   "Motivation", "Modifications", and the review thread on
 *                   the filter order (top-k renormalised before top-p).
 *   [eval guide]    "用 SGLang benchmark/uno 复现 UNO 全量数学评测：
 *                   run_math_eval 实战与源码解析" -- sections
 *                   "run_math_eval 全参数详解" (sampling-parameter checks),
 *                   "B/K/V 参数映射" and "启动期硬性约束" (tree constraints).
 * The pages name the steps but print no formula for them.  Where they are
 * silent this file takes the plainest reading that the rest supports; every
 * such reading is listed in the design notes and repeated at the function
 * that takes it.
 *
 * Every function below keeps the steps in the order the method states them,
 * with no blocking, fusion or reordering: a full sort of the row for top-k,
 * a sequential walk for top-p, a sequential inverse-CDF for sampling, a
 * sequential accept/reject loop for linear verification, a linear-scan
 * best-first expansion for the tree, and a root-to-leaf walk for tree
 * verification.
 *
 * Parity status of each function (what pins it) is listed in the file header
 * of the Python wrapper (oracle/__init__.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- identifiers of this oracle (its own copies of the definitions) ---- */
enum { REF_F32 = 0, REF_BF16 = 1 };
/* Which random draw a uniform feeds (third counter word). */
enum { DRAW_PROPOSAL = 0, DRAW_ACCEPT = 1, DRAW_RESIDUAL = 2, DRAW_TARGET = 3 };
/* Per-row / per-request data-error bits. */
#define FLAG_NONFINITE_ROW 1u        /* NaN or +inf logit, or no finite logit */
#define FLAG_DRAFT_NOT_IN_SUPPORT 2u /* draft token has q = 0: rejected w.p. 1 */
#define FLAG_RESIDUAL_EMPTY 4u       /* max(0, p - q) summed to 0: sampled p */

/* Filter order.  TOPK_FIRST: the top-p cut is taken on the top-k set
 * renormalised (the speculative-decoding convention UNO follows).  JOINT: the
 * top-p cut is taken on the full-vocabulary softmax (the order of the regular
 * autoregressive sampler the review asks UNO to align with). */
enum { ORDER_TOPK_FIRST = 0, ORDER_JOINT = 1 };

/* Return codes. */
enum { REF_OK = 0, REF_ERR_INVALID_ARG = 1, REF_ERR_UNSUPPORTED = 2, REF_ERR_NOMEM = 5 };

/* =====================================================================
 * Philox4x32-10 (Salmon, Moraes, Dror & Shaw, "Parallel random numbers:
 * as easy as 1, 2, 3", SC'11).  Ten rounds; each round multiplies words 0
 * and 2 by the two Philox multipliers, takes the high and low halves, and
 * mixes in the round key; the key is bumped by the two Weyl constants
 * before every round after the first.
 * ===================================================================== */
void uno_ref_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t prod0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
        uint64_t prod1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(prod0 >> 32), lo0 = (uint32_t)prod0;
        uint32_t hi1 = (uint32_t)(prod1 >> 32), lo1 = (uint32_t)prod1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The uniform a decision draws: Philox4x32-10 with key = the 64-bit seed
 * (low word first) and counter = (request, position, draw, cycle); the first
 * 32 bits of output followed by the top 21 bits of the second word form a
 * 53-bit integer m, and u = m * 2^-53 lies in [0, 1).  Counter-based, so any
 * draw of any cycle can be recomputed on its own. */
/* Uniform injection, for the exact-enumeration pins only: while a table is
 * set, the uniform of (request r, position i, draw d) with r < nreq and
 * i < npos is table[(r * npos + i) * 4 + d] instead of the Philox draw (seed
 * and cycle are then ignored).  Every decision of the oracle takes its
 * uniform from uno_ref_uniform, so a test can run the oracle's own decision
 * code at chosen uniforms and measure, by bisection on the 53-bit grid, the
 * exact probability of each branch. */
static const double* g_u_table = NULL;
static int64_t g_u_nreq = 0;
static int32_t g_u_npos = 0;

void uno_ref_set_uniforms(const double* table, int64_t nreq, int32_t npos)
{
    g_u_table = (table != NULL && nreq > 0 && npos > 0) ? table : NULL;
    g_u_nreq = g_u_table ? nreq : 0;
    g_u_npos = g_u_table ? npos : 0;
}

double uno_ref_uniform(uint64_t seed, uint32_t request, uint32_t position, uint32_t draw, uint32_t cycle)
{
    if (g_u_table != NULL && (int64_t)request < g_u_nreq && (int32_t)position < g_u_npos && draw < 4u)
        return g_u_table[((int64_t)request * g_u_npos + (int64_t)position) * 4 + (int64_t)draw];
    uint32_t ctr[4] = {request, position, draw, cycle};
    uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};
    uint32_t x[4];
    uno_ref_philox4x32_10(ctr, key, x);
    uint64_t m = ((uint64_t)x[0] << 21) | (uint64_t)(x[1] >> 11);
    return (double)m * 0x1p-53;
}

/* ---- logits decoding: bf16 is the top half of an IEEE binary32 ---- */
static float decode_logit(const void* base, int dtype, int64_t idx)
{
    if (dtype == REF_F32) return ((const float*)base)[idx];
    uint16_t h = ((const uint16_t*)base)[idx];
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

typedef struct {
    float v;
    int32_t id;
} ref_entry;

/* Order: raw logit descending, then token id ascending.  Ties are decided on
 * the raw logits before any temperature scaling. */
static int cmp_value_desc_id_asc(const void* pa, const void* pb)
{
    const ref_entry* a = (const ref_entry*)pa;
    const ref_entry* b = (const ref_entry*)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->id > b->id) - (a->id < b->id);
}

static int cmp_id_asc(const void* pa, const void* pb)
{
    const ref_entry* a = (const ref_entry*)pa;
    const ref_entry* b = (const ref_entry*)pb;
    return (a->id > b->id) - (a->id < b->id);
}

static double min_d(double a, double b) { return a < b ? a : b; }

/* =====================================================================
 * Filter one row: temperature, top-k, then top-p, then renormalise.
 *
 * [UNO PR, review thread on the filter order]: UNO keeps the top-k tokens,
 * renormalises over them, and applies the top-p cut to that renormalised
 * distribution (the speculative-decoding convention), so the full-vocabulary
 * softmax is never formed.  The same thread names the regular sampler's
 * "joint" order, where the top-p cut is computed from the full softmax; with
 * order = ORDER_JOINT step 4 divides by the sum over every finite token
 * instead (top-k still bounds the kept set, and the kept weights are still
 * renormalised among themselves in step 6).  [eval guide, run_math_eval
 * 全参数详解]: top_k > 0, top_p in (0, 1], temperature >= 0.
 *
 * Steps, in order:
 *  1. a NaN or +inf logit, or a row with no finite logit, makes the row
 *     non-finite: no support, flag NONFINITE_ROW;
 *  2. sort the finite logits by (logit desc, id asc) and keep the first
 *     k' = min(top_k, #finite);
 *  3. temperature 0 is greedy: the first entry alone, probability 1;
 *  4. otherwise w_j = exp((l_j - l_0) / T), S = sum_j w_j (in that order),
 *     P_j = w_j / S; under the joint order S also adds, in the same order,
 *     the weights of the finite tokens beyond the first k';
 *  5. top-p: walk in that order with the mass m accumulated before j; keep j
 *     when j = 0 or m < top_p, stop at the first j that fails; top_p >= 1
 *     keeps all k';
 *  6. renormalise: prob_j = w_j / W with W = sum of the kept w_j (in order);
 *  7. store (id, prob rounded to binary32) in ascending id order.
 * Returns the kept count.  *margin receives min |m - top_p| over the top-p
 * comparisons made (the distance of that integer decision from its flip).
 * ===================================================================== */
static int filter_row(const void* row, int dtype, int64_t vocab, double T, int32_t top_k, double top_p,
                      int order, int32_t* ids, float* probs, uint32_t* flags, double* margin, int* nomem)
{
    *margin = INFINITY;
    ref_entry* e = (ref_entry*)malloc((size_t)(vocab > 0 ? vocab : 1) * sizeof(ref_entry));
    if (!e) {
        *nomem = 1;
        return 0;
    }
    int64_t n = 0;
    int bad = 0;
    for (int64_t j = 0; j < vocab; ++j) {
        float f = decode_logit(row, dtype, j);
        if (isnan(f) || (isinf(f) && f > 0)) {
            bad = 1;
        } else if (!isinf(f)) {
            e[n].v = f;
            e[n].id = (int32_t)j;
            ++n;
        }
    }
    if (bad || n == 0) {
        *flags |= FLAG_NONFINITE_ROW;
        free(e);
        return 0;
    }
    qsort(e, (size_t)n, sizeof(ref_entry), cmp_value_desc_id_asc);
    int64_t kk = top_k < n ? top_k : n;

    double* w = (double*)malloc((size_t)kk * sizeof(double));
    if (!w) {
        free(e);
        *nomem = 1;
        return 0;
    }
    int64_t kept;
    if (T == 0.0) {
        kept = 1;
        w[0] = 1.0;
    } else {
        for (int64_t j = 0; j < kk; ++j) w[j] = exp(((double)e[j].v - (double)e[0].v) / T);
        double S = 0.0;
        for (int64_t j = 0; j < kk; ++j) S += w[j];
        if (order == ORDER_JOINT)
            for (int64_t j = kk; j < n; ++j) S += exp(((double)e[j].v - (double)e[0].v) / T);
        if (top_p >= 1.0) {
            kept = kk;
        } else {
            double m = 0.0;
            kept = 0;
            for (int64_t j = 0; j < kk; ++j) {
                if (j > 0) {
                    *margin = min_d(*margin, fabs(m - top_p));
                    if (!(m < top_p)) break;
                }
                m += w[j] / S;
                ++kept;
            }
        }
    }
    double W = 0.0;
    for (int64_t j = 0; j < kept; ++j) W += w[j];
    ref_entry* out = (ref_entry*)malloc((size_t)kept * sizeof(ref_entry));
    if (!out) {
        free(w);
        free(e);
        *nomem = 1;
        return 0;
    }
    for (int64_t j = 0; j < kept; ++j) {
        out[j] = e[j];
        out[j].v = (float)(w[j] / W); /* reuse the value slot for the probability */
    }
    qsort(out, (size_t)kept, sizeof(ref_entry), cmp_id_asc);
    for (int64_t j = 0; j < kept; ++j) {
        ids[j] = out[j].id;
        probs[j] = out[j].v;
    }
    free(out);
    free(w);
    free(e);
    return (int)kept;
}

/* =====================================================================
 * Inverse-CDF draw over a weight list in the order given (ascending token id
 * everywhere in this file): S = sum of weights in order, C_j the inclusive
 * prefix sums in order; return the first j with u*S < C_j, or, if rounding
 * leaves none, the last j whose weight is positive.  Returns -1 when every
 * weight is zero.  *margin receives min_j |u*S - C_j| / S over the internal
 * boundaries j = 0 .. n-2.
 * ===================================================================== */
static int inv_cdf(const double* wts, int n, double u, double* margin)
{
    double S = 0.0;
    for (int j = 0; j < n; ++j) S += wts[j];
    *margin = INFINITY;
    if (!(S > 0.0)) return -1;
    double x = u * S;
    double c = 0.0;
    int pick = -1;
    for (int j = 0; j < n; ++j) {
        c += wts[j];
        if (j < n - 1) *margin = min_d(*margin, fabs(x - c) / S);
        if (pick < 0 && x < c) pick = j;
    }
    if (pick < 0) {
        for (int j = n - 1; j >= 0; --j)
            if (wts[j] > 0.0) {
                pick = j;
                break;
            }
    }
    return pick;
}

/* Probability of token `tok` in a compact support (ids ascending). */
static double lookup_prob(const int32_t* ids, const float* probs, int count, int32_t tok)
{
    for (int j = 0; j < count; ++j)
        if (ids[j] == tok) return (double)probs[j];
    return 0.0;
}

static int check_params(float temperature, int32_t top_k, float top_p)
{
    /* [eval guide, run_math_eval 全参数详解]: top_k positive, top_p in (0, 1],
     * temperature non-negative. */
    if (!(temperature >= 0.0f) || isinf(temperature)) return 0;
    if (top_k < 1) return 0;
    if (!(top_p > 0.0f && top_p <= 1.0f)) return 0;
    return 1;
}

/* Sampling parameters of a call: request r uses temperature[r * stride],
 * top_k[r * stride] and top_p[r * stride] (stride 0 gives every request the
 * same values), and every row of the call is filtered in one order. */
typedef struct {
    const float* temperature;
    const int32_t* top_k;
    const float* top_p;
    int64_t stride;
    int order;
} ref_params;

static double sp_T(const ref_params* sp, int64_t r) { return (double)sp->temperature[r * sp->stride]; }
static int32_t sp_k(const ref_params* sp, int64_t r) { return sp->top_k[r * sp->stride]; }
static double sp_p(const ref_params* sp, int64_t r) { return (double)sp->top_p[r * sp->stride]; }

/* Check the parameters of requests 0 .. nreq-1 (just entry 0 when stride is
 * 0) and the order; *need receives the largest min(top_k, vocab), the
 * compact width a row of the call can fill. */
static int check_call_params(const ref_params* sp, int64_t nreq, int64_t vocab, int32_t* need)
{
    if (!sp->temperature || !sp->top_k || !sp->top_p) return 0;
    if (sp->order != ORDER_TOPK_FIRST && sp->order != ORDER_JOINT) return 0;
    int64_t n = sp->stride == 0 ? 1 : nreq;
    int64_t most = 0;
    for (int64_t r = 0; r < n; ++r) {
        if (!check_params(sp->temperature[r * sp->stride], sp->top_k[r * sp->stride], sp->top_p[r * sp->stride]))
            return 0;
        int64_t k = sp->top_k[r * sp->stride] < vocab ? sp->top_k[r * sp->stride] : vocab;
        if (k > most) most = k;
    }
    *need = (int32_t)most;
    return 1;
}

static ref_params scalar_params(const float* temperature, const int32_t* top_k, const float* top_p)
{
    ref_params sp = {temperature, top_k, top_p, 0, ORDER_TOPK_FIRST};
    return sp;
}

/* =====================================================================
 * uno_ref_filter_softmax: filter every row (see filter_row) and, when
 * has_rng, draw one token per row from the stored compact distribution by
 * inverse CDF with the uniform (seed, request, position, PROPOSAL, cycle),
 * where request = first_request + row / rows_per_request and position =
 * row % rows_per_request.  In every entry point, first_request is the global
 * index of the call's first request (the RNG counter's request word).
 * [UNO PR, Motivation]: the linear sampler draws each of the B draft tokens
 * independently from its own marginal.
 *
 * logits: rows x row_stride elements (f32 or bf16 bits); out_ids/out_probs:
 * rows x cap; out_count, out_flags: rows; out_dense (nullable): rows x vocab;
 * out_sample (nullable): rows; out_margin (nullable): rows, the smaller of
 * the top-p and the draw margins.
 *
 * uno_ref_filter_softmax_params is the same with one temperature, top_k and
 * top_p per request (arrays of ceil(rows / rows_per_request) entries) and a
 * filter order (ORDER_TOPK_FIRST or ORDER_JOINT); cap must hold the largest
 * min(top_k, vocab) of the call.
 * ===================================================================== */
static int filter_softmax_impl(const void* logits, int dtype, int64_t rows, int64_t vocab, int64_t row_stride,
                               int32_t rows_per_request, const ref_params* sp, int32_t cap, int32_t* out_ids,
                               float* out_probs, int32_t* out_count, float* out_dense, int has_rng, uint64_t seed,
                               uint32_t cycle, uint32_t first_request, int32_t* out_sample, uint32_t* out_flags,
                               double* out_margin)
{
    if (!logits || !out_ids || !out_probs || !out_count || !out_flags) return REF_ERR_INVALID_ARG;
    if (rows < 0 || vocab <= 0 || row_stride < vocab || rows_per_request < 1) return REF_ERR_INVALID_ARG;
    if (dtype != REF_F32 && dtype != REF_BF16) return REF_ERR_INVALID_ARG;
    int32_t need;
    if (!check_call_params(sp, (rows + rows_per_request - 1) / rows_per_request, vocab, &need))
        return REF_ERR_INVALID_ARG;
    if (has_rng && !out_sample) return REF_ERR_INVALID_ARG;
    if (cap < need) return REF_ERR_UNSUPPORTED;
    size_t esz = dtype == REF_F32 ? 4 : 2;
    for (int64_t r = 0; r < rows; ++r) {
        const char* row = (const char*)logits + (size_t)r * (size_t)row_stride * esz;
        int32_t* ids = out_ids + (size_t)r * (size_t)cap;
        float* probs = out_probs + (size_t)r * (size_t)cap;
        uint32_t flags = 0;
        double m_top = INFINITY, m_draw = INFINITY;
        int nomem = 0;
        int64_t rq = r / rows_per_request;
        int cnt = filter_row(row, dtype, vocab, sp_T(sp, rq), sp_k(sp, rq), sp_p(sp, rq), sp->order, ids, probs,
                             &flags, &m_top, &nomem);
        if (nomem) return REF_ERR_NOMEM;
        for (int j = cnt; j < cap; ++j) {
            ids[j] = -1;
            probs[j] = 0.0f;
        }
        out_count[r] = cnt;
        out_flags[r] = flags;
        if (out_dense) {
            float* d = out_dense + (size_t)r * (size_t)vocab;
            for (int64_t j = 0; j < vocab; ++j) d[j] = 0.0f;
            for (int j = 0; j < cnt; ++j) d[ids[j]] = probs[j];
        }
        if (has_rng) {
            int32_t tok = -1;
            if (cnt > 0) {
                double* wts = (double*)malloc((size_t)cnt * sizeof(double));
                if (!wts) return REF_ERR_NOMEM;
                for (int j = 0; j < cnt; ++j) wts[j] = (double)probs[j];
                double u = uno_ref_uniform(seed, first_request + (uint32_t)(r / rows_per_request),
                                           (uint32_t)(r % rows_per_request), DRAW_PROPOSAL, cycle);
                int pick = inv_cdf(wts, cnt, u, &m_draw);
                tok = pick >= 0 ? ids[pick] : -1;
                free(wts);
            }
            out_sample[r] = tok;
        }
        if (out_margin) out_margin[r] = min_d(m_top, m_draw);
    }
    return REF_OK;
}

int uno_ref_filter_softmax(const void* logits, int dtype, int64_t rows, int64_t vocab, int64_t row_stride,
                           int32_t rows_per_request, float temperature, int32_t top_k, float top_p, int32_t cap,
                           int32_t* out_ids, float* out_probs, int32_t* out_count, float* out_dense, int has_rng,
                           uint64_t seed, uint32_t cycle, uint32_t first_request, int32_t* out_sample,
                           uint32_t* out_flags, double* out_margin)
{
    ref_params sp = scalar_params(&temperature, &top_k, &top_p);
    return filter_softmax_impl(logits, dtype, rows, vocab, row_stride, rows_per_request, &sp, cap, out_ids,
                               out_probs, out_count, out_dense, has_rng, seed, cycle, first_request, out_sample,
                               out_flags, out_margin);
}

int uno_ref_filter_softmax_params(const void* logits, int dtype, int64_t rows, int64_t vocab, int64_t row_stride,
                                  int32_t rows_per_request, const float* temperature, const int32_t* top_k,
                                  const float* top_p, int order, int32_t cap, int32_t* out_ids, float* out_probs,
                                  int32_t* out_count, float* out_dense, int has_rng, uint64_t seed, uint32_t cycle,
                                  uint32_t first_request, int32_t* out_sample, uint32_t* out_flags,
                                  double* out_margin)
{
    ref_params sp = {temperature, top_k, top_p, 1, order};
    return filter_softmax_impl(logits, dtype, rows, vocab, row_stride, rows_per_request, &sp, cap, out_ids,
                               out_probs, out_count, out_dense, has_rng, seed, cycle, first_request, out_sample,
                               out_flags, out_margin);
}

/* =====================================================================
 * uno_ref_linear_verify: linear-mode rejection sampling for R requests.
 *
 * [UNO PR, Motivation]: UNO is lossless like speculative decoding; the
 * diffusion pathway drafts B tokens from independent marginals q_1..q_B and
 * the AR pathway verifies them.  [UNO PR, Modifications]: proposal and
 * rejection sampling for linear UNO.  The pages print no formula; the
 * standard speculative-sampling rule is the reading taken:
 *   for i = 0 .. B-1 (0-based position): x = draft_ids[r][i], a = q_i(x);
 *     a = 0 (x outside supp q_i) rejects with probability 1 (flagged);
 *     otherwise accept iff u_ACCEPT(r, i) * a < p_i(x);
 *     on the first rejection draw y from normalise(max(0, p_i - q_i)) over
 *     supp p_i with u_RESIDUAL(r, i) (if that residual sums to 0, draw from
 *     p_i instead and flag), emit x_0..x_{i-1}, y and stop;
 *   if all B are accepted, draw the bonus y from p_B with u_TARGET(r, B).
 * p_i is target row i filtered exactly as filter_row does, kept as binary32
 * probabilities; q_i is the caller's compact support (binary32).  All the
 * arithmetic of a decision is double.
 * A non-finite target row that is reached stops the request there with token
 * -1 (flag NONFINITE_ROW; every non-finite target row of the request sets it).
 *
 * target_logits: R x (B+1) x vocab; draft_ids: R x B; q_*: (R*B) x q_cap;
 * outputs: out_tokens R x (B+1) (unused slots -1), out_accept_len,
 * out_num_tokens, out_flags, out_margin (nullable): R.
 *
 * uno_ref_linear_verify_params is the same with per-request sampling
 * parameters (arrays of R) and a filter order for the target rows.
 * ===================================================================== */
static int linear_verify_impl(const void* target_logits, int dtype, int32_t R, int32_t B, int64_t vocab,
                              const ref_params* sp, const int32_t* draft_ids, const int32_t* q_ids,
                              const float* q_probs, const int32_t* q_count, int32_t q_cap, uint64_t seed,
                              uint32_t cycle, uint32_t first_request, int32_t* out_tokens, int32_t* out_accept_len,
                              int32_t* out_num_tokens, uint32_t* out_flags, double* out_margin)
{
    if (!target_logits || !draft_ids || !q_ids || !q_probs || !q_count || !out_tokens || !out_accept_len ||
        !out_num_tokens || !out_flags)
        return REF_ERR_INVALID_ARG;
    if (R < 0 || B < 1 || vocab <= 0 || q_cap < 1) return REF_ERR_INVALID_ARG;
    if (dtype != REF_F32 && dtype != REF_BF16) return REF_ERR_INVALID_ARG;
    int32_t cap;
    if (!check_call_params(sp, R, vocab, &cap)) return REF_ERR_INVALID_ARG;
    if (cap < 1) cap = 1;
    size_t esz = dtype == REF_F32 ? 4 : 2;

    int32_t* p_ids = (int32_t*)malloc((size_t)(B + 1) * (size_t)cap * sizeof(int32_t));
    float* p_probs = (float*)malloc((size_t)(B + 1) * (size_t)cap * sizeof(float));
    int* p_cnt = (int*)malloc((size_t)(B + 1) * sizeof(int));
    double* wts = (double*)malloc((size_t)cap * sizeof(double));
    if (!p_ids || !p_probs || !p_cnt || !wts) {
        free(p_ids); free(p_probs); free(p_cnt); free(wts);
        return REF_ERR_NOMEM;
    }
    for (int32_t r = 0; r < R; ++r) {
        uint32_t flags = 0;
        double margin = INFINITY;
        /* filter the B+1 target rows of this request */
        for (int32_t i = 0; i <= B; ++i) {
            const char* row = (const char*)target_logits + ((size_t)r * (size_t)(B + 1) + (size_t)i) * (size_t)vocab * esz;
            double m_top;
            int nomem = 0;
            p_cnt[i] = filter_row(row, dtype, vocab, sp_T(sp, r), sp_k(sp, r), sp_p(sp, r), sp->order,
                                  p_ids + (size_t)i * (size_t)cap, p_probs + (size_t)i * (size_t)cap, &flags,
                                  &m_top, &nomem);
            if (nomem) {
                free(p_ids); free(p_probs); free(p_cnt); free(wts);
                return REF_ERR_NOMEM;
            }
            margin = min_d(margin, m_top);
        }
        int32_t* toks = out_tokens + (size_t)r * (size_t)(B + 1);
        for (int32_t i = 0; i <= B; ++i) toks[i] = -1;
        int32_t acc = B, ntok = B + 1;
        for (int32_t i = 0; i < B; ++i) {
            const int32_t* pi_ids = p_ids + (size_t)i * (size_t)cap;
            const float* pi_pr = p_probs + (size_t)i * (size_t)cap;
            const int32_t qrow = r * B + i;
            const int32_t* qi_ids = q_ids + (size_t)qrow * (size_t)q_cap;
            const float* qi_pr = q_probs + (size_t)qrow * (size_t)q_cap;
            int qc = q_count[qrow];
            if (qc < 0) qc = 0;
            if (qc > q_cap) qc = q_cap;
            if (p_cnt[i] == 0) { /* reached a non-finite target row */
                acc = i;
                ntok = i;
                break;
            }
            int32_t x = draft_ids[(size_t)r * (size_t)B + (size_t)i];
            double a = (x >= 0 && x < vocab) ? lookup_prob(qi_ids, qi_pr, qc, x) : 0.0;
            double px = (x >= 0 && x < vocab) ? lookup_prob(pi_ids, pi_pr, p_cnt[i], x) : 0.0;
            int accept = 0;
            if (a > 0.0) {
                double u = uno_ref_uniform(seed, first_request + (uint32_t)r, (uint32_t)i, DRAW_ACCEPT, cycle);
                accept = (u * a < px);
                margin = min_d(margin, fabs(u * a - px) / a);
            } else {
                flags |= FLAG_DRAFT_NOT_IN_SUPPORT;
            }
            if (accept) {
                toks[i] = x;
                continue;
            }
            /* residual max(0, p_i - q_i) over supp p_i, ascending id */
            double tot = 0.0;
            for (int j = 0; j < p_cnt[i]; ++j) {
                double d = (double)pi_pr[j] - lookup_prob(qi_ids, qi_pr, qc, pi_ids[j]);
                wts[j] = d > 0.0 ? d : 0.0;
                tot += wts[j];
            }
            if (!(tot > 0.0)) {
                flags |= FLAG_RESIDUAL_EMPTY;
                for (int j = 0; j < p_cnt[i]; ++j) wts[j] = (double)pi_pr[j];
            }
            double u = uno_ref_uniform(seed, first_request + (uint32_t)r, (uint32_t)i, DRAW_RESIDUAL, cycle);
            double md;
            int pick = inv_cdf(wts, p_cnt[i], u, &md);
            margin = min_d(margin, md);
            toks[i] = pick >= 0 ? pi_ids[pick] : -1;
            acc = i;
            ntok = i + 1;
            break;
        }
        if (acc == B && ntok == B + 1) { /* every draft accepted: bonus from p_B */
            if (p_cnt[B] == 0) {
                ntok = B;
            } else {
                for (int j = 0; j < p_cnt[B]; ++j) wts[j] = (double)p_probs[(size_t)B * (size_t)cap + (size_t)j];
                double u = uno_ref_uniform(seed, first_request + (uint32_t)r, (uint32_t)B, DRAW_TARGET, cycle);
                double md;
                int pick = inv_cdf(wts, p_cnt[B], u, &md);
                margin = min_d(margin, md);
                toks[B] = pick >= 0 ? p_ids[(size_t)B * (size_t)cap + (size_t)pick] : -1;
            }
        }
        out_accept_len[r] = acc;
        out_num_tokens[r] = ntok;
        out_flags[r] = flags;
        if (out_margin) out_margin[r] = margin;
    }
    free(p_ids); free(p_probs); free(p_cnt); free(wts);
    return REF_OK;
}

int uno_ref_linear_verify(const void* target_logits, int dtype, int32_t R, int32_t B, int64_t vocab,
                          float temperature, int32_t top_k, float top_p, const int32_t* draft_ids,
                          const int32_t* q_ids, const float* q_probs, const int32_t* q_count, int32_t q_cap,
                          uint64_t seed, uint32_t cycle, uint32_t first_request, int32_t* out_tokens,
                          int32_t* out_accept_len, int32_t* out_num_tokens, uint32_t* out_flags,
                          double* out_margin)
{
    ref_params sp = scalar_params(&temperature, &top_k, &top_p);
    return linear_verify_impl(target_logits, dtype, R, B, vocab, &sp, draft_ids, q_ids, q_probs, q_count, q_cap,
                              seed, cycle, first_request, out_tokens, out_accept_len, out_num_tokens, out_flags,
                              out_margin);
}

int uno_ref_linear_verify_params(const void* target_logits, int dtype, int32_t R, int32_t B, int64_t vocab,
                                 const float* temperature, const int32_t* top_k, const float* top_p, int order,
                                 const int32_t* draft_ids, const int32_t* q_ids, const float* q_probs,
                                 const int32_t* q_count, int32_t q_cap, uint64_t seed, uint32_t cycle,
                                 uint32_t first_request, int32_t* out_tokens, int32_t* out_accept_len,
                                 int32_t* out_num_tokens, uint32_t* out_flags, double* out_margin)
{
    ref_params sp = {temperature, top_k, top_p, 1, order};
    return linear_verify_impl(target_logits, dtype, R, B, vocab, &sp, draft_ids, q_ids, q_probs, q_count, q_cap,
                              seed, cycle, first_request, out_tokens, out_accept_len, out_num_tokens, out_flags,
                              out_margin);
}

/* =====================================================================
 * uno_ref_linear_cycle: one linear decoding cycle in the layout the pages
 * give UNO's two forward passes.
 *
 * [UNO PR, Motivation]: a cycle runs two target-model forward passes; the
 * diffusion-pathway pass yields the first output token and a block of draft
 * proposals, the AR-pathway pass verifies the proposals.  [eval guide,
 * 单模型双前向架构]: of a request's B draft rows the first runs on the base
 * weights and the other B - 1 on the UNO adapter.  [UNO PR, Modifications,
 * and the review thread on the token counters]: the scheduler slices B + 1
 * output rows per request, num_correct_drafts = accept_len - 2 counts the
 * accepted proposals, and a request adds num_correct_drafts + 2 generated
 * tokens (two tokens of a cycle are not drafts).
 *
 * Reading taken (the pages print no formula; the decisions are those of
 * uno_ref_linear_verify):
 *   draft row i (i = 0 .. B-1) is filtered and x_i drawn from it by inverse
 *   CDF (ascending ids) with u_PROPOSAL(r, i);
 *   x_0, drawn from the base-weights row, is output token 0 with no test;
 *   target row i (i = 0 .. B-1) is the AR pathway's distribution of output
 *   token i + 1, i.e. given x_0 .. x_i;
 *   for i = 1 .. B-1: a = q_i(x_i); a = 0 rejects w.p. 1 (flagged); else
 *   accept iff u_ACCEPT(r, i) * a < p_{i-1}(x_i); on the first rejection draw
 *   y from normalise(max(0, p_{i-1} - q_i)) over supp p_{i-1} with
 *   u_RESIDUAL(r, i) (p_{i-1} itself if that sums to 0, flagged), emit y as
 *   token i and stop; if every proposal is accepted, draw token B from
 *   target row B-1 with u_TARGET(r, B).
 * accept_len = the number of tokens emitted (at most B + 1);
 * num_correct_drafts = the number of accepted proposals, which is
 * accept_len - 2 whenever every row reached is finite.  A non-finite draft
 * row 0 emits nothing; a non-finite draft row i >= 1 has no support
 * (x_i = -1) and is rejected; a non-finite target row that is reached stops
 * the request without a further token.  Every non-finite row of the request,
 * draft or target, sets NONFINITE_ROW.
 *
 * draft_logits and target_logits: R x B x vocab each; parameters: one per
 * request (arrays of R) and one filter order for the rows of both passes;
 * outputs: out_tokens R x (B+1) (unused slots -1), out_accept_len,
 * out_num_correct_drafts, out_flags, out_margin (nullable): R.
 * ===================================================================== */
int uno_ref_linear_cycle(const void* draft_logits, const void* target_logits, int dtype, int32_t R, int32_t B,
                         int64_t vocab, const float* temperature, const int32_t* top_k, const float* top_p,
                         int order, uint64_t seed, uint32_t cycle, uint32_t first_request, int32_t* out_tokens,
                         int32_t* out_accept_len, int32_t* out_num_correct_drafts, uint32_t* out_flags,
                         double* out_margin)
{
    if (!draft_logits || !target_logits || !out_tokens || !out_accept_len || !out_num_correct_drafts || !out_flags)
        return REF_ERR_INVALID_ARG;
    if (R < 0 || B < 1 || vocab <= 0) return REF_ERR_INVALID_ARG;
    if (dtype != REF_F32 && dtype != REF_BF16) return REF_ERR_INVALID_ARG;
    ref_params sp = {temperature, top_k, top_p, 1, order};
    int32_t cap;
    if (!check_call_params(&sp, R, vocab, &cap)) return REF_ERR_INVALID_ARG;
    if (cap < 1) cap = 1;
    size_t esz = dtype == REF_F32 ? 4 : 2;
    size_t n = (size_t)B * (size_t)cap;
    int32_t* q_ids = (int32_t*)malloc(n * sizeof(int32_t));
    float* q_pr = (float*)malloc(n * sizeof(float));
    int32_t* p_ids = (int32_t*)malloc(n * sizeof(int32_t));
    float* p_pr = (float*)malloc(n * sizeof(float));
    int* q_cnt = (int*)malloc((size_t)B * sizeof(int));
    int* p_cnt = (int*)malloc((size_t)B * sizeof(int));
    int32_t* x = (int32_t*)malloc((size_t)B * sizeof(int32_t));
    double* wts = (double*)malloc((size_t)cap * sizeof(double));
    int nomem = !q_ids || !q_pr || !p_ids || !p_pr || !q_cnt || !p_cnt || !x || !wts;
    for (int32_t r = 0; r < R && !nomem; ++r) {
        uint32_t flags = 0;
        double margin = INFINITY, m;
        const uint32_t req = first_request + (uint32_t)r;
        /* the draft pass: filter the B rows and draw x_0 .. x_{B-1} */
        for (int32_t i = 0; i < B && !nomem; ++i) {
            const char* row = (const char*)draft_logits + ((size_t)r * (size_t)B + (size_t)i) * (size_t)vocab * esz;
            int32_t* ids = q_ids + (size_t)i * (size_t)cap;
            float* pr = q_pr + (size_t)i * (size_t)cap;
            q_cnt[i] = filter_row(row, dtype, vocab, sp_T(&sp, r), sp_k(&sp, r), sp_p(&sp, r), order, ids, pr, &flags,
                                  &m, &nomem);
            margin = min_d(margin, m);
            x[i] = -1;
            if (q_cnt[i] > 0) {
                for (int j = 0; j < q_cnt[i]; ++j) wts[j] = (double)pr[j];
                int pick = inv_cdf(wts, q_cnt[i], uno_ref_uniform(seed, req, (uint32_t)i, DRAW_PROPOSAL, cycle), &m);
                margin = min_d(margin, m);
                x[i] = pick >= 0 ? ids[pick] : -1;
            }
        }
        /* the verify pass: filter the B target rows */
        for (int32_t i = 0; i < B && !nomem; ++i) {
            const char* row = (const char*)target_logits + ((size_t)r * (size_t)B + (size_t)i) * (size_t)vocab * esz;
            p_cnt[i] = filter_row(row, dtype, vocab, sp_T(&sp, r), sp_k(&sp, r), sp_p(&sp, r), order,
                                  p_ids + (size_t)i * (size_t)cap, p_pr + (size_t)i * (size_t)cap, &flags, &m,
                                  &nomem);
            margin = min_d(margin, m);
        }
        if (nomem) break;
        int32_t* toks = out_tokens + (size_t)r * (size_t)(B + 1);
        for (int32_t t = 0; t <= B; ++t) toks[t] = -1;
        int32_t emitted = 0, correct = 0;
        if (q_cnt[0] > 0) {
            toks[0] = x[0]; /* the base-weights token: emitted untested */
            emitted = 1;
            int stopped = 0;
            for (int32_t i = 1; i < B; ++i) {
                const int32_t* pi_ids = p_ids + (size_t)(i - 1) * (size_t)cap;
                const float* pi_pr = p_pr + (size_t)(i - 1) * (size_t)cap;
                const int32_t* qi_ids = q_ids + (size_t)i * (size_t)cap;
                const float* qi_pr = q_pr + (size_t)i * (size_t)cap;
                if (p_cnt[i - 1] == 0) { /* a non-finite target row is reached */
                    stopped = 1;
                    break;
                }
                double a = x[i] >= 0 ? lookup_prob(qi_ids, qi_pr, q_cnt[i], x[i]) : 0.0;
                double px = x[i] >= 0 ? lookup_prob(pi_ids, pi_pr, p_cnt[i - 1], x[i]) : 0.0;
                if (a > 0.0) {
                    double u = uno_ref_uniform(seed, req, (uint32_t)i, DRAW_ACCEPT, cycle);
                    margin = min_d(margin, fabs(u * a - px) / a);
                    if (u * a < px) {
                        toks[i] = x[i];
                        ++emitted;
                        ++correct;
                        continue;
                    }
                } else {
                    flags |= FLAG_DRAFT_NOT_IN_SUPPORT;
                }
                double tot = 0.0;
                for (int j = 0; j < p_cnt[i - 1]; ++j) {
                    double d = (double)pi_pr[j] - lookup_prob(qi_ids, qi_pr, q_cnt[i], pi_ids[j]);
                    wts[j] = d > 0.0 ? d : 0.0;
                    tot += wts[j];
                }
                if (!(tot > 0.0)) {
                    flags |= FLAG_RESIDUAL_EMPTY;
                    for (int j = 0; j < p_cnt[i - 1]; ++j) wts[j] = (double)pi_pr[j];
                }
                int pick = inv_cdf(wts, p_cnt[i - 1], uno_ref_uniform(seed, req, (uint32_t)i, DRAW_RESIDUAL, cycle), &m);
                margin = min_d(margin, m);
                toks[i] = pick >= 0 ? pi_ids[pick] : -1;
                ++emitted;
                stopped = 1;
                break;
            }
            if (!stopped && p_cnt[B - 1] > 0) { /* every proposal accepted: the bonus token */
                const int32_t* pb_ids = p_ids + (size_t)(B - 1) * (size_t)cap;
                const float* pb_pr = p_pr + (size_t)(B - 1) * (size_t)cap;
                for (int j = 0; j < p_cnt[B - 1]; ++j) wts[j] = (double)pb_pr[j];
                int pick = inv_cdf(wts, p_cnt[B - 1], uno_ref_uniform(seed, req, (uint32_t)B, DRAW_TARGET, cycle), &m);
                margin = min_d(margin, m);
                toks[B] = pick >= 0 ? pb_ids[pick] : -1;
                ++emitted;
            }
        }
        out_accept_len[r] = emitted;
        out_num_correct_drafts[r] = correct;
        out_flags[r] = flags;
        if (out_margin) out_margin[r] = margin;
    }
    free(q_ids); free(q_pr); free(p_ids); free(p_pr); free(q_cnt); free(p_cnt); free(x); free(wts);
    return nomem ? REF_ERR_NOMEM : REF_OK;
}

/* =====================================================================
 * uno_ref_tree_topk_expand: candidate extraction and best-first expansion.
 *
 * [UNO PR, Motivation]: the tree sampler considers V candidate sequences by
 * selecting the top K candidates from each marginal; its hyperparameters are
 * (B, K, V).  [eval guide, B/K/V 参数映射]: B is the draft width, K the number
 * of candidates kept per depth (unrelated to the request's top_k), V the
 * verification width.  [eval guide, 启动期硬性约束]: V >= B, V <= 128,
 * V*K <= 2048.  The pages fix no construction rule; the rule taken here is:
 *   cand_d = the first min(K, count_d) entries of the filtered marginal q_d
 *            ordered by (binary32 probability desc, id asc), d = 0 .. B-1;
 *   node 0 is the root (token -1, parent -1, depth 0, score 1);
 *   a node at depth t < B has one child per c in cand_t with
 *            score = parent score * q_t(c)  (double);
 *   repeatedly move the best frontier node into the tree -- highest score,
 *   then lower depth, then lower parent index, then lower candidate rank --
 *   until the tree holds V nodes (root included) or the frontier is empty.
 * Node indices are assigned in that order, so a parent precedes its child.
 * The frontier here holds every child of every tree node (a linear scan picks
 * the best), the plain form of the rule.
 *
 * q_*: (R*B) x q_cap compact marginals (ids ascending); outputs R x V each
 * (unused slots: token -1, parent -1, depth -1, score 0) and num_nodes R.
 * ===================================================================== */
typedef struct {
    double score;
    int32_t depth, parent, rank, token;
} ref_cand;

static int cand_better(const ref_cand* a, const ref_cand* b)
{
    if (a->score != b->score) return a->score > b->score;
    if (a->depth != b->depth) return a->depth < b->depth;
    if (a->parent != b->parent) return a->parent < b->parent;
    return a->rank < b->rank;
}

typedef struct {
    float p;
    int32_t id;
} ref_qent;

static int cmp_prob_desc_id_asc(const void* pa, const void* pb)
{
    const ref_qent* a = (const ref_qent*)pa;
    const ref_qent* b = (const ref_qent*)pb;
    if (a->p > b->p) return -1;
    if (a->p < b->p) return 1;
    return (a->id > b->id) - (a->id < b->id);
}

int uno_ref_tree_topk_expand(const int32_t* q_ids, const float* q_probs, const int32_t* q_count, int32_t q_cap,
                             int32_t R, int32_t B, int32_t K, int32_t V, int32_t* node_token, int32_t* node_parent,
                             int32_t* node_depth, float* node_score, int32_t* num_nodes)
{
    if (!q_ids || !q_probs || !q_count || !node_token || !node_parent || !node_depth || !node_score || !num_nodes)
        return REF_ERR_INVALID_ARG;
    if (R < 0 || B < 1 || K < 1 || V < 1 || q_cap < 1) return REF_ERR_INVALID_ARG;
    if (V < B || V > 128 || (int64_t)V * K > 2048) return REF_ERR_INVALID_ARG;

    ref_qent* cand = (ref_qent*)malloc((size_t)B * (size_t)K * sizeof(ref_qent));
    int* ncand = (int*)malloc((size_t)B * sizeof(int));
    ref_qent* tmp = (ref_qent*)malloc((size_t)q_cap * sizeof(ref_qent));
    /* every child of every tree node: at most V * K entries */
    ref_cand* front = (ref_cand*)malloc((size_t)V * (size_t)K * sizeof(ref_cand) + sizeof(ref_cand));
    int8_t* used = (int8_t*)malloc((size_t)V * (size_t)K + 1);
    double* score = (double*)malloc((size_t)V * sizeof(double));
    if (!cand || !ncand || !tmp || !front || !used || !score) {
        free(cand); free(ncand); free(tmp); free(front); free(used); free(score);
        return REF_ERR_NOMEM;
    }
    for (int32_t r = 0; r < R; ++r) {
        for (int32_t d = 0; d < B; ++d) {
            int32_t row = r * B + d;
            int c = q_count[row];
            if (c < 0) c = 0;
            if (c > q_cap) c = q_cap;
            for (int j = 0; j < c; ++j) {
                tmp[j].p = q_probs[(size_t)row * (size_t)q_cap + (size_t)j];
                tmp[j].id = q_ids[(size_t)row * (size_t)q_cap + (size_t)j];
            }
            qsort(tmp, (size_t)c, sizeof(ref_qent), cmp_prob_desc_id_asc);
            int nk = c < K ? c : K;
            for (int j = 0; j < nk; ++j) cand[(size_t)d * (size_t)K + (size_t)j] = tmp[j];
            ncand[d] = nk;
        }
        int32_t* tok = node_token + (size_t)r * (size_t)V;
        int32_t* par = node_parent + (size_t)r * (size_t)V;
        int32_t* dep = node_depth + (size_t)r * (size_t)V;
        float* sco = node_score + (size_t)r * (size_t)V;
        for (int32_t j = 0; j < V; ++j) {
            tok[j] = -1; par[j] = -1; dep[j] = -1; sco[j] = 0.0f;
        }
        int n = 1, nf = 0;
        tok[0] = -1; par[0] = -1; dep[0] = 0; sco[0] = 1.0f; score[0] = 1.0;
        /* children of the root come from marginal 0 */
        for (int j = 0; j < ncand[0]; ++j) {
            front[nf].score = 1.0 * (double)cand[j].p;
            front[nf].depth = 1; front[nf].parent = 0; front[nf].rank = j; front[nf].token = cand[j].id;
            used[nf] = 0;
            ++nf;
        }
        while (n < V) {
            int best = -1;
            for (int f = 0; f < nf; ++f) {
                if (used[f]) continue;
                if (best < 0 || cand_better(&front[f], &front[best])) best = f;
            }
            if (best < 0) break;
            used[best] = 1;
            int idx = n++;
            tok[idx] = front[best].token;
            par[idx] = front[best].parent;
            dep[idx] = front[best].depth;
            score[idx] = front[best].score;
            sco[idx] = (float)front[best].score;
            int t = front[best].depth; /* children at depth t+1 come from marginal t */
            if (t < B) {
                for (int j = 0; j < ncand[t]; ++j) {
                    front[nf].score = score[idx] * (double)cand[(size_t)t * (size_t)K + (size_t)j].p;
                    front[nf].depth = t + 1; front[nf].parent = idx; front[nf].rank = j;
                    front[nf].token = cand[(size_t)t * (size_t)K + (size_t)j].id;
                    used[nf] = 0;
                    ++nf;
                }
            }
        }
        num_nodes[r] = n;
    }
    free(cand); free(ncand); free(tmp); free(front); free(used); free(score);
    return REF_OK;
}

/* =====================================================================
 * uno_ref_tree_verify: target-only verification of the candidate tree.
 *
 * [UNO PR, Modifications]: tree UNO reuses EAGLE's tree verification, with
 * sparse (compact-support) target sampling when eligible; [eval guide,
 * 启动期硬性约束]: both acceptance thresholds are 1.0, i.e. pure target
 * sampling.  Steps: start at the root j = 0; draw y from the filtered target
 * row of node j with u_TARGET(r, j); if a child c of j carries token y, emit
 * y and continue from c; otherwise emit y and stop.  A leaf's draw is the
 * bonus token.  accept_len = emitted - 1; path_nodes[t] = the node whose row
 * produced token t.  Node rows at or beyond num_nodes[r] are never read.  A
 * non-finite row that is reached stops the request with token -1 (flag).
 *
 * target_logits: R x V x vocab (one row per node); node_*: R x V;
 * outputs R x (B+1) for tokens and path_nodes (unused slots -1), and R for
 * accept_len, num_tokens, flags, margin (nullable).
 *
 * uno_ref_tree_verify_params is the same with per-request sampling
 * parameters (arrays of R) and a filter order for the node rows.
 * ===================================================================== */
static int tree_verify_impl(const void* target_logits, int dtype, int32_t R, int32_t B, int32_t V, int64_t vocab,
                            const ref_params* sp, const int32_t* node_token, const int32_t* node_parent,
                            const int32_t* num_nodes, uint64_t seed, uint32_t cycle, uint32_t first_request,
                            int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                            int32_t* out_path_nodes, uint32_t* out_flags, double* out_margin)
{
    if (!target_logits || !node_token || !node_parent || !num_nodes || !out_tokens || !out_accept_len ||
        !out_num_tokens || !out_path_nodes || !out_flags)
        return REF_ERR_INVALID_ARG;
    if (R < 0 || B < 1 || V < 1 || vocab <= 0) return REF_ERR_INVALID_ARG;
    if (V < B || V > 128) return REF_ERR_INVALID_ARG;
    if (dtype != REF_F32 && dtype != REF_BF16) return REF_ERR_INVALID_ARG;
    int32_t cap;
    if (!check_call_params(sp, R, vocab, &cap)) return REF_ERR_INVALID_ARG;
    if (cap < 1) cap = 1;
    size_t esz = dtype == REF_F32 ? 4 : 2;
    int32_t* ids = (int32_t*)malloc((size_t)cap * sizeof(int32_t));
    float* pr = (float*)malloc((size_t)cap * sizeof(float));
    double* wts = (double*)malloc((size_t)cap * sizeof(double));
    if (!ids || !pr || !wts) {
        free(ids); free(pr); free(wts);
        return REF_ERR_NOMEM;
    }
    for (int32_t r = 0; r < R; ++r) {
        int32_t* toks = out_tokens + (size_t)r * (size_t)(B + 1);
        int32_t* path = out_path_nodes + (size_t)r * (size_t)(B + 1);
        for (int32_t t = 0; t <= B; ++t) {
            toks[t] = -1;
            path[t] = -1;
        }
        uint32_t flags = 0;
        double margin = INFINITY;
        int32_t n = num_nodes[r];
        if (n < 1) n = 1;
        if (n > V) n = V;
        const int32_t* tk = node_token + (size_t)r * (size_t)V;
        const int32_t* pa = node_parent + (size_t)r * (size_t)V;
        /* every non-finite node row of the request sets the flag */
        for (int32_t j = 0; j < n; ++j) {
            const char* row = (const char*)target_logits + ((size_t)r * (size_t)V + (size_t)j) * (size_t)vocab * esz;
            uint32_t f = 0;
            double mt;
            int nomem = 0;
            int c = filter_row(row, dtype, vocab, sp_T(sp, r), sp_k(sp, r), sp_p(sp, r), sp->order, ids, pr, &f, &mt,
                               &nomem);
            if (nomem) {
                free(ids); free(pr); free(wts);
                return REF_ERR_NOMEM;
            }
            (void)c;
            flags |= f;
        }
        int32_t j = 0, t = 0;
        int32_t ntok = 0, acc = 0;
        for (;;) {
            const char* row = (const char*)target_logits + ((size_t)r * (size_t)V + (size_t)j) * (size_t)vocab * esz;
            uint32_t f = 0;
            double mt;
            int nomem = 0;
            int c = filter_row(row, dtype, vocab, sp_T(sp, r), sp_k(sp, r), sp_p(sp, r), sp->order, ids, pr, &f, &mt,
                               &nomem);
            if (nomem) {
                free(ids); free(pr); free(wts);
                return REF_ERR_NOMEM;
            }
            margin = min_d(margin, mt);
            if (c == 0) { /* non-finite row reached: the t tokens so far were all
                             accepted drafts; stop without a further token */
                path[t] = j;
                ntok = t;
                acc = t;
                break;
            }
            for (int q = 0; q < c; ++q) wts[q] = (double)pr[q];
            double u = uno_ref_uniform(seed, first_request + (uint32_t)r, (uint32_t)j, DRAW_TARGET, cycle);
            double md;
            int pick = inv_cdf(wts, c, u, &md);
            margin = min_d(margin, md);
            int32_t y = pick >= 0 ? ids[pick] : -1;
            toks[t] = y;
            path[t] = j;
            ++t;
            ntok = t;
            acc = t - 1;
            int32_t next = -1;
            for (int32_t cnd = 1; cnd < n; ++cnd)
                if (pa[cnd] == j && tk[cnd] == y) {
                    next = cnd;
                    break;
                }
            if (next < 0 || t > B) break;
            j = next;
        }
        out_accept_len[r] = acc;
        out_num_tokens[r] = ntok;
        out_flags[r] = flags;
        if (out_margin) out_margin[r] = margin;
    }
    free(ids); free(pr); free(wts);
    return REF_OK;
}

int uno_ref_tree_verify(const void* target_logits, int dtype, int32_t R, int32_t B, int32_t V, int64_t vocab,
                        float temperature, int32_t top_k, float top_p, const int32_t* node_token,
                        const int32_t* node_parent, const int32_t* num_nodes, uint64_t seed, uint32_t cycle,
                        uint32_t first_request, int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                        int32_t* out_path_nodes, uint32_t* out_flags, double* out_margin)
{
    ref_params sp = scalar_params(&temperature, &top_k, &top_p);
    return tree_verify_impl(target_logits, dtype, R, B, V, vocab, &sp, node_token, node_parent, num_nodes, seed,
                            cycle, first_request, out_tokens, out_accept_len, out_num_tokens, out_path_nodes,
                            out_flags, out_margin);
}

int uno_ref_tree_verify_params(const void* target_logits, int dtype, int32_t R, int32_t B, int32_t V, int64_t vocab,
                               const float* temperature, const int32_t* top_k, const float* top_p, int order,
                               const int32_t* node_token, const int32_t* node_parent, const int32_t* num_nodes,
                               uint64_t seed, uint32_t cycle, uint32_t first_request, int32_t* out_tokens,
                               int32_t* out_accept_len, int32_t* out_num_tokens, int32_t* out_path_nodes,
                               uint32_t* out_flags, double* out_margin)
{
    ref_params sp = {temperature, top_k, top_p, 1, order};
    return tree_verify_impl(target_logits, dtype, R, B, V, vocab, &sp, node_token, node_parent, num_nodes, seed,
                            cycle, first_request, out_tokens, out_accept_len, out_num_tokens, out_path_nodes,
                            out_flags, out_margin);
}
