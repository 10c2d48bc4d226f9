/*
 * oracle.c -- plain, slow, single-threaded fp64 CPU oracle for batched
 * speculative-decoding verification.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or helper with the CUDA path, and it never calls it.
 *
 * What it computes (sources, by page title and section):
 *  - "Speculative decoding becomes standard: DSpark and multi-token drafters",
 *    section "Why draft-and-verify does not change the output": the target
 *    scores the drafted block; the token drafted at position j is kept with probability
 *    min(1, p/q) (p = target, q = drafter); at the first rejection a token is
 *    drawn from a residual distribution instead and the block ends there; at
 *    temperature 0 a token is kept while it is the target's own choice, and
 *    the target's choice replaces the first token that is not.
 *  - same page, section "What DSpark adds": a confidence head,
 *    s_j = sigmoid(w . h_j + b), estimates whether position j passes once the
 *    positions before it have; the verified length is derived from it.
 *  - The residual is norm(max(0, p - q)) (Leviathan, Kalman, Matias 2022); a
 *    bonus token is drawn from the target when the whole block survives.
 *
 * Every point the pages leave open is fixed by a stated reading; the list is
 * kept with the design notes.  In short:
 *  - p = softmax(l / T) and q = softmax(d / T) at the request's temperature T;
 *    T == 0 selects the greedy path, which never reads draft logits.
 *  - greedy "agreement" means x_j equals the LOWEST index attaining the row max.
 *  - accept iff u * q(x) < p(x), with u uniform in [0, 1) (53 bits).
 *  - inverse CDF: smallest t with sum_{s<=t} w_s > u * sum_s w_s (index order,
 *    strict); if rounding leaves none, the largest t with w_t > 0.
 *  - if the residual mass R is below 1e-12 the residual is numerically
 *    undefined and the token is drawn from p instead (same rule both sides).
 *  - draws: Philox4x32-10, key = (seed low, seed high), counter =
 *    (2*position + draw, global request index, step, 0); draw 0 = accept test,
 *    draw 1 = residual or bonus sample.
 *  - -inf logits are masked tokens (probability 0).  NaN or +inf in a row the
 *    chain reads, or a row whose max is -inf, makes the request fail.  Errors
 *    are found lazily, in chain order: rows past the first rejection are never
 *    examined.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define ORC_DTYPE_F32 0
#define ORC_DTYPE_BF16 1

#define ORC_ERR_BAD_TOKEN 1u
#define ORC_ERR_NONFINITE 2u
#define ORC_ERR_BAD_TEMPERATURE 4u

/* ------------------------------------------------------------------------ */
/* Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as   */
/* easy as 1, 2, 3", SC'11.  Ten rounds of the 4x32 Philox S-box with the   */
/* multipliers and Weyl key increments given in that paper.                  */
/* ------------------------------------------------------------------------ */
void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                          uint32_t out[4]) {
    uint32_t x0 = ctr_in[0], x1 = ctr_in[1], x2 = ctr_in[2], x3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        uint64_t prod_a = (uint64_t)0xD2511F53u * (uint64_t)x0;
        uint64_t prod_b = (uint64_t)0xCD9E8D57u * (uint64_t)x2;
        uint32_t hi_a = (uint32_t)(prod_a >> 32), lo_a = (uint32_t)prod_a;
        uint32_t hi_b = (uint32_t)(prod_b >> 32), lo_b = (uint32_t)prod_b;
        uint32_t y0 = hi_b ^ x1 ^ k0;
        uint32_t y1 = lo_b;
        uint32_t y2 = hi_a ^ x3 ^ k1;
        uint32_t y3 = lo_a;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
        k0 += 0x9E3779B9u;  /* golden ratio */
        k1 += 0xBB67AE85u;  /* sqrt(3) - 1 */
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* 53-bit uniform in [0, 1): 27 high bits of word 0 and 26 high bits of word 1. */
double oracle_uniform(uint64_t seed, uint32_t request, uint32_t position,
                      uint32_t draw, uint32_t step) {
    uint32_t ctr[4] = {2u * position + draw, request, step, 0u};
    uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
    uint32_t w[4];
    oracle_philox4x32_10(ctr, key, w);
    double hi = (double)(w[0] >> 5);
    double lo = (double)(w[1] >> 6);
    return (hi * 67108864.0 + lo) / 9007199254740992.0; /* / 2^53 */
}

/* The same draws over a grid of requests and positions (row-major). */
void oracle_uniform_fill(uint64_t seed, uint32_t requests, uint32_t positions, uint32_t draw,
                         uint32_t step, double* out) {
    for (uint32_t i = 0; i < requests; ++i)
        for (uint32_t j = 0; j < positions; ++j)
            out[(size_t)i * positions + j] = oracle_uniform(seed, i, j, draw, step);
}

/* ------------------------------------------------------------------------ */
/* Reading stored values exactly into double.                               */
/* ------------------------------------------------------------------------ */
static double bf16_to_double(uint16_t bits) {
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

static double load_logit(const void* base, int dtype, int64_t index) {
    if (dtype == ORC_DTYPE_BF16) return bf16_to_double(((const uint16_t*)base)[index]);
    return (double)((const float*)base)[index];
}

/* ------------------------------------------------------------------------ */
/* Confidence head: s_j = sigmoid(w . h_j + b); P_j = prod_{j'<=j} s_j';    */
/* budget = number of leading positions with P_j >= threshold.              */
/* ("What DSpark adds": survival of a position given that the earlier ones  */
/* survived, so the chance that the first j all survive is the product.)    */
/* ------------------------------------------------------------------------ */
int oracle_conf_budget(const uint16_t* hidden, const uint16_t* w, float bias, int B,
                       int kb, int H, float threshold, int32_t* out_len,
                       double* out_survival, double* out_prefix) {
    if (B < 0 || kb < 0 || H < 0) return 1;
    for (int i = 0; i < B; ++i) {
        double prefix = 1.0;
        int budget = 0;
        int counting = 1;
        for (int j = 0; j < kb; ++j) {
            const uint16_t* h = hidden + ((int64_t)i * kb + j) * H;
            double z = 0.0;
            for (int c = 0; c < H; ++c) z += bf16_to_double(w[c]) * bf16_to_double(h[c]);
            z += (double)bias;
            double s = 1.0 / (1.0 + exp(-z));
            prefix *= s;
            if (out_survival) out_survival[(int64_t)i * kb + j] = s;
            if (out_prefix) out_prefix[(int64_t)i * kb + j] = prefix;
            if (counting && prefix >= (double)threshold) budget++;
            else counting = 0;
        }
        out_len[i] = budget;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Verification.                                                             */
/* ------------------------------------------------------------------------ */
typedef struct {
    int dtype;                    /* ORC_DTYPE_F32 or ORC_DTYPE_BF16 */
    const void* target;           /* [B, k+1, V] */
    const void* draft;            /* [B, k, V]; may be NULL when every T_i == 0 */
    const int32_t* draft_tokens;  /* [B, k] */
    const int32_t* verify_len;    /* [B] or NULL (=> k) */
    const float* temperature;     /* [B] or NULL (=> 1.0) */
    const uint16_t* conf_hidden;  /* [B, conf_kb, conf_H] bf16 or NULL */
    const uint16_t* conf_w;       /* [conf_H] bf16 */
    float conf_bias;
    float conf_threshold;
    int conf_kb;
    int conf_H;
    int64_t conf_total;           /* batch-wide verify budget; <= 0: none */
    int B;
    int k;
    int64_t V;
    uint64_t seed;
    uint32_t step;
    uint32_t request_offset;      /* global index of request 0 (Philox counter) */
    const double* u_override;     /* [B, k+1, 2] or NULL */
} oracle_inputs;

typedef struct {
    int32_t* accepted;        /* [B]: n_i, or -1 on error */
    int32_t* tokens;          /* [B, k+1]: emitted tokens, -1 padded */
    double* p_x;              /* [B, k]: p_j(x_j) for evaluated j, else -1 */
    double* q_x;              /* [B, k]: q_j(x_j) for evaluated j, else -1 */
    double* accept_margin;    /* [B, k]: |u - p/q| for evaluated j, else -1 */
    double* sample_margin;    /* [B]: distance of u*W to the nearest cell edge / W, or -1 */
    int32_t* verify_len_used; /* [B]: L_i after clamping and the confidence budget */
    uint32_t* status;         /* [B]: error bits */
} oracle_outputs;

/* ------------------------------------------------------------------------ */
/* Batch-wide verify budget (the load-aware form of the confidence rule:     */
/* "Speculative decoding becomes standard: DSpark and multi-token drafters", */
/* section "What DSpark adds" -- the verified length follows the predicted   */
/* survival and the load of the batch).  Among the candidate positions       */
/* (request i, position j < cap_i) keep the `total` ones with the largest    */
/* prefix survival P_ij, ties going to the lower request index, then to the  */
/* lower position; L_i = how many of request i's positions were kept.        */
/* Because P_ij does not increase with j, the kept positions of a request    */
/* are always a leading run.  total >= number of candidates keeps them all.  */
/* Written as its definition: list the candidates, sort them, take a prefix. */
/* ------------------------------------------------------------------------ */
typedef struct {
    double P;
    int i;
    int j;
} orc_candidate;

static int candidate_order(const void* a, const void* b) {
    const orc_candidate* x = (const orc_candidate*)a;
    const orc_candidate* y = (const orc_candidate*)b;
    if (x->P != y->P) return x->P > y->P ? -1 : 1;  /* larger survival first */
    if (x->i != y->i) return x->i < y->i ? -1 : 1;  /* then lower request */
    return (x->j > y->j) - (x->j < y->j);           /* then lower position */
}

int oracle_budget_topn(const double* prefix, const int32_t* cap, int B, int kb,
                       int64_t total, int32_t* out_len) {
    if (B < 0 || kb < 0 || total < 0) return 1;
    int64_t n = 0;
    for (int i = 0; i < B; ++i) {
        if (cap[i] < 0 || cap[i] > kb) return 1;
        n += cap[i];
    }
    orc_candidate* c = (orc_candidate*)malloc((size_t)(n > 0 ? n : 1) * sizeof *c);
    if (!c) return 2;
    int64_t m = 0;
    for (int i = 0; i < B; ++i) {
        for (int j = 0; j < cap[i]; ++j) {
            c[m].P = prefix[(int64_t)i * kb + j];
            c[m].i = i;
            c[m].j = j;
            ++m;
        }
    }
    qsort(c, (size_t)n, sizeof *c, candidate_order);
    for (int i = 0; i < B; ++i) out_len[i] = 0;  /* after the last read of cap */
    for (int64_t r = 0; r < n && r < total; ++r) out_len[c[r].i]++;
    free(c);
    return 0;
}

/* Verified length of every request: verify_len clamped to [0, k], then the
 * confidence head's per-request budget, then (if conf_total > 0) the batch-wide
 * budget over the positions that survive the first two limits. */
int oracle_verify_lengths(const oracle_inputs* in, int32_t* out_len) {
    const int B = in->B, k = in->k;
    if (B < 0 || k < 0) return 1;
    for (int i = 0; i < B; ++i) {
        int L = in->verify_len ? in->verify_len[i] : k;
        if (L < 0) L = 0;
        if (L > k) L = k;
        out_len[i] = L;
    }
    if (!in->conf_hidden || B == 0) return 0;
    const int kb = in->conf_kb;
    int32_t* budget = (int32_t*)malloc((size_t)B * sizeof *budget);
    double* prefix = (double*)malloc((size_t)B * (size_t)(kb > 0 ? kb : 1) * sizeof *prefix);
    if (!budget || !prefix) { free(budget); free(prefix); return 2; }
    oracle_conf_budget(in->conf_hidden, in->conf_w, in->conf_bias, B, kb, in->conf_H,
                       in->conf_threshold, budget, NULL, prefix);
    for (int i = 0; i < B; ++i)
        if (budget[i] < out_len[i]) out_len[i] = budget[i];
    int rc = 0;
    if (in->conf_total > 0) rc = oracle_budget_topn(prefix, out_len, B, kb, in->conf_total, out_len);
    free(budget);
    free(prefix);
    return rc;
}

static double draw_uniform(const oracle_inputs* in, int i, int position, int draw) {
    if (in->u_override) return in->u_override[((int64_t)i * (in->k + 1) + position) * 2 + draw];
    return oracle_uniform(in->seed, in->request_offset + (uint32_t)i, (uint32_t)position,
                          (uint32_t)draw, in->step);
}

/* Row statistics of softmax(l / T): max of l/T and sum of exp(l/T - max).
 * Returns 0 when the row is usable, else an error bit. */
static unsigned row_softmax_stats(const void* row, int dtype, int64_t V, double T,
                                  double* out_max, double* out_sum) {
    double m = -INFINITY;
    for (int64_t t = 0; t < V; ++t) {
        double v = load_logit(row, dtype, t);
        if (isnan(v) || v == INFINITY) return ORC_ERR_NONFINITE;
        double z = v / T;
        if (z > m) m = z;
    }
    if (!(m > -INFINITY) || !isfinite(m)) return ORC_ERR_NONFINITE;
    double Z = 0.0;
    for (int64_t t = 0; t < V; ++t) Z += exp(load_logit(row, dtype, t) / T - m);
    if (!isfinite(Z) || !(Z > 0.0)) return ORC_ERR_NONFINITE;
    *out_max = m;
    *out_sum = Z;
    return 0;
}

/* Greedy token of a row: lowest index attaining the maximum stored value. */
static unsigned row_argmax(const void* row, int dtype, int64_t V, int32_t* out_index) {
    double best = -INFINITY;
    int64_t best_t = -1;
    for (int64_t t = 0; t < V; ++t) {
        double v = load_logit(row, dtype, t);
        if (isnan(v) || v == INFINITY) return ORC_ERR_NONFINITE;
        if (best_t < 0 || v > best) { best = v; best_t = t; }
    }
    if (!(best > -INFINITY)) return ORC_ERR_NONFINITE;
    *out_index = (int32_t)best_t;
    return 0;
}

/* Inverse CDF over weights produced by `weight(t)`: the smallest t whose
 * running sum exceeds u * W; if none (rounding), the largest t with w_t > 0.
 * Reports the distance from u*W to the nearest edge of the chosen cell, / W. */
typedef double (*weight_fn)(const void* ctx, int64_t t);

static int32_t inverse_cdf(weight_fn weight, const void* ctx, int64_t V, double u,
                           double* out_margin) {
    double W = 0.0;
    for (int64_t t = 0; t < V; ++t) W += weight(ctx, t);
    double target = u * W;
    double running = 0.0;
    int64_t last_positive = -1;
    for (int64_t t = 0; t < V; ++t) {
        double w = weight(ctx, t);
        if (w > 0.0) last_positive = t;
        double before = running;
        running += w;
        if (running > target) {
            double lo = target - before, hi = running - target;
            *out_margin = (lo < hi ? lo : hi) / W;
            return (int32_t)t;
        }
    }
    *out_margin = 0.0;
    return (int32_t)last_positive;
}

typedef struct {
    const void* row;
    int dtype;
    double T, m, Z;
} target_ctx;

typedef struct {
    const void* trow;
    const void* drow;
    int dtype;
    double T, mp, Zp, mq, Zq;
} residual_ctx;

/* Bonus / fallback weights: unnormalised target probabilities exp(l/T - m). */
static double target_weight(const void* vctx, int64_t t) {
    const target_ctx* c = (const target_ctx*)vctx;
    return exp(load_logit(c->row, c->dtype, t) / c->T - c->m);
}

/* Residual weights max(0, p_t - q_t) with each row normalised by its own sum. */
static double residual_weight(const void* vctx, int64_t t) {
    const residual_ctx* c = (const residual_ctx*)vctx;
    double p = exp(load_logit(c->trow, c->dtype, t) / c->T - c->mp) / c->Zp;
    double q = exp(load_logit(c->drow, c->dtype, t) / c->T - c->mq) / c->Zq;
    double r = p - q;
    return r > 0.0 ? r : 0.0;
}

static double residual_total(const residual_ctx* c, int64_t V) {
    double R = 0.0;
    for (int64_t t = 0; t < V; ++t) R += residual_weight(c, t);
    return R;
}

#define ORC_RESIDUAL_FLOOR 1e-12

static void fail_request(const oracle_inputs* in, const oracle_outputs* out, int i,
                         unsigned bits) {
    int k = in->k;
    out->accepted[i] = -1;
    for (int j = 0; j <= k; ++j) out->tokens[(int64_t)i * (k + 1) + j] = -1;
    for (int j = 0; j < k; ++j) {
        out->p_x[(int64_t)i * k + j] = -1.0;
        out->q_x[(int64_t)i * k + j] = -1.0;
        out->accept_margin[(int64_t)i * k + j] = -1.0;
    }
    out->sample_margin[i] = -1.0;
    out->status[i] |= bits;
}

static int temperature_valid(float T) {
    if (!(T >= 0.0f) || isinf(T)) return 0;
    if (T > 0.0f && T < 0x1p-100f) return 0;
    return 1;
}

int oracle_verify(const oracle_inputs* in, const oracle_outputs* out) {
    const int B = in->B, k = in->k;
    const int64_t V = in->V;
    if (B < 0 || k < 0 || V <= 0) return 1;
    {
        const int rc = oracle_verify_lengths(in, out->verify_len_used);
        if (rc) return rc;
    }
    for (int i = 0; i < B; ++i) {
        out->status[i] = 0;
        out->sample_margin[i] = -1.0;
        for (int j = 0; j <= k; ++j) out->tokens[(int64_t)i * (k + 1) + j] = -1;
        for (int j = 0; j < k; ++j) {
            out->p_x[(int64_t)i * k + j] = -1.0;
            out->q_x[(int64_t)i * k + j] = -1.0;
            out->accept_margin[(int64_t)i * k + j] = -1.0;
        }

        /* 1. verification length (computed for the whole batch above). */
        const int L = out->verify_len_used[i];

        float Tf = in->temperature ? in->temperature[i] : 1.0f;
        if (!temperature_valid(Tf)) { fail_request(in, out, i, ORC_ERR_BAD_TEMPERATURE); continue; }
        const double T = (double)Tf;
        const void* trows = (const char*)in->target +
            (int64_t)i * (k + 1) * V * (in->dtype == ORC_DTYPE_BF16 ? 2 : 4);
        const int64_t row_bytes = V * (in->dtype == ORC_DTYPE_BF16 ? 2 : 4);
        const int32_t* x = in->draft_tokens + (int64_t)i * k;
        int32_t* tok = out->tokens + (int64_t)i * (k + 1);

        if (T == 0.0) {
            /* 2. greedy: keep while x_j is the target's argmax; at the first
             *    disagreement emit the argmax; if all agree emit row L's argmax. */
            int n = L;
            unsigned err = 0;
            for (int j = 0; j < L; ++j) {
                if (x[j] < 0 || (int64_t)x[j] >= V) { err = ORC_ERR_BAD_TOKEN; break; }
                int32_t a;
                err = row_argmax((const char*)trows + j * row_bytes, in->dtype, V, &a);
                if (err) break;
                if (x[j] == a) { tok[j] = x[j]; continue; }
                tok[j] = a;
                n = j;
                break;
            }
            if (!err && n == L) {
                int32_t a;
                err = row_argmax((const char*)trows + L * row_bytes, in->dtype, V, &a);
                if (!err) tok[L] = a;
            }
            if (err) { fail_request(in, out, i, err); continue; }
            out->accepted[i] = n;
            continue;
        }

        /* 3. stochastic chain. */
        const void* drows = (const char*)in->draft + (int64_t)i * k * row_bytes;
        int n = L;
        unsigned err = 0;
        for (int j = 0; j < L; ++j) {
            if (x[j] < 0 || (int64_t)x[j] >= V) { err = ORC_ERR_BAD_TOKEN; break; }
            const void* trow = (const char*)trows + j * row_bytes;
            const void* drow = (const char*)drows + j * row_bytes;
            double mp, Zp, mq, Zq;
            err = row_softmax_stats(trow, in->dtype, V, T, &mp, &Zp);
            if (err) break;
            err = row_softmax_stats(drow, in->dtype, V, T, &mq, &Zq);
            if (err) break;
            double p = exp(load_logit(trow, in->dtype, x[j]) / T - mp) / Zp;
            double q = exp(load_logit(drow, in->dtype, x[j]) / T - mq) / Zq;
            out->p_x[(int64_t)i * k + j] = p;
            out->q_x[(int64_t)i * k + j] = q;
            double u = draw_uniform(in, i, j, 0);
            out->accept_margin[(int64_t)i * k + j] = q > 0.0 ? fabs(u - p / q) : INFINITY;
            if (u * q < p) { tok[j] = x[j]; continue; }
            /* rejection: sample from norm(max(0, p - q)) with draw 1 */
            residual_ctx rc = {trow, drow, in->dtype, T, mp, Zp, mq, Zq};
            double u2 = draw_uniform(in, i, j, 1);
            double margin;
            if (residual_total(&rc, V) >= ORC_RESIDUAL_FLOOR) {
                tok[j] = inverse_cdf(residual_weight, &rc, V, u2, &margin);
            } else {
                target_ctx tc = {trow, in->dtype, T, mp, Zp};
                tok[j] = inverse_cdf(target_weight, &tc, V, u2, &margin);
            }
            out->sample_margin[i] = margin;
            n = j;
            break;
        }
        if (!err && n == L) {
            /* 4. the whole block survived: bonus token from target row L. */
            const void* trow = (const char*)trows + L * row_bytes;
            double mp, Zp;
            err = row_softmax_stats(trow, in->dtype, V, T, &mp, &Zp);
            if (!err) {
                target_ctx tc = {trow, in->dtype, T, mp, Zp};
                double margin;
                tok[L] = inverse_cdf(target_weight, &tc, V, draw_uniform(in, i, L, 1), &margin);
                out->sample_margin[i] = margin;
            }
        }
        if (err) { fail_request(in, out, i, err); continue; }
        out->accepted[i] = n;
    }
    return 0;
}

/* Row softmax of one row, exposed so tests can compare it with a library
 * softmax: out[t] = exp(l_t/T - m) / Z.  Returns an error bit or 0. */
int oracle_row_softmax(const void* row, int dtype, int64_t V, double T, double* out) {
    double m, Z;
    unsigned err = row_softmax_stats(row, dtype, V, T, &m, &Z);
    if (err) return (int)err;
    for (int64_t t = 0; t < V; ++t) out[t] = exp(load_logit(row, dtype, t) / T - m) / Z;
    return 0;
}

/* Greedy token of one row, exposed for the same reason. */
int oracle_row_argmax(const void* row, int dtype, int64_t V, int32_t* out) {
    return (int)row_argmax(row, dtype, V, out);
}
