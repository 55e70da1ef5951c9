/*
 * CPU oracle for one TiDAR decode step -- TEST INFRASTRUCTURE ONLY (tests,
 * smoke check, benchmark CPU baseline).  Plain loops, double precision, no
 * blocking or reordering beyond the definitions.  Shares nothing with the CUDA
 * library.  See oracle.h for the layouts and the sources.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- number formats --------------------------------------------------- */

static double bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double straight to bf16 (8 significant bits), ties to even. */
static uint16_t bf16_round(double x) {
    if (isnan(x)) return 0x7FC0;
    if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
    double ax = fabs(x);
    float f;
    if (ax < 0x1p-126 || ax >= 0x1p127) {
        /* outside the normal range the float path is used (not reached by the tests) */
        f = (float)x;
        uint32_t u;
        memcpy(&u, &f, 4);
        u = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
        return (uint16_t)u;
    }
    int e;
    double m = frexp(x, &e);          /* x = m * 2^e, 0.5 <= |m| < 1 */
    double r = nearbyint(ldexp(m, 8)); /* 8 significant bits, current mode = to nearest even */
    f = (float)ldexp(r, e - 8);        /* exact in float */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

static double logit_value(const void *base, int dtype, size_t idx) {
    if (dtype == ORACLE_LOGITS_BF16) return bf16_value(((const uint16_t *)base)[idx]);
    return (double)((const float *)base)[idx];
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* ---- the structured hybrid mask -------------------------------------- */
/*
 * Decode-time layout of one forward ("并行 self-speculative 生成 (§3.2)"):
 *   partition 1, the cached prefix, is visible to every query row;
 *   partition 2, the k previous drafts, attend causally (they are verified
 *     with this step's causal logits, and their KV must equal plain AR KV);
 *   partition 3, pre-draft group j (k mask tokens), conditions on the prefix
 *     and on drafts d_1..d_j -- one group per possible accept length -- and is
 *     bidirectional inside itself (the last block of the hybrid mask is the
 *     only bidirectional one, §1.2 of the bxzpzcl.cn walkthrough).
 * mode CAUSAL replaces it by plain causal attention over prefix + R tokens,
 * the pages' "pure causal mask" likelihood mode (Table 3 discussion).
 */
int oracle_hybrid_mask(int k, int P, int mode, uint8_t *mask) {
    if (k < 1 || P < 0 || !mask) return 1;
    const int R = k * (k + 2);
    const size_t W = (size_t)P + R;
    memset(mask, 0, (size_t)R * W);
    if (mode == ORACLE_MASK_CAUSAL) {
        for (int r = 0; r < R; ++r)
            for (size_t n = 0; n <= (size_t)P + r; ++n) mask[r * W + n] = 1;
        return 0;
    }
    if (mode != ORACLE_MASK_HYBRID) return 1;
    for (int r = 0; r < R; ++r) /* partition 1: prefix */
        for (int n = 0; n < P; ++n) mask[r * W + n] = 1;
    for (int i = 0; i < k; ++i) /* partition 2: drafts, causal */
        for (int i2 = 0; i2 <= i; ++i2) mask[(size_t)i * W + P + i2] = 1;
    for (int j = 0; j <= k; ++j) /* partition 3: group j */
        for (int s = 0; s < k; ++s) {
            size_t row = (size_t)k + (size_t)j * k + s;
            for (int i2 = 0; i2 < j; ++i2) mask[row * W + P + i2] = 1;        /* d_1..d_j */
            for (int s2 = 0; s2 < k; ++s2) mask[row * W + P + k + j * k + s2] = 1; /* own group */
        }
    return 0;
}

/* The same rule as a predicate on (row r, key n). */
static int allowed_predicate(int k, int P, int mode, int r, int n) {
    if (n < P) return 1;
    const int nn = n - P;
    if (mode == ORACLE_MASK_CAUSAL) return nn <= r;
    if (r < k) return nn < k && nn <= r;
    const int j = (r - k) / k;
    if (nn < k) return nn < j;
    return (nn - k) / k == j;
}

/* ---- attention -------------------------------------------------------- */

typedef struct {
    const uint16_t *q, *k_new, *v_new, *k_cache, *v_cache;
    const int32_t *prefix_len;
    int B, Hq, Hkv, D, k, P_max, mode;
    double scale;
} attn_args;

static const uint16_t *key_row(const attn_args *a, int b, int kv, int P, int n) {
    const int R = a->k * (a->k + 2);
    if (n < P) return a->k_cache + (((size_t)b * a->Hkv + kv) * a->P_max + n) * a->D;
    return a->k_new + (((size_t)b * R + (n - P)) * a->Hkv + kv) * a->D;
}

static const uint16_t *value_row(const attn_args *a, int b, int kv, int P, int n) {
    const int R = a->k * (a->k + 2);
    if (n < P) return a->v_cache + (((size_t)b * a->Hkv + kv) * a->P_max + n) * a->D;
    return a->v_new + (((size_t)b * R + (n - P)) * a->Hkv + kv) * a->D;
}

/* softmax(q k^T * scale) v over the allowed keys of one query row. */
static void attn_row(const attn_args *a, int b, int h, int r, const uint8_t *mask_row,
                     double *s_buf, uint8_t *ok_buf, double *o_out, double *lse_out) {
    const int R = a->k * (a->k + 2);
    const int P = a->prefix_len[b];
    const int W = P + R;
    const int kv = h / (a->Hq / a->Hkv);
    const uint16_t *qr = a->q + (((size_t)b * R + r) * a->Hq + h) * a->D;
    double m = -INFINITY;
    for (int n = 0; n < W; ++n) {
        ok_buf[n] = (uint8_t)(mask_row ? mask_row[n] : allowed_predicate(a->k, P, a->mode, r, n));
        if (!ok_buf[n]) continue;
        const uint16_t *kr = key_row(a, b, kv, P, n);
        double dot = 0.0;
        for (int d = 0; d < a->D; ++d) dot += bf16_value(qr[d]) * bf16_value(kr[d]);
        s_buf[n] = dot * a->scale;
        if (s_buf[n] > m) m = s_buf[n];
    }
    double l = 0.0;
    for (int n = 0; n < W; ++n)
        if (ok_buf[n]) l += exp(s_buf[n] - m);
    const double lse = m + log(l);
    for (int d = 0; d < a->D; ++d) o_out[d] = 0.0;
    for (int n = 0; n < W; ++n) {
        if (!ok_buf[n]) continue;
        const double w = exp(s_buf[n] - lse);
        const uint16_t *vr = value_row(a, b, kv, P, n);
        for (int d = 0; d < a->D; ++d) o_out[d] += w * bf16_value(vr[d]);
    }
    *lse_out = lse;
}

static int check_attn(const attn_args *a) {
    if (a->B < 1 || a->Hq < 1 || a->Hkv < 1 || a->Hq % a->Hkv || a->D < 1 || a->k < 1) return 1;
    for (int b = 0; b < a->B; ++b)
        if (a->prefix_len[b] < 0 || a->prefix_len[b] > a->P_max) return 1;
    return 0;
}

int oracle_attn(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                const uint16_t *k_cache, const uint16_t *v_cache, const int32_t *prefix_len,
                int B, int Hq, int Hkv, int D, int k, int P_max, double scale, int mode,
                int use_dense, int nthreads, double *o, double *lse, uint16_t *o_bf16) {
    attn_args a = {q, k_new, v_new, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, k, P_max, mode, scale};
    if (check_attn(&a)) return 1;
    const int R = k * (k + 2);
    set_threads(nthreads);
    for (int b = 0; b < B; ++b) {
        const int P = prefix_len[b];
        const int W = P + R;
        uint8_t *mask = NULL;
        if (use_dense) {
            mask = (uint8_t *)malloc((size_t)R * W);
            if (!mask || oracle_hybrid_mask(k, P, mode, mask)) { free(mask); return 1; }
        }
        const long total = (long)Hq * R;
#pragma omp parallel
        {
            double *s_buf = (double *)malloc(sizeof(double) * W);
            uint8_t *ok_buf = (uint8_t *)malloc(W);
#pragma omp for schedule(dynamic, 4)
            for (long t = 0; t < total; ++t) {
                const int h = (int)(t / R), r = (int)(t % R);
                const size_t row = ((size_t)b * R + r) * Hq + h;
                attn_row(&a, b, h, r, mask ? mask + (size_t)r * W : NULL, s_buf, ok_buf, o + row * D, lse + row);
                if (o_bf16)
                    for (int d = 0; d < D; ++d) o_bf16[row * D + d] = bf16_round(o[row * D + d]);
            }
            free(s_buf);
            free(ok_buf);
        }
        free(mask);
    }
    return 0;
}

int oracle_attn_rows(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                     const uint16_t *k_cache, const uint16_t *v_cache, const int32_t *prefix_len,
                     int B, int Hq, int Hkv, int D, int k, int P_max, double scale, int mode,
                     int n, const int32_t *sel_b, const int32_t *sel_h, const int32_t *sel_r,
                     int nthreads, double *o, double *lse) {
    attn_args a = {q, k_new, v_new, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, k, P_max, mode, scale};
    if (check_attn(&a)) return 1;
    const int R = k * (k + 2);
    for (int i = 0; i < n; ++i)
        if (sel_b[i] < 0 || sel_b[i] >= B || sel_h[i] < 0 || sel_h[i] >= Hq || sel_r[i] < 0 || sel_r[i] >= R)
            return 1;
    int Wmax = 0;
    for (int b = 0; b < B; ++b)
        if (prefix_len[b] + R > Wmax) Wmax = prefix_len[b] + R;
    set_threads(nthreads);
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * Wmax);
        uint8_t *ok_buf = (uint8_t *)malloc(Wmax);
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < n; ++i)
            attn_row(&a, sel_b[i], sel_h[i], sel_r[i], NULL, s_buf, ok_buf, o + (size_t)i * D, lse + i);
        free(s_buf);
        free(ok_buf);
    }
    return 0;
}

/* ---- softmax statistics and inverse CDF ------------------------------ */

typedef struct {
    double m, Z; /* max and sum of exp(z - m) */
} row_stats;

static row_stats softmax_stats(const void *base, int dtype, size_t off, int V) {
    row_stats st = {-INFINITY, 0.0};
    for (int v = 0; v < V; ++v) {
        double z = logit_value(base, dtype, off + v);
        if (z > st.m) st.m = z;
    }
    for (int v = 0; v < V; ++v) st.Z += exp(logit_value(base, dtype, off + v) - st.m);
    return st;
}

static double log_prob(const void *base, int dtype, size_t off, row_stats st, int v) {
    return logit_value(base, dtype, off + v) - st.m - log(st.Z);
}

/*
 * The verify's target logits: lambda * z_AR + (1 - lambda) * z_diff ("Trust AR
 * vs trust diffusion logits", Fig. 6 of the summary: the AR and diffusion
 * logits are mixed with a weight lambda at verification).  lambda = 1 is the
 * AR row itself, lambda = 0 the diffusion row itself (taken as stored, so that
 * an infinite logit never meets a zero weight).
 */
typedef struct {
    const void *p, *q;
    int dtype;
    size_t off_p, off_q;
    double lambda;
} target_row;

static double target_logit(const target_row *t, int v) {
    if (t->lambda == 1.0) return logit_value(t->p, t->dtype, t->off_p + v);
    if (t->lambda == 0.0) return logit_value(t->q, t->dtype, t->off_q + v);
    return t->lambda * logit_value(t->p, t->dtype, t->off_p + v) +
           (1.0 - t->lambda) * logit_value(t->q, t->dtype, t->off_q + v);
}

static row_stats target_stats(const target_row *t, int V) {
    row_stats st = {-INFINITY, 0.0};
    for (int v = 0; v < V; ++v) {
        const double z = target_logit(t, v);
        if (z > st.m) st.m = z;
    }
    for (int v = 0; v < V; ++v) st.Z += exp(target_logit(t, v) - st.m);
    return st;
}

static double target_log_prob(const target_row *t, row_stats st, int v) {
    return target_logit(t, v) - st.m - log(st.Z);
}

/*
 * Smallest token t whose inclusive cumulative weight exceeds u * total, for
 * non-negative weights w(v).  Reports the chosen token's interval of the
 * normalised CDF in [lo, hi).  Returns -1 if the total weight is zero.
 */
typedef double (*weight_fn)(const void *ctx, int v);

static int inverse_cdf(weight_fn w, const void *ctx, int V, double u, double *lo, double *hi) {
    double total = 0.0;
    for (int v = 0; v < V; ++v) total += w(ctx, v);
    if (!(total > 0.0)) return -1;
    const double target = u * total;
    double c = 0.0;
    for (int v = 0; v < V; ++v) {
        const double wv = w(ctx, v);
        const double prev = c;
        c += wv;
        if (c > target && wv > 0.0) {
            *lo = prev / total;
            *hi = c / total;
            return v;
        }
    }
    /* u * total below total in exact arithmetic; reached only through rounding */
    for (int v = V - 1; v >= 0; --v)
        if (w(ctx, v) > 0.0) {
            *lo = 1.0;
            *hi = 1.0;
            return v;
        }
    return -1;
}

typedef struct {
    target_row t;
    row_stats sp, sq;
} residual_ctx;

/* max(0, p(v) - q(v)): the residual distribution of a rejected draft (p the verify's target). */
static double residual_weight(const void *c, int v) {
    const residual_ctx *r = (const residual_ctx *)c;
    const double pv = exp(target_log_prob(&r->t, r->sp, v));
    const double qv = exp(log_prob(r->t.q, r->t.dtype, r->t.off_q, r->sq, v));
    return pv > qv ? pv - qv : 0.0;
}

static double p_weight(const void *c, int v) {
    const residual_ctx *r = (const residual_ctx *)c;
    return exp(target_log_prob(&r->t, r->sp, v));
}

typedef struct {
    const void *z;
    int dtype;
    size_t off;
    row_stats st;
} softmax_ctx;

static double softmax_weight(const void *c, int v) {
    const softmax_ctx *s = (const softmax_ctx *)c;
    return exp(logit_value(s->z, s->dtype, s->off + v) - s->st.m);
}

/* ---- verify ------------------------------------------------------------ */
/*
 * Talk: the drafts d_1..d_k proposed from the diffusion marginals q are
 * checked against this step's AR distribution p ("并行 self-speculative 生成
 * (§3.2)": AR rejection sampling of the previous drafts).  Draft i is
 * accepted with probability min(1, p_i(d_i)/q_i(d_i)); the first rejection
 * stops the scan and a replacement is drawn from norm(max(0, p - q)) at that
 * slot.  A pre-accepted slot 1 (the previous step's resampled token) is
 * accepted unconditionally.  Slot 1's p is the AR row carried from the
 * previous forward; slot i > 1 uses the causal logits of draft row i-1.
 * With trust_ar = lambda < 1 the target p is softmax of the mixed logits
 * lambda * z_AR + (1 - lambda) * z_diff (see target_logit).
 */
int oracle_verify(const void *p_logits, const void *q_logits, int logits_dtype,
                  const int32_t *drafts, const uint8_t *preaccepted,
                  const float *u_acc, const float *u_res, int B, int k, int V, double trust_ar,
                  const int32_t *forced_accept_len, int nthreads,
                  int32_t *accept_len, int32_t *resampled, int32_t *tokens, int32_t *n_emitted,
                  double *logp_d, double *logq_d, double *ratio, double *res_lo, double *res_hi) {
    if (B < 1 || k < 1 || V < 1 || !(trust_ar >= 0.0 && trust_ar <= 1.0)) return 1;
    for (size_t i = 0; i < (size_t)B * k; ++i)
        if (drafts[i] < 0 || drafts[i] >= V) return 1;
    set_threads(nthreads);
    row_stats *sp = (row_stats *)malloc(sizeof(row_stats) * B * k);
    row_stats *sq = (row_stats *)malloc(sizeof(row_stats) * B * k);
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < 2L * B * k; ++t) {
        const long row = t / 2;
        if (t % 2 == 0) {
            const target_row tr = {p_logits, q_logits, logits_dtype, (size_t)row * V, (size_t)row * V, trust_ar};
            sp[row] = target_stats(&tr, V);
        } else
            sq[row] = softmax_stats(q_logits, logits_dtype, (size_t)row * V, V);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        int j = 0;
        int stopped = 0;
        for (int i = 0; i < k; ++i) {
            const size_t row = (size_t)b * k + i;
            const int d = drafts[row];
            const target_row tr = {p_logits, q_logits, logits_dtype, row * V, row * V, trust_ar};
            logp_d[row] = target_log_prob(&tr, sp[row], d);
            logq_d[row] = log_prob(q_logits, logits_dtype, row * V, sq[row], d);
            ratio[row] = NAN;
            if (stopped) continue;
            if (i == 0 && preaccepted[b]) {
                j = 1;
                continue;
            }
            ratio[row] = exp(logp_d[row] - logq_d[row]);
            if ((double)u_acc[row] < ratio[row])
                j = i + 1;
            else
                stopped = 1;
        }
        if (forced_accept_len && forced_accept_len[b] >= 0) j = forced_accept_len[b];
        accept_len[b] = j;
        int n = 0;
        for (int i = preaccepted[b] ? 1 : 0; i < j; ++i) tokens[(size_t)b * k + n++] = drafts[(size_t)b * k + i];
        res_lo[b] = NAN;
        res_hi[b] = NAN;
        resampled[b] = -1;
        if (j < k) {
            const size_t row = (size_t)b * k + j;
            residual_ctx rc = {{p_logits, q_logits, logits_dtype, row * V, row * V, trust_ar}, sp[row], sq[row]};
            double lo = NAN, hi = NAN;
            int t = inverse_cdf(residual_weight, &rc, V, (double)u_res[b], &lo, &hi);
            if (t < 0) t = inverse_cdf(p_weight, &rc, V, (double)u_res[b], &lo, &hi); /* p == q */
            resampled[b] = t;
            res_lo[b] = lo;
            res_hi[b] = hi;
            tokens[(size_t)b * k + n++] = t;
        }
        n_emitted[b] = n;
        for (int i = n; i < k; ++i) tokens[(size_t)b * k + i] = -1;
    }
    free(sp);
    free(sq);
    return 0;
}

/* ---- commit and next-draft selection ----------------------------------- */
/*
 * Exact KV cache (§3.2/§3.3 of the summary; §1.3 and §2.2 of the bxzpzcl.cn
 * walkthrough): the K/V of causally computed, accepted tokens are kept, those
 * of rejected drafts are dropped at once, and pre-draft tokens never enter
 * the persistent cache.  The next draft block is the pre-draft group that
 * matches the accept length, each slot drawn from its diffusion marginal
 * (one-step drafting); after a rejection the resampled token takes slot 0 and
 * is pre-accepted, since it is a final AR token.
 */
int oracle_kv_commit(uint16_t *k_caches, uint16_t *v_caches,
                     const uint16_t *k_news, const uint16_t *v_news,
                     int L, int B, int Hkv, int D, int k, int P_max,
                     int32_t *prefix_len, const int32_t *accept_len, const int32_t *resampled,
                     const void *group_logits, int logits_dtype, int V, const float *u_draft,
                     int nthreads,
                     int32_t *next_drafts, uint8_t *next_preaccepted, int32_t *next_q_group,
                     double *draft_lo, double *draft_hi) {
    if (L < 1 || B < 1 || Hkv < 1 || D < 1 || k < 1 || V < 1) return 1;
    const int R = k * (k + 2);
    for (int b = 0; b < B; ++b) {
        if (accept_len[b] < 0 || accept_len[b] > k) return 1;
        if (prefix_len[b] < 0 || prefix_len[b] + accept_len[b] > P_max) return 1;
        if (accept_len[b] < k && (resampled[b] < 0 || resampled[b] >= V)) return 1;
    }
    set_threads(nthreads);
    for (int l = 0; l < L; ++l)
        for (int b = 0; b < B; ++b)
            for (int kv = 0; kv < Hkv; ++kv)
                for (int i = 0; i < accept_len[b]; ++i) {
                    const size_t dst = ((((size_t)l * B + b) * Hkv + kv) * P_max + prefix_len[b] + i) * D;
                    const size_t src = ((((size_t)l * B + b) * R + i) * Hkv + kv) * D;
                    memcpy(k_caches + dst, k_news + src, sizeof(uint16_t) * D);
                    memcpy(v_caches + dst, v_news + src, sizeof(uint16_t) * D);
                }
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < (long)B * k; ++t) {
        const int b = (int)(t / k), s = (int)(t % k);
        const int j = accept_len[b];
        softmax_ctx sc;
        sc.z = group_logits;
        sc.dtype = logits_dtype;
        sc.off = (((size_t)b * (k + 1) + j) * k + s) * V;
        sc.st = softmax_stats(group_logits, logits_dtype, sc.off, V);
        double lo = NAN, hi = NAN;
        next_drafts[t] = inverse_cdf(softmax_weight, &sc, V, (double)u_draft[t], &lo, &hi);
        draft_lo[t] = lo;
        draft_hi[t] = hi;
    }
    for (int b = 0; b < B; ++b) {
        const int j = accept_len[b];
        next_q_group[b] = j;
        next_preaccepted[b] = j < k ? 1 : 0;
        if (j < k) {
            next_drafts[(size_t)b * k] = resampled[b];
            draft_lo[(size_t)b * k] = NAN;
            draft_hi[(size_t)b * k] = NAN;
        }
        prefix_len[b] += j;
    }
    return 0;
}

/* ---- rotary position embedding of the step's rows --------------------- */
/*
 * Positions of the R = k(k+2) rows of one step (reading of "并行 self-speculative
 * 生成 (§3.2)" of the summary, where the pages give the partitions but not the
 * positions): draft d_i (row i-1) continues the prefix at P + i - 1; pre-draft
 * group j (the continuation after j accepted drafts) puts its slot s at
 * P + j + s.
 */
int oracle_row_position(int k, int P, int r) {
    if (r < k) return P + r;
    const int j = (r - k) / k, s = (r - k) % k;
    return P + j + s;
}

/*
 * Rotary embedding with base theta, in the half-split layout of the Qwen
 * backbones the pages start from: for i < D/2 the pair (x_i, x_{i+D/2}) is
 * rotated by the angle pos * theta^(-2i/D).  qkv: bf16 [B, R, Hq + 2 Hkv, D]
 * (the fused projection output: Q heads, then K heads, then V heads); outputs
 * q [B, R, Hq, D], k_new and v_new [B, R, Hkv, D], bf16 rounded to nearest
 * even from double.  V is copied.
 */
int oracle_rope_qkv(const uint16_t *qkv, const int32_t *prefix_len, int B, int Hq, int Hkv, int D, int k,
                    double theta, uint16_t *q, uint16_t *k_new, uint16_t *v_new) {
    if (B < 1 || Hq < 1 || Hkv < 1 || k < 1 || D < 2 || D % 2 || !(theta > 1.0)) return 1;
    const int R = k * (k + 2), H = Hq + 2 * Hkv, half = D / 2;
    for (int b = 0; b < B; ++b)
        for (int r = 0; r < R; ++r) {
            const double pos = (double)oracle_row_position(k, prefix_len[b], r);
            for (int h = 0; h < H; ++h) {
                const uint16_t *x = qkv + (((size_t)b * R + r) * H + h) * D;
                uint16_t *y;
                if (h < Hq) y = q + (((size_t)b * R + r) * Hq + h) * D;
                else if (h < Hq + Hkv) y = k_new + (((size_t)b * R + r) * Hkv + (h - Hq)) * D;
                else y = v_new + (((size_t)b * R + r) * Hkv + (h - Hq - Hkv)) * D;
                if (h >= Hq + Hkv) {
                    for (int d = 0; d < D; ++d) y[d] = x[d];
                    continue;
                }
                for (int i = 0; i < half; ++i) {
                    const double ang = pos * pow(theta, -2.0 * i / D);
                    const double c = cos(ang), sn = sin(ang);
                    const double a = bf16_value(x[i]), bb = bf16_value(x[i + half]);
                    y[i] = bf16_round(a * c - bb * sn);
                    y[i + half] = bf16_round(bb * c + a * sn);
                }
            }
        }
    return 0;
}
