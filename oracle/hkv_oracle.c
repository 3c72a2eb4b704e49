/*
 * hkv_oracle.c -- plain CPU oracle for the HeadKV hot path.
 *
 * TEST INFRASTRUCTURE ONLY (see hkv_oracle.h): used by the tests, the smoke
 * check and the bench's CPU-baseline leg; never by the product path.
 *
 * Written for a reader who checks it against the explainer pages of
 * "Head-Aware Key-Value Compression for Efficient Autoregressive Image
 * Generation": every step is the plain definition, in the pages' order, in
 * double precision, with no blocking, fusion or reordering.  Where the pages
 * leave a step open, the reading taken is stated at that step.
 */
#include "hkv_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Attention                                                                */
/* ------------------------------------------------------------------------ */

/* One query row against the key rows listed in rows[0..n): softmax of the
 * scaled dot products, then the weighted sum of the value rows.
 * [Problem]: attention of the decoded token over its KV cache. */
static void attend_rows(const double* qrow, const double* K, const double* V,
                        const int32_t* rows, int32_t n, int32_t d,
                        double* o, double* p)
{
    const double scale = 1.0 / sqrt((double)d);
    double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double m = -INFINITY;
    for (int32_t i = 0; i < n; ++i) {
        const double* krow = K + (size_t)rows[i] * d;
        double dot = 0.0;
        for (int32_t c = 0; c < d; ++c) dot += qrow[c] * krow[c];
        s[i] = dot * scale;
        if (s[i] > m) m = s[i];
    }
    double l = 0.0;
    for (int32_t i = 0; i < n; ++i) {
        s[i] = exp(s[i] - m);
        l += s[i];
    }
    for (int32_t i = 0; i < n; ++i) s[i] /= l;
    if (o) {
        for (int32_t c = 0; c < d; ++c) o[c] = 0.0;
        for (int32_t i = 0; i < n; ++i) {
            const double* vrow = V + (size_t)rows[i] * d;
            for (int32_t c = 0; c < d; ++c) o[c] += s[i] * vrow[c];
        }
    }
    if (p)
        for (int32_t i = 0; i < n; ++i) p[i] = s[i];
    free(s);
}

int hkvo_causal_attention(const double* q, const double* k, const double* v,
                          int32_t n_q, int32_t n_k, int32_t d, int32_t q_pos0,
                          double* o, double* p)
{
    if (!q || !k || !v || n_q < 0 || n_k < 0 || d <= 0 || q_pos0 < 0)
        return -1;
    int32_t* rows = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_k > 0 ? n_k : 1));
    double* w = (double*)malloc(sizeof(double) * (size_t)(n_k > 0 ? n_k : 1));
    for (int32_t j = 0; j < n_k; ++j) rows[j] = j;
    for (int32_t i = 0; i < n_q; ++i) {
        int32_t pos = q_pos0 + i;
        int32_t nvis = pos + 1 < n_k ? pos + 1 : n_k;  /* keys 0..pos */
        attend_rows(q + (size_t)i * d, k, v, rows, nvis, d,
                    o ? o + (size_t)i * d : NULL, w);
        if (p) {
            double* prow = p + (size_t)i * n_k;
            for (int32_t j = 0; j < n_k; ++j) prow[j] = j < nvis ? w[j] : 0.0;
        }
    }
    free(rows);
    free(w);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Head grouping [Method/Grouping]                                          */
/* ------------------------------------------------------------------------ */

int hkvo_classify(const double* p_row, int32_t n, int32_t W, double tau,
                  int32_t* n_tau, uint8_t* label, double* c_window)
{
    if (!p_row || n <= 0 || W <= 0 || !n_tau || !label) return -1;
    /* Accumulate backward from the current position (delta = 0 is the
     * current token itself) until the sum reaches tau ("reaches": >=). */
    double c = 0.0;
    int32_t need = n;
    for (int32_t delta = 0; delta < n; ++delta) {
        c += p_row[n - 1 - delta];
        if (c >= tau) {
            need = delta + 1;
            break;
        }
    }
    *n_tau = need;
    /* "fewer tokens than the local window": strictly less than W. */
    *label = (uint8_t)(need < W ? 1 : 0);
    if (c_window) {
        double cw = 0.0;
        for (int32_t delta = 0; delta < W - 1 && delta < n; ++delta)
            cw += p_row[n - 1 - delta];
        *c_window = cw;
    }
    return 0;
}

int hkvo_class_row_from_weights(const double* w, int32_t P, int32_t nq, double* row)
{
    if (!w || !row || P <= 0 || nq < 1 || nq > P) return -1;
    for (int32_t j = 0; j < P; ++j) row[j] = 0.0;
    for (int32_t k = 0; k < nq; ++k) {
        const int32_t i = P - nq + k;  /* position of the k-th query */
        const double* wi = w + (size_t)k * P;
        /* its weight at distance delta lands where the last query's row
         * holds distance delta */
        for (int32_t delta = 0; delta <= i; ++delta) row[P - 1 - delta] += wi[i - delta];
    }
    for (int32_t j = 0; j < P; ++j) row[j] /= (double)nq;
    return 0;
}

int hkvo_class_row(const double* qh, const double* kh, const double* vh,
                   int32_t P, int32_t d, int32_t nq, double* row)
{
    if (!qh || !kh || !vh || !row || P <= 0 || d <= 0 || nq < 1 || nq > P) return -1;
    double* w = (double*)malloc(sizeof(double) * (size_t)P * (size_t)nq);
    /* weights of the queries at positions P-nq .. P-1 over positions 0..P-1
     * (0 past each query's own position) */
    hkvo_causal_attention(qh + (size_t)(P - nq) * d, kh, vh, nq, P, d, P - nq, NULL, w);
    hkvo_class_row_from_weights(w, P, nq, row);
    free(w);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Budgets [Contrib/Budgets]                                                */
/* ------------------------------------------------------------------------ */

int hkvo_budgets(const uint8_t* labels, int32_t H, int32_t L, int32_t W,
                 int32_t rho_num, int32_t rho_den,
                 int32_t* n_local, int32_t* budget_g, int64_t* total)
{
    if (!labels || H <= 0 || L <= 0 || W <= 0 || rho_num <= 0 || rho_den <= 0 ||
        rho_num > rho_den || !n_local || !budget_g)
        return -1;
    /* The compression ratio rho keeps rho of the full cache: H * L tokens per
     * (sequence, layer) at full length.  Exact rational arithmetic. */
    int64_t T = ((int64_t)H * (int64_t)L * rho_num) / rho_den;
    if (total) *total = T;
    if (T < (int64_t)H * W) return -2;
    int32_t nl = 0;
    for (int32_t h = 0; h < H; ++h) nl += labels[h] == 1;
    int32_t ng = H - nl;
    *n_local = nl;
    /* Local heads keep W; the Global heads split what is left, rounded down. */
    *budget_g = ng > 0 ? (int32_t)((T - (int64_t)nl * W) / ng) : 0;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Stratified Token Eviction [Method/STE]                                    */
/* ------------------------------------------------------------------------ */

typedef struct {
    double s;
    int32_t pos;
    int32_t idx;
} key_t_;

/* Total order of eviction: lower score first; equal scores, lower position
 * (the lower index) first. */
static int key_cmp(const void* a, const void* b)
{
    const key_t_* x = (const key_t_*)a;
    const key_t_* y = (const key_t_*)b;
    if (x->s < y->s) return -1;
    if (x->s > y->s) return 1;
    return (x->pos > y->pos) - (x->pos < y->pos);
}

static double boundary_gap(const key_t_* a, int32_t m, int32_t k)
{
    if (k <= 0 || k >= m) return INFINITY;
    double lo = a[k - 1].s, hi = a[k].s;
    if (hi > 0.0) return (hi - lo) / hi;
    return hi > lo ? INFINITY : 0.0;
}

static void evict_lowest(key_t_* a, int32_t m, int32_t k, uint8_t* evict, double* gap)
{
    qsort(a, (size_t)m, sizeof(key_t_), key_cmp);
    for (int32_t i = 0; i < k && i < m; ++i) evict[a[i].idx] = 1;
    if (gap) *gap = boundary_gap(a, m, k);
}

int hkvo_ste_select(const double* score, const int32_t* pos, int32_t n,
                    int32_t t, int32_t D, int32_t k_near, int32_t k_far,
                    int32_t stratified, uint8_t* evict,
                    double* gap_near, double* gap_far)
{
    if (!score || !pos || !evict || n < 0 || D < 0 || k_near < 0 || k_far < 0)
        return -1;
    memset(evict, 0, (size_t)n);
    key_t_* nearv = (key_t_*)malloc(sizeof(key_t_) * (size_t)(n > 0 ? n : 1));
    key_t_* farv = (key_t_*)malloc(sizeof(key_t_) * (size_t)(n > 0 ? n : 1));
    int32_t nn = 0, nf = 0;
    for (int32_t i = 0; i < n; ++i) {
        int32_t delta = t - pos[i];
        if (delta < 1) continue;  /* only past tokens are candidates */
        key_t_ e = {score[i], pos[i], i};
        if (stratified && delta <= D) nearv[nn++] = e;  /* near: delta <= D */
        else farv[nf++] = e;                            /* far: delta > D  */
    }
    if (stratified) {
        int32_t kn = k_near, kf = k_far;
        if (kn > nn) { kf += kn - nn; kn = nn; }
        if (kf > nf) { kn += kf - nf; kf = nf; if (kn > nn) kn = nn; }
        evict_lowest(nearv, nn, kn, evict, gap_near);
        evict_lowest(farv, nf, kf, evict, gap_far);
    } else {
        int32_t k = k_near + k_far;
        if (k > nf) k = nf;
        evict_lowest(farv, nf, k, evict, gap_far);
        if (gap_near) *gap_near = INFINITY;
    }
    free(nearv);
    free(farv);
    return 0;
}

int hkvo_ste_scores(const double* q_all, const double* k_all, int32_t d,
                    const int32_t* kept, int32_t n, int32_t t, int32_t r,
                    double* score)
{
    if (!q_all || !k_all || !kept || !score || d <= 0 || n < 0 || r < 0)
        return -1;
    for (int32_t i = 0; i < n; ++i) score[i] = 0.0;
    int32_t* rows = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
    int32_t* where = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
    double* w = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    /* Past query features: the queries of the last r steps.  Each one's
     * softmax runs over the cache as it stood at its own step, i.e. over the
     * cached keys whose position is not later than the query's. */
    for (int32_t step = t - r + 1; step <= t; ++step) {
        if (step < 0) continue;
        int32_t nv = 0;
        for (int32_t i = 0; i < n; ++i)
            if (kept[i] <= step) { rows[nv] = kept[i]; where[nv] = i; ++nv; }
        if (nv == 0) continue;
        attend_rows(q_all + (size_t)step * d, k_all, k_all /*unused*/, rows, nv, d,
                    NULL, w);
        for (int32_t j = 0; j < nv; ++j) score[where[j]] += w[j];
    }
    free(rows);
    free(where);
    free(w);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Whole unit                                                               */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t* kept;  /* ascending positions */
    int32_t len;
} head_state;

static int cmp_i32(const void* a, const void* b)
{
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* Is the hinted eviction a valid answer once scores within `band` of each
 * other are treated as tied?  before[0..n) are the cached positions (with
 * their scores), after[0..keep) the hinted survivors.  *excess gets the
 * largest relative amount by which an evicted score exceeds a kept score of
 * its stratum (0 when the hint orders every stratum exactly). */
static int hint_valid_in_band(const int32_t* before, const double* score, int32_t n,
                              const int32_t* after, int32_t keep, int32_t t,
                              int32_t D, int32_t k_near, int32_t k_far,
                              int32_t stratified, double band, double* excess)
{
    *excess = 0.0;
    uint8_t* gone = (uint8_t*)malloc((size_t)(n > 0 ? n : 1));
    memset(gone, 1, (size_t)n);
    int32_t found = 0;
    for (int32_t a = 0; a < keep; ++a)
        for (int32_t i = 0; i < n; ++i)
            if (before[i] == after[a] && gone[i]) { gone[i] = 0; ++found; break; }
    int ok = found == keep;
    /* same shortfall rule as hkvo_ste_select */
    int32_t nn = 0, nf = 0;
    for (int32_t i = 0; i < n; ++i) {
        int32_t delta = t - before[i];
        if (delta < 1) { if (gone[i]) ok = 0; continue; }
        if (stratified && delta <= D) ++nn; else ++nf;
    }
    int32_t kn = k_near, kf = k_far;
    if (stratified) {
        if (kn > nn) { kf += kn - nn; kn = nn; }
        if (kf > nf) { kn += kf - nf; kf = nf; if (kn > nn) kn = nn; }
    } else {
        kf = k_near + k_far; kn = 0; if (kf > nf) kf = nf;
    }
    for (int s = 0; s < 2 && ok; ++s) {
        int32_t cnt = 0;
        double max_gone = -INFINITY, min_kept = INFINITY;
        for (int32_t i = 0; i < n; ++i) {
            int32_t delta = t - before[i];
            if (delta < 1) continue;
            int in_near = stratified && delta <= D;
            if (in_near != (s == 0)) continue;
            if (gone[i]) { ++cnt; if (score[i] > max_gone) max_gone = score[i]; }
            else if (score[i] < min_kept) min_kept = score[i];
        }
        if (cnt != (s == 0 ? kn : kf)) ok = 0;
        else if (max_gone > min_kept * (1.0 + band)) ok = 0;
        else if (max_gone > min_kept) {
            const double x = (max_gone - min_kept) / min_kept;
            if (x > *excess) *excess = x;
        }
    }
    free(gone);
    return ok;
}

int hkvo_run_unit(const hkvo_unit_params* prm, const double* q,
                  const double* k, const double* v, const hkvo_hints* hints,
                  hkvo_unit_out* out)
{
    if (!prm || !q || !k || !v || !out) return -1;
    const int32_t H = prm->num_heads, d = prm->head_dim, L = prm->max_len;
    const int32_t P = prm->prefill_len, W = prm->local_window, M = prm->ste_m;
    const int32_t D = prm->near_dist, r = prm->score_window;
    if (H <= 0 || d <= 0 || P <= 0 || P >= L || W <= 0 || M < 2 || (M & 1) ||
        r <= 0 || r > M || r > P || D < 0 || !(prm->tau > 0.0 && prm->tau <= 1.0) ||
        !out->labels || !out->n_tau || !out->c_window)
        return -1;
    const size_t HL = (size_t)L * d; /* per-head stride of q, k, v */

    out->n_label_ties = out->n_label_hard = 0;
    out->n_select = out->n_select_ties = out->n_select_hard = 0;
    out->n_events = 0;
    out->first_hard_step = -1;
    out->max_label_tie_gap = 0.0;
    out->max_select_tie_gap = 0.0;

    const int32_t nq = prm->cls_queries;
    if (nq < 1 || nq > r) return -1;

    /* Step 1, cache prefilling [Method/Prefill]: uncompressed causal attention
     * over the first P tokens; the weights of the last query (the last nq
     * queries, averaged by distance) are kept for classification. */
    double* prow = (double*)malloc(sizeof(double) * (size_t)P);
    for (int32_t h = 0; h < H; ++h) {
        const double* qh = q + h * HL;
        const double* kh = k + h * HL;
        const double* vh = v + h * HL;
        if (out->o_prefill) {
            /* outputs of all prefill queries: layout [H][P][d] */
            hkvo_causal_attention(qh, kh, vh, P, P, d, 0,
                                  out->o_prefill + (size_t)h * P * d, NULL);
        }
        const double* crow = prow;
        if (prm->cls_rows) crow = prm->cls_rows + (size_t)h * P;
        else hkvo_class_row(qh, kh, vh, P, d, nq, prow);
        /* Step 2, head grouping [Method/Grouping], once, at this length. */
        hkvo_classify(crow, P, W, prm->tau, &out->n_tau[h], &out->labels[h],
                      &out->c_window[h]);
        if (prm->mode == HKVO_MODE_FULL) out->labels[h] = 2;
        if (prm->mode == HKVO_MODE_UNIFORM) out->labels[h] = 0;
        if (prm->mode == HKVO_MODE_HEADKV && hints && hints->labels &&
            hints->labels[h] != out->labels[h]) {
            if (fabs(out->c_window[h] - prm->tau) <= prm->label_band) {
                ++out->n_label_ties;
                if (fabs(out->c_window[h] - prm->tau) > out->max_label_tie_gap)
                    out->max_label_tie_gap = fabs(out->c_window[h] - prm->tau);
            } else { ++out->n_label_hard; if (out->first_hard_step < 0) out->first_hard_step = P - 1; }
            out->labels[h] = hints->labels[h];
        }
    }
    free(prow);

    /* Budgets [Contrib/Budgets]. */
    int32_t n_local = 0, budget_g = 0;
    int64_t total = 0;
    if (prm->mode == HKVO_MODE_HEADKV) {
        if (hkvo_budgets(out->labels, H, L, W, prm->rho_num, prm->rho_den,
                         &n_local, &budget_g, &total) != 0)
            return -2;
    } else if (prm->mode == HKVO_MODE_UNIFORM) {
        total = ((int64_t)H * L * prm->rho_num) / prm->rho_den;
        budget_g = (int32_t)(total / H);
        if (budget_g < 1) return -2;
    } else {
        budget_g = L;
    }
    const int32_t cap_g = prm->mode == HKVO_MODE_FULL ? L : budget_g + M;
    out->n_local = n_local;
    out->budget_g = budget_g;
    out->cap_g = cap_g;

    head_state* hs = (head_state*)calloc((size_t)H, sizeof(head_state));
    for (int32_t h = 0; h < H; ++h)
        hs[h].kept = (int32_t*)malloc(sizeof(int32_t) * (size_t)(L + 1));

    double* sc = (double*)malloc(sizeof(double) * (size_t)(L + 1));
    uint8_t* ev = (uint8_t*)malloc((size_t)(L + 1));
    int32_t* tmp = (int32_t*)malloc(sizeof(int32_t) * (size_t)(L + 1));

    /* Step 3, head-aware compression at classification time (t = P-1). */
    for (int32_t h = 0; h < H; ++h) {
        hs[h].len = 0;
        if (out->labels[h] == 1) {
            /* Local [Method/Local]: only the most recent W tokens. */
            for (int32_t p = P - W > 0 ? P - W : 0; p < P; ++p) hs[h].kept[hs[h].len++] = p;
        } else {
            for (int32_t p = 0; p < P; ++p) hs[h].kept[hs[h].len++] = p;
        }
    }

    int32_t ev_idx = 0;
    /* One STE event at step t over every Global head, evicting down to
     * `target` tokens: kn from the near stratum, kf from the far one. */
#define RUN_EVENT(t_, target_, kn_, kf_)                                          \
    do {                                                                        \
        int32_t et = (t_);                                                      \
        int hint_ok = hints && hints->kept && ev_idx < hints->n_events &&       \
                      hints->event_step[ev_idx] == et;                          \
        if (hints && hints->kept && !hint_ok) {                                 \
            ++out->n_select_hard;                                               \
            if (out->first_hard_step < 0) out->first_hard_step = et;            \
        }                                                                       \
        if (out->event_step && ev_idx < out->max_events) out->event_step[ev_idx] = et; \
        for (int32_t h = 0; h < H; ++h) {                                       \
            if (out->labels[h] != 0) continue;                                  \
            head_state* S = &hs[h];                                             \
            if (S->len <= (target_)) continue;                                  \
            hkvo_ste_scores(q + h * HL, k + h * HL, d, S->kept, S->len, et, r, sc); \
            hkvo_ste_select(sc, S->kept, S->len, et, D, (kn_), (kf_),            \
                            prm->stratified, ev, NULL, NULL);                   \
            int32_t nk = 0;                                                     \
            for (int32_t i = 0; i < S->len; ++i) if (!ev[i]) tmp[nk++] = S->kept[i]; \
            ++out->n_select;                                                    \
            if (hint_ok) {                                                      \
                const int32_t* g = hints->kept +                                \
                    ((size_t)ev_idx * H + h) * hints->kept_stride;              \
                int same = nk == (target_);                                     \
                for (int32_t i = 0; same && i < nk; ++i) same = tmp[i] == g[i]; \
                if (!same) {                                                    \
                    double xs = 0.0;                                            \
                    if (hint_valid_in_band(S->kept, sc, S->len, g, (target_), et, D, \
                                           (kn_), (kf_), prm->stratified,       \
                                           prm->select_band, &xs)) {            \
                        ++out->n_select_ties;                                   \
                        if (xs > out->max_select_tie_gap) out->max_select_tie_gap = xs; \
                    } else {                                                    \
                        ++out->n_select_hard;                                   \
                        if (out->first_hard_step < 0) out->first_hard_step = et; \
                    }                                                           \
                    nk = (target_);                                             \
                    for (int32_t i = 0; i < nk; ++i) tmp[i] = g[i];             \
                }                                                               \
            }                                                                   \
            if (out->evicted && ev_idx < out->max_events) {                     \
                int32_t* lg = out->evicted +                                    \
                    ((size_t)ev_idx * H + h) * out->evicted_stride;             \
                int32_t ne = 0, a = 0;                                          \
                for (int32_t i = 0; i < S->len; ++i) {                          \
                    if (a < nk && tmp[a] == S->kept[i]) { ++a; continue; }      \
                    if (ne < out->evicted_stride) lg[ne] = S->kept[i];          \
                    ++ne;                                                       \
                }                                                               \
                for (; ne < out->evicted_stride; ++ne) lg[ne] = -1;             \
            }                                                                   \
            memcpy(S->kept, tmp, sizeof(int32_t) * (size_t)nk);                 \
            S->len = nk;                                                        \
        }                                                                       \
        ++ev_idx;                                                               \
    } while (0)

    if (prm->mode != HKVO_MODE_FULL && P > budget_g) {
        /* A Global cache already above its budget at classification is
         * brought down to the budget by one STE of E = P - budget tokens,
         * split floor(E/2) near and ceil(E/2) far, scored by the last r
         * prefill queries. */
        int32_t E = P - budget_g;
        int any_global = 0;
        for (int32_t h = 0; h < H; ++h) any_global |= out->labels[h] == 0;
        if (any_global) RUN_EVENT(P - 1, budget_g, E / 2, E - E / 2);
    }

    /* Decode steps: append, attend, and STE when a Global cache reaches
     * budget + M. */
    for (int32_t t = P; t < L; ++t) {
        int due = 0;
        for (int32_t h = 0; h < H; ++h) {
            head_state* S = &hs[h];
            if (out->labels[h] == 1) {
                /* sliding window: drop the token that leaves the window */
                int32_t w = 0;
                for (int32_t i = 0; i < S->len; ++i)
                    if (S->kept[i] > t - W) S->kept[w++] = S->kept[i];
                S->len = w;
            }
            S->kept[S->len++] = t;
            if (out->o_decode)
                attend_rows(q + h * HL + (size_t)t * d, k + h * HL, v + h * HL,
                            S->kept, S->len, d,
                            out->o_decode + ((size_t)(t - P) * H + h) * d, NULL);
            if (out->labels[h] == 0 && prm->mode != HKVO_MODE_FULL && S->len >= cap_g)
                due = 1;
        }
        if (due) RUN_EVENT(t, budget_g, M / 2, M / 2);
    }
#undef RUN_EVENT
    out->n_events = ev_idx;

    for (int32_t h = 0; h < H; ++h) {
        qsort(hs[h].kept, (size_t)hs[h].len, sizeof(int32_t), cmp_i32);
        if (out->len_final) out->len_final[h] = hs[h].len;
        if (out->kept_final)
            for (int32_t i = 0; i < L; ++i)
                out->kept_final[(size_t)h * L + i] = i < hs[h].len ? hs[h].kept[i] : -1;
        free(hs[h].kept);
    }
    free(hs);
    free(sc);
    free(ev);
    free(tmp);
    return 0;
}
