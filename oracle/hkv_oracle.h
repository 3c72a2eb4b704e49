/*
 * hkv_oracle.h -- plain CPU oracle for the HeadKV hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this code: only the tests, the package's smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code with the CUDA library.
 *
 * What it computes follows the technical summary of the explainer pages of
 * "Head-Aware Key-Value Compression for Efficient Autoregressive Image
 * Generation" (Liang, Zhang, Wen, Ye; gist.science, ja/de/fr/ko/es pages,
 * which carry the same technical summary).  Citations below name that
 * summary's parts:
 *   [Method/Prefill]    Methodology, pipeline step 1, cache prefilling
 *   [Method/Grouping]   Methodology, pipeline step 2, head grouping
 *   [Method/Local]      Methodology, step 3, local heads (sliding window)
 *   [Method/STE]        Methodology, step 3, global heads, Stratified Token
 *                       Eviction (strata, per-stratum scores, M/2 + M/2)
 *   [Contrib/Budgets]   Main contributions, asymmetric budgets
 *   [Problem]           Problem statement (KV cache of AR decoding)
 *
 * All arithmetic is IEEE double.  Inputs are the exact values of the bf16 or
 * fp32 bits the GPU consumes, widened to double by the caller.
 *
 * Every function returns 0 on success and a negative value on a bad argument.
 */
#ifndef HKV_ORACLE_H
#define HKV_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Causal scaled-dot-product attention of n_q queries against n_k keys.
 * q [n_q][d], k [n_k][d], v [n_k][d]; query i sits at position q_pos0 + i and
 * sees key j iff j <= q_pos0 + i.  Scale 1/sqrt(d), no positional bias.
 * o [n_q][d] (nullable) gets the outputs; p [n_q][n_k] (nullable) gets the
 * normalised weights (0 where masked). */
int hkvo_causal_attention(const double* q, const double* k, const double* v,
                          int32_t n_q, int32_t n_k, int32_t d, int32_t q_pos0,
                          double* o, double* p);

/* Head grouping [Method/Grouping].  p_row[0..n) are the weights of the query
 * at position n-1 over positions 0..n-1.  Accumulates p(delta) = p_row[n-1-delta]
 * for delta = 0, 1, ... until the sum reaches tau; n_tau is the number of
 * tokens that took (n if it never does).  label = 1 (Local) iff n_tau < W,
 * else 0 (Global).  c_window = sum of the W-1 most recent weights, the
 * quantity whose comparison with tau decides the label (nullable). */
int hkvo_classify(const double* p_row, int32_t n, int32_t W, double tau,
                  int32_t* n_tau, uint8_t* label, double* c_window);

/* Classification row of one head from its last nq prefill queries
 * [Method/Grouping], the distance-averaged variant of the grouping rule.
 * The query at position i puts weight w_i(j) on position j <= i; its weight
 * at distance delta is w_i(i - delta) (0 when delta > i).  The row is the
 * mean over i = P-nq .. P-1 of those per-distance weights, written in the
 * position order hkvo_classify reads: row[P-1-delta].  nq = 1 gives the last
 * query's own weights.  qh, kh, vh: [>= P][d] rows of one head; row: [P]. */
int hkvo_class_row(const double* qh, const double* kh, const double* vh,
                   int32_t P, int32_t d, int32_t nq, double* row);

/* The same from given weights: w [nq][P], row k holding the weights of the
 * query at position P-nq+k over positions 0..P-1 (only positions up to the
 * query's own are read). */
int hkvo_class_row_from_weights(const double* w, int32_t P, int32_t nq, double* row);

/* Asymmetric budgets [Contrib/Budgets]: total T = floor(H * L * rho_num /
 * rho_den) tokens per (sequence, layer); Local heads keep W, the Global heads
 * split the rest evenly, rounded down.  budget_g = 0 when there is no Global
 * head.  Returns -2 when T < H * W (the config cannot give every head W). */
int hkvo_budgets(const uint8_t* labels, int32_t H, int32_t L, int32_t W,
                 int32_t rho_num, int32_t rho_den,
                 int32_t* n_local, int32_t* budget_g, int64_t* total);

/* Stratified Token Eviction select [Method/STE] for one head at step t.
 * score[i], pos[i] for the n cached tokens.  Candidates are past tokens
 * (delta = t - pos >= 1).  Near stratum: delta <= D; far: delta > D.  Evicts the
 * k_near lowest (score, pos) of the near stratum and the k_far lowest of the
 * far stratum; a stratum with too few candidates passes its shortfall to the
 * other.  With stratified = 0 all candidates form one stratum and
 * k_near + k_far are evicted from it.  evict[i] = 1 for evicted tokens.
 * gap_near / gap_far (nullable): relative score gap at the selection
 * boundary of each stratum, +inf when the boundary is empty. */
int hkvo_ste_select(const double* score, const int32_t* pos, int32_t n,
                    int32_t t, int32_t D, int32_t k_near, int32_t k_far,
                    int32_t stratified, uint8_t* evict,
                    double* gap_near, double* gap_far);

/* STE importance scores [Method/STE]: for each cached key j of one head at
 * step t, the sum over the last r queries tau = t-r+1 .. t of that query's
 * softmax weight on j, each softmax taken over the head's cache as it stood
 * at step tau (keys with position <= tau; nothing is evicted inside the
 * window).  q_all [L][d] holds the head's queries by position, k_all/v_all
 * its keys by position; kept[0..n) are the cached positions. */
int hkvo_ste_scores(const double* q_all, const double* k_all, int32_t d,
                    const int32_t* kept, int32_t n, int32_t t, int32_t r,
                    double* score);

enum { HKVO_MODE_HEADKV = 0, HKVO_MODE_FULL = 1, HKVO_MODE_UNIFORM = 2 };

typedef struct {
    int32_t num_heads, head_dim, max_len, prefill_len;
    int32_t local_window, ste_m, near_dist, score_window;
    int32_t rho_num, rho_den;
    int32_t mode;        /* HKVO_MODE_* */
    int32_t stratified;  /* 1: near/far strata (STE); 0: one pool */
    int32_t cls_queries; /* prefill queries whose per-distance weights are
                            averaged for grouping (1: the last one alone) */
    double tau;
    double label_band;   /* |c_window - tau| <= band: either label is valid */
    double select_band;  /* boundary scores within this relative gap: either
                            order is valid */
    const double* cls_rows; /* [H][P] classification rows to group by instead
                               of the unit's own (labels tied across a CFG
                               pair: the mean of both sequences' rows), or
                               NULL */
} hkvo_unit_params;

/* Decisions another implementation took for the same unit.  When the
 * oracle's own decision differs only inside a band (a near-tie between two
 * valid answers), it adopts the hinted one so that both stay in lock step;
 * a difference outside the band is counted as a hard mismatch. */
typedef struct {
    const uint8_t* labels;      /* [H] or NULL */
    int32_t n_events;
    const int32_t* event_step;  /* [n_events] */
    const int32_t* kept;        /* [n_events][H][kept_stride] positions kept by
                                   each Global head after the event, ascending */
    int32_t kept_stride;
} hkvo_hints;

typedef struct {
    uint8_t* labels;          /* [H] 1 = Local, 0 = Global (2 in full mode) */
    int32_t* n_tau;           /* [H] */
    double* c_window;         /* [H] */
    double* o_prefill;        /* [H][P][d] or NULL */
    double* o_decode;         /* [L-P][H][d] or NULL */
    int32_t* kept_final;      /* [H][L] ascending, or NULL */
    int32_t* len_final;       /* [H] or NULL */
    int32_t max_events;       /* capacity of the event log below */
    int32_t* event_step;      /* [max_events] or NULL */
    int32_t* evicted;         /* [max_events][H][ste_m_max] evicted positions, or NULL */
    int32_t evicted_stride;   /* >= largest eviction count of one head */
    int32_t n_local, budget_g, cap_g;
    int32_t n_events;
    int32_t n_label_ties, n_label_hard;
    int32_t n_select, n_select_ties, n_select_hard;
    int32_t first_hard_step;  /* -1 if none */
    double max_label_tie_gap;  /* largest |c_window - tau| of an adopted label */
    double max_select_tie_gap; /* largest relative excess of an evicted score
                                  over a kept one of its stratum in an
                                  adopted selection */
} hkvo_unit_out;

/* Whole hot path for one (sequence, layer) unit [Method/Prefill] ..
 * [Method/STE]: prefill attention, one-time classification of every head,
 * budgets, compression at classification, then decode steps
 * t = P .. L-1 (append, attention over the compressed cache, STE on Global
 * heads whose cache reached budget + M).  q, k, v: [H][L][d]. */
int hkvo_run_unit(const hkvo_unit_params* prm, const double* q,
                  const double* k, const double* v, const hkvo_hints* hints,
                  hkvo_unit_out* out);

#ifdef __cplusplus
}
#endif
#endif
