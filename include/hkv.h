/*
 * hkv.h -- C ABI of libhkv, a B200 (sm_100a) library for head-aware
 * key-value cache compression in autoregressive image generation (HeadKV).
 *
 * The operations follow the technical summary of the explainer pages of
 * "Head-Aware Key-Value Compression for Efficient Autoregressive Image
 * Generation" (Liang, Zhang, Wen, Ye; gist.science, ja/de/fr/ko/es pages).
 * Passages are named by that summary's parts:
 *   Methodology step 1 (cache prefilling), step 2 (head grouping),
 *   step 3 (head-specific compression: Local sliding window; Global
 *   Stratified Token Eviction), Main contributions (asymmetric budgets),
 *   Problem statement (the KV cache of autoregressive decoding).
 *
 * Conventions for every call:
 *  - Pointers named *_host are host memory; all others are device memory of
 *    the GPU the context was created on.  The library allocates nothing: the
 *    state lives in one caller-owned device buffer (the pool) and inputs and
 *    outputs are caller-owned.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call that takes one only enqueues work on it; calls on one context must
 *    be ordered (one stream, or explicit dependencies): they share scratch.
 *  - Argument errors are reported synchronously and enqueue nothing.
 *    Errors found on the device (a numeric fault, an index out of range) are
 *    latched in a device status word, never trap, and are read back by
 *    hkv_check.
 *  - Tensors are row-major.  S = num_seqs, H = num_heads, d = head_dim.
 *    Element type is the config's dtype (fp32 or bf16) unless stated.
 */
#ifndef HKV_H
#define HKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HKV_API __attribute__((visibility("default")))
#else
#define HKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HKV_OK = 0,
    HKV_ERR_INVALID_ARG = 1, /* bad pointer, size, layer or config value */
    HKV_ERR_STATE = 2,       /* call out of order (e.g. decode before classify) */
    HKV_ERR_CAPACITY = 3,    /* pool too small, sequence longer than max_len */
    HKV_ERR_NUMERIC = 4,     /* NaN/inf met in a softmax or a score */
    HKV_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
    HKV_ERR_TIMEOUT = 6      /* a bounded device wait gave up */
} hkv_status;

typedef enum { HKV_DTYPE_F32 = 0, HKV_DTYPE_BF16 = 1 } hkv_dtype;

typedef enum {
    HKV_MODE_HEADKV = 0,  /* the method: Local window / Global STE */
    HKV_MODE_FULL = 1,    /* full cache, no compression (comparison baseline) */
    HKV_MODE_UNIFORM = 2  /* one uniform budget for every head, STE eviction */
} hkv_mode;

/* Which sequences form a classifier-free-guidance pair (the conditional and
 * the unconditional stream of one image) when grouping is tied across it. */
typedef enum {
    HKV_CFG_UNTIED = 0,   /* every sequence is grouped on its own */
    HKV_CFG_HALVES = 1,   /* batch = [conditional | unconditional]: s, s + S/2 */
    HKV_CFG_ADJACENT = 2  /* streams alternate: 2i, 2i + 1 */
} hkv_cfg_pairing;

typedef struct {
    int32_t num_seqs;     /* S: independent sequences (CFG halves included) */
    int32_t num_layers;   /* layers; each keeps its own cache */
    int32_t num_heads;    /* H: attention heads (as many KV heads) */
    int32_t head_dim;     /* d: 64 or 128 */
    int32_t dtype;        /* hkv_dtype of q, k, v, outputs and the cache */
    int32_t max_len;      /* L: longest sequence (prefix + all image tokens) */
    int32_t local_window; /* W: Local heads keep the W most recent tokens */
    int32_t ste_m;        /* M: tokens one STE evicts (even; M/2 per stratum) */
    int32_t near_dist;    /* D: near stratum = distance 1..D, far = beyond */
    int32_t score_window; /* r: queries of the last r steps score tokens, r <= M */
    int32_t rho_num;      /* rho = rho_num / rho_den: kept share of the full cache */
    int32_t rho_den;
    int32_t mode;         /* hkv_mode */
    int32_t stratified;   /* 1: near/far strata (STE); 0: one pool */
    int32_t cls_queries;  /* grouping reads the per-distance weights of the
                             last cls_queries prefill queries, averaged
                             (1..r; 0 means 1 = the last query alone) */
    int32_t cfg_pairing;  /* hkv_cfg_pairing: grouping of a CFG pair by the
                             mean of both streams' rows (one label per pair);
                             S must be even unless HKV_CFG_UNTIED */
    int32_t heads_total;  /* heads of a whole (sequence, layer) when this
                             context holds only num_heads of them (heads
                             sharded over GPUs); 0 means num_heads.  Budgets
                             count all heads_total heads: T = floor(heads_total
                             * L * rho).  A sharded context prefills with
                             hkv_prefill_label + hkv_prefill_compress */
    double tau;           /* grouping threshold, 0.9 on the pages */
} hkv_config;

typedef struct hkv_ctx hkv_ctx;

/* Human-readable name of a status code (static string). */
HKV_API const char* hkv_status_string(hkv_status s);

/* Bytes of device memory the pool of `cfg` needs (state + scratch).
 * Budgets [Main contributions]: each (sequence, layer) region holds
 * floor(H * L * rho) + H * M slots for HKV_MODE_HEADKV.
 * Errors: HKV_ERR_INVALID_ARG for an unusable config, including
 * floor(H * L * rho) < H * W (the budget cannot give every head W). */
HKV_API hkv_status hkv_pool_bytes(const hkv_config* cfg, size_t* bytes);

/* Binds a context to `pool` (device memory on the current CUDA device,
 * >= hkv_pool_bytes bytes, 256-byte aligned, owned by the caller and kept
 * alive until hkv_destroy).  Enqueues the clearing of the pool's control
 * words on `stream`.  *out receives the context (host memory owned by the
 * library until hkv_destroy). */
HKV_API hkv_status hkv_create(const hkv_config* cfg, void* pool, size_t bytes, void* stream,
                      hkv_ctx** out);

/* Cache prefilling and head grouping for one layer [Methodology steps 1-2],
 * then compression at classification time [step 3].  Must be called once
 * per layer before any append or decode on it.
 *  q, k, v: S*H blocks of [prefill_len][d]; block b = s*H + h starts at
 *           element b * block_stride (block_stride >= prefill_len * d).
 *  out:     [S][H][prefill_len][d] causal attention outputs, or NULL.
 * Causal softmax(q k^T / sqrt(d)) v over the prefill tokens.  Each head is
 * then labelled from the weights of the last prefill query: Local iff the
 * newest tokens reach tau in fewer than W tokens.  With cls_queries = n > 1
 * the weight at each distance is the mean over the last n queries; with a
 * cfg_pairing the row is also averaged over the pair's two streams, which
 * then share their labels and budgets (the pair's two layers must be
 * classified by the same call: they are, as one call covers all S).  Budgets follow: Local
 * heads keep W, Global heads split floor(H*L*rho) - nL*W evenly (rounded
 * down) per (sequence, layer).  Local heads keep their last W prefill
 * tokens; Global heads keep all, or, beyond their budget, run one
 * Stratified Token Eviction (E = prefill_len - budget: floor(E/2) near,
 * ceil(E/2) far) scored by the last r prefill queries.
 * Requirements: W <= prefill_len < max_len, r <= prefill_len.
 * Errors: INVALID_ARG (pointers, sizes), STATE (layer already classified). */
HKV_API hkv_status hkv_prefill_classify(hkv_ctx* ctx, int32_t layer, const void* q, const void* k,
                                const void* v, int32_t prefill_len, int64_t block_stride,
                                void* out, void* stream);

/* The same, in two phases, for heads sharded over several contexts (one per
 * GPU), whose budgets need the Local count of every shard [Main
 * contributions: asymmetric budgets count all heads of a sequence and
 * layer].  hkv_prefill_label runs the prefill attention and the grouping of
 * the heads held here and writes, per sequence, their Local count:
 *  n_local: int32[S] device output (4-byte aligned), stream-ordered.
 * The caller sums n_local over the shards (an all-reduce; NCCL over NVLink
 * on GPUs) into n_local_total and calls hkv_prefill_compress with the same
 * layer, prefill_len, k, v and block_stride (k and v must still hold the
 * prefill tokens): budgets from the total, then the compression at
 * classification.  Between the two calls no other layer may be labelled
 * (the weight rows of the last r queries live in one shared scratch).
 * A total outside [Local count here, Local count here + heads_total -
 * num_heads] latches HKV_ERR_INVALID_ARG in the status word and is clamped
 * into that range.  With heads_total == num_heads and n_local_total =
 * n_local the pair computes exactly what hkv_prefill_classify computes;
 * hkv_prefill_classify on a context with heads_total > num_heads returns
 * INVALID_ARG.  Errors: INVALID_ARG, STATE (label: layer classified or
 * another layer labelled and not compressed; compress: layer not the one
 * labelled, or another prefill_len), CUDA. */
HKV_API hkv_status hkv_prefill_label(hkv_ctx* ctx, int32_t layer, const void* q, const void* k,
                                     const void* v, int32_t prefill_len, int64_t block_stride,
                                     void* out, int32_t* n_local, void* stream);
HKV_API hkv_status hkv_prefill_compress(hkv_ctx* ctx, int32_t layer, const void* k, const void* v,
                                        int32_t prefill_len, int64_t block_stride,
                                        const int32_t* n_local_total, void* stream);

/* Appends the next token's key and value ([S][H][d] each) to every head of
 * `layer` [step 3]: Local heads overwrite their oldest token (sliding
 * window), Global heads add it at the tail.  Errors: STATE (layer not
 * classified), CAPACITY (sequence already max_len long). */
HKV_API hkv_status hkv_append(hkv_ctx* ctx, int32_t layer, const void* k_t, const void* v_t,
                      void* stream);

/* Decode attention of the newest token over each head's compressed cache
 * [Problem statement; step 3]: o_t = softmax(q_t K^T / sqrt(d)) V over the
 * head's kept tokens (the newest included).  q_t, o_t: [S][H][d].  For a
 * Global head within r steps of its next eviction the same pass records the
 * logits the STE scores are built from [step 3, STE scores].
 * Errors: STATE (layer not classified or nothing appended yet). */
HKV_API hkv_status hkv_decode_attend(hkv_ctx* ctx, int32_t layer, const void* q_t, void* o_t,
                             void* stream);

/* hkv_append followed by hkv_decode_attend in one kernel.
 * Launch overlap: when the previous launch this context made on `stream`
 * was a decode of another layer, this launch may start before the kernel
 * in front of it has finished (programmatic dependent launch).  Before
 * that kernel finishes it reads only this layer's cache and plan in the
 * pool; q_t, k_t, v_t and o_t are touched after it, so a caller's kernel
 * may produce q_t, k_t, v_t (a projection) right before the call. */
HKV_API hkv_status hkv_decode_step(hkv_ctx* ctx, int32_t layer, const void* q_t, const void* k_t,
                           const void* v_t, void* o_t, void* stream);

/* Stratified Token Eviction [step 3, Global heads] on layers
 * [layer_begin, layer_end): every Global head whose cache reached
 * budget + M tokens splits its past tokens (distance >= 1 from the newest)
 * into near (distance <= D) and far strata, scores each token by the summed
 * softmax weight the last r queries gave it, and evicts the M/2 lowest
 * (score, position) of each stratum, ties going to the lower position; the
 * cache is compacted in place.  Heads that are not due are left untouched,
 * so one call per decode step serves every step.
 * Errors: INVALID_ARG (layer range), STATE (a layer not classified). */
HKV_API hkv_status hkv_ste_evict(hkv_ctx* ctx, int32_t layer_begin, int32_t layer_end, void* stream);

/* Head labels of one layer (1 = Local, 0 = Global, 2 = full mode) and the
 * token counts n_tau that decided them, [S][H] each (n_tau_host nullable).
 * Waits for `stream`. */
HKV_API hkv_status hkv_get_labels(hkv_ctx* ctx, int32_t layer, uint8_t* labels_host,
                          int32_t* n_tau_host, void* stream);

/* Cache lengths [S][H] and per-head budgets [S][H] (nullable) of one layer
 * as of the work enqueued so far.  Waits for `stream`. */
HKV_API hkv_status hkv_get_lens(hkv_ctx* ctx, int32_t layer, int32_t* len_host, int32_t* budget_host,
                        void* stream);

/* Positions cached by one head, ascending, into pos_host[0..capacity);
 * *len_out = how many.  Waits for `stream`.  CAPACITY if capacity < len. */
HKV_API hkv_status hkv_get_kept(hkv_ctx* ctx, int32_t seq, int32_t layer, int32_t head,
                        int32_t* pos_host, int32_t capacity, int32_t* len_out, void* stream);

/* Counters of the evictions run since hkv_create or hkv_reset, into
 * stats_host[3] (int64): Global heads evicted, cached tokens they scored
 * (their lengths at eviction), rows moved by the compaction (one K row, one
 * V row and a position each).  A head's eviction reads its positions and r
 * logits per token and each moved row's K|V pair once, and writes it once:
 * these counts give the eviction's bytes.  Waits for `stream`. */
HKV_API hkv_status hkv_get_evict_stats(hkv_ctx* ctx, int64_t* stats_host, void* stream);

/* Reads the device status word (waits for `stream`) and returns the first
 * error latched on the device, or HKV_OK.  *detail_host (nullable) gets a
 * code-specific detail (e.g. the head index). */
HKV_API hkv_status hkv_check(hkv_ctx* ctx, int32_t* detail_host, void* stream);

/* Clears a latched device error. */
HKV_API hkv_status hkv_clear_error(hkv_ctx* ctx, void* stream);

/* Starts a new generation on the same pool: enqueues the clearing of the
 * control words (positions, counters, status) on `stream` and forgets every
 * layer's classification (and a labelled layer awaiting
 * hkv_prefill_compress), so prefill_classify must run again per layer.
 * Cache contents are not cleared (they are rewritten by the next prefill). */
HKV_API hkv_status hkv_reset(hkv_ctx* ctx, void* stream);

/* Releases the context (not the pool). */
HKV_API void hkv_destroy(hkv_ctx* ctx);

/* ---- Standalone primitives on caller-supplied device arrays -------------- */

/* Head grouping rule [step 2] on n_rows weight rows (fp32, [n_rows][n]): row
 * i holds the weights of a query at position n-1 over positions 0..n-1.
 * n_tau[i] (int32) = tokens the backward accumulation needs to reach tau
 * (n if never); label[i] (uint8) = 1 iff n_tau[i] < W.  Accumulation in
 * double.  Errors: INVALID_ARG. */
HKV_API hkv_status hkv_classify_rows(const float* rows, int32_t n_rows, int32_t n, int32_t W,
                             double tau, int32_t* n_tau, uint8_t* label, void* stream);

/* Head grouping [step 2] with the averaged and tied variants, on n_units
 * blocks of kept weight rows (fp32, [n_units][r][n]): row q of a block
 * holds the weights of the query at position n - r + q over positions
 * 0..n-1 (entries past that position are not read).  The weight at
 * distance delta is the mean over the last nq queries of each query's
 * weight on the position delta back from its own; with partner (int32
 * [n_units], nullable) and partner[u] = p != u, unit u is grouped on the
 * mean of its and p's values (the lower index summed first, so u and p get
 * the same answer).  Each unit's sum over its queries runs in position
 * order in double and is divided by nq; the pair mean is taken after.
 * Outputs as hkv_classify_rows; a partner outside [0, n_units) gives
 * n_tau -1 and label 255.  Requirements: 1 <= nq <= r <= n.
 * Errors: INVALID_ARG. */
HKV_API hkv_status hkv_classify_groups(const float* rows, int32_t n_units, int32_t r, int32_t nq,
                                       int32_t n, const int32_t* partner, int32_t W, double tau,
                                       int32_t* n_tau, uint8_t* label, void* stream);

/* Stratified selection [step 3, STE] on n_probs independent problems.
 * Problem i has count[i] <= n tokens: score[i*n + j] (fp32, >= 0) and
 * pos[i*n + j] (int32, distinct); the newest position is t[i].  Evicts
 * k_near lowest (score, position) of the near stratum (distance 1..D) and
 * k_far of the far one (distance > D); a stratum short of candidates hands
 * the shortfall to the other; stratified = 0 pools them.  evict[i*n + j]
 * (uint8) = 1 for evicted tokens.  n <= 4096.  Errors: INVALID_ARG; a NaN
 * score latches nothing here (no context) and selects as the largest key. */
HKV_API hkv_status hkv_ste_select_batch(const float* score, const int32_t* pos, const int32_t* count,
                                const int32_t* t, int32_t n_probs, int32_t n, int32_t D,
                                int32_t k_near, int32_t k_far, int32_t stratified,
                                uint8_t* evict, void* stream);

/* ---- Allocation-free entry point ------------------------------------------ */

/* Prefill attention and head grouping with no device allocation at all.
 * The pages have no counterpart of this call: it exists for callers that
 * cannot allocate device memory, not even the pool of hkv_create (code that
 * runs during a global-mode CUDA graph capture, where cudaMalloc is refused;
 * runtimes whose caching allocator owns all device memory; processes that
 * may not allocate after start-up).  It computes, for n_blocks independent
 * (sequence, head) blocks, what hkv_prefill_classify computes before it
 * compresses anything: the causal attention outputs and each block's label.
 *  q, k, v:  n_blocks blocks of [prefill_len][head_dim] elements of `dtype`,
 *            block b at element b * block_stride (>= prefill_len * head_dim,
 *            16-byte multiple); 16-byte aligned device pointers.
 *  out:      [n_blocks][prefill_len][head_dim] outputs, or NULL.
 *  n_tau:    int32[n_blocks] device output: tokens the backward accumulation
 *            of the last query's weights needs to reach tau.
 *  label:    uint8[n_blocks] device output: 1 (Local) iff n_tau < local_window.
 *  status:   int32[2] device output (nullable): zeroed, then a device-side
 *            fault (HKV_ERR_TIMEOUT, block index) if one occurs.  A block
 *            whose bounded wait gave up leaves its n_tau and label computed
 *            from stale scratch, so a caller that passes NULL here cannot
 *            tell a timed-out call from a good one: pass a status buffer
 *            and read it.
 * Scratch: a fixed 8 MiB array inside the library, present on every GPU that
 * loads it until the process exits.  Limit: n_blocks * prefill_len <=
 * 2,097,088; larger calls return HKV_ERR_CAPACITY and enqueue nothing.  The
 * fp32 path also needs prefill_len <= 12,288 (its attention kernel stages
 * 16 * (head_dim + prefill_len) bytes of shared memory); longer fp32 calls
 * return HKV_ERR_INVALID_ARG and enqueue nothing.  The
 * first call on a device looks the array's address up and sets kernel
 * attributes (host-side work): make it before any stream capture.  Every
 * call reuses the same array, so calls that overlap on the GPU (other
 * streams, other threads) race; order them.  Calls no cudaMalloc/cudaFree.
 * Errors: INVALID_ARG, CAPACITY, CUDA. */
HKV_API hkv_status hkv_prefill_classify_noalloc(int32_t dtype, int32_t head_dim, int32_t n_blocks,
                                                const void* q, const void* k, const void* v,
                                                int32_t prefill_len, int64_t block_stride,
                                                int32_t local_window, double tau, void* out,
                                                int32_t* n_tau, uint8_t* label, int32_t* status,
                                                void* stream);

#ifdef __cplusplus
}
#endif
#endif /* HKV_H */
