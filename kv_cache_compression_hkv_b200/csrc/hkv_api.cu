// hkv_api.cu -- the C ABI declared in include/hkv.h: argument checks, the
// carving of the caller-owned pool, call-order bookkeeping and launches.
// Every function here only validates and enqueues; the arithmetic of the
// hot path runs in the kernels.
#include <stdlib.h>
#include <string.h>

#include <new>
#include <vector>

#include "hkv_internal.cuh"
#include "kernels.h"

using hkv::Layout;

struct hkv_ctx {
    hkv_config cfg;
    Layout lay;
    int device;
    int n_sm;
    int decode_grid;
    int evict_grid;
    hkv::DecodeShape decode_sh;
    std::vector<int> plan_for;    // per layer: step its decode plan was made for (-1: none)
    int64_t t_total;
    std::vector<int> classified;  // per layer
    std::vector<int> t_host;      // per layer: next position, as enqueued by API calls
    std::vector<int> prefill_len;
    // the last kernel this context enqueued: a decode launch of layer
    // last_decode (-1: any other kernel) on stream last_stream
    int last_decode = -1;
    void* last_stream = nullptr;
    int split_buf = 0;  // split-K buffer set of the next decode launch
    // a layer labelled by hkv_prefill_label and not yet compressed (-1: none),
    // and its prefill length; its weight rows occupy the shared row scratch
    int labelled_layer = -1;
    int labelled_len = 0;
};

namespace {

// Records a launch that is not a decode launch.
void note_other(hkv_ctx* c, void* stream) {
    c->last_decode = -1;
    c->last_stream = stream;
}

// Launches the decode kernel of `layer`, overlapping its start with the
// previous launch when that is a decode launch of another layer.
cudaError_t decode_launch(hkv_ctx* c, int layer, const void* q, const void* k, const void* v,
                          void* o, int append, void* stream) {
    const int early = c->last_stream == stream && c->last_decode >= 0 && c->last_decode != layer;
    cudaError_t e = hkv::launch_decode(c->lay, layer, q, k, v, o, append, c->decode_sh,
                                       c->decode_grid, early, c->split_buf, (cudaStream_t)stream);
    c->split_buf ^= 1;
    c->last_decode = layer;
    c->last_stream = stream;
    return e;
}

}  // namespace

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

size_t elem_size(int dtype) { return dtype == HKV_DTYPE_F32 ? 4 : 2; }

int64_t total_heads(const hkv_config* c) { return c->heads_total > 0 ? c->heads_total : c->num_heads; }

bool config_ok(const hkv_config* c, int64_t* T_out, int32_t* R_out) {
    if (!c) return false;
    if (c->num_seqs < 1 || c->num_layers < 1 || c->num_heads < 1 || c->num_heads > 32) return false;
    if (c->head_dim != 64 && c->head_dim != 128) return false;
    if (c->dtype != HKV_DTYPE_F32 && c->dtype != HKV_DTYPE_BF16) return false;
    if (c->max_len < 2 || c->max_len > 8192) return false;
    if (c->local_window < 1 || c->local_window > c->max_len) return false;
    if (c->ste_m < 2 || (c->ste_m & 1)) return false;
    if (c->near_dist < 0) return false;
    if (c->score_window < 1 || c->score_window > c->ste_m || c->score_window > 32) return false;
    if (c->rho_num < 1 || c->rho_den < c->rho_num) return false;
    if (c->mode < HKV_MODE_HEADKV || c->mode > HKV_MODE_UNIFORM) return false;
    if (c->stratified != 0 && c->stratified != 1) return false;
    if (c->cls_queries < 0 || c->cls_queries > c->score_window) return false;
    if (c->cfg_pairing < HKV_CFG_UNTIED || c->cfg_pairing > HKV_CFG_ADJACENT) return false;
    if (c->cfg_pairing != HKV_CFG_UNTIED && (c->num_seqs & 1)) return false;
    if (!(c->tau > 0.0 && c->tau <= 1.0)) return false;
    if ((int64_t)c->num_seqs * c->num_heads > 12288) return false;
    if (c->heads_total != 0 && (c->heads_total < c->num_heads || c->heads_total > 4096)) return false;
    const int64_t H = c->num_heads, L = c->max_len;
    const int64_t Ht = total_heads(c);
    // the budget of a (sequence, layer) counts all its heads, sharded or not
    const int64_t T = Ht * L * c->rho_num / c->rho_den;
    int64_t R;
    if (c->mode == HKV_MODE_HEADKV) {
        if (T < Ht * c->local_window) return false;
        // this shard's caps: nL_here*W + nG_here*(B_g + M) <= T + H*M
        R = T + H * c->ste_m;
    } else if (c->mode == HKV_MODE_UNIFORM) {
        if (T / Ht < 1) return false;
        R = (T / Ht + c->ste_m) * H;
    } else {
        R = H * L;
    }
    if (R > (int64_t)1 << 30) return false;
    if (T_out) *T_out = T;
    if (R_out) *R_out = (int32_t)R;
    return true;
}

// Carves the pool.  With base == nullptr only sizes are computed.
size_t carve(const hkv_config* c, int64_t T, int32_t R, unsigned char* base, Layout* L) {
    const size_t S = c->num_seqs, Ly = c->num_layers, H = c->num_heads, d = c->head_dim;
    const size_t r = c->score_window, Lmax = c->max_len;
    const size_t es = elem_size(c->dtype);
    const size_t nh = Ly * S * H;
    const size_t slots = Ly * S * (size_t)R;
    const size_t max_chunks = S * ((size_t)R / hkv::CHUNK + H + 1);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes);
        return base ? base + at : nullptr;
    };
    Layout l;
    memset(&l, 0, sizeof(l));
    l.status = (int32_t*)take(16);
    l.t_next = (int32_t*)take(Ly * 4);
    l.done_ctr = (int32_t*)take(Ly * 4);
    l.ticket = (int32_t*)take(2 * S * H * 4);  // two sets: consecutive decode launches alternate
    l.ev_stats = (unsigned long long*)take(3 * 8);
    const size_t ctrl_end = o;
    l.off = (int32_t*)take(nh * 4);
    l.cap = (int32_t*)take(nh * 4);
    l.budget = (int32_t*)take(nh * 4);
    l.base = (uint64_t*)take(nh * 8);
    l.n_tau = (int32_t*)take(nh * 4);
    l.label = (uint8_t*)take(nh);
    l.K = take(slots * 2 * d * es);  // K and V rows interleaved per slot
    l.V = l.K ? (unsigned char*)l.K + d * es : nullptr;
    l.pos = (int32_t*)take(slots * 4);
    l.logit = (float*)take(slots * r * 4);
    l.ml = (float2*)take(nh * r * 8);
    l.rows = (float*)take(S * H * r * Lmax * 4);
    l.partial = (float*)take(2 * 2 * (size_t)hkv::PLAN_MAX_WARPS * (d + 2) * 4);
    l.unit = (int4*)take(Ly * S * 16);
    l.plan_desc = (int4*)take(Ly * max_chunks * 16);
    l.plan_warp = (int4*)take(Ly * hkv::PLAN_MAX_WARPS * (1 + hkv::PLAN_WARP_DESC) * 16);
    l.S = c->num_seqs; l.Ly = c->num_layers; l.H = c->num_heads; l.d = c->head_dim;
    l.H_total = (int32_t)total_heads(c);
    l.L = c->max_len; l.W = c->local_window; l.M = c->ste_m; l.D = c->near_dist;
    l.r = c->score_window; l.mode = c->mode; l.stratified = c->stratified; l.dtype = c->dtype;
    l.nq = c->cls_queries > 0 ? c->cls_queries : 1; l.pairing = c->cfg_pairing;
    l.R = R; l.T_total = T; l.tau = c->tau; l.max_chunks = (int32_t)max_chunks;
    if (L) *L = l;
    (void)ctrl_end;
    return o;
}

size_t ctrl_bytes(const hkv_config* c) {
    // status, t_next, done_ctr, ticket and ev_stats are laid out first (see carve)
    size_t o = 0;
    o = align_up(o + 16);
    o = align_up(o + (size_t)c->num_layers * 4);
    o = align_up(o + (size_t)c->num_layers * 4);
    o = align_up(o + 2 * (size_t)c->num_seqs * c->num_heads * 4);
    o = align_up(o + 3 * 8);
    return o;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

hkv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? HKV_OK : HKV_ERR_CUDA; }

}  // namespace

extern "C" {

const char* hkv_status_string(hkv_status s) {
    switch (s) {
        case HKV_OK: return "HKV_OK";
        case HKV_ERR_INVALID_ARG: return "HKV_ERR_INVALID_ARG";
        case HKV_ERR_STATE: return "HKV_ERR_STATE";
        case HKV_ERR_CAPACITY: return "HKV_ERR_CAPACITY";
        case HKV_ERR_NUMERIC: return "HKV_ERR_NUMERIC";
        case HKV_ERR_CUDA: return "HKV_ERR_CUDA";
        case HKV_ERR_TIMEOUT: return "HKV_ERR_TIMEOUT";
    }
    return "HKV_ERR_UNKNOWN";
}

hkv_status hkv_pool_bytes(const hkv_config* cfg, size_t* bytes) {
    int64_t T;
    int32_t R;
    if (!bytes || !config_ok(cfg, &T, &R)) return HKV_ERR_INVALID_ARG;
    *bytes = carve(cfg, T, R, nullptr, nullptr);
    return HKV_OK;
}

hkv_status hkv_create(const hkv_config* cfg, void* pool, size_t bytes, void* stream, hkv_ctx** out) {
    int64_t T;
    int32_t R;
    if (!out || !pool || ((uintptr_t)pool % kAlign) != 0 || !config_ok(cfg, &T, &R))
        return HKV_ERR_INVALID_ARG;
    *out = nullptr;
    if (bytes < carve(cfg, T, R, nullptr, nullptr)) return HKV_ERR_CAPACITY;
    hkv_ctx* c = new (std::nothrow) hkv_ctx();
    if (!c) return HKV_ERR_CAPACITY;
    c->cfg = *cfg;
    c->t_total = T;
    carve(cfg, T, R, (unsigned char*)pool, &c->lay);
    c->classified.assign(cfg->num_layers, 0);
    c->t_host.assign(cfg->num_layers, 0);
    c->prefill_len.assign(cfg->num_layers, 0);
    cudaError_t e = cudaGetDevice(&c->device);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&c->n_sm, cudaDevAttrMultiProcessorCount, c->device);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(pool, 0, ctrl_bytes(cfg), (cudaStream_t)stream);
    if (e != cudaSuccess) {
        delete c;
        return HKV_ERR_CUDA;
    }
    if (hkv::prepare_kernels() != cudaSuccess) {
        delete c;
        return HKV_ERR_CUDA;
    }
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, c->device);
    if (hkv::plan_smem_bytes(cfg->num_seqs * cfg->num_heads, c->lay.max_chunks) > (size_t)optin - 1024) {
        delete c;
        return HKV_ERR_INVALID_ARG;  // too many heads per layer for one plan block
    }
    c->decode_sh = hkv::decode_shape(c->lay, (size_t)optin - 256);
    c->decode_grid = c->n_sm * c->decode_sh.per_sm;  // persistent: every block resident
    {
        // A small cache needs fewer blocks: the plan gives a warp at least
        // min_range_cost of work, and a layer holds at most
        // max_chunks chunks (S heads' slot regions in 32-token chunks, one
        // partial chunk per head).
        const int hc = c->decode_sh.head_cost;
        const int64_t tcost = (int64_t)hkv::CHUNK_COST * c->lay.max_chunks + (int64_t)hc * cfg->num_seqs * cfg->num_heads;
        const int64_t mrc = hkv::min_range_cost(hc);
        const int64_t warps = (tcost + mrc - 1) / mrc;
        const int64_t blocks = (warps + c->decode_sh.warps - 1) / c->decode_sh.warps;
        if (blocks < c->decode_grid) c->decode_grid = (int)(blocks < 1 ? 1 : blocks);
    }
    if (c->decode_sh.warps == 0 || c->decode_grid * c->decode_sh.warps > hkv::PLAN_MAX_WARPS) {
        delete c;
        return HKV_ERR_INVALID_ARG;
    }
    c->lay.plan_gw = c->decode_grid * c->decode_sh.warps;
    c->lay.plan_nw = c->decode_sh.warps;
    c->lay.plan_hc = c->decode_sh.head_cost;
    c->lay.plan_lw = c->decode_sh.lone_weight;
    c->plan_for.assign(cfg->num_layers, -1);
    c->evict_grid = c->n_sm * hkv::evict_blocks_per_sm(c->lay, optin);
    *out = c;
    return HKV_OK;
}

// Argument checks shared by the prefill entry points (q may be null for the
// compression phase, which reads only k and v).
static hkv_status prefill_args(const hkv_ctx* c, int32_t layer, const void* q, const void* k,
                               const void* v, int32_t P, int64_t block_stride, const void* out,
                               bool need_q) {
    if (!c || (need_q && !q) || !k || !v) return HKV_ERR_INVALID_ARG;
    const hkv_config& g = c->cfg;
    if (layer < 0 || layer >= g.num_layers) return HKV_ERR_INVALID_ARG;
    if (P < g.local_window || P >= g.max_len || P < g.score_window || P < 2)
        return HKV_ERR_INVALID_ARG;
    const size_t es = elem_size(g.dtype);
    if (block_stride < (int64_t)P * g.head_dim || (block_stride * (int64_t)es) % 16 != 0)
        return HKV_ERR_INVALID_ARG;
    if ((q && !aligned16(q)) || !aligned16(k) || !aligned16(v) || (out && !aligned16(out)))
        return HKV_ERR_INVALID_ARG;
    if (hkv::pack_smem_bytes(P) > 200 * 1024) return HKV_ERR_INVALID_ARG;
    return HKV_OK;
}

// Marks `layer` ready for appends and decodes at length P and enqueues its
// first decode plan.
static hkv_status prefill_done(hkv_ctx* c, int32_t layer, int P, void* stream) {
    if (hkv::launch_plan(c->lay, layer, layer + 1, 1, 0, (cudaStream_t)stream) != cudaSuccess)
        return HKV_ERR_CUDA;
    c->plan_for[layer] = P;
    c->classified[layer] = 1;
    c->t_host[layer] = P;
    c->prefill_len[layer] = P;
    return HKV_OK;
}

hkv_status hkv_prefill_classify(hkv_ctx* c, int32_t layer, const void* q, const void* k,
                                const void* v, int32_t prefill_len, int64_t block_stride,
                                void* out, void* stream) {
    hkv_status st = prefill_args(c, layer, q, k, v, prefill_len, block_stride, out, true);
    if (st != HKV_OK) return st;
    // sharded heads need every shard's Local count: hkv_prefill_label + _compress
    if (total_heads(&c->cfg) != c->cfg.num_heads) return HKV_ERR_INVALID_ARG;
    if (c->classified[layer] || c->labelled_layer >= 0) return HKV_ERR_STATE;
    note_other(c, stream);
    if (hkv::launch_prefill(c->lay, layer, q, k, v, prefill_len, block_stride, out,
                            (cudaStream_t)stream) != cudaSuccess)
        return HKV_ERR_CUDA;
    return prefill_done(c, layer, prefill_len, stream);
}

hkv_status hkv_prefill_label(hkv_ctx* c, int32_t layer, const void* q, const void* k,
                             const void* v, int32_t prefill_len, int64_t block_stride, void* out,
                             int32_t* n_local, void* stream) {
    hkv_status st = prefill_args(c, layer, q, k, v, prefill_len, block_stride, out, true);
    if (st != HKV_OK) return st;
    if (!n_local || ((uintptr_t)n_local & 3)) return HKV_ERR_INVALID_ARG;
    if (c->classified[layer] || c->labelled_layer >= 0) return HKV_ERR_STATE;
    note_other(c, stream);
    if (hkv::launch_prefill_label(c->lay, layer, q, k, v, prefill_len, block_stride, out, n_local,
                                  (cudaStream_t)stream) != cudaSuccess)
        return HKV_ERR_CUDA;
    c->labelled_layer = layer;
    c->labelled_len = prefill_len;
    return HKV_OK;
}

hkv_status hkv_prefill_compress(hkv_ctx* c, int32_t layer, const void* k, const void* v,
                                int32_t prefill_len, int64_t block_stride,
                                const int32_t* n_local_total, void* stream) {
    hkv_status st = prefill_args(c, layer, nullptr, k, v, prefill_len, block_stride, nullptr, false);
    if (st != HKV_OK) return st;
    if (!n_local_total || ((uintptr_t)n_local_total & 3)) return HKV_ERR_INVALID_ARG;
    if (c->labelled_layer != layer || c->labelled_len != prefill_len) return HKV_ERR_STATE;
    note_other(c, stream);
    if (hkv::launch_prefill_compress(c->lay, layer, k, v, prefill_len, block_stride, n_local_total,
                                     (cudaStream_t)stream) != cudaSuccess)
        return HKV_ERR_CUDA;
    c->labelled_layer = -1;
    return prefill_done(c, layer, prefill_len, stream);
}

static hkv_status step_check(hkv_ctx* c, int32_t layer, bool appends) {
    if (!c) return HKV_ERR_INVALID_ARG;
    if (layer < 0 || layer >= c->cfg.num_layers) return HKV_ERR_INVALID_ARG;
    if (!c->classified[layer]) return HKV_ERR_STATE;
    if (appends && c->t_host[layer] >= c->cfg.max_len) return HKV_ERR_CAPACITY;
    return HKV_OK;
}

hkv_status hkv_append(hkv_ctx* c, int32_t layer, const void* k_t, const void* v_t, void* stream) {
    hkv_status s = step_check(c, layer, true);
    if (s != HKV_OK) return s;
    if (!k_t || !v_t || !aligned16(k_t) || !aligned16(v_t)) return HKV_ERR_INVALID_ARG;
    note_other(c, stream);
    cudaError_t e = hkv::launch_append(c->lay, layer, k_t, v_t, (cudaStream_t)stream);
    if (e != cudaSuccess) return HKV_ERR_CUDA;
    c->t_host[layer] += 1;
    return HKV_OK;
}

hkv_status hkv_decode_attend(hkv_ctx* c, int32_t layer, const void* q_t, void* o_t, void* stream) {
    hkv_status s = step_check(c, layer, false);
    if (s != HKV_OK) return s;
    if (!q_t || !o_t || !aligned16(q_t) || !aligned16(o_t)) return HKV_ERR_INVALID_ARG;
    const int t = c->t_host[layer] - 1;  // newest cached position
    cudaError_t e = cudaSuccess;
    if (c->plan_for[layer] != t) {
        note_other(c, stream);
        e = hkv::launch_plan(c->lay, layer, layer + 1, 0, 0, (cudaStream_t)stream);
        c->plan_for[layer] = t;
    }
    if (e == cudaSuccess) e = decode_launch(c, layer, q_t, nullptr, nullptr, o_t, 0, stream);
    return cuda_status(e);
}

hkv_status hkv_decode_step(hkv_ctx* c, int32_t layer, const void* q_t, const void* k_t,
                           const void* v_t, void* o_t, void* stream) {
    hkv_status s = step_check(c, layer, true);
    if (s != HKV_OK) return s;
    if (!q_t || !k_t || !v_t || !o_t || !aligned16(q_t) || !aligned16(k_t) || !aligned16(v_t) ||
        !aligned16(o_t))
        return HKV_ERR_INVALID_ARG;
    const int t = c->t_host[layer];  // position this step appends
    cudaError_t e = cudaSuccess;
    if (c->plan_for[layer] != t) {
        note_other(c, stream);
        e = hkv::launch_plan(c->lay, layer, layer + 1, 1, 0, (cudaStream_t)stream);
        c->plan_for[layer] = t;
    }
    if (e == cudaSuccess) e = decode_launch(c, layer, q_t, k_t, v_t, o_t, 1, stream);
    if (e != cudaSuccess) return HKV_ERR_CUDA;
    c->t_host[layer] += 1;
    return HKV_OK;
}

hkv_status hkv_ste_evict(hkv_ctx* c, int32_t layer_begin, int32_t layer_end, void* stream) {
    if (!c || layer_begin < 0 || layer_end > c->cfg.num_layers || layer_begin >= layer_end)
        return HKV_ERR_INVALID_ARG;
    for (int l = layer_begin; l < layer_end; ++l)
        if (!c->classified[l]) return HKV_ERR_STATE;
    cudaError_t e = cudaSuccess;
    note_other(c, stream);
    if (c->cfg.mode != HKV_MODE_FULL) {
        // no more blocks than (unit, head) items: a small cache launches few
        const int64_t items = (int64_t)(layer_end - layer_begin) * c->cfg.num_seqs * c->cfg.num_heads;
        const int grid = items < c->evict_grid ? (int)items : c->evict_grid;
        e = hkv::launch_evict(c->lay, layer_begin, layer_end, grid, (cudaStream_t)stream);
    }
    // plans of the next step, made once for all these layers, with the new
    // lengths of the heads just evicted
    if (e == cudaSuccess)
        e = hkv::launch_plan(c->lay, layer_begin, layer_end, 1, c->cfg.mode != HKV_MODE_FULL,
                             (cudaStream_t)stream, c->cfg.mode != HKV_MODE_FULL);
    if (e != cudaSuccess) return HKV_ERR_CUDA;
    for (int l = layer_begin; l < layer_end; ++l) c->plan_for[l] = c->t_host[l];
    return HKV_OK;
}

static hkv_status copy_back(void* dst, const void* src, size_t bytes, void* stream) {
    cudaError_t e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    return cuda_status(e);
}

hkv_status hkv_get_labels(hkv_ctx* c, int32_t layer, uint8_t* labels_host, int32_t* n_tau_host,
                          void* stream) {
    if (!c || !labels_host || layer < 0 || layer >= c->cfg.num_layers) return HKV_ERR_INVALID_ARG;
    if (!c->classified[layer]) return HKV_ERR_STATE;
    const size_t nh = (size_t)c->cfg.num_seqs * c->cfg.num_heads;
    hkv_status s = copy_back(labels_host, c->lay.label + layer * nh, nh, stream);
    if (s == HKV_OK && n_tau_host) s = copy_back(n_tau_host, c->lay.n_tau + layer * nh, nh * 4, stream);
    return s;
}

hkv_status hkv_get_lens(hkv_ctx* c, int32_t layer, int32_t* len_host, int32_t* budget_host,
                        void* stream) {
    if (!c || !len_host || layer < 0 || layer >= c->cfg.num_layers) return HKV_ERR_INVALID_ARG;
    if (!c->classified[layer]) return HKV_ERR_STATE;
    const size_t nh = (size_t)c->cfg.num_seqs * c->cfg.num_heads;
    std::vector<uint64_t> base(nh);
    std::vector<int32_t> cap(nh), tn(1);
    std::vector<uint8_t> lab(nh);
    hkv_status s = copy_back(base.data(), c->lay.base + layer * nh, nh * 8, stream);
    if (s == HKV_OK) s = copy_back(cap.data(), c->lay.cap + layer * nh, nh * 4, stream);
    if (s == HKV_OK) s = copy_back(lab.data(), c->lay.label + layer * nh, nh, stream);
    if (s == HKV_OK) s = copy_back(tn.data(), c->lay.t_next + layer, 4, stream);
    if (s == HKV_OK && budget_host) s = copy_back(budget_host, c->lay.budget + layer * nh, nh * 4, stream);
    if (s != HKV_OK) return s;
    const int t = tn[0] - 1;  // newest cached position
    for (size_t i = 0; i < nh; ++i) {
        int n = hkv::base_len_of(base[i]) + (t - hkv::base_t_of(base[i]));
        if (lab[i] == 1 && n > cap[i]) n = cap[i];
        len_host[i] = n;
    }
    return HKV_OK;
}

hkv_status hkv_get_kept(hkv_ctx* c, int32_t seq, int32_t layer, int32_t head, int32_t* pos_host,
                        int32_t capacity, int32_t* len_out, void* stream) {
    if (!c || !pos_host || !len_out || seq < 0 || seq >= c->cfg.num_seqs || layer < 0 ||
        layer >= c->cfg.num_layers || head < 0 || head >= c->cfg.num_heads)
        return HKV_ERR_INVALID_ARG;
    if (!c->classified[layer]) return HKV_ERR_STATE;
    const size_t nh = (size_t)c->cfg.num_seqs * c->cfg.num_heads;
    std::vector<int32_t> lens(nh);
    hkv_status s = hkv_get_lens(c, layer, lens.data(), nullptr, stream);
    if (s != HKV_OK) return s;
    const size_t hi = (size_t)layer * nh + (size_t)seq * c->cfg.num_heads + head;
    int32_t off = 0;
    s = copy_back(&off, c->lay.off + hi, 4, stream);
    if (s != HKV_OK) return s;
    const int n = lens[(size_t)seq * c->cfg.num_heads + head];
    *len_out = n;
    if (n > capacity) return HKV_ERR_CAPACITY;
    const size_t slot0 = ((size_t)layer * c->cfg.num_seqs + seq) * (size_t)c->lay.R + off;
    s = copy_back(pos_host, c->lay.pos + slot0, (size_t)n * 4, stream);
    if (s != HKV_OK) return s;
    // ascending order (slot order is a ring or a compacted set)
    for (int i = 1; i < n; ++i) {
        int32_t x = pos_host[i];
        int j = i - 1;
        while (j >= 0 && pos_host[j] > x) { pos_host[j + 1] = pos_host[j]; --j; }
        pos_host[j + 1] = x;
    }
    return HKV_OK;
}

hkv_status hkv_get_evict_stats(hkv_ctx* c, int64_t* stats_host, void* stream) {
    if (!c || !stats_host) return HKV_ERR_INVALID_ARG;
    return copy_back(stats_host, c->lay.ev_stats, 3 * 8, stream);
}

hkv_status hkv_check(hkv_ctx* c, int32_t* detail_host, void* stream) {
    if (!c) return HKV_ERR_INVALID_ARG;
    int32_t w[2] = {0, 0};
    hkv_status s = copy_back(w, c->lay.status, 8, stream);
    if (s != HKV_OK) return s;
    if (detail_host) *detail_host = w[1];
    return (hkv_status)w[0];
}

hkv_status hkv_clear_error(hkv_ctx* c, void* stream) {
    if (!c) return HKV_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(c->lay.status, 0, 8, (cudaStream_t)stream));
}

hkv_status hkv_reset(hkv_ctx* c, void* stream) {
    if (!c) return HKV_ERR_INVALID_ARG;
    note_other(c, stream);
    cudaError_t e = cudaMemsetAsync(c->lay.status, 0, ctrl_bytes(&c->cfg), (cudaStream_t)stream);
    if (e != cudaSuccess) return HKV_ERR_CUDA;
    for (int l = 0; l < c->cfg.num_layers; ++l) {
        c->classified[l] = 0;
        c->t_host[l] = 0;
        c->prefill_len[l] = 0;
        c->plan_for[l] = -1;
    }
    c->labelled_layer = -1;
    return HKV_OK;
}

void hkv_destroy(hkv_ctx* c) { delete c; }

hkv_status hkv_classify_groups(const float* rows, int32_t n_units, int32_t r, int32_t nq,
                               int32_t n, const int32_t* partner, int32_t W, double tau,
                               int32_t* n_tau, uint8_t* label, void* stream) {
    if (!rows || !n_tau || !label || n_units < 0 || r < 1 || nq < 1 || nq > r || n < r || W < 1 ||
        !(tau > 0.0 && tau <= 1.0))
        return HKV_ERR_INVALID_ARG;
    if (n_units == 0) return HKV_OK;
    return cuda_status(hkv::launch_classify_groups(rows, n_units, r, nq, n, partner, W, tau, n_tau,
                                                   label, (cudaStream_t)stream));
}

hkv_status hkv_classify_rows(const float* rows, int32_t n_rows, int32_t n, int32_t W, double tau,
                             int32_t* n_tau, uint8_t* label, void* stream) {
    if (!rows || !n_tau || !label || n_rows < 0 || n < 1 || W < 1 || !(tau > 0.0 && tau <= 1.0))
        return HKV_ERR_INVALID_ARG;
    if (n_rows == 0) return HKV_OK;
    return cuda_status(hkv::launch_classify_rows(rows, n_rows, n, W, tau, n_tau, label,
                                                 (cudaStream_t)stream));
}

hkv_status hkv_ste_select_batch(const float* score, const int32_t* pos, const int32_t* count,
                                const int32_t* t, int32_t n_probs, int32_t n, int32_t D,
                                int32_t k_near, int32_t k_far, int32_t stratified, uint8_t* evict,
                                void* stream) {
    if (!score || !pos || !count || !t || !evict || n_probs < 0 || n < 1 || n > 4096 || D < 0 ||
        k_near < 0 || k_far < 0 || (stratified != 0 && stratified != 1))
        return HKV_ERR_INVALID_ARG;
    if (n_probs == 0) return HKV_OK;
    return cuda_status(hkv::launch_select_batch(score, pos, count, t, n_probs, n, D, k_near, k_far,
                                                stratified, evict, (cudaStream_t)stream));
}

}  // extern "C"
