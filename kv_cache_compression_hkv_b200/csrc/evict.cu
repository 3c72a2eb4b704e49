// evict.cu -- Stratified Token Eviction for Global heads (HeadKV technical
// summary, Methodology step 3, global heads) and the standalone grouping and
// selection primitives.
//
// One warp per due head (listed first by a scan): it turns the logits the decode kernel stored over
// the last r steps into scores (summed softmax weights, each step normalised
// by its own (max, sum) and counting only tokens already cached at that
// step), selects the M/2 lowest (score, position) of the near and the far
// strata with a warp bisection, and compacts the cache in place by moving
// the surviving tail tokens into the holes below the budget.
#include <math.h>

#include <mutex>

#include "hkv_internal.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace hkv {

// Per-warp scratch of the eviction: the select's own scratch, the (max, sum)
// of the scoring steps, the step each column holds, an mbarrier, the
// positions of the top M slots, then their K and V rows (`row_bytes` each),
// prefetched while the head is scored.
__host__ __device__ inline size_t evict_warp_bytes(int n_max, int m_rows, int row_bytes) {
    return select_scratch_bytes(n_max) + 32 * 8 + 32 * 4 + 16 + (size_t)round32(m_rows) * 4 +
           2 * (size_t)m_rows * row_bytes;
}

constexpr uint64_t EVICT_WAIT_NS = 2000000000ull;  // a copy that takes 2 s has failed

// Lists the Global heads of layers [l0, l1) whose cache reached budget + M
// (one thread per head; one atomic per warp).
__global__ void __launch_bounds__(256) evict_scan_kernel(Layout L, int l0, int l1) {
    const int n_heads = L.S * L.H;
    const int total = (l1 - l0) * n_heads;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    bool due = false;
    size_t hx = 0;
    if (i < total && L.mode != HKV_MODE_FULL) {
        const int l = l0 + i / n_heads;
        hx = (size_t)l * n_heads + (i % n_heads);
        due = L.label[hx] == 0 && len_at(L, hx, L.t_next[l] - 1) >= L.cap[hx];
    }
    const unsigned b = __ballot_sync(FULL_MASK, due);
    if (!b) return;
    const int leader = __ffs(b) - 1;  // every lane of the warp reaches here
    int base = 0;
    if (lane == leader) base = atomicAdd(L.due_ctl, __popc(b));
    base = __shfl_sync(FULL_MASK, base, leader);
    if (due) L.due_list[base + __popc(b & ((1u << lane) - 1u))] = (int)hx;
}

// Evicts every listed head, one warp per head: scores from the stored
// logits, stratified select, compaction.  The last block clears the list.
constexpr int EVICT_MAX_WARPS = 12;

template <typename T>
__global__ void __launch_bounds__(EVICT_MAX_WARPS * 32) evict_run_kernel(Layout L, int n_max) {
    extern __shared__ __align__(16) unsigned char esm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NW = blockDim.x >> 5;
    const int d = L.d;
    const int r = L.r;
    const int row_bytes = d * (int)sizeof(T);
    const int MR = L.M;  // rows above the budget of a due head
    unsigned char* wbase = esm + (size_t)warp * evict_warp_bytes(n_max, MR, row_bytes);
    SelectScratch sc = carve_select_scratch(wbase, n_max);
    float2* ml_s = reinterpret_cast<float2*>(wbase + select_scratch_bytes(n_max));
    int32_t* step_s = reinterpret_cast<int32_t*>(ml_s + 32);
    uint64_t* bar = reinterpret_cast<uint64_t*>(step_s + 32);
    int32_t* top_pos = reinterpret_cast<int32_t*>(bar + 2);
    unsigned char* kvbuf = reinterpret_cast<unsigned char*>(top_pos + round32(MR));  // K|V row pairs
    const int n_heads = L.S * L.H;
    unsigned char* KVb = reinterpret_cast<unsigned char*>(L.K);  // slot s: K|V pair at 2 row_bytes s
    const int pair = 2 * row_bytes;
    const int per_pair = pair / 16;  // 16-byte pieces per K|V pair
    const int count = L.due_ctl[0];
    if (lane == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
    }
    __syncwarp();
    uint32_t phase = 0;

    for (int e = blockIdx.x * NW + warp; e < count; e += gridDim.x * NW) {
        const size_t hx = (size_t)L.due_list[e];
        const int l = (int)(hx / n_heads);
        const int hs = (int)(hx % n_heads);
        const int s = hs / L.H;
        const int t = L.t_next[l] - 1;
        const int n = len_at(L, hx, t);
        const int target = L.budget[hx];
        if (n > n_max || n != L.cap[hx] || n - target > MR || n - target < 0) {
            if (lane == 0) latch_error(L, HKV_ERR_CAPACITY, (int)hx);
            continue;
        }
        const size_t slot0 = region_slot0(L, l, s) + L.off[hx];
        const int top = n - target;  // the slots a survivor may move from
        // the K and V rows of slots target .. n-1, while the head is scored
        if (lane == 0 && top > 0) {
            ptx::mbar_expect_tx(bar, (uint32_t)(top * pair));
            ptx::bulk_g2s(kvbuf, KVb + (slot0 + target) * pair, top * pair, bar);
        }
        // (max, 1/sum) of each scoring step, by column = step mod r, and the
        // step each column holds inside the window t-r+1 .. t
        if (lane < r) {
            const float2 ml = L.ml[hx * r + lane];
            ml_s[lane] = make_float2(ml.x, 1.0f / ml.y);
            step_s[lane] = t - (((t - lane) % r) + r) % r;
        }
        __syncwarp();
        // scores: summed softmax weight of the last r queries, each
        // counting only tokens already cached at its step.  Tokens go in
        // batches of 8 per lane whose loads are all issued before any is
        // used; every 32 of them are sorted into the strata right away.
        bool bad = false;
        int nn = 0, nf = 0;
        for (int b0 = 0; b0 < n; b0 += 32 * 8) {
            int pv[8];
            float4 la[8], lb[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int q = b0 + u * 32 + lane;
                if (q < n) {
                    pv[u] = L.pos[slot0 + q];
                    if (r == 8) {
                        const float4* lg = reinterpret_cast<const float4*>(L.logit + (slot0 + q) * 8);
                        la[u] = lg[0];
                        lb[u] = lg[1];
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int base = b0 + u * 32;
                if (base >= n) break;  // warp-uniform
                const int q = base + lane;
                const bool valid = q < n;
                const int p = valid ? pv[u] : 0;
                float acc = 0.f;
                if (valid) {
                    if (r == 8) {
                        const float v[8] = {la[u].x, la[u].y, la[u].z, la[u].w, lb[u].x, lb[u].y, lb[u].z, lb[u].w};
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            if (p <= step_s[c]) acc += exp2f(v[c] - ml_s[c].x) * ml_s[c].y;
                    } else {
                        const float* lg = L.logit + (slot0 + q) * r;
                        for (int c = 0; c < r; ++c)
                            if (p <= step_s[c]) acc += exp2f(lg[c] - ml_s[c].x) * ml_s[c].y;
                    }
                    if (isnan(acc)) bad = true;
                    if (q >= target) top_pos[q - target] = p;
                }
                warp_partition_batch(sc, n, t, L.D, L.stratified, base, valid, __float_as_uint(acc), p, nn, nf);
            }
        }
        __syncwarp();
        const int E = n - target;
        warp_select_partitioned(sc, n, nn, nf, E / 2, E - E / 2, L.stratified);
        if (__any_sync(FULL_MASK, bad) && lane == 0) latch_error(L, HKV_ERR_NUMERIC, (int)hx);
        // holes: evicted slots below the budget; movers: survivors above it
        int nh = 0, nm = 0;
        for (int b0 = 0; b0 < n; b0 += 32) {
            const int q = b0 + lane;
            const bool ev = q < n && ((sc.evict_bits[q >> 5] >> (q & 31)) & 1u);
            const bool hole = q < target && ev;
            const bool mover = q >= target && q < n && !ev;
            const unsigned bh = __ballot_sync(FULL_MASK, hole);
            const unsigned bm = __ballot_sync(FULL_MASK, mover);
            const unsigned lt = (1u << lane) - 1u;
            if (hole) sc.moves[nh + __popc(bh & lt)] = (uint16_t)q;
            if (mover) sc.moves[sc.n_max - 1 - (nm + __popc(bm & lt))] = (uint16_t)q;
            nh += __popc(bh);
            nm += __popc(bm);
        }
        __syncwarp();
        bool ok = true;
        if (top > 0) {
            ok = ptx::mbar_wait(bar, phase, EVICT_WAIT_NS);
            ok = __all_sync(FULL_MASK, ok);
            phase ^= 1u;
        }
        if (!ok) {  // the prefetch never landed: stop before reusing its buffer
            if (lane == 0) latch_error(L, HKV_ERR_TIMEOUT, (int)hx);
            break;
        }
        if (nh != nm) {
            if (lane == 0) latch_error(L, HKV_ERR_CAPACITY, (int)hx);
            continue;
        }
        // move rows: each survivor's K and V rows from shared memory into a
        // hole, in 16-byte pieces
        const int pieces = nh * per_pair;
        for (int w = lane; w < pieces; w += 32) {
            const int mv = w / per_pair, pc = w % per_pair;
            const int src = sc.moves[sc.n_max - 1 - mv] - target;
            const size_t dst = (slot0 + sc.moves[mv]) * pair + pc * 16;
            *reinterpret_cast<uint4*>(KVb + dst) =
                *reinterpret_cast<const uint4*>(kvbuf + (size_t)src * pair + pc * 16);
        }
        for (int mv = lane; mv < nh; mv += 32)
            L.pos[slot0 + sc.moves[mv]] = top_pos[sc.moves[sc.n_max - 1 - mv] - target];
        __syncwarp();
        if (lane == 0) {
            L.base_len[hx] = target;
            L.base_t[hx] = t;
        }
    }
    // the last block out clears the list for the next step
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(L.due_ctl + 1, 1) == (int)gridDim.x - 1) {
            L.due_ctl[0] = 0;
            L.due_ctl[1] = 0;
        }
    }
}

// Standalone grouping rule over weight rows, one warp per row.
__global__ void classify_rows_kernel(const float* __restrict__ rows, int n_rows, int n, int W,
                                     double tau, int32_t* __restrict__ n_tau,
                                     uint8_t* __restrict__ label) {
    const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (row >= n_rows) return;
    const int need = warp_tokens_to_tau(rows + (size_t)row * n, n, tau);
    if ((threadIdx.x & 31) == 0) {
        n_tau[row] = need;
        label[row] = need < W ? 1 : 0;
    }
}

// Standalone grouping of caller weight rows, one warp per unit: unit u is
// grouped alone or, with partner[u] = p != u, with p (the lower of the two
// first).  A partner outside [0, n_units) marks the unit: n_tau -1, label
// 255.
__global__ void classify_groups_kernel(const float* __restrict__ rows, int n_units, int r, int nq,
                                       int n, const int32_t* __restrict__ partner, int W,
                                       double tau, int32_t* __restrict__ n_tau,
                                       uint8_t* __restrict__ label) {
    const int u = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (u >= n_units) return;
    const int p = partner ? partner[u] : u;
    if (p < 0 || p >= n_units) {
        if ((threadIdx.x & 31) == 0) { n_tau[u] = -1; label[u] = 255; }
        return;
    }
    const int a = min(u, p), b = max(u, p);
    const size_t blk = (size_t)r * n;
    const int need = warp_group_need_rows(rows + (size_t)a * blk,
                                          b != a ? rows + (size_t)b * blk : nullptr, r, nq, n, tau);
    if ((threadIdx.x & 31) == 0) {
        n_tau[u] = need;
        label[u] = need < W ? 1 : 0;
    }
}

// Standalone stratified select, one warp per problem.
__global__ void __launch_bounds__(128) select_batch_kernel(
    const float* __restrict__ score, const int32_t* __restrict__ pos, const int32_t* __restrict__ count,
    const int32_t* __restrict__ tt, int n_probs, int n, int D, int k_near, int k_far, int stratified,
    uint8_t* __restrict__ evict) {
    extern __shared__ __align__(16) unsigned char ssm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int prob = blockIdx.x * (blockDim.x >> 5) + warp;
    if (prob >= n_probs) return;
    SelectScratch sc = carve_select_scratch(ssm + (size_t)warp * select_scratch_bytes(n), n);
    const int m = min(max(count[prob], 0), n);
    const float* sp = score + (size_t)prob * n;
    const int32_t* pp = pos + (size_t)prob * n;
    auto key_of = [&](int i, uint32_t& sb, int32_t& p) {
        sb = __float_as_uint(sp[i]);
        p = pp[i];
    };
    warp_stratified_select(sc, m, tt[prob], D, k_near, k_far, stratified, key_of);
    for (int i = lane; i < n; i += 32)
        evict[(size_t)prob * n + i] = i < m ? (uint8_t)((sc.evict_bits[i >> 5] >> (i & 31)) & 1u) : 0;
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

static int evict_warps(size_t per) {
    int w = (int)((200 * 1024) / per);
    return w < 1 ? 1 : (w > EVICT_MAX_WARPS ? EVICT_MAX_WARPS : w);
}

cudaError_t launch_evict(const Layout& L, int l0, int l1, int grid, cudaStream_t st) {
    const int heads = (l1 - l0) * L.S * L.H;
    evict_scan_kernel<<<(heads + 255) / 256, 256, 0, st>>>(L, l0, l1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int n_max = L.L;
    const size_t per = evict_warp_bytes(n_max, L.M, L.d * (L.dtype == HKV_DTYPE_F32 ? 4 : 2));
    const int nw = evict_warps(per);
    const size_t sm = (size_t)nw * per;
    if (L.dtype == HKV_DTYPE_BF16)
        evict_run_kernel<__nv_bfloat16><<<grid, 32 * nw, sm, st>>>(L, n_max);
    else
        evict_run_kernel<float><<<grid, 32 * nw, sm, st>>>(L, n_max);
    return cudaGetLastError();
}

cudaError_t prepare_evict(int smem) {
    cudaError_t e = allow_max_dynamic_smem(evict_run_kernel<__nv_bfloat16>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(evict_run_kernel<float>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(select_batch_kernel, smem);
    return e;
}

cudaError_t launch_classify_groups(const float* rows, int n_units, int r, int nq, int n,
                                   const int32_t* partner, int W, double tau, int32_t* n_tau,
                                   uint8_t* label, cudaStream_t st) {
    const int grid = (n_units + 7) / 8;  // 8 warps per block
    classify_groups_kernel<<<grid, 256, 0, st>>>(rows, n_units, r, nq, n, partner, W, tau, n_tau,
                                                 label);
    return cudaGetLastError();
}

cudaError_t launch_classify_rows(const float* rows, int n_rows, int n, int W, double tau,
                                 int32_t* n_tau, uint8_t* label, cudaStream_t st) {
    const int grid = (n_rows + 7) / 8;
    classify_rows_kernel<<<grid, 256, 0, st>>>(rows, n_rows, n, W, tau, n_tau, label);
    return cudaGetLastError();
}

cudaError_t launch_select_batch(const float* score, const int32_t* pos, const int32_t* count,
                                const int32_t* t, int n_probs, int n, int D, int k_near, int k_far,
                                int stratified, uint8_t* evict, cudaStream_t st) {
    const int nw = 4;
    const size_t sm = (size_t)nw * select_scratch_bytes(n);
    cudaError_t e = prepare_kernels();
    if (e != cudaSuccess) return e;
    select_batch_kernel<<<(n_probs + nw - 1) / nw, 32 * nw, sm, st>>>(
        score, pos, count, t, n_probs, n, D, k_near, k_far, stratified, evict);
    return cudaGetLastError();
}

cudaError_t prepare_kernels() {
    // Every kernel may use up to the device's opt-in shared memory.  The
    // attribute belongs to the current device, so the latch is kept per
    // device (a host-side attribute call, kept out of stream captures).
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    int dev = 0, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev]) return cudaSuccess;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = prepare_prefill(optin);
    if (e == cudaSuccess) e = prepare_prefill_umma(optin);
    if (e == cudaSuccess) e = prepare_decode(optin);
    if (e == cudaSuccess) e = prepare_evict(optin);
    if (e == cudaSuccess) done[dev] = true;
    return e;
}

}  // namespace hkv
