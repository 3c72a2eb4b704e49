// evict.cu -- Stratified Token Eviction for Global heads (HeadKV technical
// summary, Methodology step 3, global heads) and the standalone grouping and
// selection primitives.
//
// One block per due head: it turns the logits the decode kernel stored over
// the last r steps into scores (summed softmax weights, each step normalised
// by its own (max, sum) and counting only tokens already cached at that
// step), selects the M/2 lowest (score, position) of the near and the far
// strata by a block-wide threshold search, and compacts the cache in place
// by moving the surviving tail tokens into the holes below the budget.
#include <math.h>
#include <stdlib.h>

#include <mutex>

#include "hkv_internal.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace hkv {

// ---------------------------------------------------------------------------
// Eviction of the due heads of layers [l0, l1), one block per head.  A
// head's unit (layer, sequence) is due at step t when its due step (kept
// by the plan kernel; all Global heads of a unit share capacity and length)
// is t, the layer's newest position.  Block c looks at the items (unit,
// head) numbered c, c + G, c + 2G, ... (G blocks), lists the due ones among
// them in shared memory and evicts them one after the other: a unit's heads
// land on consecutive blocks.  Nothing here changes what the due test
// reads, so every block sees the same due set; the plan kernel that follows
// the eviction records the heads' new lengths.  Per head:
//  1. the rows a survivor may move from (slots budget .. len-1) are
//     prefetched into L2 while the head is scored;
//  2. every thread loads the position and the r stored logits of its tokens
//     (all loads of up to 4 tokens issued before any is used) and turns them
//     into the token's score: the summed softmax weight of the last r steps,
//     each step's weight exp2(logit - max) / sum, only for tokens already
//     cached at that step; key = (score bits, position) in shared memory;
//  3. the threshold of each stratum (near: distance 1..D; far: beyond) is
//     found by a 16-ary search on the score bits, both strata per round
//     (15 pivots each, counts reduced over the block), then the position tie
//     at the boundary; every key <= the threshold is evicted, so each
//     stratum loses exactly its share, lowest (score, position) first;
//  4. holes (evicted slots below the budget) and movers (survivors above it)
//     are listed in (thread, token) order and the i-th mover's K|V row pair
//     and position are copied into the i-th hole.
// ---------------------------------------------------------------------------
constexpr int EVB_THREADS = 256;  // threads of an eviction block
constexpr int EVB_WARPS = EVB_THREADS / 32;
__host__ __device__ inline size_t evict_group_smem(int n_max, int M);
// A stratum whose search window holds at most this many keys is finished by
// ranking those keys against each other.
constexpr int RANK_WIN = 32;
// Shared memory of the ranking: two candidate lists, their counters, the
// two thresholds.
constexpr int EVB_RANK_BYTES = 2 * RANK_WIN * 8 + 16 + 16;

// One round of the threshold search of both strata: every thread adds its
// candidate keys with score bits in [lo, hi] of their stratum to 16 bins of
// width 2^sh above lo (16-bit counters packed two to a word: a warp holds
// far fewer than 65536 keys) and counts those below lo; the totals of the
// head's group of warps (w0 .. w0 + nw - 1) are reduced through `red` (this
// round's buffer; rounds alternate between two, so one group barrier per
// round suffices).  Lane i of every warp returns {the number of keys at or
// below the top of bin i, the number below lo} (i < 16: near stratum, else
// bin i - 16 of the far stratum).
template <typename Sync>
__device__ __forceinline__ int2 group_bin_counts(const uint32_t (&ha)[8], const uint32_t (&hb)[8],
                                                int below_a, int below_b, int (*red)[32], int w0,
                                                int nw, Sync gsync) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        w[j] = __reduce_add_sync(FULL_MASK, ha[j]);
        w[8 + j] = __reduce_add_sync(FULL_MASK, hb[j]);
    }
    below_a = __reduce_add_sync(FULL_MASK, below_a);
    below_b = __reduce_add_sync(FULL_MASK, below_b);
    if (lane == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) red[warp][j] = (int)w[j];
        red[warp][16] = below_a;
        red[warp][17] = below_b;
    }
    gsync();
    // lane i: bin i & 15 of stratum i >> 4, summed over the group's warps
    int tot = 0, below = 0;
    const int word = lane >> 1, sh = 16 * (lane & 1);
    for (int v = w0; v < w0 + nw; ++v) {
        tot += ((uint32_t)red[v][word] >> sh) & 0xffffu;
        below += red[v][16 + (lane >> 4)];
    }
    // inclusive prefix over the 16 bins of each stratum
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
        const int y = __shfl_up_sync(FULL_MASK, tot, o);
        if ((lane & 15) >= o) tot += y;
    }
    return make_int2(tot + below, below);
}

// Adds one candidate key to its stratum's packed bins.
__device__ __forceinline__ void bin_add(uint32_t (&h)[8], int& below, uint32_t sb, uint32_t lo,
                                        uint32_t hi, int sh) {
    if (sb < lo) { ++below; return; }
    if (sb > hi) return;
    const uint32_t b = (sb - lo) >> sh;  // 0 .. 15
    const uint32_t inc = 1u << (16 * (b & 1));
    const uint32_t wi = b >> 1;
#pragma unroll
    for (int j = 0; j < 8; ++j) h[j] += wi == (uint32_t)j ? inc : 0u;
}

// Bin width (log2) that splits [lo, hi] into at most 16 bins.
__device__ __forceinline__ int bin_shift(uint32_t lo, uint32_t hi) {
    const uint32_t w = hi - lo;
    const int bits = w ? 32 - __clz(w) : 0;
    return bits > 4 ? bits - 4 : 0;
}

template <typename T>
__global__ void __launch_bounds__(EVB_THREADS, 2) evict_block_kernel(Layout L, int l0, int l1, int n_max,
                                                                    int GW) {
    extern __shared__ __align__(16) unsigned char ebs[];
    __shared__ float2 ml_all[EVB_WARPS][32];
    __shared__ int step_all[EVB_WARPS][32];
    __shared__ int red[2][EVB_WARPS][32];
    __shared__ int lists[2][EVB_WARPS];
    __shared__ int4 due_items[EVB_THREADS];  // {head, due step, budget, Global mask}
    __shared__ int n_due;
    __shared__ int flag_all[EVB_WARPS];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int BT = blockDim.x, NW = BT >> 5;
    // the block's warps work in groups of GW, one due head per group
    const int GT = 32 * GW, ngroups = NW / GW, grp = warp / GW, gw0 = grp * GW, gtid = tid % GT;
    const int r = L.r, M = L.M;
    unsigned char* gbase = ebs + (size_t)grp * evict_group_smem(n_max, M);
    uint64_t* keys = reinterpret_cast<uint64_t*>(gbase);          // [n_max]
    int32_t* holes = reinterpret_cast<int32_t*>(keys + n_max);    // [M]
    int32_t* movers = holes + M;                                  // [M]
    int32_t* mpos = movers + M;                                   // [M]
    uint64_t* cand = reinterpret_cast<uint64_t*>(gbase + ((size_t)n_max * 8 + (size_t)M * 12 + 15) / 16 * 16);
    int* ccnt = reinterpret_cast<int*>(cand + 2 * RANK_WIN);      // [2] (+ 2 spare)
    uint64_t* thr_sm = reinterpret_cast<uint64_t*>(ccnt + 4);     // [2]
    float2* ml_s = ml_all[grp];
    int* step_s = step_all[grp];
    // barrier of the head's group (one warp: the warp itself)
    auto gsync = [&]() {
        if (GW == 1) __syncwarp();
        else asm volatile("bar.sync %0, %1;" ::"r"(grp + 1), "r"(GT) : "memory");
    };
    // OR of a flag over the group
    auto gany = [&](bool x) -> bool {
        const bool wx = __any_sync(FULL_MASK, x);
        if (GW == 1) return wx;
        if (lane == 0) flag_all[warp] = wx;
        gsync();
        bool any = false;
        for (int w = gw0; w < gw0 + GW; ++w) any |= flag_all[w] != 0;
        gsync();  // the flags are read before they are written again
        return any;
    };
    const int n_heads = L.S * L.H;
    const int pair = 2 * L.d * (int)sizeof(T);                    // bytes of a K|V row pair
    const int per_pair = pair / 16;          // a power of two: 16 .. 64
    const int pp_shift = __ffs(per_pair) - 1;
    unsigned char* KVb = reinterpret_cast<unsigned char*>(L.K);
    int par = 0;  // reduction buffer of the next round
    const int64_t items = (int64_t)(l1 - l0) * L.S * L.H;
    const int64_t G = gridDim.x;
    if ((int64_t)blockIdx.x >= items) ptx::grid_dep_trigger();

    for (int64_t k0 = 0; (int64_t)blockIdx.x + k0 * G < items; k0 += BT) {
        // this block's next BT items: the due ones, in item order, each with
        // its unit's step, budget and Global mask (no per-head metadata)
        {
            const int64_t i = (int64_t)blockIdx.x + (k0 + tid) * G;
            bool due = false;
            int4 item = make_int4(0, 0, 0, 0);
            if (i < items) {
                const int64_t u = i / L.H;  // unit within the range
                const int h = (int)(i % L.H);
                const int l = l0 + (int)(u / L.S), s = (int)(u % L.S);
                const size_t uu = (size_t)l * L.S + s;
                const int4 rec = L.unit[uu];
                due = rec.x == L.t_next[l] - 1 && (((uint32_t)rec.y >> h) & 1u);
                item = make_int4((int)(uu * L.H + h), rec.x, rec.z, rec.y);
            }
            const unsigned b = __ballot_sync(FULL_MASK, due);
            __syncthreads();  // the previous round's list is no longer read
            if (lane == 0) lists[0][warp] = __popc(b);
            __syncthreads();
            int o = __popc(b & ((1u << lane) - 1u)), tot = 0;
            for (int w = 0; w < NW; ++w) {
                if (w < warp) o += lists[0][w];
                tot += lists[0][w];
            }
            if (due) due_items[o] = item;
            if (tid == 0) n_due = tot;
            __syncthreads();
        }
        // every unit record this block reads has been read: the plan
        // launched after this kernel (which commits the new lengths and due
        // steps) may start
        if ((int64_t)blockIdx.x + (k0 + BT) * G >= items) ptx::grid_dep_trigger();
        const int nd = n_due;
        for (int e = grp; e < nd; e += ngroups) {
            const int4 item = due_items[e];
            const size_t hx = (size_t)item.x;
            const int l = (int)(hx / n_heads);
            const int s = (int)(hx % n_heads) / L.H;
            const int h = (int)(hx % L.H);
            const int t = item.y;                 // the due step: the newest position
            const int target = item.z;            // the budget
            const int n = target + M;             // the capacity, reached at the due step
            const uint32_t gm = (uint32_t)item.w, below = (1u << h) - 1u;
            // first slot: Local heads before h hold W slots, Global ones n
            const size_t slot0 = region_slot0(L, l, s) + (size_t)__popc(~gm & below) * L.W +
                                 (size_t)__popc(gm & below) * n;
            gsync();  // the previous head's lists and keys are no longer read
            if (n > n_max) {
                if (gtid == 0) latch_error(L, HKV_ERR_CAPACITY, (int)hx);
                continue;
            }
            // every load of the head at once: thread 0 the L2 prefetch of the
            // rows a survivor may move from (slots budget .. n-1) and the
            // head's length record (checked below), threads < r the (max, sum)
            // of the scoring steps, every thread the positions and logits of
            // its first two tokens
            bool head_bad = false;
            if (gtid == 0) {
                ptx::bulk_prefetch_l2(KVb + (slot0 + target) * pair, (uint32_t)(M * pair));
                // the head's length record, before or after the plan kernel
                // running next to this one commits it
                const uint64_t b = L.base[hx];
                head_bad = !(base_len_of(b) + (t - base_t_of(b)) == n || b == base_pack(target, t));
            }
            if (gtid < r) {
                const float2 ml = L.ml[hx * r + gtid];
                ml_s[gtid] = make_float2(ml.x, 1.0f / ml.y);
                step_s[gtid] = t - (((t - gtid) % r) + r) % r;  // the step column gtid holds
            }
            const bool strat = L.stratified != 0;
            // two tokens of this thread: position and r = 8 logits each
            struct Two {
                int p[2];
                float4 a[2], b[2];
            };
            auto load2 = [&](int b0, Two& x) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int q = b0 + u * GT + gtid;
                    if (q < n) {
                        x.p[u] = L.pos[slot0 + q];
                        if (r == 8) {
                            const float4* p4 = reinterpret_cast<const float4*>(L.logit + (slot0 + q) * 8);
                            x.a[u] = p4[0];
                            x.b[u] = p4[1];
                        }
                    }
                }
            };
            Two cur, nxt;
            load2(0, cur);
            gsync();  // ml_s, step_s
            // the r = 8 scoring steps' (max, 1/sum) and positions in registers
            float mx[8], il[8];
            int stp[8];
            if (r == 8) {
#pragma unroll
                for (int c = 0; c < 8; ++c) { mx[c] = ml_s[c].x; il[c] = ml_s[c].y; stp[c] = step_s[c]; }
            }

            // scores and stratum counts; keys into shared memory; the next
            // two tokens' loads go out before this pair is used
            bool bad = false;
            int nn = 0, nf = 0;
            uint32_t alo = 0xffffffffu, ahi = 0u, blo = 0xffffffffu, bhi = 0u;
            for (int b0 = 0; b0 < n; b0 += 2 * GT) {
                if (b0 + 2 * GT < n) load2(b0 + 2 * GT, nxt);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int q = b0 + u * GT + gtid;
                    if (q >= n) continue;
                    const int p = cur.p[u];
                    float acc = 0.f;
                    if (r == 8) {
                        const float v[8] = {cur.a[u].x, cur.a[u].y, cur.a[u].z, cur.a[u].w,
                                            cur.b[u].x, cur.b[u].y, cur.b[u].z, cur.b[u].w};
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            if (p <= stp[c]) acc += exp2f(v[c] - mx[c]) * il[c];
                    } else {
                        const float* lp = L.logit + (slot0 + q) * r;
                        for (int c = 0; c < r; ++c)
                            if (p <= step_s[c]) acc += exp2f(lp[c] - ml_s[c].x) * ml_s[c].y;
                    }
                    if (isnan(acc)) bad = true;
                    const uint32_t sb = __float_as_uint(acc);
                    keys[q] = ((uint64_t)sb << 32) | (uint32_t)p;
                    const int delta = t - p;
                    if (delta >= 1) {
                        if (strat && delta <= L.D) { ++nn; alo = min(alo, sb); ahi = max(ahi, sb); }
                        else { ++nf; blo = min(blo, sb); bhi = max(bhi, sb); }
                    }
                }
                cur = nxt;
            }
            if (gany(bad) && gtid == 0) latch_error(L, HKV_ERR_NUMERIC, (int)hx);
            if (gany(head_bad)) {  // the head's length disagrees with its unit's record
                if (gtid == 0) latch_error(L, HKV_ERR_CAPACITY, (int)hx);
                continue;
            }
            // block totals: counts and score-bit ranges of both strata
            {
                nn = __reduce_add_sync(FULL_MASK, nn);
                nf = __reduce_add_sync(FULL_MASK, nf);
                alo = __reduce_min_sync(FULL_MASK, alo);
                ahi = __reduce_max_sync(FULL_MASK, ahi);
                blo = __reduce_min_sync(FULL_MASK, blo);
                bhi = __reduce_max_sync(FULL_MASK, bhi);
                int (*rb)[32] = red[par];
                if (lane == 0) {
                    rb[warp][0] = nn; rb[warp][1] = nf;
                    rb[warp][2] = (int)alo; rb[warp][3] = (int)ahi;
                    rb[warp][4] = (int)blo; rb[warp][5] = (int)bhi;
                }
                gsync();
                nn = nf = 0;
                alo = blo = 0xffffffffu;
                ahi = bhi = 0u;
                for (int w = gw0; w < gw0 + GW; ++w) {
                    nn += rb[w][0]; nf += rb[w][1];
                    alo = min(alo, (uint32_t)rb[w][2]); ahi = max(ahi, (uint32_t)rb[w][3]);
                    blo = min(blo, (uint32_t)rb[w][4]); bhi = max(bhi, (uint32_t)rb[w][5]);
                }
                par ^= 1;
            }
            // shares of the strata (a stratum short of candidates hands its
            // shortfall to the other); unstratified: one pool, all "far"
            const int E = n - target;
            int ka = E / 2, kb = E - E / 2;
            if (strat) {
                if (ka > nn) { kb += ka - nn; ka = nn; }
                if (kb > nf) { ka += kb - nf; kb = nf; if (ka > nn) ka = nn; }
            } else {
                kb = E < nf ? E : nf;
                ka = 0;
            }
            // threshold of each partial stratum (0 < k < m): the k-th smallest
            // key.  A window of score bits [lo, hi] that holds it shrinks
            // 16-fold per round until it holds at most RANK_WIN keys (or one
            // score value); those keys are then ranked against each other
            const bool a_part = ka > 0 && ka < nn, b_part = kb > 0 && kb < nf;
            int bel_a = 0, win_a = nn, bel_b = 0, win_b = nf;  // keys below / inside the window
            bool sa_on = a_part && alo < ahi && win_a > RANK_WIN;
            bool sb_on = b_part && blo < bhi && win_b > RANK_WIN;
            while (sa_on || sb_on) {
                const int sa = bin_shift(alo, ahi), sbh = bin_shift(blo, bhi);
                uint32_t ha[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u}, hb[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                int below_a = 0, below_b = 0;
                for (int q = gtid; q < n; q += GT) {
                    const uint64_t key = keys[q];
                    const uint32_t sb = (uint32_t)(key >> 32);
                    const int delta = t - (int32_t)(uint32_t)key;
                    if (delta < 1) continue;
                    if (strat && delta <= L.D) { if (sa_on) bin_add(ha, below_a, sb, alo, ahi, sa); }
                    else if (sb_on) bin_add(hb, below_b, sb, blo, bhi, sbh);
                }
                const int2 cb = group_bin_counts(ha, hb, below_a, below_b, red[par], gw0, GW, gsync);
                par ^= 1;
                const int cum = cb.x;
                // first bin whose cumulative count reaches the share; the keys
                // before it (the bin before's total, or those below lo)
                const unsigned ma = __ballot_sync(FULL_MASK, lane < 16 && cum >= ka);
                const unsigned mb = __ballot_sync(FULL_MASK, lane >= 16 && cum >= kb);
                const int ja = ma ? __ffs(ma) - 1 : 0, jb = mb ? __ffs(mb >> 16) - 1 : 0;
                const int at_a = __shfl_sync(FULL_MASK, cum, ja), at_b = __shfl_sync(FULL_MASK, cum, 16 + jb);
                const int pre_a = __shfl_sync(FULL_MASK, ja ? cum : cb.y, ja ? ja - 1 : 0);
                const int pre_b = __shfl_sync(FULL_MASK, jb ? cum : cb.y, jb ? 15 + jb : 16);
                if (sa_on) {
                    const uint64_t top = (uint64_t)alo + ((uint64_t)(ja + 1) << sa) - 1;
                    alo = alo + ((uint32_t)ja << sa);
                    ahi = top < ahi ? (uint32_t)top : ahi;
                    bel_a = pre_a;
                    win_a = at_a - pre_a;
                    sa_on = alo < ahi && win_a > RANK_WIN;
                }
                if (sb_on) {
                    const uint64_t top = (uint64_t)blo + ((uint64_t)(jb + 1) << sbh) - 1;
                    blo = blo + ((uint32_t)jb << sbh);
                    bhi = top < bhi ? (uint32_t)top : bhi;
                    bel_b = pre_b;
                    win_b = at_b - pre_b;
                    sb_on = blo < bhi && win_b > RANK_WIN;
                }
            }
            const int need_a = ka - bel_a, need_b = kb - bel_b;  // rank in the window, 1..win
            // every key <= thr of its stratum is evicted
            uint64_t thr_a = a_part ? 0ull : (ka >= nn && ka > 0 ? ~0ull : 0ull);
            uint64_t thr_b = b_part ? 0ull : (kb >= nf && kb > 0 ? ~0ull : 0ull);
            const bool none_a = ka <= 0, none_b = kb <= 0;
            const bool rank_a = a_part && win_a <= RANK_WIN, rank_b = b_part && win_b <= RANK_WIN;
            if (rank_a || rank_b) {
                // the window's keys into two lists, ranked by the group's first warp
                if (gtid < 2) ccnt[gtid] = 0;
                gsync();
                for (int q = gtid; q < n; q += GT) {
                    const uint64_t key = keys[q];
                    const uint32_t sb = (uint32_t)(key >> 32);
                    const int delta = t - (int32_t)(uint32_t)key;
                    if (delta < 1) continue;
                    if (strat && delta <= L.D) {
                        if (rank_a && sb >= alo && sb <= ahi) {
                            const int i = atomicAdd(&ccnt[0], 1);
                            if (i < RANK_WIN) cand[i] = key;
                        }
                    } else if (rank_b && sb >= blo && sb <= bhi) {
                        const int i = atomicAdd(&ccnt[1], 1);
                        if (i < RANK_WIN) cand[RANK_WIN + i] = key;
                    }
                }
                gsync();
                if (warp == gw0) {
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        const bool on = x == 0 ? rank_a : rank_b;
                        const int cnt = x == 0 ? win_a : win_b, need = x == 0 ? need_a : need_b;
                        if (!on) continue;
                        const uint64_t* cl = cand + x * RANK_WIN;
                        const uint64_t mine = lane < cnt ? cl[lane] : ~0ull;
                        int rk = 0;
                        for (int j = 0; j < cnt; ++j) rk += cl[j] < mine;
                        if (lane < cnt && rk == need - 1) thr_sm[x] = mine;
                    }
                }
                gsync();
                if (rank_a) thr_a = thr_sm[0];
                if (rank_b) thr_b = thr_sm[1];
            }
            const bool tie_a = a_part && !rank_a, tie_b = b_part && !rank_b;  // one score, many keys
            if (tie_a || tie_b) {
                // the need lowest positions among the keys at the one score s*
                uint32_t plo_a = 0xffffffffu, phi_a = 0u, plo_b = 0xffffffffu, phi_b = 0u;
                for (int q = gtid; q < n; q += GT) {
                    const uint64_t key = keys[q];
                    const uint32_t sb = (uint32_t)(key >> 32), p = (uint32_t)key;
                    const int delta = t - (int32_t)p;
                    if (delta < 1) continue;
                    if (strat && delta <= L.D) {
                        if (sb == alo) { plo_a = min(plo_a, p); phi_a = max(phi_a, p); }
                    } else if (sb == blo) {
                        plo_b = min(plo_b, p); phi_b = max(phi_b, p);
                    }
                }
                int (*rb)[32] = red[par];
                plo_a = __reduce_min_sync(FULL_MASK, plo_a); phi_a = __reduce_max_sync(FULL_MASK, phi_a);
                plo_b = __reduce_min_sync(FULL_MASK, plo_b); phi_b = __reduce_max_sync(FULL_MASK, phi_b);
                if (lane == 0) {
                    rb[warp][4] = (int)plo_a; rb[warp][5] = (int)phi_a;
                    rb[warp][6] = (int)plo_b; rb[warp][7] = (int)phi_b;
                }
                gsync();
                par ^= 1;
                plo_a = plo_b = 0xffffffffu;
                phi_a = phi_b = 0u;
                for (int w = gw0; w < gw0 + GW; ++w) {
                    plo_a = min(plo_a, (uint32_t)rb[w][4]); phi_a = max(phi_a, (uint32_t)rb[w][5]);
                    plo_b = min(plo_b, (uint32_t)rb[w][6]); phi_b = max(phi_b, (uint32_t)rb[w][7]);
                }
                // bisection on positions (every key of the window has score s*)
                while ((tie_a && plo_a < phi_a) || (tie_b && plo_b < phi_b)) {
                    const uint32_t mid_a = plo_a + ((phi_a - plo_a) >> 1);
                    const uint32_t mid_b = plo_b + ((phi_b - plo_b) >> 1);
                    int da = 0, db = 0;
                    for (int q = gtid; q < n; q += GT) {
                        const uint64_t key = keys[q];
                        const uint32_t sb = (uint32_t)(key >> 32), p = (uint32_t)key;
                        const int delta = t - (int32_t)p;
                        if (delta < 1) continue;
                        if (strat && delta <= L.D) da += sb == alo && p <= mid_a;
                        else db += sb == blo && p <= mid_b;
                    }
                    da = __reduce_add_sync(FULL_MASK, da);
                    db = __reduce_add_sync(FULL_MASK, db);
                    int (*rr)[32] = red[par];
                    if (lane == 0) { rr[warp][0] = da; rr[warp][1] = db; }
                    gsync();
                    par ^= 1;
                    da = db = 0;
                    for (int w = gw0; w < gw0 + GW; ++w) { da += rr[w][0]; db += rr[w][1]; }
                    if (tie_a && plo_a < phi_a) { if (da >= need_a) phi_a = mid_a; else plo_a = mid_a + 1; }
                    if (tie_b && plo_b < phi_b) { if (db >= need_b) phi_b = mid_b; else plo_b = mid_b + 1; }
                }
                if (tie_a) thr_a = ((uint64_t)alo << 32) | plo_a;
                if (tie_b) thr_b = ((uint64_t)blo << 32) | plo_b;
            }
            // holes and movers, listed in (thread, token) order
            int nh_mine = 0, nm_mine = 0;
            for (int q = gtid; q < n; q += GT) {
                const uint64_t key = keys[q];
                const int delta = t - (int32_t)(uint32_t)key;
                bool ev = false;
                if (delta >= 1) {
                    if (strat && delta <= L.D) ev = !none_a && key <= thr_a;
                    else ev = !none_b && key <= thr_b;
                }
                nh_mine += ev && q < target;
                nm_mine += !ev && q >= target;
            }
            int xh = nh_mine, xm = nm_mine;  // inclusive scans over the warp
    #pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int yh = __shfl_up_sync(FULL_MASK, xh, o), ym = __shfl_up_sync(FULL_MASK, xm, o);
                if (lane >= o) { xh += yh; xm += ym; }
            }
            if (lane == 31) { lists[0][warp] = xh; lists[1][warp] = xm; }
            gsync();
            int oh = xh - nh_mine, om = xm - nm_mine, nh = 0, nm = 0;
            for (int w = gw0; w < gw0 + GW; ++w) {
                if (w < warp) { oh += lists[0][w]; om += lists[1][w]; }
                nh += lists[0][w];
                nm += lists[1][w];
            }
            if (nh != nm || nh > M) {
                if (gtid == 0) latch_error(L, HKV_ERR_CAPACITY, (int)hx);
                continue;
            }
            for (int q = gtid; q < n; q += GT) {
                const uint64_t key = keys[q];
                const int delta = t - (int32_t)(uint32_t)key;
                bool ev = false;
                if (delta >= 1) {
                    if (strat && delta <= L.D) ev = !none_a && key <= thr_a;
                    else ev = !none_b && key <= thr_b;
                }
                if (ev && q < target) holes[oh++] = q;
                if (!ev && q >= target) { movers[om] = q; mpos[om] = (int32_t)(uint32_t)key; ++om; }
            }
            gsync();
            // row moves: the i-th mover's K|V pair into the i-th hole, 16-byte
            // pieces, up to 4 loads in flight per thread
            const int pieces = nh * per_pair;
            for (int w0 = 0; w0 < pieces; w0 += 4 * GT) {
                uint4 x[4];
    #pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int w = w0 + u * GT + gtid;
                    if (w < pieces) {
                        const int i = w >> pp_shift, pc = w & (per_pair - 1);
                        x[u] = *reinterpret_cast<const uint4*>(KVb + (slot0 + movers[i]) * pair + pc * 16);
                    }
                }
    #pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int w = w0 + u * GT + gtid;
                    if (w < pieces) {
                        const int i = w >> pp_shift, pc = w & (per_pair - 1);
                        *reinterpret_cast<uint4*>(KVb + (slot0 + holes[i]) * pair + pc * 16) = x[u];
                    }
                }
            }
            for (int i = gtid; i < nh; i += GT) L.pos[slot0 + holes[i]] = mpos[i];
            if (gtid == 0) {
                atomicAdd(L.ev_stats + 0, 1ull);
                atomicAdd(L.ev_stats + 1, (unsigned long long)n);
                atomicAdd(L.ev_stats + 2, (unsigned long long)nh);
            }
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

// Shared memory of one group of an eviction block: keys of up to n_max
// tokens, then the hole, mover and mover-position lists of up to M entries.
__host__ __device__ inline size_t evict_group_smem(int n_max, int M) {
    return ((size_t)n_max * 8 + (size_t)M * 12 + 15) / 16 * 16 + EVB_RANK_BYTES;
}

// Warps per head: enough for about 256 cached tokens per warp at the usual
// Global capacity floor(H_total * L * rho) / H_total + M (a power of two,
// 1 .. 8), more while the groups' shared memory would not fit two blocks per
// SM.
int evict_group_warps(const Layout& L) {
    const int64_t cap = L.T_total / (L.H_total > 0 ? L.H_total : L.H) + L.M;
    // HKV_EVICT_WARPS (1, 2, 4 or 8) sets the least group size (tuning)
    static const int least = [] {
        const char* v = getenv("HKV_EVICT_WARPS");
        const int x = v ? atoi(v) : 1;
        return (x == 2 || x == 4 || x == 8) ? x : 1;
    }();
    int gw = least < EVB_WARPS ? least : EVB_WARPS;
    while (gw < EVB_WARPS && cap > 256 * gw) gw *= 2;
    while (gw < EVB_WARPS && (EVB_WARPS / gw) * evict_group_smem(L.L, L.M) > 100 * 1024) gw *= 2;
    return gw;
}

static size_t evict_block_smem(const Layout& L) {
    return (size_t)(EVB_WARPS / evict_group_warps(L)) * evict_group_smem(L.L, L.M);
}

int evict_blocks_per_sm(const Layout& L, int optin) {
    const size_t sm = evict_block_smem(L) + 12 * 1024;  // + static
    int by_threads = 2;  // registers: see the kernel's launch bounds
    int by_smem = (int)((size_t)optin / sm);
    int b = by_threads < by_smem ? by_threads : by_smem;
    return b < 1 ? 1 : b;
}

cudaError_t launch_evict(const Layout& L, int l0, int l1, int grid, cudaStream_t st) {
    const int n_max = L.L;
    const int gw = evict_group_warps(L);
    const size_t sm = evict_block_smem(L);
    if (L.dtype == HKV_DTYPE_BF16)
        evict_block_kernel<__nv_bfloat16><<<grid, EVB_THREADS, sm, st>>>(L, l0, l1, n_max, gw);
    else
        evict_block_kernel<float><<<grid, EVB_THREADS, sm, st>>>(L, l0, l1, n_max, gw);
    return cudaGetLastError();
}

cudaError_t prepare_evict(int smem) {
    cudaError_t e = allow_max_dynamic_smem(evict_block_kernel<__nv_bfloat16>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(evict_block_kernel<float>, smem);
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
