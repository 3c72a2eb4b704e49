// hkv_internal.cuh -- device-side layout of the cache pool and helpers shared
// by the kernels of libhkv.  Everything here runs on sm_100a.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hkv.h"

namespace hkv {

constexpr unsigned FULL_MASK = 0xffffffffu;
constexpr float LOG2E = 1.4426950408889634f;
constexpr int CHUNK = 32;  // tokens one warp handles per decode work item
constexpr int PLAN_MAX_WARPS = 2048;  // capacity of a decode plan's warp table
constexpr int PLAN_WARP_DESC = 7;     // descriptors copied into each warp's plan block
constexpr int PLAN_DESC_PARTS = 4;    // blocks per layer of the plan kernel
constexpr int RANK_MAX = 32;          // strata up to this size are selected by ranking
// Costs in the plan's balancing of the warp ranges: a decode chunk costs
// CHUNK_COST, the end of a head's segment (reductions, output, a merge
// when split) HEAD_COST by default.  Per-warp timings of the decode launch
// put a head's end at about two thirds of a chunk on average; launch times
// are shortest with it weighted higher (the warps that end a launch are the
// ones with many head ends: 5 / 3 gave 2-5% shorter launches than 1 / 3 on
// the Lumina-mGPT-768 and LlamaGen-XL shapes).
constexpr int CHUNK_COST = 3;
constexpr int HEAD_COST = 5;
// Least cost of a warp's range (two chunks of one head): small layers use
// fewer warps rather than thinner ranges, and a small cache fewer blocks.
__host__ __device__ constexpr int min_range_cost(int head_cost) { return 2 * CHUNK_COST + head_cost; }
// Weights of a decode warp's share of a layer when a block's warps do not
// spread evenly over the SM's four sub-partitions (six warps: two share
// each of sub-partitions 0 and 1, two are alone on 2 and 3).  Per-warp
// timestamps of the decode launch on a d = 128 cache: 2.14 us per chunk
// for a warp alone, 2.33 for one that shares (about 12 : 11); launch times
// on the Lumina-mGPT-768 shape: 22.68 / 22.48 / 22.36 / 22.39 us at 11 /
// 12 / 13 / 14 against 11 (13 counts the warp's share of the block's end).
constexpr int SHARED_WEIGHT = 11;
constexpr int LONE_WEIGHT = 13;

// Everything a kernel needs to find the state of a (layer, sequence, head).
// The pool is one caller-owned device buffer carved into these regions.
struct Layout {
    int32_t S, Ly, H, d, L, W, M, D, r;
    int32_t H_total;    // heads of a whole (sequence, layer): H, or more when heads are sharded
    int32_t mode, stratified, dtype;
    int32_t nq;         // prefill queries whose per-distance weights group a head
    int32_t pairing;    // hkv_cfg_pairing: grouping tied across a CFG pair
    int32_t R;          // slots per (sequence, layer) region
    int64_t T_total;    // floor(H * L * rho): tokens one (sequence, layer) keeps
    double tau;
    // control words
    int32_t* status;    // [0] first error code, [1] detail
    int32_t* t_next;    // [Ly] position the next append writes
    int32_t* done_ctr;  // [Ly] CTA arrivals of the running decode launch
    unsigned long long* ev_stats;  // [3] heads evicted, tokens scored, rows moved
    // per (layer, sequence, head) metadata, index (l*S + s)*H + h
    int32_t* off;       // first slot of the head inside its region
    int32_t* cap;       // slots reserved for the head
    int32_t* budget;    // tokens kept after an eviction (W for Local heads)
    uint64_t* base;     // cache length at step t0 (low 32 bits) and t0 (high
                        // 32 bits): the length grows by one per step after t0;
                        // one 64-bit word, so a reader never sees half of an
                        // update (see base_pack / base_len_of / base_t_of)
    uint8_t* label;     // 1 Local, 0 Global, 2 full cache
    int32_t* n_tau;
    // per (layer, sequence): step at which its Global heads reach their cap
    // cache rows, slot index (l*S + s)*R + slot
    void* K;            // [Ly][S][R][2][d]: per slot its K row, then its V row
    void* V;            // K + d elements (same row stride 2 d)
    int32_t* pos;       // [Ly][S][R]
    float* logit;       // [Ly][S][R][r]   exp2-domain logits of scoring steps
    float2* ml;         // [Ly][S][H][r]   (max, sum) of those steps' softmax
    // scratch, reused by every call
    float* rows;        // [S*H][r][prefill_len] weights of the last r prefill queries
    float* partial;     // [2][PLAN_MAX_WARPS][2][d + 2] split-K partial states
    int32_t* ticket;    // [2][S*H] arrivals per head of the running decode launch
    // per (layer, sequence) "unit", index l*S + s: {x: the step at which its
    // Global heads reach their capacity (INT32_MAX: none; advanced by the
    // plan kernel after each eviction), y: the Global heads held here as a
    // bit mask (H <= 32), z: their budget, w: their capacity}.  The Global
    // heads of a unit share budget, capacity and length, and a head's first
    // slot follows from the mask (Local heads hold W slots, Global ones w).
    int4* unit;
    // decode plan per layer, for the step it was made for (see plan_kernel)
    int4* plan_desc;     // [Ly][max_chunks] one descriptor per chunk
    // [Ly][PLAN_MAX_WARPS][1 + PLAN_WARP_DESC]: per warp {first chunk, end
    // chunk, total, 0} and copies of its range's first descriptors
    int4* plan_warp;
    int32_t plan_gw;     // warps of one decode launch
    int32_t plan_nw;     // warps of one decode block
    int32_t plan_hc;     // cost of a head's end in the plan's balancing
    int32_t plan_lw;     // weight of a warp alone on its SM sub-partition
                         // (the others weigh SHARED_WEIGHT) in the plan
    int32_t max_chunks;
};

__host__ __device__ __forceinline__ uint64_t base_pack(int len, int t0) {
    return (uint64_t)(uint32_t)len | ((uint64_t)(uint32_t)t0 << 32);
}
__host__ __device__ __forceinline__ int base_len_of(uint64_t b) { return (int)(uint32_t)b; }
__host__ __device__ __forceinline__ int base_t_of(uint64_t b) { return (int)(uint32_t)(b >> 32); }

__device__ __forceinline__ size_t head_index(const Layout& L, int l, int s, int h) {
    return ((size_t)l * L.S + s) * L.H + h;
}
__device__ __forceinline__ size_t region_slot0(const Layout& L, int l, int s) {
    return ((size_t)l * L.S + s) * (size_t)L.R;
}

// Cache length of a head at step t: one token joins per step after its t0;
// a Local head's ring stops growing at its capacity W.
__device__ __forceinline__ int len_at(const Layout& L, size_t hi, int t) {
    const uint64_t b = L.base[hi];
    int n = base_len_of(b) + (t - base_t_of(b));
    if (L.label[hi] == 1 && n > L.cap[hi]) n = L.cap[hi];
    return n;
}

// Slot (within the head) that the token of position t occupies when appended.
__device__ __forceinline__ int append_slot_of(int label, int cap, int t, int len_after) {
    return label == 1 ? t % cap : len_after - 1;
}
__device__ __forceinline__ int append_slot(const Layout& L, size_t hi, int t, int len_after) {
    return append_slot_of(L.label[hi], L.cap[hi], t, len_after);
}

__device__ __forceinline__ void latch_error(const Layout& L, int code, int detail) {
    if (atomicCAS(L.status, 0, code) == 0) atomicExch(L.status + 1, detail);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_float(float& dst, float x) { dst = x; }
__device__ __forceinline__ void from_float(__nv_bfloat16& dst, float x) { dst = __float2bfloat16_rn(x); }

// ---------------------------------------------------------------------------
// Warp-level bottom-k selection (Stratified Token Eviction).
//
// keys[i] = (bits(score) << 32) | position, score >= +0 so the bit pattern
// orders like the value; the total order is (score, position), i.e. equal
// scores evict the lower position first.  The k lowest keys of a stratum
// are found by ranking (at most RANK_MAX keys), by a register-resident
// 4-ary search on the score bits (at most 256 keys), or by an MSB-first
// radix select on the score bits (four 8-bit digits, a shared-memory
// histogram per digit); the two searches resolve a score tie at the
// boundary by bisection on positions.  Every key <= the threshold found is
// evicted.
// ---------------------------------------------------------------------------
struct KthSearch {
    const uint64_t* keys;
    int m, k;          // set size, rank wanted (1 <= k < m)
    uint32_t lo;       // score bits of the k-th smallest
    uint64_t thr;      // result
};

// Resolves the position tie at score bits s.lo and sets s.thr.
__device__ __forceinline__ void kth_finish(KthSearch& s) {
    const int lane = threadIdx.x & 31;
    const uint32_t s_star = s.lo;
    unsigned c_lt = 0, c_eq = 0;
    uint32_t plo = 0xffffffffu, phi = 0u;
    for (int i = lane; i < s.m; i += 32) {
        const uint32_t sb = (uint32_t)(s.keys[i] >> 32);
        const uint32_t p = (uint32_t)s.keys[i];
        c_lt += sb < s_star;
        if (sb == s_star) { ++c_eq; plo = min(plo, p); phi = max(phi, p); }
    }
    c_lt = __reduce_add_sync(FULL_MASK, c_lt);
    c_eq = __reduce_add_sync(FULL_MASK, c_eq);
    plo = __reduce_min_sync(FULL_MASK, plo);
    phi = __reduce_max_sync(FULL_MASK, phi);
    const int need = s.k - (int)c_lt;  // 1 <= need <= c_eq
    if (need < (int)c_eq) {
        while (plo < phi) {
            const uint32_t mid = plo + ((phi - plo) >> 1);
            unsigned c = 0;
            for (int i = lane; i < s.m; i += 32)
                c += ((uint32_t)(s.keys[i] >> 32) == s_star) && ((uint32_t)s.keys[i] <= mid);
            c = __reduce_add_sync(FULL_MASK, c);
            if ((int)c >= need) phi = mid; else plo = mid + 1;
        }
    } else {
        plo = phi;  // every tied key goes
    }
    s.thr = ((uint64_t)s_star << 32) | plo;
}

// Score bits of the k-th smallest key (1 <= k <= m): four passes, each
// histogramming the next 8-bit digit of the keys that match the digits
// chosen so far (one shared-memory atomic per distinct digit per 32 keys)
// and choosing the digit whose cumulative count reaches the wanted rank.
__device__ inline uint32_t warp_radix_kth_score(const uint64_t* keys, int m, int k, uint32_t* hist) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, pmask = 0;
    int want = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
        for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0u;
        __syncwarp();
        for (int i0 = 0; i0 < m; i0 += 32) {
            const int i = i0 + lane;
            const uint32_t sb = i < m ? (uint32_t)(keys[i] >> 32) : 0u;
            const bool in = i < m && (sb & pmask) == prefix;
            const uint32_t dg = in ? (sb >> shift) & 255u : 256u;
            const unsigned same = __match_any_sync(FULL_MASK, dg);
            if (in && (__ffs(same) - 1) == lane) atomicAdd(&hist[dg], (uint32_t)__popc(same));
        }
        __syncwarp();
        uint32_t c[8], sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) { c[j] = hist[lane * 8 + j]; sum += c[j]; }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(FULL_MASK, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - sum;
        const bool mine = excl < (uint32_t)want && (uint32_t)want <= incl;
        const unsigned bm = __ballot_sync(FULL_MASK, mine);
        int digit = 0, below = 0;
        if (mine) {
            uint32_t run = excl;
            bool found = false;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (!found && run + c[j] >= (uint32_t)want) { digit = lane * 8 + j; below = (int)run; found = true; }
                run += c[j];
            }
        }
        const int src = bm ? __ffs(bm) - 1 : 0;
        digit = __shfl_sync(FULL_MASK, digit, src);
        below = __shfl_sync(FULL_MASK, below, src);
        want -= below;
        prefix |= (uint32_t)digit << shift;
        pmask |= 255u << shift;
        __syncwarp();  // every lane has read the histogram
    }
    return prefix;
}

// 64-bit load from a shared-memory address.
__device__ __forceinline__ uint64_t lds_u64(uint32_t addr) {
    uint64_t v;
    asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(addr));
    return v;
}

// Marks the k lowest of m <= 32 * U distinct keys: lane l ranks keys
// l, l + 32, ... (held in registers) against every key in one pass of
// shared-memory broadcast reads; rank < k is exactly the k lowest.

template <int U>
__device__ inline void warp_rank_evict(const uint64_t* keys, const uint16_t* slots, int m, int k,
                                       uint32_t* evict_bits) {
    const int lane = threadIdx.x & 31;
    const uint32_t kbase = (uint32_t)__cvta_generic_to_shared(keys);  // keys live in shared memory
    uint64_t mine[U];
    int rk[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int i = lane + 32 * u;
        mine[u] = i < m ? lds_u64(kbase + 8 * i) : ~0ull;
        rk[u] = 0;
    }
    int j = 0;
    for (; j + 8 <= m; j += 8) {  // eight broadcast reads in flight
        uint64_t kj[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) kj[v] = lds_u64(kbase + 8 * (j + v));
#pragma unroll
        for (int v = 0; v < 8; ++v)
#pragma unroll
            for (int u = 0; u < U; ++u) rk[u] += kj[v] < mine[u];
    }
    for (; j < m; ++j) {
        const uint64_t kj = lds_u64(kbase + 8 * j);
#pragma unroll
        for (int u = 0; u < U; ++u) rk[u] += kj < mine[u];
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int i = lane + 32 * u;
        if (i < m && rk[u] < k) atomicOr(&evict_bits[slots[i] >> 5], 1u << (slots[i] & 31));
    }
}

// Thresholds of two strata at once, with each lane's keys in registers
// (stratum a: keys l, l + 32, ... of a set of ma; likewise b), for 1 <= k < m
// in each active stratum: a 4-ary search on the score bits (three pivots
// per round, counts by warp reductions), then the position tie at the
// boundary.  Every key <= the returned threshold is evicted.  Lanes hold
// ~0 for absent keys (scores are >= +0, so their bits stay below 2^31).
template <int U>
__device__ inline void warp_kth_regs2(const uint64_t (&ka)[U], int ka_k, bool a_on,
                                      const uint64_t (&kb)[U], int kb_k, bool b_on,
                                      uint64_t& thr_a, uint64_t& thr_b) {
    uint32_t alo = 0xffffffffu, ahi = 0u, blo = 0xffffffffu, bhi = 0u;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const uint32_t sa = (uint32_t)(ka[u] >> 32), sb = (uint32_t)(kb[u] >> 32);
        if (ka[u] != ~0ull) { alo = min(alo, sa); ahi = max(ahi, sa); }
        if (kb[u] != ~0ull) { blo = min(blo, sb); bhi = max(bhi, sb); }
    }
    alo = __reduce_min_sync(FULL_MASK, alo);
    ahi = __reduce_max_sync(FULL_MASK, ahi);
    blo = __reduce_min_sync(FULL_MASK, blo);
    bhi = __reduce_max_sync(FULL_MASK, bhi);
    if (!a_on) alo = ahi = 0;
    if (!b_on) blo = bhi = 0;
    while (alo < ahi || blo < bhi) {
        const uint32_t a1 = alo + ((ahi - alo) >> 2), a2 = alo + ((ahi - alo) >> 1),
                       a3 = alo + (uint32_t)(((uint64_t)(ahi - alo) * 3) >> 2);
        const uint32_t b1 = blo + ((bhi - blo) >> 2), b2 = blo + ((bhi - blo) >> 1),
                       b3 = blo + (uint32_t)(((uint64_t)(bhi - blo) * 3) >> 2);
        unsigned ca1 = 0, ca2 = 0, ca3 = 0, cb1 = 0, cb2 = 0, cb3 = 0;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t sa = (uint32_t)(ka[u] >> 32), sb = (uint32_t)(kb[u] >> 32);
            ca1 += sa <= a1; ca2 += sa <= a2; ca3 += sa <= a3;
            cb1 += sb <= b1; cb2 += sb <= b2; cb3 += sb <= b3;
        }
        ca1 = __reduce_add_sync(FULL_MASK, ca1);
        ca2 = __reduce_add_sync(FULL_MASK, ca2);
        ca3 = __reduce_add_sync(FULL_MASK, ca3);
        cb1 = __reduce_add_sync(FULL_MASK, cb1);
        cb2 = __reduce_add_sync(FULL_MASK, cb2);
        cb3 = __reduce_add_sync(FULL_MASK, cb3);
        if (alo < ahi) {
            if ((int)ca1 >= ka_k) ahi = a1;
            else if ((int)ca2 >= ka_k) { alo = a1 + 1; ahi = a2; }
            else if ((int)ca3 >= ka_k) { alo = a2 + 1; ahi = a3; }
            else alo = a3 + 1;
        }
        if (blo < bhi) {
            if ((int)cb1 >= kb_k) bhi = b1;
            else if ((int)cb2 >= kb_k) { blo = b1 + 1; bhi = b2; }
            else if ((int)cb3 >= kb_k) { blo = b2 + 1; bhi = b3; }
            else blo = b3 + 1;
        }
    }
    // the position tie at the boundary score s* of each stratum: need =
    // k - (keys below s*) of the tied keys go, lowest positions first
    auto finish = [&](const uint64_t (&kk)[U], int k, uint32_t sstar) -> uint64_t {
        unsigned c_lt = 0, c_eq = 0;
        uint32_t plo = 0xffffffffu, phi = 0u;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t sc = (uint32_t)(kk[u] >> 32), p = (uint32_t)kk[u];
            if (kk[u] == ~0ull) continue;
            c_lt += sc < sstar;
            if (sc == sstar) { ++c_eq; plo = min(plo, p); phi = max(phi, p); }
        }
        c_lt = __reduce_add_sync(FULL_MASK, c_lt);
        c_eq = __reduce_add_sync(FULL_MASK, c_eq);
        plo = __reduce_min_sync(FULL_MASK, plo);
        phi = __reduce_max_sync(FULL_MASK, phi);
        const int need = k - (int)c_lt;  // 1 <= need <= c_eq
        if (need < (int)c_eq) {
            while (plo < phi) {
                const uint32_t mid = plo + ((phi - plo) >> 1);
                unsigned c = 0;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    c += kk[u] != ~0ull && (uint32_t)(kk[u] >> 32) == sstar && (uint32_t)kk[u] <= mid;
                c = __reduce_add_sync(FULL_MASK, c);
                if ((int)c >= need) phi = mid; else plo = mid + 1;
            }
        } else {
            plo = phi;  // every tied key goes
        }
        return ((uint64_t)sstar << 32) | plo;
    };
    thr_a = a_on ? finish(ka, ka_k, alo) : 0ull;
    thr_b = b_on ? finish(kb, kb_k, blo) : 0ull;
}

// Both strata (at most 32 * U keys each) selected by warp_kth_regs2: keys
// read once into registers, evict bits set from the thresholds.
template <int U>
__device__ inline void warp_select_regs(const uint64_t* keys_a, const uint16_t* slots_a, int ma, int ka_k,
                                        const uint64_t* keys_b, const uint16_t* slots_b, int mb, int kb_k,
                                        uint32_t* evict_bits) {
    const int lane = threadIdx.x & 31;
    uint64_t ka[U], kb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int i = lane + 32 * u;
        ka[u] = i < ma ? keys_a[i] : ~0ull;
        kb[u] = i < mb ? keys_b[i] : ~0ull;
    }
    const bool a_on = ka_k > 0 && ka_k < ma, b_on = kb_k > 0 && kb_k < mb;
    uint64_t ta = 0, tb = 0;
    warp_kth_regs2<U>(ka, ka_k, a_on, kb, kb_k, b_on, ta, tb);
    if (ka_k >= ma) ta = ~0ull;  // the whole stratum goes
    if (kb_k >= mb) tb = ~0ull;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int i = lane + 32 * u;
        if (i < ma && ka_k > 0 && ka[u] <= ta) atomicOr(&evict_bits[slots_a[i] >> 5], 1u << (slots_a[i] & 31));
        if (i < mb && kb_k > 0 && kb[u] <= tb) atomicOr(&evict_bits[slots_b[i] >> 5], 1u << (slots_b[i] & 31));
    }
}

// Scratch of one warp's stratified select over up to n_max tokens.  The
// near keys fill keys[] from the front and the far keys from the back; the
// same for slot[] and for the hole / mover lists of the compaction.
struct SelectScratch {
    uint64_t* keys;        // [n_max]
    uint32_t* hist;        // [256] digit histogram of the radix select
    uint16_t* slot;        // [n_max]
    uint32_t* evict_bits;  // [n_max / 32]
    uint16_t* moves;       // [n_max]: holes from the front, movers from the back
    int n_max;
};

__host__ __device__ inline int round32(int n) { return (n + 31) / 32 * 32; }

__host__ __device__ inline size_t select_scratch_bytes(int n_max) {
    size_t n = (size_t)round32(n_max);
    return (n * 8 + 1024 + n * 2 + (n / 32) * 4 + n * 2 + 15) / 16 * 16;  // 16-byte multiple
}

__device__ inline SelectScratch carve_select_scratch(unsigned char* base, int n_max) {
    const int n = round32(n_max);
    SelectScratch s;
    s.keys = reinterpret_cast<uint64_t*>(base);
    s.hist = reinterpret_cast<uint32_t*>(s.keys + n);
    s.slot = reinterpret_cast<uint16_t*>(s.hist + 256);
    s.evict_bits = reinterpret_cast<uint32_t*>(s.slot + n);
    s.moves = reinterpret_cast<uint16_t*>(s.evict_bits + n / 32);
    s.n_max = n;
    return s;
}

// One batch of 32 tokens (token base + lane) into the strata: near keys
// fill keys[] from the front, far keys from the back (nn, nf: counts so far,
// updated); the batch's evict-bit word is cleared.  All lanes call it.
__device__ __forceinline__ void warp_partition_batch(const SelectScratch& sc, int n, int t, int D,
                                                     int stratified, int base, bool valid,
                                                     uint32_t sb, int32_t p, int& nn, int& nf) {
    const int lane = threadIdx.x & 31;
    const int i = base + lane;
    bool is_near = false, is_far = false;
    const uint64_t key = ((uint64_t)sb << 32) | (uint32_t)p;
    if (valid) {
        const int delta = t - p;
        if (delta >= 1) {
            if (stratified && delta <= D) is_near = true; else is_far = true;
        }
    }
    const unsigned bn = __ballot_sync(FULL_MASK, is_near);
    const unsigned bf = __ballot_sync(FULL_MASK, is_far);
    const unsigned lt = (1u << lane) - 1u;
    if (is_near) {
        const int o = nn + __popc(bn & lt);
        sc.keys[o] = key;
        sc.slot[o] = (uint16_t)i;
    }
    if (is_far) {
        const int o = n - 1 - (nf + __popc(bf & lt));
        sc.keys[o] = key;
        sc.slot[o] = (uint16_t)i;
    }
    nn += __popc(bn);
    nf += __popc(bf);
    if (lane == 0) sc.evict_bits[base >> 5] = 0u;
}

__device__ int warp_select_partitioned(const SelectScratch& sc, int n, int nn, int nf, int k_near,
                                       int k_far, int stratified);

// Stratified select over tokens 0..n) whose keys a functor provides:
// key_of(i, score_bits, pos).  Candidates: t - pos >= 1; near: t - pos <= D
// (every candidate is "far" when !stratified).  k_near / k_far lowest keys
// of each stratum are evicted, a stratum short of candidates handing its
// shortfall to the other.  Sets evict_bits; returns the number evicted.
// All 32 lanes call it; n <= 65535.
template <typename KeyOf>
__device__ int warp_stratified_select(const SelectScratch& sc, int n, int t, int D, int k_near,
                                      int k_far, int stratified, KeyOf key_of) {
    const int lane = threadIdx.x & 31;
    int nn = 0, nf = 0;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        uint32_t sb = 0;
        int32_t p = 0;
        if (i < n) key_of(i, sb, p);
        warp_partition_batch(sc, n, t, D, stratified, base, i < n, sb, p, nn, nf);
    }
    __syncwarp();
    return warp_select_partitioned(sc, n, nn, nf, k_near, k_far, stratified);
}

// The selection once the strata are partitioned (nn near keys at the
// front of keys[], nf far keys at the back, evict bits cleared).
__device__ inline int warp_select_partitioned(const SelectScratch& sc, int n, int nn, int nf, int k_near,
                                              int k_far, int stratified) {
    const int lane = threadIdx.x & 31;
    int kn = k_near, kf = k_far;
    if (stratified) {
        if (kn > nn) { kf += kn - nn; kn = nn; }
        if (kf > nf) { kn += kf - nf; kf = nf; if (kn > nn) kn = nn; }
    } else {
        kf = k_near + k_far;
        kn = 0;
        if (kf > nf) kf = nf;
    }
    // Both strata of at most 256 keys, one of them over RANK_MAX: keys in
    // registers, thresholds by a joint 4-ary search.
    const int mm = max(nn, nf);
    if (mm > RANK_MAX && mm <= 256) {
        const uint64_t* kf_keys = sc.keys + (n - nf);
        const uint16_t* kf_slots = sc.slot + (n - nf);
        if (mm <= 64) warp_select_regs<2>(sc.keys, sc.slot, nn, kn, kf_keys, kf_slots, nf, kf, sc.evict_bits);
        else if (mm <= 128) warp_select_regs<4>(sc.keys, sc.slot, nn, kn, kf_keys, kf_slots, nf, kf, sc.evict_bits);
        else warp_select_regs<8>(sc.keys, sc.slot, nn, kn, kf_keys, kf_slots, nf, kf, sc.evict_bits);
        __syncwarp();
        return kn + kf;
    }
    // Otherwise each stratum alone: at most RANK_MAX keys by ranking every
    // key against all keys of its stratum (keys are distinct, so rank < k is
    // exactly the k lowest); larger by the radix select; none evicted
    // (k <= 0), all evicted (k >= m).
    for (int which = 0; which < 2; ++which) {
        const int k = which == 0 ? kn : kf;
        const int m = which == 0 ? nn : nf;
        const uint64_t* keys = which == 0 ? sc.keys : sc.keys + (n - nf);
        const uint16_t* slots = which == 0 ? sc.slot : sc.slot + (n - nf);
        if (k <= 0) continue;
        const bool by_rank = k < m && m <= RANK_MAX;
        uint64_t thr = ~0ull;
        if (k < m && !by_rank) {
            KthSearch q{keys, m, k, warp_radix_kth_score(keys, m, k, sc.hist), 0};
            kth_finish(q);
            thr = q.thr;
        }
        if (by_rank) {
            if (m <= 64) warp_rank_evict<2>(keys, slots, m, k, sc.evict_bits);
            else if (m <= 128) warp_rank_evict<4>(keys, slots, m, k, sc.evict_bits);
            else warp_rank_evict<8>(keys, slots, m, k, sc.evict_bits);
        } else {
            for (int i = lane; i < m; i += 32)
                if (keys[i] <= thr) atomicOr(&sc.evict_bits[slots[i] >> 5], 1u << (slots[i] & 31));
        }
    }
    __syncwarp();
    return kn + kf;
}

// Backward accumulation of the head-grouping rule on one weight row
// (row[j] = weight of the query at position n-1 on position j): the number
// of tokens, newest first, whose weights first sum to >= tau (n if never).
// Double-precision running sum.  All lanes call it; all get the answer.
__device__ __forceinline__ int warp_tokens_to_tau(const float* row, int n, double tau) {
    const int lane = threadIdx.x & 31;
    double carry = 0.0;
    for (int base = 0; base < n; base += 32) {
        const int delta = base + lane;
        double x = delta < n ? (double)row[n - 1 - delta] : 0.0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(FULL_MASK, x, o);
            if (lane >= o) x += y;
        }
        const double c = carry + x;
        const unsigned hit = __ballot_sync(FULL_MASK, delta < n && c >= tau);
        if (hit) return base + __ffs(hit);  // delta = 0 .. first hit
        carry += __shfl_sync(FULL_MASK, x, 31);
    }
    return n;
}

// Head grouping over kept weight rows (Methodology step 2, with the
// averaged and tied variants).  ra and rb (nullable) are [r][n] blocks of
// fp32 weights, row q holding the query at position n - r + q over
// positions 0..n-1.  The weight at distance delta is the mean over the last
// nq queries i of row i's weight on position i - delta (none when
// delta > i), per block; with rb, the mean of the two blocks' values.  Each
// block's sum runs over the queries in position order and is divided by
// nq, the pair's mean is halved after, all in double.  Summed newest first
// until the total reaches tau.  All lanes of the warp call it and get the
// number of tokens that took (n if never).
__device__ __forceinline__ int warp_group_need_rows(const float* ra, const float* rb, int r,
                                                    int nq, int n, double tau) {
    const int lane = threadIdx.x & 31;
    double carry = 0.0;
    for (int base = 0; base < n; base += 32) {
        const int delta = base + lane;
        double x = 0.0;
        if (delta < n) {
            double xa = 0.0, xb = 0.0;
            for (int q = r - nq; q < r; ++q) {
                const int i = n - r + q;
                if (delta <= i) {
                    xa += (double)ra[(size_t)q * n + (i - delta)];
                    if (rb) xb += (double)rb[(size_t)q * n + (i - delta)];
                }
            }
            x = rb ? (xa / nq + xb / nq) * 0.5 : xa / nq;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(FULL_MASK, x, o);
            if (lane >= o) x += y;
        }
        const double c = carry + x;
        const unsigned hit = __ballot_sync(FULL_MASK, delta < n && c >= tau);
        if (hit) return base + __ffs(hit);  // delta = 0 .. first hit
        carry += __shfl_sync(FULL_MASK, x, 31);
    }
    return n;
}

// Allows `func` as much dynamic shared memory as the device's opt-in limit
// leaves next to its static shared memory, and asks for the largest shared
// memory carve-out: the kernels of a decode step then all run under the same
// L1 / shared split, and an SM does not repartition between them.
template <typename F>
inline cudaError_t allow_max_dynamic_smem(F* func, int optin) {
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, func);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - (int)a.sharedSizeBytes);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout,
                                (int)cudaSharedmemCarveoutMaxShared);
}

}  // namespace hkv
