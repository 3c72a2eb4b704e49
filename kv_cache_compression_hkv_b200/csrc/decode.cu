// decode.cu -- per-step cache append and decode attention over the ragged,
// head-aware compressed cache (HeadKV technical summary: Problem statement;
// Methodology step 3, Local sliding window and Global STE scoring).
//
// Work decomposition: every head's cache is cut into chunks of 32 tokens.
// A plan (plan_kernel, once per step and layer) prefix-sums the heads' chunk
// counts, writes one descriptor per chunk and cuts the layer's chunk list
// into equal contiguous ranges, one per warp of the persistent decode grid.
// Each warp walks its range with a pipeline of shared-memory stages filled
// by bulk copies (TMA engine) and keeps the online softmax of the current
// head in registers across that head's chunks; it finishes a head it holds
// entirely, and a head split between warps leaves one partial per warp, the
// last to arrive (atomic ticket, no spinning) merging them.  Global heads
// within r steps of their eviction also store their exp2-domain logits per
// slot, which the eviction normalises with the (max, sum) stored here.
#include <math.h>
#include <stdlib.h>

#include <cuda/atomic>

#include "hkv_internal.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace hkv {

// Headroom (log2 units) a logit may exceed the running softmax reference by
// before the reference is raised: weights stay below 2^8, far from fp32 range.
constexpr float RESCALE = 8.f;
// Most pipeline stages a decode warp keeps in flight.
constexpr int MAX_STAGES = 4;
// Most warps of one decode block (one block per SM).
constexpr int DECODE_MAX_WARPS = 12;

// Most chunks a range starting a decode block moves to avoid cutting a head.
constexpr int SNAP_MAX = 2;


// Packed storage of DPL consecutive elements of one row.
template <typename T, int DPL> struct Raw;
template <int DPL> struct Raw<__nv_bfloat16, DPL> {
    static constexpr int W = DPL / 2;
    uint32_t w[W];
    __device__ __forceinline__ void load(const __nv_bfloat16* p) {
        if constexpr (W == 2) { uint2 v = __ldg(reinterpret_cast<const uint2*>(p)); w[0] = v.x; w[1] = v.y; }
        else if constexpr (W == 1) { w[0] = __ldg(reinterpret_cast<const unsigned int*>(p)); }
        else {
#pragma unroll
            for (int i = 0; i < W; ++i) w[i] = __ldg(reinterpret_cast<const unsigned int*>(p) + i);
        }
    }
    __device__ __forceinline__ void load_shared(const __nv_bfloat16* p) {
        if constexpr (W == 2) { uint2 v = *reinterpret_cast<const uint2*>(p); w[0] = v.x; w[1] = v.y; }
        else if constexpr (W == 1) { w[0] = *reinterpret_cast<const unsigned int*>(p); }
        else {
#pragma unroll
            for (int i = 0; i < W; ++i) w[i] = reinterpret_cast<const unsigned int*>(p)[i];
        }
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < W; ++i) w[i] = 0;
    }
    __device__ __forceinline__ float get(int i) const { return (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]); }
    __device__ __forceinline__ void store(__nv_bfloat16* p) const {
        if constexpr (W == 2) *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
        else if constexpr (W == 1) *reinterpret_cast<unsigned int*>(p) = w[0];
        else {
#pragma unroll
            for (int i = 0; i < W; ++i) reinterpret_cast<unsigned int*>(p)[i] = w[i];
        }
    }
};
template <int DPL> struct Raw<float, DPL> {
    float w[DPL];
    __device__ __forceinline__ void load(const float* p) {
        if constexpr (DPL == 4) { float4 v = __ldg(reinterpret_cast<const float4*>(p)); w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w; }
        else if constexpr (DPL == 2) { float2 v = __ldg(reinterpret_cast<const float2*>(p)); w[0] = v.x; w[1] = v.y; }
        else {
#pragma unroll
            for (int i = 0; i < DPL; ++i) w[i] = __ldg(p + i);
        }
    }
    __device__ __forceinline__ void load_shared(const float* p) {
        if constexpr (DPL == 4) { float4 v = *reinterpret_cast<const float4*>(p); w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w; }
        else if constexpr (DPL == 2) { float2 v = *reinterpret_cast<const float2*>(p); w[0] = v.x; w[1] = v.y; }
        else {
#pragma unroll
            for (int i = 0; i < DPL; ++i) w[i] = p[i];
        }
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < DPL; ++i) w[i] = 0.f;
    }
    __device__ __forceinline__ float get(int i) const { return w[i]; }
    __device__ __forceinline__ void store(float* p) const {
#pragma unroll
        for (int i = 0; i < DPL; ++i) p[i] = w[i];
    }
};

// Stores DPL floats as the row's element type (bf16 pairs packed).
template <typename T, int DPL>
__device__ __forceinline__ void store_row(T* p, const float (&x)[DPL]) {
    if constexpr (sizeof(T) == 2) {
        uint32_t w[DPL / 2];
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i) {
            __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&b);
        }
        if constexpr (DPL == 8) *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
        else if constexpr (DPL == 4) *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
        else if constexpr (DPL == 2) *reinterpret_cast<uint32_t*>(p) = w[0];
        else {
#pragma unroll
            for (int i = 0; i < DPL / 2; ++i) reinterpret_cast<uint32_t*>(p)[i] = w[i];
        }
    } else if constexpr (DPL == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) reinterpret_cast<float*>(p)[i] = x[i];
    }
}

// ---------------------------------------------------------------------------
// Chunk descriptors.  The plan describes every chunk of a layer in one int4:
//   x: layer-relative row of the chunk's first token
//   y: head (s * H + h)
//   z: rows n (bits 0-5) | appended row + 1 (bits 6-11, 0: none) | first
//      chunk of its head (bit 12) | last chunk (bit 13) | scoring head
//      (bit 14) | non-empty warp ranges holding the head (bits 16-31)
//   w: first warp range holding the head | (last - first) << 12
// ---------------------------------------------------------------------------
struct ChunkDesc {
    int row, head, n, a, first, last, scoring, segs, wa, wb;
    __device__ __forceinline__ static ChunkDesc of(const int4& v) {
        ChunkDesc c;
        c.row = v.x;
        c.head = v.y;
        c.n = v.z & 63;
        c.a = ((v.z >> 6) & 63) - 1;
        c.first = (v.z >> 12) & 1;
        c.last = (v.z >> 13) & 1;
        c.scoring = (v.z >> 14) & 1;
        c.segs = (int)((uint32_t)v.z >> 16);
        c.wa = v.w & 0xfff;
        c.wb = c.wa + (v.w >> 12);
        return c;
    }
};

__device__ __forceinline__ int4 shfl_int4(const int4& v, int src) {
    return make_int4(__shfl_sync(FULL_MASK, v.x, src), __shfl_sync(FULL_MASK, v.y, src),
                     __shfl_sync(FULL_MASK, v.z, src), __shfl_sync(FULL_MASK, v.w, src));
}

// Warp ranges over the chunk list (see plan_kernel): the warps w whose
// boundary falls in head i's cost interval start in head i, at the first of
// its chunks whose cost starts at or after the boundary.  Equal shares: the
// boundary of warp w is w * tcost / GWe.  U: an unsigned type that holds
// tcost * (GWe + 1).
template <typename U>
__device__ __forceinline__ void cut_ranges(const int32_t* cnt, int n, int HC, U tcost, int GWe,
                                           int32_t* wbeg, int32_t* whead) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int c0 = i ? cnt[i - 1] : 0, c1 = cnt[i];
        const U e0 = (U)CHUNK_COST * (U)c0 + (U)HC * (U)i;
        const U e1 = (U)CHUNK_COST * (U)c1 + (U)HC * (U)(i + 1);
        const int w_lo = (int)((e0 * (U)GWe + tcost - 1) / tcost);
        const int w_hi = min((int)((e1 * (U)GWe + tcost - 1) / tcost), GWe);  // exclusive
        for (int w = w_lo; w < w_hi; ++w) {
            const U bnd = (U)w * tcost / (U)GWe;
            // chunks of head i whose cost starts before the boundary
            const int k = bnd > e0 ? (int)((bnd - e0 + CHUNK_COST - 1) / CHUNK_COST) : 0;
            wbeg[w] = c0 + min(k, c1 - c0);
            whead[w] = i;
        }
    }
}

// Weighted shares: warp k of a block (NW warps) weighs wt[k]; warp w =
// b NW + k starts at unit u(w) = b S + pre[k] of U = (GW / NW) S units
// (S = the block's total weight, pre = the prefix of wt), i.e. at cost
// u(w) tcost / U.  The heads' cost intervals, scaled to units, cut [0, U)
// into consecutive pieces, so every warp gets exactly one start.  V: an
// unsigned type that holds tcost * (U + 1).
template <typename V>
__device__ __forceinline__ void cut_ranges_weighted(const int32_t* cnt, int n, int HC, V tcost, V U,
                                                    int NW, const int* pre, int32_t* wbeg,
                                                    int32_t* whead) {
    const int S = pre[NW];
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int c0 = i ? cnt[i - 1] : 0, c1 = cnt[i];
        const V e0 = (V)CHUNK_COST * (V)c0 + (V)HC * (V)i;
        const V e1 = (V)CHUNK_COST * (V)c1 + (V)HC * (V)(i + 1);
        const V x_lo = (e0 * U + tcost - 1) / tcost;  // first unit whose cost is >= e0
        const V x_hi = min((e1 * U + tcost - 1) / tcost, U);
        if (x_lo >= x_hi) continue;
        int b = (int)(x_lo / (V)S), k = 0;
        const int r = (int)(x_lo - (V)b * (V)S);
        while (k < NW && pre[k] < r) ++k;
        if (k == NW) { ++b; k = 0; }
        for (;;) {
            const V u = (V)b * (V)S + (V)pre[k];
            if (u >= x_hi) break;
            const int w = b * NW + k;
            const V bnd = u * tcost / U;
            const int kk = bnd > e0 ? (int)((bnd - e0 + CHUNK_COST - 1) / CHUNK_COST) : 0;
            wbeg[w] = c0 + min(kk, c1 - c0);
            whead[w] = i;
            if (++k == NW) { ++b; k = 0; }
        }
    }
}

// ---------------------------------------------------------------------------
// The plan of a layer's decode launch at step t (ahead = 1: the step of the
// next append, t_next; ahead = 0: the newest cached position, t_next - 1).
// Blocks (layer, part): every block computes the layer's per-head facts,
// the chunk-count prefix and the warp ranges in shared memory; part p then
// writes the descriptors of the p-th slice of the chunks and the records of
// the p-th slice of the warps (each warp: its range and copies of the first
// PLAN_WARP_DESC descriptors of its range).
// ---------------------------------------------------------------------------
// With commit (the launch right after an eviction at step t_next - 1), the
// Global heads that were due at that step get their new length first (the
// budget, from that step on) and each unit its next due step; part 0 writes
// them, every part plans with them.
//
// With after_evict, the launch may start while the eviction kernel ahead of
// it still moves rows (programmatic dependent launch; the plan reads none of
// what the eviction writes); it completes only after that kernel, so a
// decode launch that waits for the plan sees the compacted cache too.
__global__ void __launch_bounds__(1024) plan_kernel(Layout L, int l0, int ahead, int commit,
                                                    int after_evict) {
    extern __shared__ int32_t psm[];
    __shared__ int wsum[32];
    const int layer = l0 + blockIdx.x;
    const int n = L.S * L.H;
    int32_t* cnt = psm;            // chunk counts, then their inclusive prefix
    int32_t* hslot = psm + n;      // layer-relative row of the head's first token
    int32_t* hlen = psm + 2 * n;   // len << 16 | appended slot
    int32_t* hscore = psm + 3 * n; // scoring flag
    const int GW = L.plan_gw;
    int32_t* wbeg = psm + 4 * n;   // [GW + 1] first chunk of each warp's range
    int32_t* whead = wbeg + PLAN_MAX_WARPS + 1;  // [GW] the head holding that chunk
    uint16_t* own = reinterpret_cast<uint16_t*>(whead + PLAN_MAX_WARPS);  // [total] warp of each chunk
    const int parts = gridDim.y, part = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, NW = blockDim.x >> 5;
    // per-warp weights of a decode block (see the range cutting below)
    __shared__ int pre[DECODE_MAX_WARPS + 1];
    const int NWb = L.plan_nw;
    const bool uneven = NWb > 0 && NWb <= DECODE_MAX_WARPS && L.plan_gw % NWb == 0 &&
                        L.plan_lw != SHARED_WEIGHT && NWb >= 4 && NWb % 4 != 0;
    if (tid == 0 && uneven) {
        int per[4] = {0, 0, 0, 0}, top = 0;
        for (int k = 0; k < NWb; ++k) ++per[k & 3];
        for (int q = 0; q < 4; ++q) top = max(top, per[q]);
        pre[0] = 0;
        for (int k = 0; k < NWb; ++k) pre[k + 1] = pre[k] + (per[k & 3] < top ? L.plan_lw : SHARED_WEIGHT);
    }
    // block (0, 0) completes only after the eviction kernel ahead of it
    struct AfterEvict {
        bool on;
        __device__ ~AfterEvict() {
            if (on) ptx::grid_dep_wait();
        }
    } after{after_evict && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0};
    const int te = L.t_next[layer] - 1;  // newest cached position
    const int t = te + ahead;
    const size_t hbase = (size_t)layer * n;
    const bool complete = t >= L.L;  // the sequence is complete: no step left to plan
    for (int i = tid; i < n; i += blockDim.x) {
        const size_t hx = hbase + i;
        const int cap = L.cap[hx];
        const int lab = L.label[hx];
        const uint64_t b = L.base[hx];
        int bl = base_len_of(b), bt = base_t_of(b);
        if (commit && lab == 0 && L.mode != HKV_MODE_FULL) {
            // a head evicted at te: length = budget from te on (part 0 writes
            // it; another part may read either pair: the same length), due
            // again M steps later (written once per unit)
            if (bl + (te - bt) >= cap) {
                bl = L.budget[hx];
                bt = te;
                if (part == 0) L.base[hx] = base_pack(bl, bt);
            }
            if (part == 0) {
                int4* ur = L.unit + (size_t)layer * L.S + i / L.H;
                const uint32_t gm = (uint32_t)ur->y;
                if (gm && (i % L.H) == __ffs(gm) - 1) ur->x = bt + (cap - bl);
            }
        }
        if (complete) continue;
        int len = bl + (t - bt);
        if (lab == 1 && len > cap) len = cap;
        int c = (len + CHUNK - 1) / CHUNK;
        if (len > cap || len < 1) {
            if (part == 0) latch_error(L, HKV_ERR_CAPACITY, (int)hx);
            c = 0;
        }
        const int jn = append_slot_of(lab, cap, t, len);
        hscore[i] = lab == 0 && L.mode != HKV_MODE_FULL && len > cap - L.r;
        hslot[i] = (i / L.H) * L.R + L.off[hx];
        hlen[i] = (len << 16) | (jn & 0xffff);
        cnt[i] = c;
    }
    if (complete) return;
    __syncthreads();
    // inclusive scan: contiguous runs per thread, then the warps
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int i0 = min(tid * per, n), i1 = min(i0 + per, n);
    int local = 0;
    for (int i = i0; i < i1; ++i) { local += cnt[i]; cnt[i] = local; }
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL_MASK, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NW ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(FULL_MASK, w, o);
            if (lane >= o) w += y;
        }
        wsum[lane] = w;
    }
    __syncthreads();
    const int offset = x - local + (warp ? wsum[warp - 1] : 0);
    for (int i = i0; i < i1; ++i) cnt[i] += offset;
    __syncthreads();
    const int total = cnt[n - 1];
    if (total > L.max_chunks) {  // cannot happen for a consistent cache
        if (tid == 0 && part == 0) latch_error(L, HKV_ERR_STATE, layer);
        return;
    }
    // Warp ranges of equal cost: a chunk costs CHUNK_COST units and the end
    // of a head HC more (reductions, output, a merge when split), so that
    // warps holding many short heads get fewer chunks.  Head i's cost
    // interval is [E(i-1), E(i)), E(i) = CHUNK_COST * cnt[i] + HC (i + 1);
    // the warps w whose boundary w * cost / GW falls in it start in head i,
    // at the first of its chunks whose cost starts at or after the
    // boundary.  (Every warp start found by arithmetic, no search.)
    // A small layer uses only the first GWe warps, about two chunks of work
    // each or more: ranges thinner than that would split its heads into
    // one-chunk segments whose merges cost more than the chunks.
    const int HC = L.plan_hc;
    const int64_t tcost = (int64_t)CHUNK_COST * total + (int64_t)HC * n;
    const int64_t mrc = min_range_cost(HC);
    const int GWe = (int)min((int64_t)GW, max((int64_t)1, (tcost + mrc - 1) / mrc));
    // A full grid whose blocks load the SM's sub-partitions unevenly weighs
    // its warps (the prefix `pre` of LONE_WEIGHT / SHARED_WEIGHT, made at the
    // start); otherwise equal shares, in 32-bit arithmetic whenever every
    // product fits (the usual case: 64-bit divisions cost several times more).
    const bool weighted = uneven && GWe == GW;
    if (weighted) {
        const uint64_t U = (uint64_t)(GW / L.plan_nw) * pre[L.plan_nw];
        if ((uint64_t)tcost * (U + 1) < (1ull << 32))
            cut_ranges_weighted<uint32_t>(cnt, n, HC, (uint32_t)tcost, (uint32_t)U, L.plan_nw, pre, wbeg, whead);
        else
            cut_ranges_weighted<uint64_t>(cnt, n, HC, (uint64_t)tcost, U, L.plan_nw, pre, wbeg, whead);
    } else if ((uint64_t)tcost * (uint64_t)(GWe + 1) < (1ull << 32))
        cut_ranges<uint32_t>(cnt, n, HC, (uint32_t)tcost, GWe, wbeg, whead);
    else
        cut_ranges<uint64_t>(cnt, n, HC, (uint64_t)tcost, GWe, wbeg, whead);
    for (int w = GWe + threadIdx.x; w <= GW; w += blockDim.x) wbeg[w] = total;  // idle warps
    __syncthreads();
    // A range starting a decode block moves to the nearer end of the head
    // it would cut (at most SNAP_MAX chunks, staying between its neighbours'
    // starts), so that heads seldom span two blocks and their split
    // segments meet in shared memory.  Neighbours of a block start are not
    // block starts, so the entries read here are not being written.
    const int NWB = L.plan_nw;
    if (NWB > 1)
        for (int w = NWB * (threadIdx.x + 1); w < GWe; w += NWB * blockDim.x) {
            const int lo = whead[w], c = wbeg[w];
            const int c0 = lo ? cnt[lo - 1] : 0, c1 = cnt[lo];
            if (c > c0 && c < c1) {
                const int prev = wbeg[w - 1], next = wbeg[w + 1];
                const int down = c - c0, up = c1 - c;
                if (down <= up && down <= SNAP_MAX && c0 >= prev) wbeg[w] = c0;
                else if (up <= SNAP_MAX && c1 <= next) wbeg[w] = c1;
                else if (down <= SNAP_MAX && c0 >= prev) wbeg[w] = c0;
            }
        }
    __syncthreads();
    // the warp whose range holds each chunk
    for (int w = threadIdx.x; w < GW; w += blockDim.x)
        for (int c = wbeg[w]; c < wbeg[w + 1]; ++c) own[c] = (uint16_t)w;
    __syncthreads();
    constexpr int PB = 1 + PLAN_WARP_DESC;
    int4* dsc = L.plan_desc + (size_t)layer * L.max_chunks;
    int4* pw = L.plan_warp + (size_t)layer * PLAN_MAX_WARPS * PB;
    // part p writes the descriptors of the p-th slice of the chunks, one
    // chunk per thread (a head's chunks are spread over threads)
    const int c_lo = (int)((int64_t)part * total / parts), c_hi = (int)((int64_t)(part + 1) * total / parts);
    for (int c = c_lo + threadIdx.x; c < c_hi; c += blockDim.x) {
        int i = 0;  // the head holding chunk c: the first with cnt[i] > c
        for (int hi = n - 1; i < hi;) {
            const int mid = (i + hi) >> 1;
            if (cnt[mid] > c) hi = mid;
            else i = mid + 1;
        }
        const int c1 = cnt[i], c0 = i ? cnt[i - 1] : 0;
        const int wa = own[c0], wb = own[c1 - 1], w = own[c];  // w: the warp holding chunk c
        int segs = 0;
        for (int u = wa; u <= wb; ++u) segs += wbeg[u] < wbeg[u + 1];
        const int hw = wa | ((wb - wa) << 12);
        const int hl = hlen[i];
        const int len = hl >> 16, jn = (int)(int16_t)(hl & 0xffff);
        const int k = c - c0;
        const int tok0 = k * CHUNK;
        const int nr = min(CHUNK, len - tok0);
        const int a = jn - tok0;
        const int z = nr | ((a >= 0 && a < nr ? a + 1 : 0) << 6) | ((k == 0) << 12) |
                      ((c == c1 - 1) << 13) | (hscore[i] << 14) | (segs << 16);
        const int4 d = make_int4(hslot[i] + tok0, i, z, hw);
        dsc[c] = d;
        if (c - wbeg[w] < PLAN_WARP_DESC) pw[PB * w + 1 + (c - wbeg[w])] = d;
    }
    const int w0 = (int)((int64_t)part * GW / parts), w1 = (int)((int64_t)(part + 1) * GW / parts);
    for (int w = w0 + threadIdx.x; w < w1; w += blockDim.x)
        pw[PB * w] = make_int4(wbeg[w], wbeg[w + 1], total, 0);
}

// d = a * b + d on two fp32 lanes at once (packed FMA; each lane rounds as a
// scalar fmaf would).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
    asm("{.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rc;}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// d0 += lo(w) * lo(q) and d1 += hi(w) * hi(q) for two packed bf16 pairs: the
// products of bf16 values are exact in fp32, so this equals unpacking both
// operands and a scalar fmaf, without the unpacking.
__device__ __forceinline__ void fma_bf16x2(float& d0, float& d1, uint32_t w, uint32_t q) {
    asm("{.reg .b16 wl, wh, ql, qh;\n\t"
        "mov.b32 {wl, wh}, %2;\n\t"
        "mov.b32 {ql, qh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, wl, ql, %0;\n\t"
        "fma.rn.f32.bf16 %1, wh, qh, %1;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "r"(w), "r"(q));
}

// The elements of one 16-byte piece as floats (8 bf16 or 4 fp32).
template <typename T>
__device__ __forceinline__ void unpack16(const uint4& w, float (&x)[16 / sizeof(T)]) {
    if constexpr (sizeof(T) == 2) {
        x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
        x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z); x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
    } else {
        x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y);
        x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
    }
}

// Shared memory of one decode warp: its stages, one mbarrier per stage, the
// softmax numerators of the current chunk, two split-head partial states and
// a ticket.
__host__ __device__ inline size_t decode_warp_bytes(int d, int es, int nstage) {
    const size_t row = (size_t)d * es;
    return (size_t)nstage * (2 * CHUNK + 1) * row + (size_t)nstage * 8 + CHUNK * 4 +
           2 * (size_t)(d + 2) * 4 + 16;
}

constexpr uint64_t DECODE_WAIT_NS = 2000000000ull;  // a copy that takes 2 s has failed

template <typename T, int DPL>
__global__ void __launch_bounds__(DECODE_MAX_WARPS * 32, 1)
    decode_kernel(Layout L, int layer, const T* __restrict__ q_t, const T* __restrict__ k_t,
                  const T* __restrict__ v_t, T* __restrict__ o_t, int append, int nstage,
                  int early, int buf, int prologue, int l2_hint) {
    extern __shared__ __align__(128) unsigned char dsm[];
    const int n_heads = L.S * L.H;
    constexpr int D = DPL * 32;
    constexpr int ROW = D * (int)sizeof(T);           // bytes of one cache row
    constexpr int PPR = ROW / 16;                     // 16-byte pieces per row
    constexpr int KVR = 2 * ROW;                      // bytes of one K|V row pair
    constexpr int STAGE = CHUNK * KVR + ROW;          // K|V row pairs, the query
    constexpr int E = 16 / (int)sizeof(T);            // elements per 16-byte piece
    constexpr int G = PPR;                            // lanes covering one row
    constexpr int TPI = 32 / G;                       // rows per pass
    constexpr int NPASS = CHUNK / TPI;                // passes per chunk (= G)
    static_assert(PPR == 8 || PPR == 16 || PPR == 32, "rows are 8, 16 or 32 pieces");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NW = blockDim.x >> 5;
    const int GW = gridDim.x * NW;
    const int gw = blockIdx.x * NW + warp;
    const int vg = lane / G, vc = lane % G;  // row group and piece of this lane
    const size_t hbase = (size_t)layer * n_heads;
    const size_t lrow = (size_t)layer * L.S * L.R;    // first slot of the layer
    const T* KVp = reinterpret_cast<const T*>(L.K);  // slot s: K at 2 D s, V at 2 D s + D
    const float qscale = LOG2E / sqrtf((float)D);

    // Launched as a programmatic dependent of the previous launch in the
    // stream.  With `early` the plan, the cache and t_next of this layer are
    // read before the wait for that launch (the host sets it only when that
    // launch is a decode launch of another layer, which writes none of them);
    // q_t, k_t, v_t, o_t and the split-K buffers are touched only after it.
    // Every thread waits before it triggers the next launch, so that launch
    // can only ever overlap this one, whose split-K buffers (set `buf`) it
    // does not share.
    if (!early) ptx::grid_dep_wait();
    const int t = append ? L.t_next[layer] : L.t_next[layer] - 1;
    const int col = t % L.r;
    int* ticket = L.ticket + (size_t)buf * n_heads;
    float* partial = L.partial + (size_t)buf * 2 * PLAN_MAX_WARPS * (D + 2);

    // shared memory: stages of all warps, then per warp its barriers,
    // numerators, partial states and ticket
    unsigned char* my = dsm + (size_t)warp * nstage * STAGE;
    unsigned char* tail = dsm + (size_t)NW * nstage * STAGE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(tail) + warp * MAX_STAGES;
    float* myp = reinterpret_cast<float*>(tail + (size_t)NW * MAX_STAGES * 8) + warp * CHUNK;
    float* lpart = reinterpret_cast<float*>(tail + (size_t)NW * (MAX_STAGES * 8 + CHUNK * 4));
    int* ltick = reinterpret_cast<int*>(lpart + (size_t)NW * 2 * (D + 2));

    if (GW != L.plan_gw || nstage > MAX_STAGES) {
        if (early) ptx::grid_dep_wait();
        if (threadIdx.x == 0 && blockIdx.x == 0) latch_error(L, HKV_ERR_STATE, layer);
        return;
    }
    // this warp's plan block: lane 0 its range, lanes 1.. its first
    // descriptors (loaded before the block barrier, which hides its latency)
    constexpr int PB = 1 + PLAN_WARP_DESC;
    const int4* pw = L.plan_warp + (size_t)layer * PLAN_MAX_WARPS * PB;
    const int4 blk = lane < PB ? pw[(size_t)gw * PB + lane] : make_int4(0, 0, 0, 0);
    // The same warp's plan block of the next layer (same step): once this
    // warp's range is done, its first chunks are prefetched into L2 for the
    // decode launch that usually follows (layer + 1), while slower warps
    // finish.  Only a hint: a different call order merely wastes the copy.
    const bool hint = l2_hint && append && layer + 1 < L.Ly;
    const int4 nblk = hint && lane < PB ? pw[(size_t)PLAN_MAX_WARPS * PB + (size_t)gw * PB + lane]
                                        : make_int4(0, 0, 0, 0);
    if (lane == 0) {
        for (int s = 0; s < nstage; ++s) ptx::mbar_init(&bars[s], 1);
        ptx::fence_mbar_init();
    }
    if (threadIdx.x < NW) ltick[threadIdx.x] = 0;
    __syncthreads();

    const int4 wrec = shfl_int4(blk, 0);
    const int c_begin = wrec.x, c_end = wrec.y;
    const int4* dsc = L.plan_desc + (size_t)layer * L.max_chunks;

    if (c_begin < c_end) {
        // Lane 0's copies of one chunk into a stage: its cached rows, the
        // appended row from k_t / v_t in its place, and the query when q is
        // set.  part 1 issues only the cached rows (before the wait on the
        // previous launch), part 2 only the rest, part 0 all.
        auto copy_chunk = [&](int stage, int part, const ChunkDesc& c, int q) {
            if (lane != 0) return;
            unsigned char* kd = my + (size_t)stage * STAGE;
            uint64_t* bar = &bars[stage];
            const int a = append ? c.a : -1;
            if (part != 2) {
                ptx::mbar_expect_tx(bar, (uint32_t)(2 * c.n + q) * ROW);
                const size_t row0 = lrow + c.row;
                const int lo = a < 0 ? c.n : a;  // cached rows [0, lo) and (a, n)
                if (lo > 0) {
                    ptx::bulk_g2s(kd, KVp + row0 * 2 * D, lo * KVR, bar);
                }
                if (a >= 0 && a + 1 < c.n) {
                    ptx::bulk_g2s(kd + (a + 1) * KVR, KVp + (row0 + a + 1) * 2 * D, (c.n - a - 1) * KVR, bar);
                }
            }
            if (part != 1) {
                if (a >= 0) {
                    ptx::bulk_g2s(kd + a * KVR, k_t + (size_t)c.head * D, ROW, bar);
                    ptx::bulk_g2s(kd + a * KVR + ROW, v_t + (size_t)c.head * D, ROW, bar);
                }
                if (q) ptx::bulk_g2s(kd + CHUNK * KVR, q_t + (size_t)c.head * D, ROW, bar);
            }
        };
        // descriptors of the range, 32 chunks per window, lane k holding
        // chunk base + k; the producer (ip) and the consumer (i) keep their
        // own window
        auto window = [&](int base) -> int4 {
            return base + lane < c_end ? dsc[base + lane] : make_int4(0, 0, 0, 0);
        };
        int pbase = c_begin, cbase = c_begin;
        // first window: the plan block's copies (lane k < PLAN_WARP_DESC
        // holds chunk c_begin + k), the rest loaded
        const int4 head = shfl_int4(blk, min(lane + 1, 31));
        int4 pwin = head;
        if (lane >= PLAN_WARP_DESC)
            pwin = c_begin + lane < c_end ? dsc[c_begin + lane] : make_int4(0, 0, 0, 0);
        int4 cwin = pwin;
        // With many warps per SM the first stage only (the others once it
        // has landed: with every warp of the GPU asking at once, a single
        // stage each reaches the warps sooner and the queue stays short);
        // with few, every stage (fewer bytes would be in flight otherwise).
        // With `early` their cached rows go before the wait on the previous
        // launch, queries and appended rows after it.
        const int npro = (prologue == 1 || (prologue == 0 && NW >= 8)) ? 1 : min(nstage, c_end - c_begin);
        if (early) {
            for (int s = 0; s < npro; ++s) {
                const ChunkDesc c = ChunkDesc::of(shfl_int4(head, s));
                copy_chunk(s, 1, c, c.first || s == 0);
            }
            ptx::grid_dep_wait();
            ptx::grid_dep_trigger();
            for (int s = 0; s < npro; ++s) {
                const ChunkDesc c = ChunkDesc::of(shfl_int4(head, s));
                copy_chunk(s, 2, c, c.first || s == 0);
            }
        } else {
            ptx::grid_dep_trigger();
            for (int s = 0; s < npro; ++s) {
                const ChunkDesc c = ChunkDesc::of(shfl_int4(head, s));
                copy_chunk(s, 0, c, c.first || s == 0);
            }
        }
        int ip = c_begin + npro;
        auto issue = [&](int stage) {
            if (ip - pbase >= 32) { pbase += 32; pwin = window(pbase); }
            const ChunkDesc c = ChunkDesc::of(shfl_int4(pwin, ip - pbase));
            copy_chunk(stage, 0, c, c.first || ip == c_begin);
            ++ip;
        };

        uint32_t phase = 0;  // bit s: parity of stage s's next phase
        bool failed = false;
        // m: the warp's reference maximum (log2 domain), raised only when a
        // logit passes it by more than RESCALE; ls: this lane's share of the
        // softmax denominator; qw: this lane's 16-byte piece of the query;
        // acc: this lane's piece of the weighted V sum over its row group
        float m = -INFINITY, ls = 0.f, acc[E];
        uint4 qw = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
        bool seg_start = true;   // chunk i starts this warp's segment of its head
        bool seg_whole = false;  // that segment starts at the head's first chunk

        int i = c_begin;
        for (; i < c_end; ++i) {
            const int k = i - c_begin;
            const int stage = k % nstage;
            if (i - cbase >= 32) { cbase += 32; cwin = window(cbase); }
            const ChunkDesc c = ChunkDesc::of(shfl_int4(cwin, i - cbase));
            const bool ok = ptx::mbar_wait_sleep(&bars[stage], (phase >> stage) & 1u, DECODE_WAIT_NS);
            if (__any_sync(FULL_MASK, !ok)) {  // the whole warp stops
                if (lane == 0) latch_error(L, HKV_ERR_TIMEOUT, (int)(hbase + c.head));
                failed = true;
                break;
            }
            phase ^= 1u << stage;
            if (k == 0 && npro == 1)  // the first chunk has landed: fill the other stages
                for (int s2 = 1; s2 < nstage && ip < c_end; ++s2) issue(s2);
            const int n = c.n;
            const unsigned char* kst = my + (size_t)stage * STAGE;
            const unsigned char* vst = kst + ROW;  // V half of each row pair
            if (seg_start) {  // a new head: this lane's piece of its query
                qw = *reinterpret_cast<const uint4*>(kst + CHUNK * KVR + vc * 16);
                seg_whole = c.first;
            }
            // QK: pass p, lane (vg, vc) takes piece vc of row p * TPI + vg;
            // a butterfly over the G lanes of a group then leaves lane
            // (vg, vc) the whole dot product of row j = vc * TPI + vg.  All
            // 32 rows are read (no branches between the loads): a row past n
            // holds an earlier chunk's data, only ever added into its own
            // row's sum, which is dropped below.
            float part[NPASS];
#pragma unroll
            for (int p = 0; p < NPASS; ++p) {
                const int row = p * TPI + vg;
                float a0 = 0.f, a1 = 0.f;
                const uint4 kw = *reinterpret_cast<const uint4*>(kst + row * KVR + vc * 16);
                if constexpr (sizeof(T) == 2) {
                    fma_bf16x2(a0, a1, kw.x, qw.x);
                    fma_bf16x2(a0, a1, kw.y, qw.y);
                    fma_bf16x2(a0, a1, kw.z, qw.z);
                    fma_bf16x2(a0, a1, kw.w, qw.w);
                } else {
                    ffma2(a0, a1, __uint_as_float(qw.x), __uint_as_float(qw.y),
                          __uint_as_float(kw.x), __uint_as_float(kw.y));
                    ffma2(a0, a1, __uint_as_float(qw.z), __uint_as_float(qw.w),
                          __uint_as_float(kw.z), __uint_as_float(kw.w));
                }
                part[p] = a0 + a1;
            }
#pragma unroll
            for (int h = NPASS / 2; h >= 1; h >>= 1) {
                const bool upper = (vc & h) != 0;
#pragma unroll
                for (int u = 0; u < h; ++u) {
                    const float send = upper ? part[u] : part[u + h];
                    const float keep = upper ? part[u + h] : part[u];
                    part[u] = keep + __shfl_xor_sync(FULL_MASK, send, h);
                }
            }
            const int j = vc * TPI + vg;  // this lane's row
            const float sl = j < n ? part[0] * qscale : -INFINITY;
            const size_t row0 = lrow + c.row;
            if (c.scoring && j < n) L.logit[(row0 + j) * L.r + col] = sl;
            // raise the reference only when some logit passes it by more than
            // RESCALE (weights stay below 2^RESCALE); one vote otherwise
            if (__any_sync(FULL_MASK, sl > m + RESCALE)) {
                float cm = sl;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(FULL_MASK, cm, o));
                const float mn = fmaxf(m, cm);
                const float alpha = exp2f(m - mn);
                ls *= alpha;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] *= alpha;
                m = mn;
            }
            const float pj_own = j < n ? exp2f(sl - m) : 0.f;
            ls += pj_own;
            myp[j] = pj_own;
            __syncwarp();
            // PV: lane (vg, vc) adds p_j times piece vc of rows j = vg (mod TPI)
            // (rows past n are skipped: their stale V may be anything)
            float pa[2][E];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int e = 0; e < E; ++e) pa[u][e] = 0.f;
            auto pv_row = [&](int p) {
                const int jr = p * TPI + vg;
                const float pj = myp[jr];
                float x[E];
                unpack16<T>(*reinterpret_cast<const uint4*>(vst + jr * KVR + vc * 16), x);
                float* pu = pa[p & 1];
#pragma unroll
                for (int e = 0; e < E; e += 2) ffma2(pu[e], pu[e + 1], pj, pj, x[e], x[e + 1]);
            };
            if (n == CHUNK) {
#pragma unroll
                for (int p = 0; p < NPASS; ++p) pv_row(p);
            } else {
#pragma unroll
                for (int p = 0; p < NPASS; ++p)
                    if (p * TPI + vg < n) pv_row(p);
            }
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += pa[0][e] + pa[1][e];
            // the appended token joins the cache
            if (append && c.a >= 0) {
                const int a = c.a;
                Raw<T, DPL> kr, vr;
                kr.load_shared(reinterpret_cast<const T*>(kst + a * KVR) + lane * DPL);
                vr.load_shared(reinterpret_cast<const T*>(vst + a * KVR) + lane * DPL);
                kr.store(reinterpret_cast<T*>(L.K) + (row0 + a) * 2 * D + lane * DPL);
                vr.store(reinterpret_cast<T*>(L.K) + (row0 + a) * 2 * D + D + lane * DPL);
                if (lane == 0) L.pos[row0 + a] = t;
            }
            __syncwarp();  // every lane is done with this stage
            if (ip < c_end) issue(stage);
            seg_start = c.last || i + 1 == c_end;
            if (!seg_start) continue;  // the head goes on in this warp

            // end of this warp's segment of head c.head: add up the row
            // groups and the lanes' denominators
#pragma unroll
            for (int o = G; o < 32; o <<= 1)
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] += __shfl_xor_sync(FULL_MASK, acc[e], o);
            float l = ls;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(FULL_MASK, l, o);
            const int hc = c.head;
            const size_t hx = hbase + hc;
            if (!(l > 0.f) || isinf(l)) latch_error(L, HKV_ERR_NUMERIC, (int)hx);
            if (seg_whole && c.last) {
                const float inv = 1.0f / l;
                float o[E];
#pragma unroll
                for (int e = 0; e < E; ++e) o[e] = acc[e] * inv;
                if (lane < G) store_row<T, E>(o_t + (size_t)hc * D + vc * E, o);
                if (c.scoring && lane == 0) L.ml[hx * L.r + col] = make_float2(m, l);
            } else {
                const int segs = c.segs, w_a = c.wa, w_b = c.wb;
                // A split head's segments are named by (warp, side): side 1 for
                // the warp holding the head's first chunk (its segment ends its
                // range), 0 for the others (theirs start their range); a warp
                // has at most one segment of each side.  Segments all in this
                // block meet in shared memory, the others in global memory;
                // the last one in merges (no waiting).
                const bool local = w_a / NW == (int)blockIdx.x && w_b / NW == (int)blockIdx.x;
                const int side = gw == w_a ? 1 : 0;
                float* pp = local ? lpart + (size_t)(warp * 2 + side) * (D + 2)
                                  : partial + (size_t)(gw * 2 + side) * (D + 2);
                if (lane == 0) { pp[0] = m; pp[1] = l; }
                if (lane < G) {
#pragma unroll
                    for (int e = 0; e < E; ++e) pp[2 + vc * E + e] = acc[e];
                }
                __syncwarp();  // the lanes' partial stores precede lane 0's release
                int prev = 0;
                if (lane == 0) {
                    if (local) {
                        __threadfence_block();
                        prev = atomicAdd(&ltick[w_a % NW], 1);
                        __threadfence_block();
                    } else {
                        // release: this warp's partial before the ticket;
                        // acquire: the other segments' for the last one in
                        cuda::atomic_ref<int, cuda::thread_scope_device> tk(ticket[hc]);
                        prev = tk.fetch_add(1, cuda::memory_order_acq_rel);
                    }
                }
                prev = __shfl_sync(FULL_MASK, prev, 0);
                __syncwarp();  // lane 0's acquire before every lane's partial loads
                if (prev == segs - 1) {
                    if (lane == 0 && !local) ticket[hc] = 0;
                    auto slot_of = [&](int w) -> const float* {
                        const int sd = w == w_a ? 1 : 0;
                        return local ? lpart + (size_t)((w % NW) * 2 + sd) * (D + 2)
                                     : partial + (size_t)(w * 2 + sd) * (D + 2);
                    };
                    // online merge of the segments, four at a time with all
                    // their loads issued first; warp ranges between w_a and
                    // w_b are all non-empty unless segs says otherwise
                    const bool dense = segs == w_b - w_a + 1;
                    float M = -INFINITY, Ls = 0.f, o[E];
#pragma unroll
                    for (int e = 0; e < E; ++e) o[e] = 0.f;
                    for (int w0 = w_a; w0 <= w_b; w0 += 4) {
                        float pm[4], pl[4], px[4][E];
                        bool ok[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int w = w0 + u;
                            ok[u] = w <= w_b;
                            if (ok[u] && !dense) {
                                const int2 r = *reinterpret_cast<const int2*>(pw + (size_t)PB * w);
                                ok[u] = r.x < r.y;
                            }
                            pm[u] = -INFINITY;
                            pl[u] = 0.f;
#pragma unroll
                            for (int e = 0; e < E; ++e) px[u][e] = 0.f;
                            if (ok[u]) {
                                const float* pi = slot_of(w);
                                if (local) {
                                    pm[u] = pi[0];
                                    pl[u] = pi[1];
#pragma unroll
                                    for (int e = 0; e < E; ++e) px[u][e] = pi[2 + vc * E + e];
                                } else {
                                    pm[u] = __ldcg(pi);
                                    pl[u] = __ldcg(pi + 1);
#pragma unroll
                                    for (int e = 0; e < E; ++e) px[u][e] = __ldcg(pi + 2 + vc * E + e);
                                }
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (!ok[u]) continue;
                            const float mn = fmaxf(M, pm[u]);
                            const float fa = exp2f(M - mn), fb = exp2f(pm[u] - mn);
                            Ls = Ls * fa + pl[u] * fb;
#pragma unroll
                            for (int e = 0; e < E; ++e) o[e] = o[e] * fa + px[u][e] * fb;
                            M = mn;
                        }
                    }
                    const float inv = 1.0f / Ls;
#pragma unroll
                    for (int e = 0; e < E; ++e) o[e] *= inv;
                    if (lane < G) store_row<T, E>(o_t + (size_t)hc * D + vc * E, o);
                    if (c.scoring && lane == 0) L.ml[hx * L.r + col] = make_float2(M, Ls);
                }
            }
            // the next chunk starts a new segment
            m = -INFINITY;
            ls = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = 0.f;
        }
        if (failed) {
            // copies still in flight into this warp's stages: wait for them
            // (briefly) before the block's shared memory is given up
            for (int k = i - c_begin; k < ip - c_begin; ++k) {
                const int stage = k % nstage;
                if (!ptx::mbar_wait(&bars[stage], (phase >> stage) & 1u, DECODE_WAIT_NS / 8)) break;
                phase ^= 1u << stage;
            }
        }
    } else {
        if (early) ptx::grid_dep_wait();
        ptx::grid_dep_trigger();
    }
    if (hint) {
        // L2 prefetch of the next layer's first chunks of this warp number
        const int4 nrec = shfl_int4(nblk, 0);
        const int nc = min(min(nrec.y - nrec.x, l2_hint == 1 ? nstage : l2_hint), PLAN_WARP_DESC);
        const size_t nrow = (size_t)(layer + 1) * L.S * L.R;
        for (int k = 0; k < nc; ++k) {
            const ChunkDesc c = ChunkDesc::of(shfl_int4(nblk, k + 1));
            if (lane == 0 && c.n > 0)
                ptx::bulk_prefetch_l2(KVp + (nrow + c.row) * 2 * D, (uint32_t)(c.n * KVR));
        }
    }
    if (append) {
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            if (atomicAdd(&L.done_ctr[layer], 1) == (int)gridDim.x - 1) {
                L.done_ctr[layer] = 0;
                L.t_next[layer] = t + 1;
            }
        }
    }
}

// Appends one token to every head of a layer, one warp per head
// (Methodology step 3: ring overwrite for Local heads, tail for Global).
template <typename T, int DPL>
__global__ void __launch_bounds__(256) append_kernel(Layout L, int layer, const T* __restrict__ k_t,
                                                     const T* __restrict__ v_t) {
    const int n_heads = L.S * L.H;
    const int lane = threadIdx.x & 31;
    const int h = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int t = L.t_next[layer];
    if (h < n_heads) {
        const size_t hx = (size_t)layer * n_heads + h;
        const int len = len_at(L, hx, t);
        if (len > L.cap[hx]) {
            if (lane == 0) latch_error(L, HKV_ERR_CAPACITY, (int)hx);
        } else {
            const int s = h / L.H;
            const size_t slot = region_slot0(L, layer, s) + L.off[hx] + append_slot(L, hx, t, len);
            Raw<T, DPL> kr, vr;
            kr.load(k_t + (size_t)h * L.d + lane * DPL);
            vr.load(v_t + (size_t)h * L.d + lane * DPL);
            kr.store(reinterpret_cast<T*>(L.K) + slot * 2 * L.d + lane * DPL);
            vr.store(reinterpret_cast<T*>(L.K) + slot * 2 * L.d + L.d + lane * DPL);
            if (lane == 0) L.pos[slot] = t;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&L.done_ctr[layer], 1) == (int)gridDim.x - 1) {
            L.done_ctr[layer] = 0;
            L.t_next[layer] = t + 1;
        }
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

// Positive integer from the environment, or 0 when unset or invalid.
static int env_int(const char* name) {
    const char* v = getenv(name);
    if (!v) return 0;
    const int x = atoi(v);
    return x > 0 ? x : 0;
}

DecodeShape decode_shape(const Layout& L, size_t smem_limit) {
    // As many warps as fit (up to DECODE_MAX_WARPS) with two stages each:
    // the kernel is latency-bound, so warps matter more than prefetch depth
    // (one chunk in flight per warp covers the HBM latency at the rate a
    // warp consumes chunks); a third stage only when it costs no warp.
    // Tuning overrides (read once per context): HKV_DECODE_WARPS caps the
    // warps per block, HKV_DECODE_STAGES fixes the stages per warp (1 ..
    // MAX_STAGES), HKV_DECODE_PROLOGUE sets DecodeShape::prologue (1 or 2),
    // HKV_DECODE_L2_HINT=0 / =1 turns the next-layer L2 prefetch off / on
    // (=k > 1: up to k chunks per warp instead of the stage count),
    // HKV_DECODE_HEAD_COST (1 .. 4 CHUNK_COST) sets DecodeShape::head_cost,
    // HKV_DECODE_LONE_WEIGHT (SHARED_WEIGHT .. 2 SHARED_WEIGHT; SHARED_WEIGHT:
    // equal shares) DecodeShape::lone_weight.
    const int es = L.dtype == HKV_DTYPE_F32 ? 4 : 2;
    const int max_w = env_int("HKV_DECODE_WARPS");
    const int fix_s = env_int("HKV_DECODE_STAGES");
    const int pro = env_int("HKV_DECODE_PROLOGUE");
    // the next-layer L2 prefetch pays off with many warps per block
    // (LlamaGen-XL shape: 11.15 against 12.05 us per launch) and not with
    // the six of a d = 128 cache (Lumina-mGPT-768 shape: 25.04 against
    // 24.75 us): on when the block has 8 or more warps, unless overridden
    const char* hint_env = getenv("HKV_DECODE_L2_HINT");
    const int hint_val = hint_env ? atoi(hint_env) : 0;
    const int hint_set = hint_env ? (hint_env[0] == '0' && hint_env[1] == 0 ? 0 : (hint_val > 1 ? hint_val : 1)) : -1;
    DecodeShape best{0, 0, 0, 1, pro <= 2 ? pro : 0, 0, HEAD_COST};
    for (int ns = fix_s == 1 ? 1 : 2; ns <= MAX_STAGES; ++ns) {
        if (fix_s && ns != fix_s) continue;
        // the per-warp tail regions are laid out for MAX_STAGES barriers
        const size_t per = decode_warp_bytes(L.d, es, ns) + (MAX_STAGES - ns) * 8;
        int w = (int)((smem_limit - 1024) / per);
        if (w > DECODE_MAX_WARPS) w = DECODE_MAX_WARPS;
        if (max_w && w > max_w) w = max_w;
        if (w >= 1 && w >= best.warps)
            best = DecodeShape{w, ns, 1024 + (size_t)w * per, 1, best.prologue, 0, HEAD_COST};
    }
    best.l2_hint = hint_set >= 0 ? hint_set : (best.warps >= 8 ? 1 : 0);
    best.lone_weight = LONE_WEIGHT;
    const int lw = env_int("HKV_DECODE_LONE_WEIGHT");
    if (lw >= SHARED_WEIGHT && lw <= 2 * SHARED_WEIGHT) best.lone_weight = lw;
    const int hc = env_int("HKV_DECODE_HEAD_COST");
    if (hc > 0 && hc <= 4 * CHUNK_COST) best.head_cost = hc;
    return best;
}

template <typename T, int DPL>
static cudaError_t launch_decode_t(const Layout& L, int layer, const void* q, const void* k,
                                   const void* v, void* o, int append, const DecodeShape& sh,
                                   int grid, int early, int buf, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(32 * sh.warps);
    cfg.dynamicSmemBytes = sh.smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<T, DPL>, L, layer, (const T*)q, (const T*)k,
                              (const T*)v, (T*)o, append, sh.nstage, early, buf, sh.prologue,
                              sh.l2_hint);
}

cudaError_t launch_decode(const Layout& L, int layer, const void* q, const void* k, const void* v,
                          void* o, int append, const DecodeShape& sh, int grid, int early, int buf,
                          cudaStream_t st) {
    if (sh.nstage < 1 || sh.nstage > MAX_STAGES) return cudaErrorInvalidValue;
    if (L.dtype == HKV_DTYPE_BF16) {
        if (L.d == 64) return launch_decode_t<__nv_bfloat16, 2>(L, layer, q, k, v, o, append, sh, grid, early, buf, st);
        if (L.d == 128) return launch_decode_t<__nv_bfloat16, 4>(L, layer, q, k, v, o, append, sh, grid, early, buf, st);
    } else {
        if (L.d == 64) return launch_decode_t<float, 2>(L, layer, q, k, v, o, append, sh, grid, early, buf, st);
        if (L.d == 128) return launch_decode_t<float, 4>(L, layer, q, k, v, o, append, sh, grid, early, buf, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_plan(const Layout& L, int l0, int l1, int ahead, int commit, cudaStream_t st,
                        int after_evict) {
    cudaLaunchConfig_t cfg = {};
    // blocks per layer: PLAN_DESC_PARTS, or HKV_PLAN_PARTS (1 .. 32; tuning)
    static const int parts = [] {
        const int v = env_int("HKV_PLAN_PARTS");
        return v >= 1 && v <= 32 ? v : PLAN_DESC_PARTS;
    }();
    cfg.gridDim = dim3(l1 - l0, parts);
    cfg.blockDim = dim3(1024);
    cfg.dynamicSmemBytes = plan_smem_bytes(L.S * L.H, L.max_chunks);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = after_evict ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, plan_kernel, L, l0, ahead, commit, after_evict);
}

cudaError_t launch_append(const Layout& L, int layer, const void* k, const void* v, cudaStream_t st) {
    const int n_heads = L.S * L.H;
    const int grid = (n_heads + 7) / 8;
    if (L.dtype == HKV_DTYPE_BF16) {
        if (L.d == 64) append_kernel<__nv_bfloat16, 2><<<grid, 256, 0, st>>>(L, layer, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v);
        else append_kernel<__nv_bfloat16, 4><<<grid, 256, 0, st>>>(L, layer, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v);
    } else {
        if (L.d == 64) append_kernel<float, 2><<<grid, 256, 0, st>>>(L, layer, (const float*)k, (const float*)v);
        else append_kernel<float, 4><<<grid, 256, 0, st>>>(L, layer, (const float*)k, (const float*)v);
    }
    return cudaGetLastError();
}

cudaError_t prepare_decode(int smem) {
    cudaError_t e = allow_max_dynamic_smem(decode_kernel<__nv_bfloat16, 2>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(decode_kernel<__nv_bfloat16, 4>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(decode_kernel<float, 2>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(decode_kernel<float, 4>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(plan_kernel, smem);
    return e;
}

}  // namespace hkv
