// decode.cu -- per-step cache append and decode attention over the ragged,
// head-aware compressed cache (HeadKV technical summary: Problem statement;
// Methodology step 3, Local sliding window and Global STE scoring).
//
// Work decomposition: every head's cache is cut into chunks of 32 tokens.
// A plan (plan_kernel, once per step and layer) prefix-sums the heads' chunk
// counts and cuts the layer's chunk list into equal contiguous ranges, one
// per warp of the persistent decode grid.  Each warp walks its range with a
// pipeline of shared-memory stages filled by per-lane 16-byte cp.async
// copies, keeps the online softmax of the current head in registers across
// that head's chunks, and finishes a head it holds entirely; a head split
// between warps leaves one partial per warp and the last to arrive (atomic
// ticket, no spinning) merges them.  Global heads within r steps of their
// eviction also store their exp2-domain logits per slot, which the eviction
// normalises with the (max, sum) stored here.
#include <math.h>

#include <cuda/atomic>

#include "hkv_internal.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace hkv {

// Headroom (log2 units) a logit may exceed the running softmax reference by
// before the reference is raised: weights stay below 2^8, far from fp32 range.
constexpr float RESCALE = 8.f;
// Most pipeline stages a decode warp keeps in flight.
constexpr int MAX_STAGES = 3;

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

// First chunk of warp w's range when `total` chunks go to `gw` warps.
__device__ __forceinline__ int range_begin(int w, int total, int gw) {
    return (int)((int64_t)w * total / gw);
}
// Warp whose range holds chunk c.
__device__ __forceinline__ int range_owner(int c, int total, int gw) {
    return (int)(((int64_t)(c + 1) * gw - 1) / total);
}

// ---------------------------------------------------------------------------
// The plan of a layer's decode launch at step t (ahead = 1: the step of the
// next append, t_next; ahead = 0: the newest cached position, t_next - 1).
// One block per layer: per-head facts, the chunk-count prefix, and for every
// warp of the decode grid its first chunk and the head holding it.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) plan_kernel(Layout L, int l0, int ahead) {
    extern __shared__ int32_t cnt[];
    __shared__ int wsum[32];
    const int layer = l0 + blockIdx.x;
    const int n = L.S * L.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, NW = blockDim.x >> 5;
    const int t = L.t_next[layer] - 1 + ahead;
    if (t >= L.L) return;  // the sequence is complete: no step left to plan
    const size_t hbase = (size_t)layer * n;
    for (int i = tid; i < n; i += blockDim.x) {
        const size_t hx = hbase + i;
        const int len = len_at(L, hx, t);
        const int cap = L.cap[hx];
        int c = (len + CHUNK - 1) / CHUNK;
        if (len > cap || len < 1) {
            latch_error(L, HKV_ERR_CAPACITY, (int)hx);
            c = 0;
        }
        const int jn = append_slot(L, hx, t, len);
        const int scoring = L.label[hx] == 0 && L.mode != HKV_MODE_FULL && len > cap - L.r;
        const int slot = (i / L.H) * L.R + L.off[hx];
        L.plan_head[hbase + i] = make_int4(slot, (len << 16) | (jn & 0xffff), scoring, 0);
        cnt[i] = c;
    }
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
    for (int i = tid; i < n; i += blockDim.x) L.plan_pre[hbase + i] = cnt[i];
    const int GW = L.plan_gw;
    int32_t* pw = L.plan_warp + (size_t)layer * (PLAN_MAX_WARPS + 1);
    int32_t* ph = L.plan_whead + (size_t)layer * PLAN_MAX_WARPS;
    for (int w = tid; w <= GW; w += blockDim.x) {
        const int cb = range_begin(w, total, GW);
        pw[w] = cb;
        if (w < GW) {
            int lo = 0, hi = n - 1;  // head holding chunk cb
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (cnt[mid] > cb) hi = mid; else lo = mid + 1;
            }
            ph[w] = lo;
        }
    }
}

// Head facts of the 32 heads [base, base + 32) of a layer, lane i holding
// head base + i.
struct HeadCache {
    int base;
    int slot, lenjn, scoring, pre, first;
    __device__ void load(const Layout& L, size_t hbase, int n, int b) {
        const int lane = threadIdx.x & 31;
        base = b;
        const int h = b + lane;
        if (h < n) {
            const int4 v = L.plan_head[hbase + h];
            slot = v.x; lenjn = v.y; scoring = v.z;
            pre = L.plan_pre[hbase + h];
            first = h ? L.plan_pre[hbase + h - 1] : 0;
        } else {
            slot = 0; lenjn = 0; scoring = 0; pre = 0x7fffffff; first = 0x7fffffff;
        }
    }
    // facts of head h (base <= h < base + 32), broadcast to every lane
    __device__ void get(int h, int& o_slot, int& o_len, int& o_jn, int& o_scoring, int& o_pre,
                        int& o_first) const {
        const int src = h - base;
        o_slot = __shfl_sync(FULL_MASK, slot, src);
        const int lj = __shfl_sync(FULL_MASK, lenjn, src);
        o_len = lj >> 16;
        o_jn = (int)(int16_t)(lj & 0xffff);
        o_scoring = __shfl_sync(FULL_MASK, scoring, src);
        o_pre = __shfl_sync(FULL_MASK, pre, src);
        o_first = __shfl_sync(FULL_MASK, first, src);
    }
};

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
__global__ void __launch_bounds__(256, 1)
    decode_kernel(Layout L, int layer, const T* __restrict__ q_t, const T* __restrict__ k_t,
                  const T* __restrict__ v_t, T* __restrict__ o_t, int append, int nstage,
                  int early, int buf) {
    extern __shared__ __align__(128) unsigned char dsm[];
    const int n_heads = L.S * L.H;
    constexpr int D = DPL * 32;
    constexpr int ROW = D * (int)sizeof(T);           // bytes of one cache row
    constexpr int PPR = ROW / 16;                     // 16-byte pieces per row
    constexpr int STAGE = (2 * CHUNK + 1) * ROW;      // K rows, V rows, the query
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
    const T* Kp = reinterpret_cast<const T*>(L.K);
    const T* Vp = reinterpret_cast<const T*>(L.V);
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
    float* partial = L.partial + (size_t)buf * L.max_chunks * (D + 2);

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
    if (lane == 0) {
        for (int s = 0; s < nstage; ++s) ptx::mbar_init(&bars[s], 1);
        ptx::fence_mbar_init();
    }
    if (threadIdx.x < NW) ltick[threadIdx.x] = 0;
    __syncthreads();

    const int32_t* pw = L.plan_warp + (size_t)layer * (PLAN_MAX_WARPS + 1);
    const int c_begin = pw[gw], c_end = pw[gw + 1], total = pw[GW];

    if (c_begin < c_end) {
        const int h_begin = L.plan_whead[(size_t)layer * PLAN_MAX_WARPS + gw];
        HeadCache pc, cc;  // producer's and consumer's view of the heads
        pc.load(L, hbase, n_heads, h_begin);
        cc = pc;

        // Producer cursor: chunk ip of head hp.  issue() fills a stage with
        // bulk copies from lane 0: the cached rows of the chunk, the appended
        // row from k_t / v_t in its place, and the query for the first chunk
        // of a head in this range.  part 1 issues only the cached rows (before
        // the wait on the previous launch), part 2 only the rest, part 0 all.
        int ip = c_begin, hp = h_begin;
        int4 held = make_int4(0, -1, 0, 0);  // part 1's chunk: head, appended row, query wanted
        auto issue = [&](int stage, int part) {
            int slot, len, jn, sc_, pre, first;
            if (hp - pc.base >= 32) pc.load(L, hbase, n_heads, hp);
            pc.get(hp, slot, len, jn, sc_, pre, first);
            const int tok0 = (ip - first) * CHUNK;
            const int n = min(CHUNK, len - tok0);
            int a = append ? jn - tok0 : -1;  // appended row within the chunk
            if (a >= n) a = -1;
            const int needq = ip == first || ip == c_begin;
            unsigned char* kd = my + (size_t)stage * STAGE;
            unsigned char* vd = kd + CHUNK * ROW;
            unsigned char* qd = vd + CHUNK * ROW;
            uint64_t* bar = &bars[stage];
            if (lane == 0) {
                if (part != 2) {
                    const uint32_t bytes = (uint32_t)(2 * n + needq) * ROW;
                    ptx::mbar_expect_tx(bar, bytes);
                    const size_t row0 = lrow + slot + tok0;
                    const int lo = a < 0 ? n : a;      // cached rows [0, lo) and (a, n)
                    if (lo > 0) {
                        ptx::bulk_g2s(kd, Kp + row0 * D, lo * ROW, bar);
                        ptx::bulk_g2s(vd, Vp + row0 * D, lo * ROW, bar);
                    }
                    if (a >= 0 && a + 1 < n) {
                        ptx::bulk_g2s(kd + (a + 1) * ROW, Kp + (row0 + a + 1) * D, (n - a - 1) * ROW, bar);
                        ptx::bulk_g2s(vd + (a + 1) * ROW, Vp + (row0 + a + 1) * D, (n - a - 1) * ROW, bar);
                    }
                }
                if (part != 1) {
                    if (a >= 0) {
                        ptx::bulk_g2s(kd + a * ROW, k_t + (size_t)hp * D, ROW, bar);
                        ptx::bulk_g2s(vd + a * ROW, v_t + (size_t)hp * D, ROW, bar);
                    }
                    if (needq) ptx::bulk_g2s(qd, q_t + (size_t)hp * D, ROW, bar);
                }
            }
            held = make_int4(hp, a, needq, 0);
            ++ip;
            if (ip < c_end && pre <= ip) ++hp;
            while (ip < c_end) {  // skip heads with no chunk (capacity errors)
                if (hp - pc.base >= 32) pc.load(L, hbase, n_heads, hp);
                int s2, l2, j2, c2, p2, f2;
                pc.get(hp, s2, l2, j2, c2, p2, f2);
                if (p2 > ip) break;
                ++hp;
            }
        };
        // the rest of part 1's chunk, after the wait
        auto finish_held = [&](int stage) {
            if (lane == 0) {
                unsigned char* kd = my + (size_t)stage * STAGE;
                unsigned char* vd = kd + CHUNK * ROW;
                uint64_t* bar = &bars[stage];
                if (held.y >= 0) {
                    ptx::bulk_g2s(kd + held.y * ROW, k_t + (size_t)held.x * D, ROW, bar);
                    ptx::bulk_g2s(vd + held.y * ROW, v_t + (size_t)held.x * D, ROW, bar);
                }
                if (held.z) ptx::bulk_g2s(vd + CHUNK * ROW, q_t + (size_t)held.x * D, ROW, bar);
            }
        };
        if (early) {
            issue(0, 1);
            ptx::grid_dep_wait();
            ptx::grid_dep_trigger();
            finish_held(0);
        } else {
            ptx::grid_dep_trigger();
            issue(0, 0);
        }
        for (int s = 1; s < nstage && ip < c_end; ++s) issue(s, 0);

        int hc = h_begin;
        int seg0 = c_begin;
        uint32_t phase = 0;  // bit s: parity of stage s's next phase
        bool failed = false;
        // m: the warp's reference maximum (log2 domain), raised only when a
        // logit passes it by more than RESCALE; ls: this lane's share of the
        // softmax denominator; qv: this lane's piece of the pre-scaled query;
        // acc: this lane's piece of the weighted V sum over its row group
        float m = -INFINITY, ls = 0.f, acc[E], qv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
        int slot, len, jn, scoring, pre, first;
        cc.get(hc, slot, len, jn, scoring, pre, first);
        while (pre <= c_begin) {  // heads with no chunk before the first one
            ++hc;
            if (hc - cc.base >= 32) cc.load(L, hbase, n_heads, hc);
            cc.get(hc, slot, len, jn, scoring, pre, first);
        }

        int i = c_begin;
        for (; i < c_end; ++i) {
            const int k = i - c_begin;
            const int stage = k % nstage;
            const bool ok = ptx::mbar_wait(&bars[stage], (phase >> stage) & 1u, DECODE_WAIT_NS);
            if (__any_sync(FULL_MASK, !ok)) {  // the whole warp stops
                if (lane == 0) latch_error(L, HKV_ERR_TIMEOUT, (int)(hbase + hc));
                failed = true;
                break;
            }
            phase ^= 1u << stage;
            const int tok0 = (i - first) * CHUNK;
            const int n = min(CHUNK, len - tok0);
            const unsigned char* kst = my + (size_t)stage * STAGE;
            const unsigned char* vst = kst + CHUNK * ROW;
            if (i == seg0) {  // a new head: this lane's piece of its query
                float x[E];
                unpack16<T>(*reinterpret_cast<const uint4*>(vst + CHUNK * ROW + vc * 16), x);
#pragma unroll
                for (int e = 0; e < E; ++e) qv[e] = x[e] * qscale;
            }
            // QK: pass p, lane (vg, vc) takes piece vc of row p * TPI + vg;
            // a butterfly over the G lanes of a group then leaves lane
            // (vg, vc) the whole dot product of row j = vc * TPI + vg
            float part[NPASS];
#pragma unroll
            for (int p = 0; p < NPASS; ++p) {
                const int row = p * TPI + vg;
                float a0 = 0.f, a1 = 0.f;
                if (p * TPI < n) {
                    float x[E];
                    unpack16<T>(*reinterpret_cast<const uint4*>(kst + row * ROW + vc * 16), x);
#pragma unroll
                    for (int e = 0; e < E; e += 2) ffma2(a0, a1, qv[e], qv[e + 1], x[e], x[e + 1]);
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
            const float sl = j < n ? part[0] : -INFINITY;
            const size_t row0 = lrow + slot + tok0;
            if (scoring && j < n) L.logit[(row0 + j) * L.r + col] = sl;
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
            float pa[2][E];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int e = 0; e < E; ++e) pa[u][e] = 0.f;
#pragma unroll
            for (int p = 0; p < NPASS; ++p) {
                const int jr = p * TPI + vg;
                if (p * TPI < n && jr < n) {
                    const float pj = myp[jr];
                    float x[E];
                    unpack16<T>(*reinterpret_cast<const uint4*>(vst + jr * ROW + vc * 16), x);
                    float* pu = pa[p & 1];
#pragma unroll
                    for (int e = 0; e < E; e += 2) ffma2(pu[e], pu[e + 1], pj, pj, x[e], x[e + 1]);
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += pa[0][e] + pa[1][e];
            // the appended token joins the cache
            const int a = jn - tok0;
            if (append && a >= 0 && a < n) {
                Raw<T, DPL> kr, vr;
                kr.load_shared(reinterpret_cast<const T*>(kst + a * ROW) + lane * DPL);
                vr.load_shared(reinterpret_cast<const T*>(vst + a * ROW) + lane * DPL);
                kr.store(reinterpret_cast<T*>(L.K) + (row0 + a) * D + lane * DPL);
                vr.store(reinterpret_cast<T*>(L.V) + (row0 + a) * D + lane * DPL);
                if (lane == 0) L.pos[row0 + a] = t;
            }
            __syncwarp();  // every lane is done with this stage
            if (ip < c_end) issue(stage, 0);
            if (i + 1 < c_end && pre > i + 1) continue;  // head goes on

            // end of this warp's segment of head hc: add up the row groups
            // and the lanes' denominators
#pragma unroll
            for (int o = G; o < 32; o <<= 1)
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] += __shfl_xor_sync(FULL_MASK, acc[e], o);
            float l = ls;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(FULL_MASK, l, o);
            const size_t hx = hbase + hc;
            if (!(l > 0.f) || isinf(l)) latch_error(L, HKV_ERR_NUMERIC, (int)hx);
            const bool whole = seg0 == first && i + 1 == pre;
            if (whole) {
                const float inv = 1.0f / l;
                float o[E];
#pragma unroll
                for (int e = 0; e < E; ++e) o[e] = acc[e] * inv;
                if (lane < G) store_row<T, E>(o_t + (size_t)hc * D + vc * E, o);
                if (scoring && lane == 0) L.ml[hx * L.r + col] = make_float2(m, l);
            } else {
                const int w_a = range_owner(first, total, GW);
                const int w_b = range_owner(pre - 1, total, GW);
                int segs = 0;
                for (int w = w_a; w <= w_b; ++w)
                    segs += range_begin(w, total, GW) < range_begin(w + 1, total, GW);
                // segments all in this block meet in shared memory, others in
                // global memory; the last one in merges (no waiting)
                const bool local = w_a / NW == (int)blockIdx.x && w_b / NW == (int)blockIdx.x;
                float* pp = local ? lpart + (size_t)(warp * 2 + (seg0 == c_begin ? 0 : 1)) * (D + 2)
                                  : partial + (size_t)seg0 * (D + 2);
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
                    auto part_of = [&](int w) -> const float* {
                        const int rb = range_begin(w, total, GW);
                        if (local)
                            return lpart + (size_t)((w % NW) * 2 + (max(rb, first) == rb ? 0 : 1)) * (D + 2);
                        return partial + (size_t)max(rb, first) * (D + 2);
                    };
                    float M = -INFINITY;
                    for (int w = w_a + lane; w <= w_b; w += 32)
                        if (range_begin(w, total, GW) < range_begin(w + 1, total, GW))
                            M = fmaxf(M, local ? *part_of(w) : __ldcg(part_of(w)));
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL_MASK, M, o));
                    float Ls = 0.f, o[E];
#pragma unroll
                    for (int e = 0; e < E; ++e) o[e] = 0.f;
                    for (int w = w_a; w <= w_b; ++w) {
                        if (range_begin(w, total, GW) >= range_begin(w + 1, total, GW)) continue;
                        const float* pi = part_of(w);
                        if (local) {
                            const float wt = exp2f(pi[0] - M);
                            Ls = fmaf(pi[1], wt, Ls);
#pragma unroll
                            for (int e = 0; e < E; ++e) o[e] = fmaf(pi[2 + vc * E + e], wt, o[e]);
                        } else {
                            const float wt = exp2f(__ldcg(pi) - M);
                            Ls = fmaf(__ldcg(pi + 1), wt, Ls);
#pragma unroll
                            for (int e = 0; e < E; ++e) o[e] = fmaf(__ldcg(pi + 2 + vc * E + e), wt, o[e]);
                        }
                    }
                    const float inv = 1.0f / Ls;
#pragma unroll
                    for (int e = 0; e < E; ++e) o[e] *= inv;
                    if (lane < G) store_row<T, E>(o_t + (size_t)hc * D + vc * E, o);
                    if (scoring && lane == 0) L.ml[hx * L.r + col] = make_float2(M, Ls);
                }
            }
            // next head holding chunk i + 1
            seg0 = i + 1;
            m = -INFINITY;
            ls = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = 0.f;
            if (i + 1 < c_end) {
                do {
                    ++hc;
                    if (hc - cc.base >= 32) cc.load(L, hbase, n_heads, hc);
                    cc.get(hc, slot, len, jn, scoring, pre, first);
                } while (pre <= i + 1);
            }
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
            kr.store(reinterpret_cast<T*>(L.K) + slot * L.d + lane * DPL);
            vr.store(reinterpret_cast<T*>(L.V) + slot * L.d + lane * DPL);
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

DecodeShape decode_shape(const Layout& L, size_t smem_limit) {
    const int es = L.dtype == HKV_DTYPE_F32 ? 4 : 2;
    DecodeShape sh{0, 0, 0};
    for (int ns = MAX_STAGES; ns >= 2 && sh.warps == 0; --ns) {
        // the per-warp tail regions are laid out for MAX_STAGES barriers
        const size_t per = decode_warp_bytes(L.d, es, ns) + (MAX_STAGES - ns) * 8;
        int w = (int)((smem_limit - 1024) / per);
        if (w > 8) w = 8;
        if (w >= (ns == MAX_STAGES ? 6 : 1)) sh = DecodeShape{w, ns, 1024 + (size_t)w * per};
    }
    return sh;
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
                              (const T*)v, (T*)o, append, sh.nstage, early, buf);
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

cudaError_t launch_plan(const Layout& L, int l0, int l1, int ahead, cudaStream_t st) {
    const size_t sm = (size_t)L.S * L.H * sizeof(int32_t);
    plan_kernel<<<l1 - l0, 1024, sm, st>>>(L, l0, ahead);
    return cudaGetLastError();
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
