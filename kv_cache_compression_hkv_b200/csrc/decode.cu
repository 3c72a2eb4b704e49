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

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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
    constexpr int G = PPR;                            // lanes covering one row (PV)
    constexpr int TPI = 32 / G;                       // rows per PV step
    constexpr int RPI = 32 / PPR;                     // rows per copy step
    static_assert(PPR % 8 == 0 && PPR <= 32, "rows are 8, 16 or 32 pieces");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NW = blockDim.x >> 5;
    const int t = append ? L.t_next[layer] : L.t_next[layer] - 1;
    const int col = t % L.r;
    const int GW = gridDim.x * NW;
    const int gw = blockIdx.x * NW + warp;
    const size_t hbase = (size_t)layer * n_heads;
    const size_t lrow = (size_t)layer * L.S * L.R;    // first slot of the layer
    T* Kp = reinterpret_cast<T*>(L.K);
    T* Vp = reinterpret_cast<T*>(L.V);
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
    int* ticket = L.ticket + (size_t)buf * n_heads;
    float* partial = L.partial + (size_t)buf * L.max_chunks * (D + 2);
    if (GW != L.plan_gw) {
        if (early) ptx::grid_dep_wait();
        if (threadIdx.x == 0 && blockIdx.x == 0) latch_error(L, HKV_ERR_STATE, layer);
        return;
    }
    const int32_t* pw = L.plan_warp + (size_t)layer * (PLAN_MAX_WARPS + 1);
    const int c_begin = pw[gw], c_end = pw[gw + 1], total = pw[GW];

    unsigned char* my = dsm + (size_t)warp * nstage * STAGE;
    float* myq = reinterpret_cast<float*>(dsm + (size_t)NW * nstage * STAGE) + warp * (D + CHUNK);
    float* myp = myq + D;  // this chunk's softmax numerators

    if (c_begin < c_end) {
        const int h_begin = L.plan_whead[(size_t)layer * PLAN_MAX_WARPS + gw];
        HeadCache pc, cc;  // producer's and consumer's view of the heads
        pc.load(L, hbase, n_heads, h_begin);
        cc = pc;

        // producer cursor: chunk ip of head hp; lane copies piece pc_ of rows
        // pr_, pr_ + RPI, ...
        int ip = c_begin, hp = h_begin;
        const int pc_ = lane % PPR, pr_ = lane / PPR;
        // Issues the copies of chunk ip into `stage`.  With `prior` (before the
        // wait on the previous launch) the query and the appended row are left
        // out; the returned (head, appended row or -1, query wanted) lets the
        // caller put them in after the wait.
        auto issue = [&](int stage, bool prior) -> int3 {
            int slot, len, jn, sc_, pre, first;
            if (hp - pc.base >= 32) pc.load(L, hbase, n_heads, hp);
            pc.get(hp, slot, len, jn, sc_, pre, first);
            const int tok0 = (ip - first) * CHUNK;
            const int n = min(CHUNK, len - tok0);
            const int a = append ? jn - tok0 : -1;  // appended row within the chunk (or outside)
            const size_t row0 = lrow + slot + tok0;
            unsigned char* kd = my + (size_t)stage * STAGE;
            unsigned char* vd = kd + CHUNK * ROW;
            unsigned char* qd = vd + CHUNK * ROW;
            const T* kf = k_t + (size_t)hp * D + pc_ * E;
            const T* vf = v_t + (size_t)hp * D + pc_ * E;
            const bool needq = ip == first || ip == c_begin;  // the head's first chunk here
            for (int row = pr_; row < n; row += RPI) {
                const bool fresh = row == a;
                if (prior && fresh) continue;
                const T* ks = fresh ? kf : Kp + (row0 + row) * D + pc_ * E;
                const T* vs = fresh ? vf : Vp + (row0 + row) * D + pc_ * E;
                cp_async16(kd + row * ROW + ((pc_ ^ (row & 7)) << 4), ks);
                cp_async16(vd + row * ROW + (pc_ << 4), vs);
            }
            if (!prior && needq)
                for (int c = lane; c < PPR; c += 32) cp_async16(qd + c * 16, q_t + (size_t)hp * D + c * E);
            cp_async_commit();
            const int3 rec = make_int3(hp, (a >= 0 && a < n) ? a : -1, needq);
            ++ip;
            if (ip < c_end && pre <= ip) ++hp;
            while (ip < c_end) {  // skip heads with no chunk (capacity errors)
                if (hp - pc.base >= 32) pc.load(L, hbase, n_heads, hp);
                int s2, l2, j2, c2, p2, f2;
                pc.get(hp, s2, l2, j2, c2, p2, f2);
                if (p2 > ip) break;
                ++hp;
            }
            return rec;
        };
        // prologue: cached rows of the first stages, then the wait, then the
        // query and appended rows of those stages with plain loads
        int3 pro[MAX_STAGES];
        int npro = 0;
#pragma unroll
        for (int s = 0; s < MAX_STAGES; ++s)
            if (s < nstage && ip < c_end) { pro[s] = issue(s, true); npro = s + 1; }
        if (early) ptx::grid_dep_wait();
        ptx::grid_dep_trigger();
        if (lane < PPR) {
            uint4 wq[MAX_STAGES], wk[MAX_STAGES], wv[MAX_STAGES];
#pragma unroll
            for (int s = 0; s < MAX_STAGES; ++s) {
                if (s >= npro) continue;
                const size_t at = (size_t)pro[s].x * D + lane * E;
                if (pro[s].z) wq[s] = *reinterpret_cast<const uint4*>(q_t + at);
                if (pro[s].y >= 0) {
                    wk[s] = *reinterpret_cast<const uint4*>(k_t + at);
                    wv[s] = *reinterpret_cast<const uint4*>(v_t + at);
                }
            }
#pragma unroll
            for (int s = 0; s < MAX_STAGES; ++s) {
                if (s >= npro) continue;
                unsigned char* kd = my + (size_t)s * STAGE;
                unsigned char* vd = kd + CHUNK * ROW;
                if (pro[s].z) *reinterpret_cast<uint4*>(vd + CHUNK * ROW + lane * 16) = wq[s];
                const int a = pro[s].y;
                if (a >= 0) {
                    *reinterpret_cast<uint4*>(kd + a * ROW + ((lane ^ (a & 7)) << 4)) = wk[s];
                    *reinterpret_cast<uint4*>(vd + a * ROW + lane * 16) = wv[s];
                }
            }
        }

        int hc = h_begin;
        int seg0 = c_begin;
        // PV accumulators: lane (vg, vc) = (lane / G, lane % G) sums rows
        // j = vg (mod TPI) of its 16-byte piece vc; the groups are added up once
        // per head
        const int vg = lane / G, vc = lane % G;
        // m: the warp's reference maximum (log2 domain), raised only when a
        // logit passes it by more than RESCALE; ls: this lane's share of the
        // softmax denominator; qv: the pre-scaled query of the current head
        float m = -INFINITY, ls = 0.f, acc[E], qv[D];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
        int slot, len, jn, scoring, pre, first;
        cc.get(hc, slot, len, jn, scoring, pre, first);
        while (pre <= c_begin) {  // heads with no chunk before the first one
            ++hc;
            if (hc - cc.base >= 32) cc.load(L, hbase, n_heads, hc);
            cc.get(hc, slot, len, jn, scoring, pre, first);
        }

        for (int i = c_begin; i < c_end; ++i) {
            const int k = i - c_begin;
            const int stage = k % nstage;
            const int pending = (ip - c_begin) - (k + 1);  // groups issued after this one
            if (pending >= 2) cp_async_wait<2>();
            else if (pending == 1) cp_async_wait<1>();
            else cp_async_wait<0>();
            __syncwarp();
            const int tok0 = (i - first) * CHUNK;
            const int n = min(CHUNK, len - tok0);
            const unsigned char* kst = my + (size_t)stage * STAGE;
            const unsigned char* vst = kst + CHUNK * ROW;
            if (i == seg0) {
                // a new head: every lane reads the whole query (broadcast reads)
                const unsigned char* qs = vst + CHUNK * ROW;
#pragma unroll
                for (int c = 0; c < PPR; ++c) {
                    const uint4 w = *reinterpret_cast<const uint4*>(qs + c * 16);
                    if constexpr (sizeof(T) == 2) {
                        qv[c * 8 + 0] = bf16_lo(w.x) * qscale; qv[c * 8 + 1] = bf16_hi(w.x) * qscale;
                        qv[c * 8 + 2] = bf16_lo(w.y) * qscale; qv[c * 8 + 3] = bf16_hi(w.y) * qscale;
                        qv[c * 8 + 4] = bf16_lo(w.z) * qscale; qv[c * 8 + 5] = bf16_hi(w.z) * qscale;
                        qv[c * 8 + 6] = bf16_lo(w.w) * qscale; qv[c * 8 + 7] = bf16_hi(w.w) * qscale;
                    } else {
                        qv[c * 4 + 0] = __uint_as_float(w.x) * qscale;
                        qv[c * 4 + 1] = __uint_as_float(w.y) * qscale;
                        qv[c * 4 + 2] = __uint_as_float(w.z) * qscale;
                        qv[c * 4 + 3] = __uint_as_float(w.w) * qscale;
                    }
                }
            }
            // lane j: dot product of the query with row j; row j's pieces sit
            // at piece ^ (j & 7), so the lanes of a quarter-warp read 8
            // different bank groups while all reading the same query piece
            float sl = -INFINITY;
            if (lane < n) {
                const unsigned char* krow = kst + lane * ROW;
                const int sw = lane & 7;
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                for (int c = 0; c < PPR; ++c) {
                    const uint4 kw = *reinterpret_cast<const uint4*>(krow + ((c ^ sw) << 4));
                    if constexpr (sizeof(T) == 2) {
                        a0 = fmaf(qv[c * 8 + 0], bf16_lo(kw.x), a0);
                        a1 = fmaf(qv[c * 8 + 1], bf16_hi(kw.x), a1);
                        a2 = fmaf(qv[c * 8 + 2], bf16_lo(kw.y), a2);
                        a3 = fmaf(qv[c * 8 + 3], bf16_hi(kw.y), a3);
                        a0 = fmaf(qv[c * 8 + 4], bf16_lo(kw.z), a0);
                        a1 = fmaf(qv[c * 8 + 5], bf16_hi(kw.z), a1);
                        a2 = fmaf(qv[c * 8 + 6], bf16_lo(kw.w), a2);
                        a3 = fmaf(qv[c * 8 + 7], bf16_hi(kw.w), a3);
                    } else {
                        a0 = fmaf(qv[c * 4 + 0], __uint_as_float(kw.x), a0);
                        a1 = fmaf(qv[c * 4 + 1], __uint_as_float(kw.y), a1);
                        a2 = fmaf(qv[c * 4 + 2], __uint_as_float(kw.z), a2);
                        a3 = fmaf(qv[c * 4 + 3], __uint_as_float(kw.w), a3);
                    }
                }
                sl = (a0 + a1) + (a2 + a3);
            }
            const size_t row0 = lrow + slot + tok0;
            if (scoring && lane < n) L.logit[(row0 + lane) * L.r + col] = sl;
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
            const float p = lane < n ? exp2f(sl - m) : 0.f;
            ls += p;
            // weighted V: p_j parked in shared memory; each lane group reads
            // whole 16-byte pieces of its rows; two accumulator chains
            myp[lane] = p;
            __syncwarp();
            float pa[2][E];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int e = 0; e < E; ++e) pa[u][e] = 0.f;
#pragma unroll
            for (int jb = 0; jb < CHUNK; jb += TPI) {
                const int j = jb + vg;
                if (jb < n && j < n) {
                    const float pj = myp[j];
                    const uint4 vw = *reinterpret_cast<const uint4*>(vst + j * ROW + vc * 16);
                    float* pu = pa[(jb / TPI) & 1];
                    if constexpr (sizeof(T) == 2) {
                        pu[0] = fmaf(pj, bf16_lo(vw.x), pu[0]); pu[1] = fmaf(pj, bf16_hi(vw.x), pu[1]);
                        pu[2] = fmaf(pj, bf16_lo(vw.y), pu[2]); pu[3] = fmaf(pj, bf16_hi(vw.y), pu[3]);
                        pu[4] = fmaf(pj, bf16_lo(vw.z), pu[4]); pu[5] = fmaf(pj, bf16_hi(vw.z), pu[5]);
                        pu[6] = fmaf(pj, bf16_lo(vw.w), pu[6]); pu[7] = fmaf(pj, bf16_hi(vw.w), pu[7]);
                    } else {
                        pu[0] = fmaf(pj, __uint_as_float(vw.x), pu[0]);
                        pu[1] = fmaf(pj, __uint_as_float(vw.y), pu[1]);
                        pu[2] = fmaf(pj, __uint_as_float(vw.z), pu[2]);
                        pu[3] = fmaf(pj, __uint_as_float(vw.w), pu[3]);
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += pa[0][e] + pa[1][e];
            // the appended token joins the cache
            const int a = jn - tok0;
            if (append && a >= 0 && a < n) {
                constexpr int LB = DPL * (int)sizeof(T);  // bytes per lane, within one piece
                const int b = lane * LB;
                Raw<T, DPL> kr, vr;
                kr.load_shared(reinterpret_cast<const T*>(kst + a * ROW + ((((b >> 4) ^ (a & 7)) << 4) | (b & 15))));
                vr.load_shared(reinterpret_cast<const T*>(vst + a * ROW + b));
                kr.store(Kp + (row0 + a) * D + lane * DPL);
                vr.store(Vp + (row0 + a) * D + lane * DPL);
                if (lane == 0) L.pos[row0 + a] = t;
            }
            __syncwarp();
            if (ip < c_end) issue(stage, false);
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
                float* pp = partial + (size_t)seg0 * (D + 2);
                if (lane == 0) { pp[0] = m; pp[1] = l; }
                if (lane < G) {
#pragma unroll
                    for (int e = 0; e < E; ++e) pp[2 + vc * E + e] = acc[e];
                }
                __syncwarp();  // the lanes' partial stores precede lane 0's release
                const int w_a = range_owner(first, total, GW);
                const int w_b = range_owner(pre - 1, total, GW);
                int segs = 0;
                for (int w = w_a; w <= w_b; ++w)
                    segs += range_begin(w, total, GW) < range_begin(w + 1, total, GW);
                int prev = 0;
                if (lane == 0) {
                    // release: this warp's partial before the ticket; acquire:
                    // the other segments' partials for the last one in
                    cuda::atomic_ref<int, cuda::thread_scope_device> tk(ticket[hc]);
                    prev = tk.fetch_add(1, cuda::memory_order_acq_rel);
                }
                prev = __shfl_sync(FULL_MASK, prev, 0);
                __syncwarp();  // lane 0's acquire before every lane's partial loads
                if (prev == segs - 1) {
                    // last segment in: merge (lane-parallel over segments)
                    if (lane == 0) ticket[hc] = 0;
                    float M = -INFINITY;
                    for (int w = w_a + lane; w <= w_b; w += 32) {
                        const int rb = range_begin(w, total, GW);
                        if (rb < range_begin(w + 1, total, GW))
                            M = fmaxf(M, __ldcg(partial + (size_t)max(rb, first) * (D + 2)));
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL_MASK, M, o));
                    float Ls = 0.f, o[E];
#pragma unroll
                    for (int e = 0; e < E; ++e) o[e] = 0.f;
                    for (int w = w_a; w <= w_b; ++w) {
                        const int rb = range_begin(w, total, GW);
                        if (rb >= range_begin(w + 1, total, GW)) continue;
                        const float* pi = partial + (size_t)max(rb, first) * (D + 2);
                        const float wt = exp2f(__ldcg(pi) - M);
                        Ls = fmaf(__ldcg(pi + 1), wt, Ls);
#pragma unroll
                        for (int e = 0; e < E; ++e) o[e] = fmaf(__ldcg(pi + 2 + vc * E + e), wt, o[e]);
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
        cp_async_wait<0>();
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
    const size_t row = (size_t)L.d * (L.dtype == HKV_DTYPE_F32 ? 4 : 2);
    const size_t stage = (2 * CHUNK + 1) * row;
    DecodeShape sh{0, 0, 0};
    for (int ns = 3; ns >= 2 && sh.warps == 0; --ns) {
        const size_t per = ns * stage + (size_t)(L.d + CHUNK) * 4;
        int w = (int)((smem_limit - 1024) / per);
        if (w > 8) w = 8;
        if (w >= (ns == 3 ? 6 : 1)) sh = DecodeShape{w, ns, 1024 + (size_t)w * per};
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
