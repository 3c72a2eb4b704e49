// decode.cu -- per-step cache append and decode attention over the ragged,
// head-aware compressed cache (HeadKV technical summary: Problem statement;
// Methodology step 3, Local sliding window and Global STE scoring).
//
// Work decomposition: every head's cache is cut into chunks of 32 tokens;
// one warp owns one chunk.  A persistent grid walks the chunk list of the
// layer (chunk counts prefix-summed per block from the device-side lengths,
// so no host sync is needed).  Each warp computes its chunk's logits with a
// lane-transposed reduction (lane j ends with token j's logit), its
// softmax partial (max, sum, weighted V) and either finishes the head (one
// chunk) or leaves a partial; the last warp to arrive for a head (atomic
// ticket, no spinning) merges the partials.  Global heads within r steps of
// their eviction also store their exp2-domain logits per slot, which the
// eviction normalises with the (max, sum) stored here.
#include <math.h>

#include "hkv_internal.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace hkv {

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
        if constexpr (DPL == 4) *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
        else if constexpr (DPL == 2) *reinterpret_cast<uint32_t*>(p) = w[0];
        else {
#pragma unroll
            for (int i = 0; i < DPL / 2; ++i) reinterpret_cast<uint32_t*>(p)[i] = w[i];
        }
    } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) reinterpret_cast<float*>(p)[i] = x[i];
    }
}

// Per-head facts of one decode launch, cached in shared memory by every
// block: inclusive prefix of chunk counts, slot offset in the layer, cache
// length, slot of the appended token (-1: none) and whether the head records
// STE logits this step.
struct HeadTable {
    int32_t* pre;
    int64_t* slot0;
    int16_t* len;
    int16_t* jn;
    uint8_t* scoring;
    __host__ __device__ static size_t bytes(int n) { return (size_t)n * (4 + 8 + 2 + 2 + 1) + 64; }
};

__device__ HeadTable carve_table(unsigned char* p, int n) {
    HeadTable t;
    t.slot0 = reinterpret_cast<int64_t*>(p);
    t.pre = reinterpret_cast<int32_t*>(t.slot0 + n);
    t.len = reinterpret_cast<int16_t*>(t.pre + n);
    t.jn = t.len + n;
    t.scoring = reinterpret_cast<uint8_t*>(t.jn + n);
    return t;
}

// Fills the table (coalesced, independent loads) and prefix-sums the chunk
// counts; returns the layer's chunk count.  Heads past their capacity latch
// HKV_ERR_CAPACITY and get no work.
__device__ int build_table(const Layout& L, int layer, int t, int append, HeadTable tb) {
    __shared__ int wsum[32];
    const int n_heads = L.S * L.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int NW = blockDim.x >> 5;
    const size_t hbase = (size_t)layer * n_heads;
#pragma unroll 4
    for (int i = tid; i < n_heads; i += blockDim.x) {
        const size_t hx = hbase + i;
        const int n = len_at(L, hx, t);
        const int cap = L.cap[hx];
        int c = (n + CHUNK - 1) / CHUNK;
        if (n > cap || n < 1) {
            if (blockIdx.x == 0) latch_error(L, HKV_ERR_CAPACITY, (int)hx);
            c = 0;
        }
        tb.pre[i] = c;
        tb.len[i] = (int16_t)n;
        tb.slot0[i] = (int64_t)region_slot0(L, layer, i / L.H) + L.off[hx];
        tb.jn[i] = (int16_t)(append ? append_slot(L, hx, t, n) : -1);
        tb.scoring[i] = L.label[hx] == 0 && L.mode != HKV_MODE_FULL && n > cap - L.r;
    }
    __syncthreads();
    const int per = (n_heads + blockDim.x - 1) / blockDim.x;
    const int i0 = min(tid * per, n_heads), i1 = min(i0 + per, n_heads);
    int local = 0;
    for (int i = i0; i < i1; ++i) {
        local += tb.pre[i];
        tb.pre[i] = local;
    }
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(FULL_MASK, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NW ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(FULL_MASK, w, o);
            if (lane >= o) w += y;
        }
        wsum[lane] = w;
    }
    __syncthreads();
    const int offset = x - local + (warp ? wsum[warp - 1] : 0);
    for (int i = i0; i < i1; ++i) tb.pre[i] += offset;
    __syncthreads();
    return tb.pre[n_heads - 1];
}

// Head holding chunk c: smallest h with pre[h] > c.
__device__ __forceinline__ int head_of(const int32_t* pre, int n, int c) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] > c) hi = mid; else lo = mid + 1;
    }
    return lo;
}

// First chunk of warp w's range when `total` chunks go to `gw` warps.
__device__ __forceinline__ int range_begin(int w, int total, int gw) {
    return (int)((int64_t)w * total / gw);
}
// Warp whose range holds chunk c.
__device__ __forceinline__ int range_owner(int c, int total, int gw) {
    return (int)(((int64_t)(c + 1) * gw - 1) / total);
}

template <typename T, int DPL>
__global__ void __launch_bounds__(256, 1)
    decode_kernel(Layout L, int layer, const T* __restrict__ q_t, const T* __restrict__ k_t,
                  const T* __restrict__ v_t, T* __restrict__ o_t, int append, int nstage) {
    extern __shared__ __align__(128) unsigned char dsm[];
    const int n_heads = L.S * L.H;
    constexpr int D = DPL * 32;
    constexpr int ROW = D * (int)sizeof(T);           // bytes of one cache row
    constexpr int STAGE = (2 * CHUNK + 1) * ROW;       // K rows, V rows, the query
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NW = blockDim.x >> 5;
    const int t = append ? L.t_next[layer] : L.t_next[layer] - 1;
    const int col = t % L.r;

    unsigned char* stages = dsm;
    uint64_t* bars = reinterpret_cast<uint64_t*>(stages + (size_t)NW * nstage * STAGE);
    float* qbuf = reinterpret_cast<float*>(                     // [NW][D] fp32 queries
        ((uintptr_t)(bars + NW * nstage) + 15) & ~(uintptr_t)15);
    HeadTable tb = carve_table(reinterpret_cast<unsigned char*>(qbuf + NW * D), n_heads);
    const int total = build_table(L, layer, t, append, tb);
    constexpr int NPIECE = ROW / 16;  // 16-byte pieces per row

    const int GW = gridDim.x * NW;
    const int gw = blockIdx.x * NW + warp;
    const int c_begin = total > 0 ? range_begin(gw, total, GW) : 0;
    const int c_end = total > 0 ? range_begin(gw + 1, total, GW) : 0;
    T* Kp = reinterpret_cast<T*>(L.K);
    T* Vp = reinterpret_cast<T*>(L.V);
    const size_t hbase = (size_t)layer * n_heads;
    const float qscale = LOG2E / sqrtf((float)D);
    constexpr uint64_t WAIT_NS = 2000000000ull;

    if (c_begin < c_end) {
        unsigned char* my = stages + (size_t)warp * nstage * STAGE;
        uint64_t* bar = bars + warp * nstage;
        float* myq = qbuf + warp * D;
        if (lane == 0) {
            for (int s = 0; s < nstage; ++s) ptx::mbar_init(bar + s, 1);
            ptx::fence_mbar_init();
        }
        __syncwarp();

        // producer cursor (lane 0 issues): chunk ip of head hp
        int ip = c_begin, hp = head_of(tb.pre, n_heads, c_begin);
        auto issue = [&](int stage) {
            if (lane == 0) {
                const int first = hp ? tb.pre[hp - 1] : 0;
                const int tok0 = (ip - first) * CHUNK;
                const int n = min(CHUNK, (int)tb.len[hp] - tok0);
                const int jn = tb.jn[hp];
                const size_t row0 = (size_t)tb.slot0[hp] + tok0;
                unsigned char* kd = my + (size_t)stage * STAGE;
                unsigned char* vd = kd + CHUNK * ROW;
                unsigned char* qd = vd + CHUNK * ROW;
                uint64_t* b = bar + stage;
                ptx::mbar_expect_tx(b, (uint32_t)(2 * n + 1) * ROW);
                ptx::bulk_g2s(qd, q_t + (size_t)hp * D, ROW, b);
                const int a = jn - tok0;
                if (a >= 0 && a < n) {
                    if (a > 0) {
                        ptx::bulk_g2s(kd, Kp + row0 * D, a * ROW, b);
                        ptx::bulk_g2s(vd, Vp + row0 * D, a * ROW, b);
                    }
                    ptx::bulk_g2s(kd + a * ROW, k_t + (size_t)hp * D, ROW, b);
                    ptx::bulk_g2s(vd + a * ROW, v_t + (size_t)hp * D, ROW, b);
                    if (n - a - 1 > 0) {
                        ptx::bulk_g2s(kd + (a + 1) * ROW, Kp + (row0 + a + 1) * D, (n - a - 1) * ROW, b);
                        ptx::bulk_g2s(vd + (a + 1) * ROW, Vp + (row0 + a + 1) * D, (n - a - 1) * ROW, b);
                    }
                } else {
                    ptx::bulk_g2s(kd, Kp + row0 * D, n * ROW, b);
                    ptx::bulk_g2s(vd, Vp + row0 * D, n * ROW, b);
                }
            }
            ++ip;
            if (ip < c_end && tb.pre[hp] <= ip) hp = head_of(tb.pre, n_heads, ip);
        };
        for (int s = 0; s < nstage && ip < c_end; ++s) issue(s);

        int hc = head_of(tb.pre, n_heads, c_begin);
        int seg0 = c_begin;
        float m = -INFINITY, l = 0.f, acc[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
        bool failed = false;

        for (int i = c_begin; i < c_end; ++i) {
            const int k = i - c_begin;
            const int stage = k % nstage;
            if (!ptx::mbar_wait(bar + stage, (uint32_t)((k / nstage) & 1), WAIT_NS)) {
                failed = true;
                break;
            }
            const int first = hc ? tb.pre[hc - 1] : 0;
            const int tok0 = (i - first) * CHUNK;
            const int len = tb.len[hc];
            const int n = min(CHUNK, len - tok0);
            const unsigned char* kst = my + (size_t)stage * STAGE;
            const unsigned char* vst = kst + CHUNK * ROW;
            if (i == seg0) {
                // a new head: its query, pre-scaled, in fp32 shared memory
                const T* qs = reinterpret_cast<const T*>(vst + CHUNK * ROW);
                Raw<T, DPL> qr;
                qr.load_shared(qs + lane * DPL);
#pragma unroll
                for (int e = 0; e < DPL; ++e) myq[lane * DPL + e] = qr.get(e) * qscale;
                __syncwarp();
            }
            // lane j: dot product of the query with row j, reading the row's
            // 16-byte pieces in a lane-rotated order (no bank conflicts)
            float sl = -INFINITY;
            if (lane < n) {
                const unsigned char* krow = kst + lane * ROW;
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int cc = 0; cc < NPIECE; ++cc) {
                    const int c = (cc + lane) & (NPIECE - 1);
                    const uint4 kw = *reinterpret_cast<const uint4*>(krow + c * 16);
                    if constexpr (sizeof(T) == 2) {
                        const float4 qa = *reinterpret_cast<const float4*>(myq + c * 8);
                        const float4 qb = *reinterpret_cast<const float4*>(myq + c * 8 + 4);
                        a0 = fmaf(qa.x, bf16_lo(kw.x), a0);
                        a1 = fmaf(qa.y, bf16_hi(kw.x), a1);
                        a0 = fmaf(qa.z, bf16_lo(kw.y), a0);
                        a1 = fmaf(qa.w, bf16_hi(kw.y), a1);
                        a0 = fmaf(qb.x, bf16_lo(kw.z), a0);
                        a1 = fmaf(qb.y, bf16_hi(kw.z), a1);
                        a0 = fmaf(qb.z, bf16_lo(kw.w), a0);
                        a1 = fmaf(qb.w, bf16_hi(kw.w), a1);
                    } else {
                        const float4 qa = *reinterpret_cast<const float4*>(myq + c * 4);
                        a0 = fmaf(qa.x, __uint_as_float(kw.x), a0);
                        a1 = fmaf(qa.y, __uint_as_float(kw.y), a1);
                        a0 = fmaf(qa.z, __uint_as_float(kw.z), a0);
                        a1 = fmaf(qa.w, __uint_as_float(kw.w), a1);
                    }
                }
                sl = a0 + a1;
            }
            const int64_t row0 = tb.slot0[hc] + tok0;
            if (tb.scoring[hc] && lane < n) L.logit[(size_t)(row0 + lane) * L.r + col] = sl;
            float cm = sl;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(FULL_MASK, cm, o));
            const float mn = fmaxf(m, cm);
            const float alpha = exp2f(m - mn);
            const float p = lane < n ? exp2f(sl - mn) : 0.f;
            float ps = p;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(FULL_MASK, ps, o);
            l = l * alpha + ps;
            m = mn;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[e] *= alpha;
#pragma unroll
            for (int j = 0; j < CHUNK; ++j) {
                if (j < n) {
                    const float pj = __shfl_sync(FULL_MASK, p, j);
                    Raw<T, DPL> vr;
                    vr.load_shared(reinterpret_cast<const T*>(vst + j * ROW) + lane * DPL);
#pragma unroll
                    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(pj, vr.get(e), acc[e]);
                }
            }
            // the appended token joins the cache
            const int a = tb.jn[hc] - tok0;
            if (a >= 0 && a < n) {
                Raw<T, DPL> kr, vr;
                kr.load_shared(reinterpret_cast<const T*>(kst + a * ROW) + lane * DPL);
                vr.load_shared(reinterpret_cast<const T*>(vst + a * ROW) + lane * DPL);
                kr.store(Kp + (size_t)(row0 + a) * D + lane * DPL);
                vr.store(Vp + (size_t)(row0 + a) * D + lane * DPL);
                if (lane == 0) L.pos[row0 + a] = t;
            }
            __syncwarp();
            if (ip < c_end) {
                ptx::fence_proxy_async();  // this stage's reads before its refill
                issue(stage);
            }
            if (i + 1 < c_end && tb.pre[hc] > i + 1) continue;  // head goes on

            // end of this warp's segment of head hc
            const size_t hx = hbase + hc;
            if (!(l > 0.f) || isinf(l)) latch_error(L, HKV_ERR_NUMERIC, (int)hx);
            const bool whole = seg0 == first && i + 1 == tb.pre[hc];
            if (whole) {
                const float inv = 1.0f / l;
                float o[DPL];
#pragma unroll
                for (int e = 0; e < DPL; ++e) o[e] = acc[e] * inv;
                store_row<T, DPL>(o_t + (size_t)hc * D + lane * DPL, o);
                if (tb.scoring[hc] && lane == 0) L.ml[hx * L.r + col] = make_float2(m, l);
            } else {
                float* pp = L.partial + (size_t)seg0 * (D + 2);
                if (lane == 0) { pp[0] = m; pp[1] = l; }
#pragma unroll
                for (int e = 0; e < DPL; ++e) pp[2 + lane * DPL + e] = acc[e];
                __threadfence();
                const int w_a = range_owner(first, total, GW);
                const int w_b = range_owner(tb.pre[hc] - 1, total, GW);
                int segs = 0;
                for (int w = w_a; w <= w_b; ++w)
                    segs += range_begin(w, total, GW) < range_begin(w + 1, total, GW);
                int prev = 0;
                if (lane == 0) prev = atomicAdd(&L.ticket[hc], 1);
                prev = __shfl_sync(FULL_MASK, prev, 0);
                if (prev == segs - 1) {
                    // last segment in: merge (lane-parallel over segments)
                    __threadfence();
                    if (lane == 0) L.ticket[hc] = 0;
                    float M = -INFINITY;
                    for (int w = w_a + lane; w <= w_b; w += 32) {
                        const int rb = range_begin(w, total, GW);
                        if (rb < range_begin(w + 1, total, GW))
                            M = fmaxf(M, __ldcg(L.partial + (size_t)max(rb, first) * (D + 2)));
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL_MASK, M, o));
                    float Ls = 0.f, o[DPL];
#pragma unroll
                    for (int e = 0; e < DPL; ++e) o[e] = 0.f;
                    for (int w = w_a; w <= w_b; ++w) {
                        const int rb = range_begin(w, total, GW);
                        if (rb >= range_begin(w + 1, total, GW)) continue;
                        const float* pi = L.partial + (size_t)max(rb, first) * (D + 2);
                        const float wt = exp2f(__ldcg(pi) - M);
                        Ls = fmaf(__ldcg(pi + 1), wt, Ls);
#pragma unroll
                        for (int e = 0; e < DPL; ++e) o[e] = fmaf(__ldcg(pi + 2 + lane * DPL + e), wt, o[e]);
                    }
                    const float inv = 1.0f / Ls;
#pragma unroll
                    for (int e = 0; e < DPL; ++e) o[e] *= inv;
                    store_row<T, DPL>(o_t + (size_t)hc * D + lane * DPL, o);
                    if (tb.scoring[hc] && lane == 0) L.ml[hx * L.r + col] = make_float2(M, Ls);
                }
            }
            // next head
            seg0 = i + 1;
            if (i + 1 < c_end) hc = head_of(tb.pre, n_heads, i + 1);
            m = -INFINITY;
            l = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
        }
        if (failed) {
            if (lane == 0) latch_error(L, HKV_ERR_TIMEOUT, (int)(hbase + hc));
            // let this warp's outstanding copies land before the block exits
            for (int k = 0; k < nstage; ++k) {
                const int j = ip - 1 - k;
                if (j < c_begin) break;
                const int kk = j - c_begin;
                ptx::mbar_wait(bar + kk % nstage, (uint32_t)((kk / nstage) & 1), WAIT_NS);
            }
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

// Launch shape of the decode kernel: warps per block and pipeline stages per
// warp that fit the shared memory next to the head table.
struct DecodeShape {
    int warps, nstage;
    size_t smem;
};

static DecodeShape decode_shape(const Layout& L, size_t smem_limit) {
    const size_t row = (size_t)L.d * (L.dtype == HKV_DTYPE_F32 ? 4 : 2);
    const size_t stage = (2 * CHUNK + 1) * row;
    const size_t fixed = HeadTable::bytes(L.S * L.H) + 128;
    DecodeShape sh{0, 0, 0};
    for (int ns = 3; ns >= 2 && sh.warps == 0; --ns) {
        const size_t per = ns * (stage + 8) + (size_t)L.d * 4;
        int w = smem_limit > fixed ? (int)((smem_limit - fixed) / per) : 0;
        if (w > 8) w = 8;
        if (w >= (ns == 3 ? 6 : 1)) sh = DecodeShape{w, ns, fixed + (size_t)w * per};
    }
    return sh;
}

template <typename T, int DPL>
static cudaError_t launch_decode_t(const Layout& L, int layer, const void* q, const void* k,
                                   const void* v, void* o, int append, int grid, cudaStream_t st) {
    static size_t limit = 0;
    if (!limit) {
        int dev = 0, optin = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        limit = (size_t)optin - 256;  // room for the kernel's static shared memory
    }
    const DecodeShape sh = decode_shape(L, limit);
    if (sh.warps == 0) return cudaErrorInvalidConfiguration;
    decode_kernel<T, DPL><<<grid, 32 * sh.warps, sh.smem, st>>>(L, layer, (const T*)q, (const T*)k,
                                                                (const T*)v, (T*)o, append, sh.nstage);
    return cudaGetLastError();
}

cudaError_t launch_decode(const Layout& L, int layer, const void* q, const void* k, const void* v,
                          void* o, int append, int grid, cudaStream_t st) {
    if (L.dtype == HKV_DTYPE_BF16) {
        if (L.d == 64) return launch_decode_t<__nv_bfloat16, 2>(L, layer, q, k, v, o, append, grid, st);
        if (L.d == 128) return launch_decode_t<__nv_bfloat16, 4>(L, layer, q, k, v, o, append, grid, st);
    } else {
        if (L.d == 64) return launch_decode_t<float, 2>(L, layer, q, k, v, o, append, grid, st);
        if (L.d == 128) return launch_decode_t<float, 4>(L, layer, q, k, v, o, append, grid, st);
    }
    return cudaErrorInvalidValue;
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
    return e;
}

}  // namespace hkv
