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

// Block-wide inclusive prefix of the chunk counts of all heads of a layer
// into pre[0..n_heads).  Heads whose length exceeds their capacity latch
// HKV_ERR_CAPACITY and contribute no work.
__device__ int chunk_prefix(const Layout& L, int layer, int t, int32_t* pre) {
    __shared__ int wsum[32];
    const int n_heads = L.S * L.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int NW = blockDim.x >> 5;
    const size_t hbase = (size_t)layer * n_heads;
    // chunk counts, coalesced (independent iterations: loads overlap)
#pragma unroll 4
    for (int i = tid; i < n_heads; i += blockDim.x) {
        const size_t hx = hbase + i;
        const int n = len_at(L, hx, t);
        int c = (n + CHUNK - 1) / CHUNK;
        if (n > L.cap[hx] || n < 0) {
            if (blockIdx.x == 0) latch_error(L, HKV_ERR_CAPACITY, (int)hx);
            c = 0;
        }
        pre[i] = c;
    }
    __syncthreads();
    // block-wide inclusive scan: contiguous runs per thread, then the warps
    const int per = (n_heads + blockDim.x - 1) / blockDim.x;
    const int i0 = min(tid * per, n_heads), i1 = min(i0 + per, n_heads);
    int local = 0;
    for (int i = i0; i < i1; ++i) {
        local += pre[i];
        pre[i] = local;
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
    for (int i = i0; i < i1; ++i) pre[i] += offset;
    __syncthreads();
    return pre[n_heads - 1];
}

template <typename T, int DPL>
__global__ void __launch_bounds__(256, 1)
    decode_kernel(Layout L, int layer, const T* __restrict__ q_t, const T* __restrict__ k_t,
                  const T* __restrict__ v_t, T* __restrict__ o_t, int append) {
    extern __shared__ int32_t pre[];
    const int n_heads = L.S * L.H;
    const int d = L.d;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NW = blockDim.x >> 5;
    const int t = append ? L.t_next[layer] : L.t_next[layer] - 1;
    const int total = chunk_prefix(L, layer, t, pre);
    const size_t hbase = (size_t)layer * n_heads;
    const float qscale = LOG2E / sqrtf((float)d);
    T* Kp = reinterpret_cast<T*>(L.K);
    T* Vp = reinterpret_cast<T*>(L.V);
    const int col = t % L.r;

    for (int cid = blockIdx.x * NW + warp; cid < total; cid += gridDim.x * NW) {
        int lo = 0, hi = n_heads - 1;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] > cid) hi = mid; else lo = mid + 1;
        }
        const int h = lo;  // s * H + head
        const int c0 = h ? pre[h - 1] : 0;
        const int c = cid - c0;
        const size_t hx = hbase + h;
        const int len = len_at(L, hx, t);
        const int nch = (len + CHUNK - 1) / CHUNK;
        const int s = h / L.H;
        const size_t slot0 = region_slot0(L, layer, s) + L.off[hx];
        const int jn = append ? append_slot(L, hx, t, len) : -1;
        const int tok0 = c * CHUNK;
        const int n = min(CHUNK, len - tok0);
        const bool scoring = L.label[hx] == 0 && L.mode != HKV_MODE_FULL && len > L.cap[hx] - L.r;

        float qv[DPL];
        {
            Raw<T, DPL> qr;
            qr.load(q_t + (size_t)h * d + lane * DPL);
#pragma unroll
            for (int i = 0; i < DPL; ++i) qv[i] = qr.get(i) * qscale;
        }
        // issue every load of the chunk first
        Raw<T, DPL> kr[CHUNK], vr[CHUNK];
#pragma unroll
        for (int j = 0; j < CHUNK; ++j) {
            const int sj = tok0 + j;
            if (j < n) {
                const T* kp = sj == jn ? k_t + (size_t)h * d : Kp + (slot0 + sj) * d;
                const T* vp = sj == jn ? v_t + (size_t)h * d : Vp + (slot0 + sj) * d;
                kr[j].load(kp + lane * DPL);
                vr[j].load(vp + lane * DPL);
            } else {
                kr[j].zero();
                vr[j].zero();
            }
        }
        // partial dot products, then the lane-transposed butterfly sum:
        // afterwards part[0] on lane j holds the logit of token j.
        float part[CHUNK];
#pragma unroll
        for (int j = 0; j < CHUNK; ++j) {
            float a = 0.f;
#pragma unroll
            for (int i = 0; i < DPL; ++i) a = fmaf(qv[i], kr[j].get(i), a);
            part[j] = a;
        }
#pragma unroll
        for (int w = 16; w >= 1; w >>= 1) {
            const bool upper = lane & w;
#pragma unroll
            for (int i = 0; i < w; ++i) {
                const float send = upper ? part[i] : part[i + w];
                const float keep = upper ? part[i + w] : part[i];
                part[i] = keep + __shfl_xor_sync(FULL_MASK, send, w);
            }
        }
        const float sl = lane < n ? part[0] : -INFINITY;
        if (scoring && lane < n) L.logit[(slot0 + tok0 + lane) * L.r + col] = sl;
        float m = sl;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL_MASK, m, o));
        const float p = lane < n ? exp2f(sl - m) : 0.f;
        float l = p;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(FULL_MASK, l, o);
        float acc[DPL];
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
#pragma unroll
        for (int j = 0; j < CHUNK; ++j) {
            const float pj = __shfl_sync(FULL_MASK, p, j);
#pragma unroll
            for (int i = 0; i < DPL; ++i) acc[i] = fmaf(pj, vr[j].get(i), acc[i]);
            if (tok0 + j == jn) {  // the appended token joins the cache
                kr[j].store(Kp + (slot0 + jn) * d + lane * DPL);
                vr[j].store(Vp + (slot0 + jn) * d + lane * DPL);
                if (lane == 0) L.pos[slot0 + jn] = t;
            }
        }
        if (!(l > 0.f) || isinf(l)) latch_error(L, HKV_ERR_NUMERIC, (int)hx);
        if (nch == 1) {
            const float inv = 1.0f / l;
            float o[DPL];
#pragma unroll
            for (int i = 0; i < DPL; ++i) o[i] = acc[i] * inv;
            store_row<T, DPL>(o_t + (size_t)h * d + lane * DPL, o);
            if (scoring && lane == 0) L.ml[hx * L.r + col] = make_float2(m, l);
            continue;
        }
        float* pp = L.partial + (size_t)cid * (d + 2);
        if (lane == 0) { pp[0] = m; pp[1] = l; }
#pragma unroll
        for (int i = 0; i < DPL; ++i) pp[2 + lane * DPL + i] = acc[i];
        __threadfence();
        int prev = 0;
        if (lane == 0) prev = atomicAdd(&L.ticket[h], 1);
        prev = __shfl_sync(FULL_MASK, prev, 0);
        if (prev != nch - 1) continue;
        // last arrival for this head: merge the partials
        __threadfence();
        if (lane == 0) L.ticket[h] = 0;
        const float* pb = L.partial + (size_t)c0 * (d + 2);
        // (max, sum) of the partials, lane-parallel; then the weighted sum
        float M = -INFINITY;
        for (int i = lane; i < nch; i += 32) M = fmaxf(M, __ldcg(pb + (size_t)i * (d + 2)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL_MASK, M, o));
        float Ls = 0.f;
        for (int i = lane; i < nch; i += 32)
            Ls += __ldcg(pb + (size_t)i * (d + 2) + 1) * exp2f(__ldcg(pb + (size_t)i * (d + 2)) - M);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(FULL_MASK, Ls, o);
        float o[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[e] = 0.f;
#pragma unroll 4
        for (int i = 0; i < nch; ++i) {
            const float* pi = pb + (size_t)i * (d + 2);
            const float w = exp2f(__ldcg(pi) - M);
            float a[DPL];
#pragma unroll
            for (int e = 0; e < DPL; ++e) a[e] = __ldcg(pi + 2 + lane * DPL + e);
#pragma unroll
            for (int e = 0; e < DPL; ++e) o[e] = fmaf(a[e], w, o[e]);
        }
        const float inv = 1.0f / Ls;
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[e] *= inv;
        store_row<T, DPL>(o_t + (size_t)h * d + lane * DPL, o);
        if (scoring && lane == 0) L.ml[hx * L.r + col] = make_float2(M, Ls);
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

template <typename T, int DPL>
static cudaError_t launch_decode_t(const Layout& L, int layer, const void* q, const void* k,
                                   const void* v, void* o, int append, int grid, cudaStream_t st) {
    const size_t sm = (size_t)L.S * L.H * sizeof(int32_t);
    decode_kernel<T, DPL><<<grid, 256, sm, st>>>(L, layer, (const T*)q, (const T*)k, (const T*)v,
                                                 (T*)o, append);
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
