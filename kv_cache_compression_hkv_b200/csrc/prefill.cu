// prefill.cu -- cache prefilling, head grouping and compression at
// classification time (HeadKV technical summary, Methodology steps 1-3).
#include <math.h>

#include "hkv_internal.cuh"
#include "kernels.h"

namespace hkv {

// Eight consecutive elements as floats (p aligned to 16 bytes for bf16,
// 32 bytes for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 w = *reinterpret_cast<const uint4*>(p);
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z); x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}
__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
    float4 a = *reinterpret_cast<const float4*>(p);
    float4 b = *reinterpret_cast<const float4*>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Causal attention over the prefill tokens on CUDA cores, one warp per
// query (Methodology step 1, cache prefilling).  Writes the outputs (if out)
// and the normalised weights of the last r queries into rows[b][i][0..P).
// fp32 arithmetic throughout; used for fp32 caches.
template <typename T>
__global__ void __launch_bounds__(128) prefill_attn_simt(const T* __restrict__ q,
                                                         const T* __restrict__ k,
                                                         const T* __restrict__ v, int P, int d,
                                                         int64_t block_stride, int r,
                                                         T* __restrict__ out,
                                                         float* __restrict__ rows) {
    extern __shared__ float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int i = blockIdx.y * 4 + warp;
    if (i >= P) return;  // whole warp leaves; no block barrier follows
    float* qs = smem + warp * (d + P);
    float* ps = qs + d;
    const T* qb = q + (size_t)b * block_stride;
    const T* kb = k + (size_t)b * block_stride;
    const T* vb = v + (size_t)b * block_stride;
    for (int c = lane; c < d; c += 32) qs[c] = to_float(qb[(size_t)i * d + c]);
    __syncwarp();
    const float scale = 1.0f / sqrtf((float)d);
    float m = -INFINITY;
    for (int j = lane; j <= i; j += 32) {
        const T* kr = kb + (size_t)j * d;
        float acc = 0.f;
        for (int c = 0; c < d; c += 8) {
            float x[8];
            load8(kr + c, x);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(qs[c + e], x[e], acc);
        }
        float s = acc * scale;
        ps[j] = s;
        m = fmaxf(m, s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL_MASK, m, o));
    float l = 0.f;
    for (int j = lane; j <= i; j += 32) {
        float e = expf(ps[j] - m);
        ps[j] = e;
        l += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(FULL_MASK, l, o);
    __syncwarp();
    const float inv_l = 1.0f / l;
    if (out) {
        T* ob = out + ((size_t)b * P + i) * d;
        for (int c = lane; c < d; c += 32) {
            float acc = 0.f;
            for (int j = 0; j <= i; ++j) acc = fmaf(ps[j], to_float(vb[(size_t)j * d + c]), acc);
            from_float(ob[c], acc * inv_l);
        }
    }
    if (i >= P - r) {
        float* row = rows + ((size_t)b * r + (i - (P - r))) * P;
        for (int j = lane; j < P; j += 32) row[j] = j <= i ? ps[j] * inv_l : 0.f;
    }
}

// The other stream of sequence s's classifier-free-guidance pair (s itself
// when grouping is not tied).
__device__ __forceinline__ int cfg_partner(const Layout& L, int s) {
    if (L.pairing == HKV_CFG_HALVES) return s < L.S / 2 ? s + L.S / 2 : s - L.S / 2;
    if (L.pairing == HKV_CFG_ADJACENT) return s ^ 1;
    return s;
}

// Budgets (Main contributions: asymmetric budgets) and the slot layout of
// the heads of (layer, s) held here, from their labels lab[] and the Local
// count nl of the whole (sequence, layer): every shard of its heads.
// Local heads keep W; Global heads split T - nl*W evenly over the
// H_total - nl Global heads, rounded down.  One thread.
__device__ void lay_out_heads(const Layout& L, int layer, int s, int P, const uint8_t* lab,
                              const int32_t* ntau, int nl) {
    const int ng = L.H_total - nl;
    int bg;
    if (L.mode == HKV_MODE_HEADKV) bg = ng > 0 ? (int)((L.T_total - (int64_t)nl * L.W) / ng) : 0;
    else if (L.mode == HKV_MODE_UNIFORM) bg = (int)(L.T_total / L.H_total);
    else bg = L.L;
    int o = 0;
    uint32_t gmask = 0;
    for (int j = 0; j < L.H; ++j) {
        const size_t hi = head_index(L, layer, s, j);
        int cap, budget, len0;
        if (lab[j] == 1) { cap = L.W; budget = L.W; len0 = P < L.W ? P : L.W; }
        else if (lab[j] == 2) { cap = L.L; budget = L.L; len0 = P; }
        else { cap = bg + L.M; budget = bg; len0 = P < bg ? P : bg; gmask |= 1u << j; }
        L.off[hi] = o;
        L.cap[hi] = cap;
        L.budget[hi] = budget;
        L.base[hi] = base_pack(len0, P - 1);
        L.label[hi] = lab[j];
        L.n_tau[hi] = ntau[j];
        o += cap;
    }
    if (o > L.R) latch_error(L, HKV_ERR_CAPACITY, layer * L.S + s);
    // the Global heads of a unit share capacity and length: one due step
    const size_t u = (size_t)layer * L.S + s;
    const int len0_g = P < bg ? P : bg;
    L.unit[u] = make_int4(gmask ? (P - 1) + (bg + L.M - len0_g) : INT32_MAX, (int)gmask, bg, bg + L.M);
    if (s == 0) L.t_next[layer] = P;
}

// Head grouping (Methodology step 2) for one (layer, sequence) per block,
// one warp per head; the backward accumulation runs in double.  With
// n_local == nullptr the budgets and slot layout follow at once from this
// block's own Local count (every head of the sequence is here).  Otherwise
// the labels are stored and n_local[s] receives the Local count of the
// heads held here, for the caller to sum over the shards of the heads.
__global__ void classify_kernel(Layout L, int layer, int P, int32_t* n_local) {
    __shared__ uint8_t lab[32];
    __shared__ int32_t ntau[32];
    const int s = blockIdx.x;
    const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int need = P;
    uint8_t label = 0;
    if (L.mode == HKV_MODE_HEADKV) {
        // the pair's lower sequence first, so both streams sum alike
        const int sp = cfg_partner(L, s), sa = min(s, sp), sb = max(s, sp);
        const size_t blk = (size_t)L.r * P;
        need = warp_group_need_rows(L.rows + (size_t)(sa * L.H + h) * blk,
                                    sb != sa ? L.rows + (size_t)(sb * L.H + h) * blk : nullptr,
                                    L.r, L.nq, P, L.tau);
        label = need < L.W ? 1 : 0;  // fewer tokens than the window: Local
    } else if (L.mode == HKV_MODE_FULL) {
        label = 2;
    }
    if (lane == 0) { lab[h] = label; ntau[h] = need; }
    __syncthreads();
    if (threadIdx.x != 0) return;
    int nl = 0;
    for (int j = 0; j < L.H; ++j) nl += lab[j] == 1;
    if (n_local) {
        for (int j = 0; j < L.H; ++j) {
            const size_t hi = head_index(L, layer, s, j);
            L.label[hi] = lab[j];
            L.n_tau[hi] = ntau[j];
        }
        n_local[s] = nl;
        return;
    }
    lay_out_heads(L, layer, s, P, lab, ntau, nl);
}

// Budgets and slot layout of sharded heads (one block per sequence), once
// the caller has summed the shards' Local counts into n_local_total.  A
// count outside what the labels held here allow latches
// HKV_ERR_INVALID_ARG and is clamped into that range.
__global__ void layout_kernel(Layout L, int layer, int P, const int32_t* __restrict__ n_local_total) {
    __shared__ uint8_t lab[32];
    __shared__ int32_t ntau[32];
    const int s = blockIdx.x;
    if (threadIdx.x < L.H) {
        const size_t hi = head_index(L, layer, s, threadIdx.x);
        lab[threadIdx.x] = L.label[hi];
        ntau[threadIdx.x] = L.n_tau[hi];
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    int here = 0;
    for (int j = 0; j < L.H; ++j) here += lab[j] == 1;
    int nl = n_local_total[s];
    const int hi_bound = here + (L.H_total - L.H);  // every other shard's heads Local
    if (nl < here || nl > hi_bound) {
        latch_error(L, HKV_ERR_INVALID_ARG, layer * L.S + s);
        nl = nl < here ? here : hi_bound;
    }
    lay_out_heads(L, layer, s, P, lab, ntau, nl);
}

// Bytes of the pack kernel's kept-position list, rounded so that the select
// scratch behind it starts 16-byte aligned.
__host__ __device__ inline size_t pack_kept_bytes(int P) { return ((size_t)P * 4 + 15) / 16 * 16; }

// Copies the tokens each head keeps at classification time into its slots
// (Methodology step 3): the last W prefill tokens of a Local head into its
// ring (slot = position mod W); every prefill token of a Global head, or,
// beyond its budget, the survivors of one Stratified Token Eviction scored
// by the last r prefill queries.  One block per head.
template <typename T>
__global__ void __launch_bounds__(128) pack_kernel(Layout L, int layer, const T* __restrict__ k,
                                                   const T* __restrict__ v, int P,
                                                   int64_t block_stride) {
    extern __shared__ __align__(16) unsigned char psm[];
    const int b = blockIdx.x;
    const int s = b / L.H, h = b % L.H;
    const size_t hi = head_index(L, layer, s, h);
    const uint8_t lab = L.label[hi];
    const int budget = L.budget[hi];
    const int d = L.d;
    int32_t* kept = reinterpret_cast<int32_t*>(psm);  // [P] position of each slot
    int n_keep;
    int first = 0;
    if (lab == 1) {
        first = P > L.W ? P - L.W : 0;
        n_keep = P - first;
        for (int i = threadIdx.x; i < n_keep; i += blockDim.x) kept[(first + i) % L.W] = first + i;
    } else if (lab == 2 || P <= budget) {
        n_keep = P;
        for (int i = threadIdx.x; i < n_keep; i += blockDim.x) kept[i] = i;
    } else {
        n_keep = budget;
        if (threadIdx.x < 32) {
            SelectScratch sc = carve_select_scratch(psm + pack_kept_bytes(P), P);
            const float* rb = L.rows + (size_t)b * L.r * P;
            const int r = L.r;
            auto key_of = [&](int i, uint32_t& sb, int32_t& p) {
                float sc_ = 0.f;
                for (int q = 0; q < r; ++q) sc_ += rb[(size_t)q * P + i];
                sb = __float_as_uint(sc_);
                p = i;
            };
            const int E = P - budget;
            warp_stratified_select(sc, P, P - 1, L.D, E / 2, E - E / 2, L.stratified, key_of);
            // survivors in ascending position fill slots 0..budget)
            int o = 0;
            const int lane = threadIdx.x;
            for (int base = 0; base < P; base += 32) {
                const int i = base + lane;
                const bool keep = i < P && !((sc.evict_bits[i >> 5] >> (i & 31)) & 1u);
                const unsigned bal = __ballot_sync(FULL_MASK, keep);
                if (keep) {
                    const int dst = o + __popc(bal & ((1u << lane) - 1u));
                    if (dst < budget) kept[dst] = i;
                }
                o += __popc(bal);
            }
            if (lane == 0 && o != budget) latch_error(L, HKV_ERR_CAPACITY, (int)hi);
        }
    }
    __syncthreads();
    // row copies: 16-byte pieces
    const int piece = 16 / (int)sizeof(T);
    const int per_row = d / piece;
    const size_t slot0 = region_slot0(L, layer, s) + L.off[hi];
    const int n_slots = lab == 1 ? (n_keep < L.W ? n_keep : L.W) : n_keep;
    T* KVp = reinterpret_cast<T*>(L.K);  // slot s: K at 2 d s, V at 2 d s + d
    const T* kb = k + (size_t)b * block_stride;
    const T* vb = v + (size_t)b * block_stride;
    for (int w = threadIdx.x; w < n_slots * per_row; w += blockDim.x) {
        const int slot = w / per_row, c = (w % per_row) * piece;
        const int p = kept[slot];
        *reinterpret_cast<uint4*>(KVp + (slot0 + slot) * 2 * d + c) =
            *reinterpret_cast<const uint4*>(kb + (size_t)p * d + c);
        *reinterpret_cast<uint4*>(KVp + (slot0 + slot) * 2 * d + d + c) =
            *reinterpret_cast<const uint4*>(vb + (size_t)p * d + c);
    }
    for (int i = threadIdx.x; i < n_slots; i += blockDim.x) L.pos[slot0 + i] = kept[i];
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

size_t pack_smem_bytes(int P) { return pack_kept_bytes(P) + select_scratch_bytes(P); }

// Causal prefill attention of every (sequence, head) block; the weights of
// the last r queries land in L.rows.
static cudaError_t launch_attention(const Layout& L, const void* q, const void* k, const void* v,
                                    int P, int64_t block_stride, void* out, cudaStream_t st) {
    const int nb = L.S * L.H;
    dim3 grid(nb, (P + 3) / 4);
    size_t sm = (size_t)4 * (L.d + P) * sizeof(float);
    if (L.dtype == HKV_DTYPE_F32) {
        // fp32 caches keep fp32 products: CUDA cores
        prefill_attn_simt<float><<<grid, 128, sm, st>>>(
            (const float*)q, (const float*)k, (const float*)v, P, L.d, block_stride, L.r,
            (float*)out, L.rows);
        return cudaGetLastError();
    }
    // bf16 caches: tcgen05 tensor cores
    return launch_prefill_umma(L, q, k, v, P, block_stride, out, st);
}

// Compression at classification time: each head's kept prefill tokens into
// its slots.
static cudaError_t launch_pack(const Layout& L, int layer, const void* k, const void* v, int P,
                               int64_t block_stride, cudaStream_t st) {
    const int nb = L.S * L.H;
    size_t psm = pack_smem_bytes(P);
    if (L.dtype == HKV_DTYPE_F32)
        pack_kernel<float><<<nb, 128, psm, st>>>(L, layer, (const float*)k, (const float*)v, P,
                                                  block_stride);
    else
        pack_kernel<__nv_bfloat16><<<nb, 128, psm, st>>>(
            L, layer, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, P, block_stride);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const Layout& L, int layer, const void* q, const void* k, const void* v,
                           int P, int64_t block_stride, void* out, cudaStream_t st) {
    cudaError_t e = launch_attention(L, q, k, v, P, block_stride, out, st);
    if (e != cudaSuccess) return e;
    classify_kernel<<<L.S, 32 * L.H, 0, st>>>(L, layer, P, nullptr);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_pack(L, layer, k, v, P, block_stride, st);
}

cudaError_t launch_prefill_label(const Layout& L, int layer, const void* q, const void* k,
                                 const void* v, int P, int64_t block_stride, void* out,
                                 int32_t* n_local, cudaStream_t st) {
    cudaError_t e = launch_attention(L, q, k, v, P, block_stride, out, st);
    if (e != cudaSuccess) return e;
    classify_kernel<<<L.S, 32 * L.H, 0, st>>>(L, layer, P, n_local);
    return cudaGetLastError();
}

cudaError_t launch_prefill_compress(const Layout& L, int layer, const void* k, const void* v, int P,
                                    int64_t block_stride, const int32_t* n_local_total,
                                    cudaStream_t st) {
    layout_kernel<<<L.S, 32, 0, st>>>(L, layer, P, n_local_total);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_pack(L, layer, k, v, P, block_stride, st);
}

// CUDA-core causal prefill of n_blocks caller blocks writing the weights of
// their last r queries to `rows` ([n_blocks][r][P] fp32) and, if out is not
// null, the outputs.  Used by the allocation-free entry point.
cudaError_t launch_prefill_rows_simt(int dtype, int d, int n_blocks, const void* q, const void* k,
                                     const void* v, int P, int64_t block_stride, int r, void* out,
                                     float* rows, cudaStream_t st) {
    dim3 grid(n_blocks, (P + 3) / 4);
    const size_t sm = (size_t)4 * (d + P) * sizeof(float);
    if (dtype == HKV_DTYPE_F32)
        prefill_attn_simt<float><<<grid, 128, sm, st>>>((const float*)q, (const float*)k,
                                                         (const float*)v, P, d, block_stride, r,
                                                         (float*)out, rows);
    else
        prefill_attn_simt<__nv_bfloat16><<<grid, 128, sm, st>>>(
            (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, P, d,
            block_stride, r, (__nv_bfloat16*)out, rows);
    return cudaGetLastError();
}

cudaError_t prepare_prefill(int smem) {
    cudaError_t e = allow_max_dynamic_smem(prefill_attn_simt<float>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(pack_kernel<float>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(prefill_attn_simt<__nv_bfloat16>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(pack_kernel<__nv_bfloat16>, smem);
    return e;
}

}  // namespace hkv
