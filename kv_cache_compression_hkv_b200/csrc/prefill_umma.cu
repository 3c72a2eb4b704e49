// prefill_umma.cu -- causal prefill attention on the 5th-generation tensor
// cores (tcgen05) for bf16 caches (HeadKV technical summary, Methodology
// step 1, cache prefilling: its weights feed step 2, head grouping).
//
// One CTA (4 warps) per (sequence*head block, 128-query tile).  TMA brings
// the Q tile (128 x d) once and the K / V tiles (64 keys x d) per key tile,
// all with the 128-byte swizzle the tensor cores read.  Two passes over the
// key tiles (keys up to the tile's causal limit):
//   pass 1: S = Q K^T (M=128, N=64) into TMEM; thread i owns query row i
//           (TMEM lane i) and keeps its running max and sum;
//   pass 2: S again; P = exp2(S - max) / sum exactly normalised, written as
//           bf16 into shared memory in the canonical K-major layout; the
//           last r query rows also store their fp32 weights for the
//           grouping; O += P V (V as the MN-major operand) in TMEM.
// The epilogue reads O from TMEM and stores bf16 rows.  Every wait on an
// mbarrier is bounded in time; a wait that gives up latches HKV_ERR_TIMEOUT,
// waits (bounded) for the block's own copies, frees TMEM and returns.
#include <cuda.h>
#include <math.h>

#include "hkv_internal.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace hkv {
namespace umma {

constexpr int QT = 128;   // query rows per CTA (MMA M)
constexpr int KT = 64;    // keys per key tile (MMA N of S, K of P V)
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t O_COL = 128;  // O accumulator columns start here; S uses 0..63

using ptx::smem_u32;
using ptx::mbar_init;
using ptx::mbar_expect_tx;
using ptx::mbar_wait;

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
using ptx::fence_proxy_async;

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fff);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3fff) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3fff) << 32;
    d |= (uint64_t)1 << 46;  // version
    d |= (uint64_t)2 << 61;  // SWIZZLE_128B
    return d;
}
// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn_major) {
    return (1u << 4)                     // D fp32
           | (1u << 7) | (1u << 10)      // A, B bf16
           | ((b_mn_major ? 1u : 0u) << 16)
           | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(QT >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

struct Smem {
    // 1024-byte aligned tiles (128B swizzle atoms)
    __host__ __device__ static constexpr int q_bytes(int d) { return QT * d * 2; }
    __host__ __device__ static constexpr int kv_bytes(int d) { return KT * d * 2; }
    __host__ __device__ static constexpr int p_bytes() { return QT * KT * 2; }
    __host__ __device__ static constexpr int total(int d) { return 1024 + q_bytes(d) + 2 * kv_bytes(d) + p_bytes() + 64; }
};

template <int D>
__global__ void __launch_bounds__(128) prefill_attn_umma(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
    const __grid_constant__ CUtensorMap vmap, int P, int r, __nv_bfloat16* __restrict__ out,
    float* __restrict__ rows, int32_t* __restrict__ status) {
    extern __shared__ unsigned char raw[];
    unsigned char* base = reinterpret_cast<unsigned char*>(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
    unsigned char* q_s = base;
    unsigned char* k_s = q_s + Smem::q_bytes(D);
    unsigned char* v_s = k_s + Smem::kv_bytes(D);
    unsigned char* p_s = v_s + Smem::kv_bytes(D);
    uint64_t* bars = reinterpret_cast<uint64_t*>(p_s + Smem::p_bytes());
    uint64_t* bar_q = bars + 0;
    uint64_t* bar_k = bars + 1;
    uint64_t* bar_v = bars + 2;
    uint64_t* bar_m = bars + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int b = blockIdx.x;            // sequence * H + head
    const int q0 = blockIdx.y * QT;      // first query of the tile
    const int n_keys = min(P, q0 + QT);  // causal limit of the tile
    const int nkt = (n_keys + KT - 1) / KT;
    constexpr int NSUB = D / 64;         // 64-column swizzle sub-tiles
    constexpr uint64_t WAIT_NS = 2000000000ull;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_k, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_m, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's lane quarter

    uint32_t ph_k = 0, ph_v = 0, ph_m = 0;
    bool fail = false;
    int pending_k = 0, pending_v = 0, pending_q = 0;

    if (tid == 0) {
        mbar_expect_tx(bar_q, Smem::q_bytes(D));
        for (int s = 0; s < NSUB; ++s) tma_load_3d(q_s + s * QT * 128, &qmap, bar_q, s * 64, q0, b);
    }
    pending_q = 1;

    const float scale = LOG2E / sqrtf((float)D);
    const int row = tid;  // query q0 + row, TMEM lane = row
    const int qpos = q0 + row;
    float m = -INFINITY, l = 0.f;
    constexpr uint32_t IDESC_S = idesc_bf16(KT, false);
    constexpr uint32_t IDESC_O = idesc_bf16(D, true);

    for (int pass = 0; pass < 2 && !fail; ++pass) {
        for (int j = 0; j < nkt; ++j) {
            if (tid == 0) {
                mbar_expect_tx(bar_k, Smem::kv_bytes(D));
                for (int s = 0; s < NSUB; ++s) tma_load_3d(k_s + s * KT * 128, &kmap, bar_k, s * 64, j * KT, b);
                if (pass == 1) {
                    mbar_expect_tx(bar_v, Smem::kv_bytes(D));
                    for (int s = 0; s < NSUB; ++s)
                        tma_load_3d(v_s + s * KT * 128, &vmap, bar_v, s * 64, j * KT, b);
                }
            }
            pending_k = 1;
            pending_v = pass == 1;
            bool ok = true;
            if (pending_q) { ok = mbar_wait(bar_q, 0, WAIT_NS); pending_q = 0; }
            ok = ok && mbar_wait(bar_k, ph_k, WAIT_NS);
            if (ok) { ph_k ^= 1; pending_k = 0; }
            if (__syncthreads_or(!ok)) { fail = true; break; }
            // S = Q K^T
            if (tid == 0) {
                fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qa = smem_u32(q_s) + (kk / 4) * (QT * 128) + (kk % 4) * 32;
                    const uint32_t ka = smem_u32(k_s) + (kk / 4) * (KT * 128) + (kk % 4) * 32;
                    mma_bf16(tmem, sw128_desc(qa, 16, 1024), sw128_desc(ka, 16, 1024), IDESC_S, kk > 0);
                }
                mma_commit(bar_m);
            }
            ok = mbar_wait(bar_m, ph_m, WAIT_NS);
            if (ok) ph_m ^= 1;
            if (__syncthreads_or(!ok)) { fail = true; break; }
            fence_after();
            uint32_t sr[2][32];
            tmem_ld32(t_row + 0, sr[0]);
            tmem_ld32(t_row + 32, sr[1]);
            tmem_ld_wait();
            if (pass == 0) {
                float mx = m;
#pragma unroll
                for (int c = 0; c < KT; ++c) {
                    const int key = j * KT + c;
                    const float s = (key <= qpos && key < P) ? __uint_as_float(sr[c >> 5][c & 31]) * scale : -INFINITY;
                    mx = fmaxf(mx, s);
                }
                float acc = l * exp2f(m - mx);
                if (mx == -INFINITY) acc = 0.f;
#pragma unroll
                for (int c = 0; c < KT; ++c) {
                    const int key = j * KT + c;
                    if (key <= qpos && key < P) acc += exp2f(__uint_as_float(sr[c >> 5][c & 31]) * scale - mx);
                }
                l = acc;
                m = mx;
                fence_before();
                __syncthreads();
                continue;
            }
            // pass 2: exact weights -> bf16 P tile (K-major, 128B swizzle)
            const float inv_l = 1.0f / l;
            const bool keep_row = qpos >= P - r && qpos < P;
            float* rrow = keep_row ? rows + ((size_t)b * r + (qpos - (P - r))) * P : nullptr;
#pragma unroll
            for (int ch = 0; ch < KT / 8; ++ch) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float pv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int c = ch * 8 + e * 2 + u;
                        const int key = j * KT + c;
                        const bool valid = key <= qpos && key < P;
                        pv[u] = valid ? exp2f(__uint_as_float(sr[c >> 5][c & 31]) * scale - m) * inv_l : 0.f;
                        if (rrow && key < P) rrow[key] = pv[u];
                    }
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(pv[0], pv[1]);
                    w[e] = *reinterpret_cast<uint32_t*>(&h2);
                }
                const uint32_t off = row * 128 + ((ch ^ (row & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(p_s) + off),
                             "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                             : "memory");
            }
            fence_proxy_async();
            fence_before();
            ok = mbar_wait(bar_v, ph_v, WAIT_NS);
            if (ok) { ph_v ^= 1; pending_v = 0; }
            if (__syncthreads_or(!ok)) { fail = true; break; }
            // O += P V
            if (tid == 0) {
                fence_after();
#pragma unroll
                for (int kk = 0; kk < KT / 16; ++kk) {
                    const uint32_t pa = smem_u32(p_s) + kk * 32;
                    const uint32_t va = smem_u32(v_s) + kk * 16 * 128;
                    mma_bf16(tmem + O_COL, sw128_desc(pa, 16, 1024), sw128_desc(va, KT * 128, 1024),
                             IDESC_O, (j > 0 || kk > 0));
                }
                mma_commit(bar_m);
            }
            ok = mbar_wait(bar_m, ph_m, WAIT_NS);
            if (ok) ph_m ^= 1;
            if (__syncthreads_or(!ok)) { fail = true; break; }
        }
    }

    if (!fail) {
        // weights of the kept rows past this tile's causal limit are zero
        if (qpos >= P - r && qpos < P)
            for (int key = n_keys; key < P; ++key) rows[((size_t)b * r + (qpos - (P - r))) * P + key] = 0.f;
        fence_after();
        if (out != nullptr) {
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(t_row + O_COL + c0, o);
                tmem_ld_wait();
                if (qpos < P) {
                    __nv_bfloat16* orow = out + ((size_t)b * P + qpos) * D + c0;
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint32_t w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[e + 2 * u]),
                                                                      __uint_as_float(o[e + 2 * u + 1]));
                            w[u] = *reinterpret_cast<uint32_t*>(&h2);
                        }
                        *reinterpret_cast<uint4*>(orow + e) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
        }
    } else {
        if (tid == 0) {
            if (atomicCAS(status, 0, HKV_ERR_TIMEOUT) == 0) atomicExch(status + 1, b);
            // let the block's own copies land before its shared memory is released
            if (pending_q) mbar_wait(bar_q, 0, WAIT_NS);
            if (pending_k) mbar_wait(bar_k, ph_k, WAIT_NS);
            if (pending_v) mbar_wait(bar_v, ph_v, WAIT_NS);
        }
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
}

}  // namespace umma

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [blocks][P rows][d] bf16 with the block stride given in elements; box of
// 64 columns x box_rows rows, 128-byte swizzle, zero fill past P.
static bool make_map(CUtensorMap* m, const void* ptr, int d, int P, int nblk, int64_t block_stride,
                     int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)P, (cuuint64_t)nblk};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)block_stride * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_prefill_umma(const Layout& L, const void* q, const void* k, const void* v, int P,
                                int64_t block_stride, void* out, cudaStream_t st) {
    const int nblk = L.S * L.H;
    CUtensorMap qm, km, vm;
    if (!make_map(&qm, q, L.d, P, nblk, block_stride, umma::QT) ||
        !make_map(&km, k, L.d, P, nblk, block_stride, umma::KT) ||
        !make_map(&vm, v, L.d, P, nblk, block_stride, umma::KT))
        return cudaErrorInvalidValue;
    dim3 grid(nblk, (P + umma::QT - 1) / umma::QT);
    const size_t sm = umma::Smem::total(L.d);
    if (L.d == 128)
        umma::prefill_attn_umma<128><<<grid, 128, sm, st>>>(qm, km, vm, P, L.r, (__nv_bfloat16*)out,
                                                           L.rows, L.status);
    else
        umma::prefill_attn_umma<64><<<grid, 128, sm, st>>>(qm, km, vm, P, L.r, (__nv_bfloat16*)out,
                                                          L.rows, L.status);
    return cudaGetLastError();
}

cudaError_t prepare_prefill_umma(int smem) {
    cudaError_t e = allow_max_dynamic_smem(umma::prefill_attn_umma<128>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(umma::prefill_attn_umma<64>, smem);
    return e;
}

}  // namespace hkv
