// prefill_umma.cu -- causal prefill attention on the 5th-generation tensor
// cores (tcgen05) for bf16 caches (HeadKV technical summary, Methodology
// step 1, cache prefilling: its weights feed step 2, head grouping).
//
// One CTA per (sequence*head block, 128-query tile), one pass over the key
// tiles (64 keys each, up to the tile's causal limit) with the work split
// by role: a TMA warp brings the Q tile once and the K / V tiles into three
// or four stages (128-byte swizzle, the layout the tensor cores read); an
// MMA warp issues S = Q K^T (M=128, N=64) into one of two TMEM slots and
// O += P V (V as the MN-major operand) into TMEM accumulators; one or two
// groups of four row warps (thread i of a group owns query row i = TMEM
// lane i; a group takes its share of every S tile's columns and has its
// own O) turn S into bf16 weights P with an online maximum and sum.  The
// tensor cores work on tiles j and j-1 while the rows work on tile j.  The
// epilogue combines the groups, reads O from TMEM and stores bf16 rows, and
// the whole block normalises the fp32 weights of the last r query rows over
// every key for the grouping.  Every wait on an mbarrier is
// bounded in time; a wait that gives up latches HKV_ERR_TIMEOUT, the block
// waits (bounded) for its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <math.h>

#include "hkv_internal.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace hkv {
namespace umma {

constexpr int QT = 128;   // query rows per CTA (MMA M)
constexpr int KT = 64;    // keys per key tile (MMA N of S, K of P V)
constexpr uint32_t O_COL = 128;  // O accumulators start here; S uses 0..127 (two slots)

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

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 2^x by the SFU's approximation (PTX ex2.approx.ftz: relative error about
// 2^-22, results below 2^-126 flushed to zero); the weights it makes are
// rounded to bf16 right after.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Roles of a CTA's warps: NH groups of four row warps own the 128 query
// rows (TMEM lane = row; group g takes columns [g KT / NH, (g + 1) KT / NH)
// of every S tile and has an O accumulator of its own) and do the softmax
// and the epilogue; the next warp's lane 0 issues the TMA copies, the last
// warp's lane 0 the MMAs.  d = 128 has two groups: its shared memory
// allows one CTA per SM, and one row warp per SM sub-partition left the
// softmax latency-bound (about 1.2 of the 1.4 us a key tile took); d = 64
// has one group and two CTAs per SM.
template <int D> struct Roles {
    static constexpr int NH = D == 128 ? 2 : 1;
    static constexpr int ROW_THREADS = 128 * NH;
    static constexpr int PRODUCER_WARP = 4 * NH;
    static constexpr int MMA_WARP = 4 * NH + 1;
    static constexpr int NTHREADS = 32 * (4 * NH + 2);
    static constexpr uint32_t TMEM_COLS = NH == 2 ? 512 : 256;  // S slots, then NH O accumulators
};
// A row's reference maximum (log2 domain) is raised, and O rescaled, only
// when a logit passes it by more than this: the weights stay below 2^16
// (bf16 P and the fp32 sums have range to spare; bf16 rounding is relative,
// so its error does not grow with them).  A rescale waits for the previous
// tile's P V and rewrites O in TMEM; with 8 a quarter of the (warp, tile)
// pairs of Lumina-mGPT-768-shaped inputs rescaled, with 16 a few in a
// thousand.
constexpr float RESCALE = 16.f;

// K / V tiles in flight: key tile j uses stage j % nkv(d).  (S slots in
// TMEM and P tiles have two stages, j % 2.)  With two, a stage came free only
// once P V of its tile was done, and a copy's latency sat in every other
// tile's critical path; three let the copies of tile j + 2 start while
// tiles j and j + 1 are in the tensor cores and the rows, and at d = 128
// (one CTA per SM, shared memory to spare) four cover the HBM latency of a
// head's first query tile, whose K and V are not yet in L2.
__host__ __device__ constexpr int nkv(int d) { return d == 128 ? 4 : 3; }
constexpr int NKV_MAX = 4;

// Barriers of the pipeline.
enum Bar {
    B_Q = 0,
    B_KFULL = 1,                 // +kv stage: K tile landed
    B_VFULL = B_KFULL + NKV_MAX,   // +kv stage: V tile landed
    B_KVFREE = B_VFULL + NKV_MAX,  // +kv stage: P V of its tile done, K and V free
    B_SFULL = B_KVFREE + NKV_MAX,  // +slot: S = Q K^T of the slot's tile in TMEM
    B_SFREE = B_SFULL + 2,       // +slot: the row threads have read that S (ROW_THREADS arrivals)
    B_PFULL = B_SFREE + 2,       // +2 group + p stage: the group's columns of P written, its O
                                 // rescaled (128 arrivals)
    B_PVDONE = B_PFULL + 4,      // +p stage: O += P V of the tile done, P free
    B_XCH = B_PVDONE + 2,        // every row's (max, sum) of each group in shared memory
                                 // (ROW_THREADS arrivals)
    B_COUNT = B_XCH + 1
};

struct Smem {
    // 1024-byte aligned tiles (128B swizzle atoms): Q, K[nkv], V[nkv], P[2]
    __host__ __device__ static constexpr int q_bytes(int d) { return QT * d * 2; }
    __host__ __device__ static constexpr int kv_bytes(int d) { return KT * d * 2; }
    __host__ __device__ static constexpr int p_bytes() { return QT * KT * 2; }
    __host__ __device__ static constexpr int total(int d) {
        return 1024 + q_bytes(d) + 2 * nkv(d) * kv_bytes(d) + 2 * p_bytes() + B_COUNT * 8 + 16 + 3 * QT * 8;
    }
};

// Causal attention of one (block, 128-query tile) in one pass over the key
// tiles, pipelined:
//   producer: K_j, V_j into stage j % NKV once O += P V of tile j-NKV is
//             done;
//   MMA:      S_j = Q K_j^T into TMEM columns 64 (j % 2) (once the rows
//             have read S_{j-2}), then, group by group, O_g += P_{j-1} V_{j-1}
//             over the group's keys into its columns 128 + g d .. (once the
//             group has written its part of P_{j-1}), so the rows' work on
//             tile j overlaps the tensor cores' work on tiles j and j-1;
//   rows:     read their columns of S_j, raise the reference maximum m only
//             when a logit passes it by more than RESCALE (then O_g, once
//             P_{j-1} V_{j-1} is in, is rescaled in TMEM), P_j = exp2(S_j - m)
//             as bf16 into stage j % 2 of P (once P_{j-2} V_{j-2} is done),
//             running sum l.
// Epilogue: per row, M = max of the groups' m and O = sum of O_g 2^(m_g - M)
// over L = sum of l_g 2^(m_g - M), as bf16 rows; the last r rows' fp32
// weights exp2(s - M) / L over every key (their scaled logits were kept in
// `rows` during the pass and are normalised in place by the whole block).
template <int D>
__global__ void __launch_bounds__(Roles<D>::NTHREADS) prefill_attn_umma(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
    const __grid_constant__ CUtensorMap vmap, int P, int r, __nv_bfloat16* __restrict__ out,
    float* __restrict__ rows, int32_t* __restrict__ status) {
    extern __shared__ unsigned char raw[];
    unsigned char* base = reinterpret_cast<unsigned char*>(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
    unsigned char* q_s = base;
    constexpr int NKV = nkv(D);
    unsigned char* k_s = q_s + Smem::q_bytes(D);          // [NKV] stages
    unsigned char* v_s = k_s + NKV * Smem::kv_bytes(D);   // [NKV]
    unsigned char* p_s = v_s + NKV * Smem::kv_bytes(D);   // [2]
    uint64_t* bars = reinterpret_cast<uint64_t*>(p_s + 2 * Smem::p_bytes());
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
    float2* ml_s = reinterpret_cast<float2*>(tmem_slot + 4);  // [QT] kept rows' (max, 1 / sum)
    float2* xch = ml_s + QT;                                  // [2][QT] groups' (max, sum)
    using R = Roles<D>;
    constexpr int NH = R::NH, CW = KT / NH;  // column groups, S columns per group

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the query tiles of one (sequence, head) block are neighbours in the
    // grid, so its K and V tiles are read from HBM once and then from L2;
    // the longest (last) tile first
    const int b = blockIdx.y;                           // sequence * H + head
    const int q0 = (gridDim.x - 1 - blockIdx.x) * QT;   // first query of the tile
    const int n_keys = min(P, q0 + QT);  // causal limit of the tile
    const int nkt = (n_keys + KT - 1) / KT;
    constexpr int NSUB = D / 64;         // 64-column swizzle sub-tiles
    constexpr uint64_t WAIT_NS = 2000000000ull;
    constexpr int KVB = Smem::kv_bytes(D), PB = Smem::p_bytes();

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(R::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            // every other barrier: one arrival, a copy's or a commit's
            const int n = (i == B_SFREE || i == B_SFREE + 1 || i == B_XCH) ? R::ROW_THREADS
                          : (i >= B_PFULL && i < B_PFULL + 4) ? QT : 1;
            mbar_init(bars + i, n);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot;
    bool fail = false;

    if (warp == R::PRODUCER_WARP) {
        // --- TMA producer -------------------------------------------------
        uint32_t issued = 0;    // bit s: kv stage s has a load that may be in flight
        uint32_t last_par = 0;  // bit s: parity of that load's phase
        if (lane == 0) {
            mbar_expect_tx(bars + B_Q, Smem::q_bytes(D));
            for (int sub = 0; sub < NSUB; ++sub)
                tma_load_3d(q_s + sub * QT * 128, &qmap, bars + B_Q, sub * 64, q0, b);
            for (int j = 0; j < nkt && !fail; ++j) {
                const int st = j % NKV, u = j / NKV;
                if (j >= NKV && !mbar_wait(bars + B_KVFREE + st, (u - 1) & 1, WAIT_NS)) { fail = true; break; }
                mbar_expect_tx(bars + B_KFULL + st, KVB);
                for (int sub = 0; sub < NSUB; ++sub)
                    tma_load_3d(k_s + st * KVB + sub * KT * 128, &kmap, bars + B_KFULL + st, sub * 64, j * KT, b);
                mbar_expect_tx(bars + B_VFULL + st, KVB);
                for (int sub = 0; sub < NSUB; ++sub)
                    tma_load_3d(v_s + st * KVB + sub * KT * 128, &vmap, bars + B_VFULL + st, sub * 64, j * KT, b);
                issued |= 1u << st;
                last_par = (last_par & ~(1u << st)) | ((uint32_t)(u & 1) << st);
            }
            if (fail) {
                // the block's own copies land before its shared memory goes
                mbar_wait(bars + B_Q, 0, WAIT_NS);
                for (int st = 0; st < NKV; ++st)
                    if (issued & (1u << st)) {
                        mbar_wait(bars + B_KFULL + st, (last_par >> st) & 1, WAIT_NS);
                        mbar_wait(bars + B_VFULL + st, (last_par >> st) & 1, WAIT_NS);
                    }
            }
        }
    } else if (warp == R::MMA_WARP) {
        // --- MMA issuer ---------------------------------------------------
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16(KT, false);
            constexpr uint32_t IDESC_O = idesc_bf16(D, true);
            int committed = -1;  // last tile whose P V was committed
            int s_issued = -1;   // last tile whose S was committed
            if (!mbar_wait(bars + B_Q, 0, WAIT_NS)) fail = true;
            for (int j = 0; j <= nkt && !fail; ++j) {
                if (j < nkt) {
                    const int st = j & 1, k = j >> 1;           // S slot
                    const int kv = j % NKV, ku = j / NKV;       // K stage
                    if (!mbar_wait(bars + B_KFULL + kv, ku & 1, WAIT_NS)) { fail = true; break; }
                    if (j >= 2 && !mbar_wait(bars + B_SFREE + st, (k - 1) & 1, WAIT_NS)) { fail = true; break; }
                    fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t qa = smem_u32(q_s) + (kk / 4) * (QT * 128) + (kk % 4) * 32;
                        const uint32_t ka = smem_u32(k_s + kv * KVB) + (kk / 4) * (KT * 128) + (kk % 4) * 32;
                        mma_bf16(tmem + st * KT, sw128_desc(qa, 16, 1024), sw128_desc(ka, 16, 1024), IDESC_S,
                                 kk > 0);
                    }
                    mma_commit(bars + B_SFULL + st);
                    s_issued = j;
                }
                if (j >= 1) {
                    const int jp = j - 1, sp = jp & 1, kp = jp >> 1;  // P stage
                    const int kv = jp % NKV, ku = jp / NKV;           // V stage
                    if (!mbar_wait(bars + B_VFULL + kv, ku & 1, WAIT_NS)) { fail = true; break; }
                    // group g's keys of the tile into its own O accumulator,
                    // as soon as the group has written its columns of P
                    bool ok = true;
#pragma unroll
                    for (int g = 0; g < NH; ++g) {
                        if (!mbar_wait(bars + B_PFULL + 2 * g + sp, kp & 1, WAIT_NS)) { ok = false; break; }
                        fence_after();
#pragma unroll
                        for (int kk = g * (CW / 16); kk < (g + 1) * (CW / 16); ++kk) {
                            const uint32_t pa = smem_u32(p_s + sp * PB) + kk * 32;
                            const uint32_t va = smem_u32(v_s + kv * KVB) + kk * 16 * 128;
                            mma_bf16(tmem + O_COL + g * D, sw128_desc(pa, 16, 1024),
                                     sw128_desc(va, KT * 128, 1024), IDESC_O, (jp > 0 || kk > g * (CW / 16)));
                        }
                    }
                    // (on a failed wait the commits still cover what was issued)
                    mma_commit(bars + B_PVDONE + sp);
                    mma_commit(bars + B_KVFREE + kv);
                    committed = jp;
                    if (!ok) { fail = true; break; }
                }
            }
            // the tensor cores finish what was issued before TMEM is freed
            // (a commit covers every MMA issued before it), and the last
            // commit's arrivals land before the shared memory goes
            if (s_issued > committed)
                mbar_wait(bars + B_SFULL + (s_issued & 1), (s_issued >> 1) & 1, WAIT_NS);
            if (committed >= 0) {
                mbar_wait(bars + B_PVDONE + (committed & 1), (committed >> 1) & 1, WAIT_NS);
                mbar_wait(bars + B_KVFREE + committed % NKV, (committed / NKV) & 1, WAIT_NS);
            }
        }
    } else {
        // --- rows: softmax and epilogue ------------------------------------
        const int grp = warp >> 2;             // column group
        const int row = tid & (QT - 1);        // query q0 + row, TMEM lane = row
        const int qpos = q0 + row;
        const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's lane quarter
        const uint32_t o_col = O_COL + grp * D;  // the group's O accumulator
        const float scale = LOG2E / sqrtf((float)D);
        const bool keep_row = qpos >= P - r && qpos < P;
        float* rrow = keep_row ? rows + ((size_t)b * r + (qpos - (P - r))) * P : nullptr;
        // m: the reference maximum of the row over the group's columns
        // (-inf until one of them holds a key at or before the query)
        float m = -INFINITY, l = 0.f;
        // every branch around the warp-wide tcgen05.ld / tcgen05.st below is
        // taken by the whole warp: waits and decisions are warp votes
        for (int j = 0; j < nkt; ++j) {
            const int st = j & 1, k = j >> 1;
            const int kb = j * KT + grp * CW;  // key of the group's first column
            if (__any_sync(FULL_MASK, !mbar_wait(bars + B_SFULL + st, k & 1, WAIT_NS))) { fail = true; break; }
            fence_after();
            uint32_t sr[CW / 32][32];
#pragma unroll
            for (int u = 0; u < CW / 32; ++u) tmem_ld32(t_row + st * KT + grp * CW + u * 32, sr[u]);
            tmem_ld_wait();
            fence_before();
            mbar_arrive(bars + B_SFREE + st);
            // scaled logits and their maximum (eight independent chains and a
            // tree)
            // (no per-key test where every key of the group's slice is at or
            // before every query of the warp and inside P: all but the
            // diagonal tiles)
            const bool whole = kb + CW - 1 <= q0 + (warp & 3) * 32 && kb + CW <= P;
            float x[CW], mx[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
            if (whole) {
#pragma unroll
                for (int c = 0; c < CW; ++c) {
                    x[c] = __uint_as_float(sr[c >> 5][c & 31]) * scale;
                    mx[c & 7] = fmaxf(mx[c & 7], x[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < CW; ++c) {
                    const int key = kb + c;
                    x[c] = (key <= qpos && key < P) ? __uint_as_float(sr[c >> 5][c & 31]) * scale : -INFINITY;
                    mx[c & 7] = fmaxf(mx[c & 7], x[c]);
                }
            }
            const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
            if (rrow) {  // normalised after the pass
                if ((P & 3) == 0) {  // 16-byte rows: whole float4 groups
#pragma unroll
                    for (int c = 0; c < CW; c += 4) {
                        const int key = kb + c;
                        if (key < P)
                            *reinterpret_cast<float4*>(rrow + key) = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < CW; ++c) {
                        const int key = kb + c;
                        if (key < P) rrow[key] = x[c];
                    }
                }
            }
            if (__any_sync(FULL_MASK, mt > m + RESCALE)) {
                // the warp raises its rows' references together (a row whose
                // maximum did not grow keeps m: alpha = 1)
                const float mn = fmaxf(m, mt);
                const float alpha = mn == -INFINITY ? 1.f : exp2f(m - mn);  // 0 while m is -inf
                if (j > 0) {
                    // O holds P V up to tile j-1: rescale it once that is in
                    const int jp = j - 1;
                    if (__any_sync(FULL_MASK, !mbar_wait(bars + B_PVDONE + (jp & 1), (jp >> 1) & 1, WAIT_NS))) {
                        fail = true;
                        break;
                    }
                    fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t o[32];
                        tmem_ld32(t_row + o_col + c0, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(t_row + o_col + c0, o);
                    }
                    tmem_st_wait();
                }
                l *= alpha;
                m = mn;
            }
            // stage st of P is free once P V of tile j-2 is done
            if (j >= 2 && __any_sync(FULL_MASK, !mbar_wait(bars + B_PVDONE + st, (k - 1) & 1, WAIT_NS))) {
                fail = true;
                break;
            }
            // the weights as packed bf16 pairs (the sum over four chains),
            // then the stores into the group's chunks of the swizzled P tile
            const float mb = m == -INFINITY ? 0.f : m;  // every logit is -inf then: weight 0
            uint32_t w[CW / 2];
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c2 = 0; c2 < CW / 2; ++c2) {
                const float p0 = ex2_approx(x[2 * c2] - mb), p1 = ex2_approx(x[2 * c2 + 1] - mb);
                ls[c2 & 3] += p0 + p1;
                __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                w[c2] = *reinterpret_cast<uint32_t*>(&h2);
            }
            l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            unsigned char* pst = p_s + st * PB;
#pragma unroll
            for (int ch = 0; ch < CW / 8; ++ch) {
                const int gch = grp * (CW / 8) + ch;  // 16-byte chunk of the 128-byte row
                const uint32_t off = row * 128 + ((gch ^ (row & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(pst) + off),
                             "r"(w[4 * ch]), "r"(w[4 * ch + 1]), "r"(w[4 * ch + 2]), "r"(w[4 * ch + 3])
                             : "memory");
            }
            fence_proxy_async();
            fence_before();
            mbar_arrive(bars + B_PFULL + 2 * grp + st);
        }
        if (!fail && nkt > 0) {
            const int jl = nkt - 1;
            if (__any_sync(FULL_MASK, !mbar_wait(bars + B_PVDONE + (jl & 1), (jl >> 1) & 1, WAIT_NS)))
                fail = true;
        }
        // The row's maximum and sum over both groups (every row thread
        // arrives once, even after a failed wait, so no wait here depends
        // on a thread that left).
        float M = m, fa = 1.f, fb = 0.f, Lsum = l;
        if constexpr (NH == 2) {
            xch[grp * QT + row] = make_float2(m, l);
            mbar_arrive(bars + B_XCH);
            if (!fail && __any_sync(FULL_MASK, !mbar_wait(bars + B_XCH, 0, WAIT_NS))) fail = true;
            if (!fail) {
                const float2 a = xch[row], c = xch[QT + row];  // group 0 holds key 0: a.x is finite
                M = fmaxf(a.x, c.x);
                fa = exp2f(a.x - M);
                fb = c.x == -INFINITY ? 0.f : exp2f(c.x - M);
                Lsum = a.y * fa + c.y * fb;
            }
        }
        if (!fail) {
            fence_after();
            const float inv_l = 1.0f / Lsum;
            if (rrow && grp == 0) ml_s[row] = make_float2(M, inv_l);  // normalised below, by the whole block
            if (out != nullptr) {
                // group g writes the output columns [g D / NH, (g + 1) D / NH)
#pragma unroll
                for (int c0 = grp * (D / NH); c0 < (grp + 1) * (D / NH); c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(t_row + O_COL + c0, o);
                    if constexpr (NH == 2) {
                        uint32_t o2[32];
                        tmem_ld32(t_row + O_COL + D + c0, o2);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * fa + __uint_as_float(o2[e]) * fb);
                    } else {
                        tmem_ld_wait();
                    }
                    if (qpos < P) {
                        __nv_bfloat16* orow = out + ((size_t)b * P + qpos) * D + c0;
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint32_t w[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[e + 2 * u]) * inv_l,
                                                                          __uint_as_float(o[e + 2 * u + 1]) * inv_l);
                                w[u] = *reinterpret_cast<uint32_t*>(&h2);
                            }
                            *reinterpret_cast<uint4*>(orow + e) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            }
        }
    }
    if (__syncthreads_or(fail)) {
        if (tid == 0 && atomicCAS(status, 0, HKV_ERR_TIMEOUT) == 0) atomicExch(status + 1, b);
    } else {
        // The kept rows' weights over every key, exactly normalised: every
        // thread of the block takes a share of the rows' keys (coalesced,
        // independent loads of the logits the pass stored).  The kept rows
        // of the tile are consecutive rows of `rows`.
        const int k0 = max(q0, P - r), k1 = min(q0 + QT, P);
        if (k0 < k1) {
            float* kr0 = rows + ((size_t)b * r + (k0 - (P - r))) * P;
            if ((P & 3) == 0) {
                const int P4 = P >> 2, total = (k1 - k0) * P4;
#pragma unroll 4
                for (int e = tid; e < total; e += R::NTHREADS) {
                    const int kr = e / P4, key = (e - kr * P4) * 4, qs = k0 + kr;
                    const float2 mi = ml_s[qs - q0];
                    float4* p4 = reinterpret_cast<float4*>(kr0 + (size_t)kr * P + key);
                    float4 x4 = *p4;
                    x4.x = key <= qs ? exp2f(x4.x - mi.x) * mi.y : 0.f;
                    x4.y = key + 1 <= qs ? exp2f(x4.y - mi.x) * mi.y : 0.f;
                    x4.z = key + 2 <= qs ? exp2f(x4.z - mi.x) * mi.y : 0.f;
                    x4.w = key + 3 <= qs ? exp2f(x4.w - mi.x) * mi.y : 0.f;
                    *p4 = x4;
                }
            } else {
                const int total = (k1 - k0) * P;
#pragma unroll 4
                for (int e = tid; e < total; e += R::NTHREADS) {
                    const int kr = e / P, key = e - kr * P, qs = k0 + kr;
                    const float2 mi = ml_s[qs - q0];
                    float* p1 = kr0 + (size_t)kr * P + key;
                    *p1 = key <= qs ? exp2f(*p1 - mi.x) * mi.y : 0.f;
                }
            }
        }
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(R::TMEM_COLS));
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
    if (nblk > 65535) return cudaErrorInvalidValue;
    dim3 grid((P + umma::QT - 1) / umma::QT, nblk);
    const size_t sm = umma::Smem::total(L.d);
    if (L.d == 128)
        umma::prefill_attn_umma<128><<<grid, umma::Roles<128>::NTHREADS, sm, st>>>(qm, km, vm, P, L.r, (__nv_bfloat16*)out,
                                                           L.rows, L.status);
    else
        umma::prefill_attn_umma<64><<<grid, umma::Roles<64>::NTHREADS, sm, st>>>(qm, km, vm, P, L.r, (__nv_bfloat16*)out,
                                                          L.rows, L.status);
    return cudaGetLastError();
}

cudaError_t prepare_prefill_umma(int smem) {
    cudaError_t e = allow_max_dynamic_smem(umma::prefill_attn_umma<128>, smem);
    if (e == cudaSuccess) e = allow_max_dynamic_smem(umma::prefill_attn_umma<64>, smem);
    return e;
}

}  // namespace hkv
