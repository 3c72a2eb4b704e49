// kernels.h -- launchers of libhkv's kernels (host side, internal).
#pragma once

#include <cuda_runtime.h>

#include "hkv_internal.cuh"

namespace hkv {


// Raises the dynamic shared-memory limits the kernels of this layout need
// (a host call that must not run inside a stream capture; hkv_create makes it).
cudaError_t prepare_kernels();
cudaError_t prepare_prefill(int smem);
cudaError_t prepare_decode(int smem);
cudaError_t prepare_evict(int smem);
cudaError_t prepare_prefill_umma(int smem);
size_t pack_smem_bytes(int P);
cudaError_t launch_prefill_umma(const Layout& L, const void* q, const void* k, const void* v, int P,
                                int64_t block_stride, void* out, cudaStream_t st);
cudaError_t launch_prefill(const Layout& L, int layer, const void* q, const void* k, const void* v,
                           int P, int64_t block_stride, void* out, cudaStream_t st);
// Sharded heads: attention and labels, with each sequence's Local count of
// the heads held here in n_local[S]; then budgets from the all-shards count
// n_local_total[S] and the compression at classification.
cudaError_t launch_prefill_label(const Layout& L, int layer, const void* q, const void* k,
                                 const void* v, int P, int64_t block_stride, void* out,
                                 int32_t* n_local, cudaStream_t st);
cudaError_t launch_prefill_compress(const Layout& L, int layer, const void* k, const void* v, int P,
                                    int64_t block_stride, const int32_t* n_local_total,
                                    cudaStream_t st);
// Launch shape of the decode kernel: warps per block, pipeline stages per
// warp, dynamic shared memory.
struct DecodeShape {
    int warps, nstage;
    size_t smem;
    int per_sm;    // resident blocks per SM
    int prologue;  // stages a warp fills before its first chunk lands:
                   // 0 one when the block has 8 or more warps, else all;
                   // 1 one; 2 all
    int l2_hint;   // 1: finished warps prefetch the next layer's first chunks into L2
    int head_cost; // cost of a head's end in the plan's balancing (CHUNK_COST per chunk)
    int lone_weight;  // plan weight of a warp alone on its SM sub-partition
};
DecodeShape decode_shape(const Layout& L, size_t smem_limit);
// early: the previous launch in `st` is a decode launch of another layer (the
// plan and cache may then be read before waiting for it); buf: which of the
// two split-K buffer sets to use (consecutive decode launches alternate).
cudaError_t launch_decode(const Layout& L, int layer, const void* q, const void* k, const void* v,
                          void* o, int append, const DecodeShape& sh, int grid, int early, int buf,
                          cudaStream_t st);
// commit: the launch right after an eviction (see plan_kernel)
// after_evict: launched right behind the eviction kernel, which it may
// overlap (see plan_kernel)
cudaError_t launch_plan(const Layout& L, int l0, int l1, int ahead, int commit, cudaStream_t st,
                        int after_evict = 0);
// Shared memory of the plan kernel: four words per head of a layer, two per
// warp of the decode grid (and one more), two bytes per chunk.
inline size_t plan_smem_bytes(int heads_per_layer, int max_chunks) {
    return (size_t)heads_per_layer * 16 + (2 * PLAN_MAX_WARPS + 1) * 4 + ((size_t)max_chunks * 2 + 15) / 16 * 16;
}
cudaError_t launch_prefill_rows_simt(int dtype, int d, int n_blocks, const void* q, const void* k,
                                     const void* v, int P, int64_t block_stride, int r, void* out,
                                     float* rows, cudaStream_t st);
cudaError_t launch_append(const Layout& L, int layer, const void* k, const void* v, cudaStream_t st);
cudaError_t launch_evict(const Layout& L, int l0, int l1, int grid, cudaStream_t st);
// Eviction blocks one SM holds at once (the eviction grid is this times the SMs).
int evict_blocks_per_sm(const Layout& L, int optin);
cudaError_t launch_classify_groups(const float* rows, int n_units, int r, int nq, int n,
                                   const int32_t* partner, int W, double tau, int32_t* n_tau,
                                   uint8_t* label, cudaStream_t st);
cudaError_t launch_classify_rows(const float* rows, int n_rows, int n, int W, double tau,
                                 int32_t* n_tau, uint8_t* label, cudaStream_t st);
cudaError_t launch_select_batch(const float* score, const int32_t* pos, const int32_t* count,
                                const int32_t* t, int n_probs, int n, int D, int k_near, int k_far,
                                int stratified, uint8_t* evict, cudaStream_t st);

}  // namespace hkv
