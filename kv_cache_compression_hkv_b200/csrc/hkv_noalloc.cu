// hkv_noalloc.cu -- prefill attention + head grouping without any device
// allocation, for callers that cannot allocate device memory at all.
//
// The context-based path needs a pool the caller allocates (hkv_pool_bytes
// bytes).  Some callers cannot do that: code that runs while a CUDA graph is
// being captured in global mode (where cudaMalloc is refused), runtimes whose
// caching allocator owns all device memory and forbids raw allocations, and
// real-time or certified processes that may not allocate after start-up.
// This entry point needs no pool: its only scratch (the weights of each
// block's last query, plus a status word) lives in a fixed array compiled
// into the library, which every GPU that loads the library holds until the
// process exits.
#include <string.h>

#include <mutex>

#include "hkv_internal.cuh"
#include "kernels.h"

namespace {

// 8 MiB: 256 bytes of status words, then fp32 weights, n_blocks * P floats.
constexpr size_t kScratchBytes = size_t(8) << 20;
constexpr size_t kStatusBytes = 256;
constexpr size_t kMaxWeights = (kScratchBytes - kStatusBytes) / sizeof(float);
// Longest prefill of the fp32 path: its attention kernel stages 16 (d + P)
// bytes of shared memory per block (198,656 bytes at d = 128).
constexpr int kMaxPrefillF32 = 12288;

static __device__ __align__(256) unsigned char hkv_noalloc_scratch[kScratchBytes];

// Device address of the array, looked up once per device.  In host code the
// array's name is only a stand-in; kernels must get this address.
constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch[kMaxDevices] = {nullptr};

hkv_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HKV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, hkv_noalloc_scratch) != cudaSuccess || !p) return HKV_ERR_CUDA;
        if (hkv::prepare_kernels() != cudaSuccess) return HKV_ERR_CUDA;
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return HKV_OK;
}

}  // namespace

extern "C" hkv_status hkv_prefill_classify_noalloc(int32_t dtype, int32_t head_dim,
                                                   int32_t n_blocks, const void* q, const void* k,
                                                   const void* v, int32_t prefill_len,
                                                   int64_t block_stride, int32_t local_window,
                                                   double tau, void* out, int32_t* n_tau,
                                                   uint8_t* label, int32_t* status, void* stream) {
    const int P = prefill_len;
    if (!q || !k || !v || !n_tau || !label || n_blocks < 1 || P < 1 || local_window < 1 ||
        !(tau > 0.0 && tau <= 1.0) || (head_dim != 64 && head_dim != 128) ||
        (dtype != HKV_DTYPE_F32 && dtype != HKV_DTYPE_BF16))
        return HKV_ERR_INVALID_ARG;
    const int64_t es = dtype == HKV_DTYPE_F32 ? 4 : 2;
    if (block_stride < (int64_t)P * head_dim || (block_stride * es) % 16 != 0) return HKV_ERR_INVALID_ARG;
    if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)out) & 15) return HKV_ERR_INVALID_ARG;
    if (dtype == HKV_DTYPE_F32 && P > kMaxPrefillF32) return HKV_ERR_INVALID_ARG;
    if ((size_t)n_blocks * (size_t)P > kMaxWeights) return HKV_ERR_CAPACITY;  // beyond the array
    void* base = nullptr;
    hkv_status s = scratch_address(&base);
    if (s != HKV_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    int32_t* stat = status ? status : reinterpret_cast<int32_t*>(base);
    float* rows = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + kStatusBytes);
    // the status words start every call at zero; the weights are fully rewritten
    if (cudaMemsetAsync(stat, 0, 8, st) != cudaSuccess) return HKV_ERR_CUDA;
    cudaError_t e;
    if (dtype == HKV_DTYPE_BF16) {
        hkv::Layout L;
        memset(&L, 0, sizeof(L));
        L.S = n_blocks;
        L.H = 1;
        L.d = head_dim;
        L.r = 1;
        L.dtype = dtype;
        L.rows = rows;
        L.status = stat;
        e = hkv::launch_prefill_umma(L, q, k, v, P, block_stride, out, st);
    } else {
        e = hkv::launch_prefill_rows_simt(dtype, head_dim, n_blocks, q, k, v, P, block_stride, 1, out,
                                          rows, st);
    }
    if (e == cudaSuccess) e = hkv::launch_classify_rows(rows, n_blocks, P, local_window, tau, n_tau, label, st);
    return e == cudaSuccess ? HKV_OK : HKV_ERR_CUDA;
}
