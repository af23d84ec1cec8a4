// csa2_index_score_topk_noalloc: the indexer-score + Top-K operation for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or get a workspace from anyone who does): plugins
// and custom layers hosted by an inference engine or framework that owns every device
// allocation and forbids direct cudaMalloc, and latency-critical serving loops where an
// allocation (which may synchronise the device) is not acceptable. This entry point serves
// them with scratch space that lives in a fixed, file-scope device array instead of a
// caller-supplied workspace. The caller still passes every input and output buffer.
//
// The array is kNoallocBytes (16 MiB) and exists on every GPU that loads the library until
// the process exits. Requests whose workspace would exceed it are rejected with
// CSA2_ERR_WORKSPACE before anything is launched. Every call shares the array and it keeps
// the previous call's contents: the operation itself zeroes the histograms and counters it
// relies on, and this wrapper clears the device status word at the start of every call.
// Calls that overlap on the GPU (different streams, or different host threads without
// ordering) race on the array; order them on one stream.
//
// The device address of the array is looked up once per device, with that device current,
// by the first call on that device; make that first call before any stream capture.
#include <mutex>

#include "csa2.h"
#include "csa2_common.cuh"

namespace csa2 {

constexpr size_t kNoallocBytes = (size_t)16 << 20;
constexpr int kMaxDevices = 64;

// Host code must not use this name as a device address: it is a host-side stand-in. The
// address comes from cudaGetSymbolAddress() below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocBytes];

static void* g_scratch_addr[kMaxDevices] = {};
static std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (nullptr on failure).
static void* scratch_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

// OR the call's device status word into the caller's word.
__global__ void noalloc_status_kernel(const int32_t* word, int32_t* out) {
    const int32_t v = *word;
    if (v) atomicOr(out, v);
}

}  // namespace csa2

extern "C" CSA2_API csa2_status_t csa2_index_score_topk_noalloc(
    csa2_mode_t mode, int B, int T, int H_I, csa2_dtype_t qk_dtype, const void* q_I,
    const float* w, const void* k_I, int64_t cap, const int32_t* n_vis0, int ratio,
    const int32_t* q_pos0, int K, const int32_t* pool_in, int P_in, int32_t* pool_out,
    int pool_blocks, int32_t* idx_out, float* scores_out, int32_t* status, void* stream) {
    using namespace csa2;
    if (mode == CSA2_MODE_REUSE)
        return csa2_index_score_topk(mode, B, T, H_I, qk_dtype, q_I, w, k_I, cap, n_vis0, ratio,
                                     q_pos0, K, pool_in, P_in, pool_out, pool_blocks, idx_out,
                                     scores_out, nullptr, 0, stream);
    const int64_t rows = mode == CSA2_MODE_REINDEX ? P_in : cap;
    const size_t need = csa2_workspace_bytes(CSA2_OP_INDEX_SCORE_TOPK, B, T, H_I, rows, K,
                                             pool_out ? pool_blocks : 0);
    if (need == 0) return CSA2_ERR_ARG;
    if (need > kNoallocBytes) return CSA2_ERR_WORKSPACE;
    void* ws = scratch_for_current_device();
    if (!ws) return CSA2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(int32_t), st) != cudaSuccess) return CSA2_ERR_CUDA;
    const csa2_status_t s =
        csa2_index_score_topk(mode, B, T, H_I, qk_dtype, q_I, w, k_I, cap, n_vis0, ratio, q_pos0,
                              K, pool_in, P_in, pool_out, pool_blocks, idx_out, scores_out, ws,
                              kNoallocBytes, stream);
    if (s != CSA2_OK) return s;
    if (status) {
        noalloc_status_kernel<<<1, 1, 0, st>>>(reinterpret_cast<const int32_t*>(ws), status);
        if (cudaGetLastError() != cudaSuccess) return CSA2_ERR_CUDA;
    }
    return CSA2_OK;
}
