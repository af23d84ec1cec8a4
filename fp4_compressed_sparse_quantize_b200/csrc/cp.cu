// Context parallelism for long contexts: every GPU owns a contiguous range (a shard) of each
// sequence's compressed entries, scans it with the ordinary Full-mode indexer and keeps its
// own Top-K and candidate pool. These kernels turn a shard's selections into candidate lists
// with global indices, merge the lists gathered from all shards (e.g. by an NCCL all-gather)
// into the exact global Top-K, and expand merged pool blocks into entry positions.
//
// "DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale LLM Serving", Compressed Sparse
// Attention 2 (CSA2): a Full layer scores every visible compressed entry and keeps the
// highest (512); the decoder's Hierarchical Sparse Indexer keeps a candidate pool of the
// 2,048 blocks of 8 positions with the highest block maxima. Both selections are decomposable: an entry in the global Top-K is in its shard's
// Top-K, and a block in the global pool is in its shard's pool, as long as shards start at
// multiples of 8. The order (score descending, index ascending) is a total order, so the
// merge reproduces the single-GPU result exactly when every shard scores its entries the
// same way the single-GPU scan does (it does: a score depends only on its own entry).
#include <climits>
#include <cstdint>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

constexpr int kCpThreads = 1024;
constexpr int kCpMaxCand = 16384;  // candidates per row the merge accepts (8 x 2,048 pool blocks)

// exclusive prefix sum of v over the CTA (blockDim.x == kCpThreads); *total gets the sum
__device__ __forceinline__ int cp_excl_scan(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        warp_sums[lane] = s;   // inclusive over warps
    }
    __syncthreads();
    const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
    *total = warp_sums[31];
    __syncthreads();   // warp_sums may be reused by the caller's next scan
    return before;
}

// (score, global index) of every selected entry of a shard's Top-K list; -1 entries give
// (0, -1).
__global__ void __launch_bounds__(256) cp_topk_candidates_kernel(
    const float* scores, int64_t ld, const int32_t* idx, int K,
    int64_t offset, float* __restrict__ cand_score, int32_t* __restrict__ cand_idx) {
    grid_dep_launch();
    grid_dep_wait();
    const int64_t r = blockIdx.x;
    for (int i = threadIdx.x; i < K; i += blockDim.x) {
        const int32_t j = idx[r * K + i];
        float s = 0.f;
        int32_t g = -1;
        if (j >= 0) {
            s = scores[r * ld + j];
            g = (int32_t)(offset + j);
        }
        cand_score[r * K + i] = s;
        cand_idx[r * K + i] = g;
    }
}

// (block maximum, global block) of every block of a shard's pool (positions ascending, all
// visible positions of a chosen block present, -1 padded); at most nb blocks per row, the
// rest of the row is (0, -1).
__global__ void __launch_bounds__(kCpThreads) cp_pool_candidates_kernel(
    const float* scores, int64_t ld, const int32_t* pool, int P,
    int nb, int64_t offset, float* __restrict__ cand_bmax, int32_t* __restrict__ cand_block) {
    __shared__ int warp_sums[32];
    grid_dep_launch();
    grid_dep_wait();
    const int64_t r = blockIdx.x;
    const int32_t* pr = pool + r * P;
    int base = 0;
    for (int i0 = 0; i0 < P; i0 += kCpThreads) {
        const int i = i0 + (int)threadIdx.x;
        const int32_t p = i < P ? pr[i] : -1;
        const int32_t prev = (i > 0 && i < P) ? pr[i - 1] : -1;
        const bool start = p >= 0 && (prev < 0 || (prev >> 3) != (p >> 3));
        int total;
        const int slot = base + cp_excl_scan(start ? 1 : 0, warp_sums, &total);
        if (start && slot < nb) {
            float m = scores[r * ld + p];
            for (int k = i + 1; k < P && k < i + 8; ++k) {
                const int32_t q = pr[k];
                if (q < 0 || (q >> 3) != (p >> 3)) break;
                m = fmaxf(m, scores[r * ld + q]);
            }
            cand_bmax[r * nb + slot] = m;
            cand_block[r * nb + slot] = (int32_t)((offset >> 3) + (p >> 3));
        }
        base += total;
    }
    for (int i = base + (int)threadIdx.x; i < nb; i += kCpThreads) {
        cand_bmax[r * nb + i] = 0.f;
        cand_block[r * nb + i] = -1;
    }
}

// The K best candidates of a row by (score descending, index ascending), written in
// ascending index order and -1 padded. Candidates are sorted as unique 64-bit keys
// (order-preserving score bits, then the complemented index) by a bitonic network in shared
// memory; the chosen indices are sorted again, ascending.
__global__ void __launch_bounds__(kCpThreads) cp_merge_kernel(
    const float* cand_score, const int32_t* cand_idx, int n_cand,
    int n2, int K, int k2, int32_t* __restrict__ idx_out) {
    extern __shared__ __align__(16) uint64_t key[];   // [n2], then uint32 [k2]
    uint32_t* sel = reinterpret_cast<uint32_t*>(key + n2);
    grid_dep_launch();
    grid_dep_wait();
    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    for (int i = tid; i < n2; i += kCpThreads) {
        uint64_t v = 0ull;   // no candidate: below every real key
        if (i < n_cand) {
            const int32_t g = cand_idx[r * n_cand + i];
            if (g >= 0)
                v = ((uint64_t)score_key(cand_score[r * n_cand + i]) << 32) |
                    (uint64_t)(0xFFFFFFFFu - (uint32_t)g);
        }
        key[i] = v;
    }
    __syncthreads();
    // descending bitonic sort
    for (int k = 2; k <= n2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < n2; i += kCpThreads) {
                const int l = i ^ j;
                if (l > i) {
                    const uint64_t a = key[i], b = key[l];
                    const bool desc = (i & k) == 0;
                    if (desc ? (a < b) : (a > b)) {
                        key[i] = b;
                        key[l] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = tid; i < k2; i += kCpThreads) {
        const uint64_t v = i < K ? key[i] : 0ull;
        sel[i] = v ? 0xFFFFFFFFu - (uint32_t)v : 0xFFFFFFFFu;   // no candidate sorts last
    }
    __syncthreads();
    // ascending bitonic sort of the chosen indices
    for (int k = 2; k <= k2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < k2; i += kCpThreads) {
                const int l = i ^ j;
                if (l > i) {
                    const uint32_t a = sel[i], b = sel[l];
                    const bool asc = (i & k) == 0;
                    if (asc ? (a > b) : (a < b)) {
                        sel[i] = b;
                        sel[l] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = tid; i < K; i += kCpThreads)
        idx_out[r * K + i] = sel[i] == 0xFFFFFFFFu ? -1 : (int32_t)sel[i];
}

// Entry positions of merged pool blocks (ascending, -1 padded): block b gives the visible
// positions among 8b .. 8b+7.
__global__ void __launch_bounds__(kCpThreads) cp_pool_expand_kernel(
    const int32_t* blocks, int nb, const int32_t* n_row, int P,
    int32_t* __restrict__ pool_out) {
    __shared__ int warp_sums[32];
    grid_dep_launch();
    grid_dep_wait();
    const int64_t r = blockIdx.x;
    const int64_t nv = n_row ? (int64_t)n_row[r] : INT64_MAX;
    int base = 0;
    for (int i0 = 0; i0 < nb; i0 += kCpThreads) {
        const int i = i0 + (int)threadIdx.x;
        const int32_t b = i < nb ? blocks[r * nb + i] : -1;
        int cnt = 0;
        if (b >= 0) {
            const int64_t left = nv - 8 * (int64_t)b;
            cnt = left <= 0 ? 0 : (left >= 8 ? 8 : (int)left);
        }
        int total;
        const int at = base + cp_excl_scan(cnt, warp_sums, &total);
        for (int c = 0; c < cnt && at + c < P; ++c) pool_out[r * P + at + c] = 8 * b + c;
        base += total;
    }
    for (int i = base + (int)threadIdx.x; i < P; i += kCpThreads) pool_out[r * P + i] = -1;
}

// Global selected indices -> this shard's local indices (-1 outside [lo, hi)), for the
// shard's partial attention over the rows it holds.
__global__ void __launch_bounds__(256) cp_local_idx_kernel(const int32_t* idx,
                                                           int64_t n, int64_t lo, int64_t hi,
                                                           int32_t* __restrict__ out) {
    grid_dep_launch();
    grid_dep_wait();
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t v = idx[i];
        out[i] = (v >= lo && v < hi) ? (int32_t)(v - lo) : -1;
    }
}

static int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

}  // namespace csa2

using namespace csa2;

extern "C" {

CSA2_API csa2_status_t csa2_cp_topk_candidates(int rows, const float* scores, int64_t ld_scores,
                                               const int32_t* idx, int K, int64_t offset,
                                               float* cand_score, int32_t* cand_idx,
                                               void* stream) {
    if (rows < 1 || K < 1 || ld_scores < 1 || offset < 0) return CSA2_ERR_ARG;
    if (!scores || !idx || !cand_score || !cand_idx) return CSA2_ERR_ARG;
    if (offset + ld_scores > (int64_t)INT_MAX) return CSA2_ERR_UNSUPPORTED;
    const cudaError_t e = launch_pdl(cp_topk_candidates_kernel, dim3((unsigned)rows), dim3(256), 0,
                                     reinterpret_cast<cudaStream_t>(stream), scores, ld_scores,
                                     idx, K, offset, cand_score, cand_idx);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

CSA2_API csa2_status_t csa2_cp_pool_candidates(int rows, const float* scores, int64_t ld_scores,
                                               const int32_t* pool, int P, int max_blocks,
                                               int64_t offset, float* cand_bmax,
                                               int32_t* cand_block, void* stream) {
    if (rows < 1 || P < 1 || max_blocks < 1 || ld_scores < 1 || offset < 0 || (offset & 7))
        return CSA2_ERR_ARG;
    if (!scores || !pool || !cand_bmax || !cand_block) return CSA2_ERR_ARG;
    if (offset + ld_scores > (int64_t)INT_MAX) return CSA2_ERR_UNSUPPORTED;
    const cudaError_t e = launch_pdl(cp_pool_candidates_kernel, dim3((unsigned)rows),
                                     dim3(kCpThreads), 0, reinterpret_cast<cudaStream_t>(stream),
                                     scores, ld_scores, pool, P, max_blocks, offset, cand_bmax,
                                     cand_block);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

CSA2_API csa2_status_t csa2_cp_merge(int rows, int n_cand, const float* cand_score,
                                     const int32_t* cand_idx, int K, int32_t* idx_out,
                                     void* stream) {
    if (rows < 1 || n_cand < 1 || K < 1 || K > n_cand) return CSA2_ERR_ARG;
    if (!cand_score || !cand_idx || !idx_out) return CSA2_ERR_ARG;
    if (n_cand > kCpMaxCand) return CSA2_ERR_UNSUPPORTED;
    const int n2 = pow2_at_least(n_cand), k2 = pow2_at_least(K);
    const size_t smem = (size_t)n2 * 8 + (size_t)k2 * 4;
    cudaError_t e = cudaFuncSetAttribute(cp_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    e = launch_pdl(cp_merge_kernel, dim3((unsigned)rows), dim3(kCpThreads), smem,
                   reinterpret_cast<cudaStream_t>(stream), cand_score, cand_idx, n_cand, n2, K,
                   k2, idx_out);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

CSA2_API csa2_status_t csa2_cp_pool_expand(int rows, const int32_t* blocks, int nb,
                                           const int32_t* n_row, int P, int32_t* pool_out,
                                           void* stream) {
    if (rows < 1 || nb < 1 || P < 1 || !blocks || !pool_out) return CSA2_ERR_ARG;
    const cudaError_t e = launch_pdl(cp_pool_expand_kernel, dim3((unsigned)rows),
                                     dim3(kCpThreads), 0, reinterpret_cast<cudaStream_t>(stream),
                                     blocks, nb, n_row, P, pool_out);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

CSA2_API csa2_status_t csa2_cp_local_idx(int64_t n, const int32_t* idx, int64_t lo, int64_t hi,
                                         int32_t* idx_local, void* stream) {
    if (n < 0 || lo < 0 || hi < lo || !idx || !idx_local) return CSA2_ERR_ARG;
    if (n == 0) return CSA2_OK;
    const int64_t blocks = (n + 255) / 256;
    const cudaError_t e = launch_pdl(cp_local_idx_kernel,
                                     dim3((unsigned)(blocks < 4096 ? blocks : 4096)), dim3(256), 0,
                                     reinterpret_cast<cudaStream_t>(stream), idx, n, lo, hi,
                                     idx_local);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

}  // extern "C"
