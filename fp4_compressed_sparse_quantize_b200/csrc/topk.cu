// Exact Top-K selection over rows of indexer scores (or of candidate-pool block maxima).
//
// "DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale LLM Serving", Compressed Sparse
// Attention 2 (CSA2): each Full / Reindex layer selects fresh Top-512 indices;
// "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (AI summary),
// Methodology in Plain English: the candidate pool keeps the blocks with the highest
// maximum index score (e.g. 2,048 blocks of 8 positions).
//
// Order: (score descending, position ascending), exactly; the output lists the chosen
// positions in ascending order, padded with -1.
//
// Radix select on an order-preserving 32-bit key of the fp32 score, extended to a unique
// 64-bit composite  (key << 32) | ~id  so that "larger composite" is the required order:
//   1. the scan kernel already histogrammed the top 12 key bits of every row;
//   2. collect (grid = chunks x rows): every element whose digit is above the threshold
//      digit d0 is a sure winner (fewer than K of them), every element with digit d0 is a
//      candidate; both are appended to per-row lists with warp-aggregated atomics;
//   3. finalize (one CTA per row): sort the candidates in shared memory when they fit
//      (bitonic), otherwise refine with further 12-bit radix passes over the candidate list
//      (or, if even that overflowed, over the row), take the `need` best, merge with the
//      winners and sort the chosen ids ascending.
#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

constexpr int kBinsT = 4096;
constexpr int kSortCap = 4096;   // candidates sorted in shared memory
constexpr int kRankCap = 64;     // candidates selected by rank counting
constexpr int kCollectChunk = 8192;   // elements per collect CTA (32 per thread)
constexpr int kMaxK = 2048;

struct TopkDev {
    int R, K;
    const float* scores;
    const uint32_t* keys;
    int64_t ld;
    const int32_t* n_row;
    int n_row_div;
    const int32_t* ids;
    const int32_t* id_limit;
    const uint32_t* hist;
    int32_t* out;
    bool expand8;
    const int32_t* expand_limit;
    uint32_t* counters;
    uint64_t* winners;
    uint64_t* cands;
    int ccap;
    int bitmap_words;        // > 0: order the picks through a shared bitmap of ids
    int32_t* status;
};

__device__ __forceinline__ int64_t row_len(const TopkDev& a, int r) {
    if (a.ids) return a.ld;
    const int64_t n = __ldg(a.n_row + r);
    return (n + a.n_row_div - 1) / a.n_row_div;
}

// element i of row r: returns false when it is not a valid candidate
__device__ __forceinline__ bool load_elem(const TopkDev& a, int r, int64_t i, uint64_t& comp) {
    uint32_t id = (uint32_t)i;
    if (a.ids) {
        const int32_t v = __ldg(a.ids + (int64_t)r * a.ld + i);
        if (v < 0 || v >= __ldg(a.id_limit + r)) return false;
        id = (uint32_t)v;
    }
    uint32_t key;
    if (a.scores)
        key = score_key(__ldg(a.scores + (int64_t)r * a.ld + i));
    else
        key = __ldg(a.keys + (int64_t)r * a.ld + i);
    comp = ((uint64_t)key << 32) | (uint64_t)(~id);
    return true;
}

// Find digit d in hist[0..nb) (counts) such that above(d) = sum_{e > d} hist[e] < rem <=
// above(d) + hist[d]. Block-wide; every thread gets the result. Returns false when the
// total is < rem (then d = -1 and above = total).
__device__ bool find_digit(const uint32_t* hist, int nb, uint32_t rem, int& d_out,
                           uint32_t& above_out, uint32_t* red /*>= 34 words*/) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (nb + nt - 1) / nt;
    const int lo = tid * per, hi = min(nb, lo + per);
    uint32_t local = 0;
    if (per % 4 == 0 && hi - lo == per) {
        // whole 16-byte groups: issue every load before summing
        const uint4* h4 = reinterpret_cast<const uint4*>(hist + lo);
        uint4 t[8];
        const int n4 = per / 4;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k < n4) t[k] = h4[k];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k < n4) local += t[k].x + t[k].y + t[k].z + t[k].w;
        for (int k = 8; k < n4; ++k) local += h4[k].x + h4[k].y + h4[k].z + h4[k].w;
    } else {
        for (int i = lo; i < hi; ++i) local += hist[i];
    }
    // inclusive suffix sum over threads: reverse thread order
    const int lane = tid & 31, wid = tid >> 5, nw = (nt + 31) >> 5;
    uint32_t v = local;
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t u = __shfl_down_sync(0xffffffffu, v, o);
        if (lane + o < 32) v += u;
    }
    if (lane == 0) red[wid] = v;  // sum of lanes >= 0 in this warp
    __syncthreads();
    if (tid == 0) {
        uint32_t acc = 0;
        for (int w2 = nw - 1; w2 >= 0; --w2) {
            const uint32_t t = red[w2];
            red[w2] = acc;  // sum of warps strictly after w2
            acc += t;
        }
        red[32] = acc;  // total
        red[33] = 0xFFFFFFFFu;
    }
    __syncthreads();
    const uint32_t suffix_incl = v + red[wid];  // sum over threads >= tid
    const uint32_t suffix_excl = suffix_incl - local;
    const uint32_t total = red[32];
    __syncthreads();
    if (total < rem) {
        d_out = -1;
        above_out = total;
        return false;
    }
    if (suffix_incl >= rem && suffix_excl < rem) {
        uint32_t acc = suffix_excl;
        for (int i = hi - 1; i >= lo; --i) {
            if (acc + hist[i] >= rem) {
                red[33] = (uint32_t)i;
                red[32] = acc;
                break;
            }
            acc += hist[i];
        }
    }
    __syncthreads();
    d_out = (int)red[33];
    above_out = red[32];
    __syncthreads();
    return true;
}

__global__ void __launch_bounds__(256) topk_collect_kernel(const TopkDev a) {
    __shared__ uint32_t red[40];
    const int r = blockIdx.y;
    const int64_t n = row_len(a, r);
    const int64_t start = (int64_t)blockIdx.x * kCollectChunk;
    if (start >= n) return;
    const int64_t end = min(n, start + kCollectChunk);
    int d0;
    uint32_t above;
    const bool many = find_digit(a.hist + (int64_t)r * kBinsT, kBinsT, (uint32_t)a.K + 0u, d0,
                                 above, red);
    // many == false: at most K valid elements, all of them win
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    uint32_t* cnt = a.counters + (int64_t)r * 4;
    constexpr int kPer = kCollectChunk / 256;
    // every load of this thread in flight before any is used
    uint64_t comp[kPer];
    uint32_t valid = 0;
    if (a.scores && !a.ids) {
        // Full rows: plain score loads, all issued before any key is formed
        float sv[kPer];
        const float* row = a.scores + (int64_t)r * a.ld;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int64_t i = start + (int64_t)k * blockDim.x + threadIdx.x;
            sv[k] = (i < end) ? __ldg(row + i) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int64_t i = start + (int64_t)k * blockDim.x + threadIdx.x;
            comp[k] = ((uint64_t)score_key(sv[k]) << 32) | (uint64_t)(~(uint32_t)i);
            if (i < end) valid |= 1u << k;
        }
    } else {
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int64_t i = start + (int64_t)k * blockDim.x + threadIdx.x;
            comp[k] = 0;
            if (i < end && load_elem(a, r, i, comp[k])) valid |= 1u << k;
        }
    }
    // pass 1: this CTA's winner / candidate counts, one global atomic per list per CTA
    const int wid = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    uint32_t mw[kPer], mc[kPer];
    uint32_t cw = 0, cc = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const bool ok = (valid >> k) & 1u;
        const int dig = (int)(comp[k] >> 52);
        mw[k] = __ballot_sync(0xffffffffu, ok && (!many || dig > d0));
        mc[k] = __ballot_sync(0xffffffffu, ok && many && dig == d0);
        cw += __popc(mw[k]);
        cc += __popc(mc[k]);
    }
    __shared__ uint32_t wsum[2][32], wbase[2];
    if (lane == 0) {
        wsum[0][wid] = cw;
        wsum[1][wid] = cc;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t tw = 0, tc = 0;
        for (int w = 0; w < nwarps; ++w) {
            const uint32_t a0 = wsum[0][w], a1 = wsum[1][w];
            wsum[0][w] = tw;
            wsum[1][w] = tc;
            tw += a0;
            tc += a1;
        }
        wbase[0] = tw ? atomicAdd(cnt + 0, tw) : 0u;
        wbase[1] = tc ? atomicAdd(cnt + 1, tc) : 0u;
    }
    __syncthreads();
    // pass 2: write at the reserved offsets
    uint32_t pw = wbase[0] + wsum[0][wid], pc = wbase[1] + wsum[1][wid];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        if ((mw[k] >> lane) & 1u) {
            const uint32_t pos = pw + __popc(mw[k] & lt);
            if (pos < (uint32_t)a.K) a.winners[(int64_t)r * a.K + pos] = comp[k];
        }
        if ((mc[k] >> lane) & 1u) {
            const uint32_t pos = pc + __popc(mc[k] & lt);
            if (pos < (uint32_t)a.ccap) a.cands[(int64_t)r * a.ccap + pos] = comp[k];
        }
        pw += __popc(mw[k]);
        pc += __popc(mc[k]);
    }
}

// ---- shared-memory bitonic sorts ------------------------------------------------------------

__device__ void bitonic_desc_u64(uint64_t* v, int n) {
    for (int k = 2; k <= n; k <<= 1)
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n; i += blockDim.x) {
                const int x = i ^ j;
                if (x > i) {
                    const uint64_t p = v[i], q = v[x];
                    const bool desc = (i & k) == 0;
                    if (desc ? (p < q) : (p > q)) {
                        v[i] = q;
                        v[x] = p;
                    }
                }
            }
            __syncthreads();
        }
}

__device__ __forceinline__ int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

// Source of candidate composites for the refinement passes: the global candidate list or,
// after an overflow of that list, the whole row filtered to digit d0.
struct CandSource {
    const uint64_t* list;
    int64_t n;
    bool from_row;
    int d0;
};

__device__ __forceinline__ bool cand_at(const TopkDev& a, int r, const CandSource& s,
                                        int64_t i, uint64_t& c) {
    if (!s.from_row) {
        c = s.list[i];
        return true;
    }
    if (!load_elem(a, r, i, c)) return false;
    return (int)(c >> 52) == s.d0;
}

__global__ void __launch_bounds__(512) topk_finalize_kernel(const TopkDev a) {
    extern __shared__ uint8_t sm[];
    uint64_t* sortbuf = reinterpret_cast<uint64_t*>(sm);                 // kSortCap
    uint32_t* hist = reinterpret_cast<uint32_t*>(sortbuf + kSortCap);    // kBinsT
    int32_t* ids = reinterpret_cast<int32_t*>(hist + kBinsT);            // kMaxK
    __shared__ uint32_t red[40];
    __shared__ uint32_t nsel_s, ncoll_s;

    const int r = blockIdx.x;
    const int K = a.K;
    int d0;
    uint32_t above;
    const bool many = find_digit(a.hist + (int64_t)r * kBinsT, kBinsT, (uint32_t)K, d0, above,
                                 red);
    const uint32_t* cnt = a.counters + (int64_t)r * 4;
    const uint32_t nwin = min(__ldcg(cnt + 0), (uint32_t)K);
    for (uint32_t i = threadIdx.x; i < nwin; i += blockDim.x)
        ids[i] = (int32_t)(~(uint32_t)(a.winners[(int64_t)r * K + i] & 0xFFFFFFFFu));
    uint32_t total = nwin;
    if (many) {
        const uint32_t need = (uint32_t)K - above;
        if (nwin != above) set_status(a.status, CSA2_DEV_BAD_COUNT);  // internal consistency
        const uint32_t ncand = __ldcg(cnt + 1);
        CandSource src;
        src.list = a.cands + (int64_t)r * a.ccap;
        src.n = ncand;
        src.from_row = ncand > (uint32_t)a.ccap;
        src.d0 = d0;
        if (src.from_row) src.n = row_len(a, r);
        uint64_t thresh = 0;
        const bool small = !src.from_row && ncand <= (uint32_t)kRankCap;
        if (small) {
            // rank of each candidate among the candidates (composites are unique): the
            // `need` largest take slots nwin + rank directly
            for (int i = threadIdx.x; i < (int)ncand; i += blockDim.x) sortbuf[i] = src.list[i];
            __syncthreads();
            for (int i = threadIdx.x; i < (int)ncand; i += blockDim.x) {
                const uint64_t c = sortbuf[i];
                uint32_t rank = 0;
#pragma unroll 8
                for (int j = 0; j < (int)ncand; ++j) rank += sortbuf[j] > c;
                if (rank < need) ids[nwin + rank] = (int32_t)(~(uint32_t)(c & 0xFFFFFFFFu));
            }
            __syncthreads();
        } else if (!src.from_row && ncand <= (uint32_t)kSortCap) {
            const int n2 = pow2_at_least((int)ncand);
            for (int i = threadIdx.x; i < n2; i += blockDim.x)
                sortbuf[i] = (i < (int)ncand) ? src.list[i] : 0ull;
            __syncthreads();
            bitonic_desc_u64(sortbuf, n2);
            thresh = sortbuf[need - 1];
            __syncthreads();
        } else {
            // radix refinement on the bits below the first digit
            uint64_t prefix = (uint64_t)d0;
            int shift = 52;
            uint32_t rem = need;
            while (true) {
                const int nb = shift < 12 ? shift : 12;
                for (int i = threadIdx.x; i < kBinsT; i += blockDim.x) hist[i] = 0;
                __syncthreads();
                for (int64_t i = threadIdx.x; i < src.n; i += blockDim.x) {
                    uint64_t c;
                    if (cand_at(a, r, src, i, c) && (c >> shift) == prefix)
                        atomicAdd(&hist[(c >> (shift - nb)) & ((1u << nb) - 1u)], 1u);
                }
                __syncthreads();
                int d;
                uint32_t ab;
                if (!find_digit(hist, 1 << nb, rem, d, ab, red)) {
                    set_status(a.status, CSA2_DEV_BAD_COUNT);  // counts disagree: give up
                    break;
                }
                const uint32_t inbin = hist[d];
                __syncthreads();
                rem -= ab;
                prefix = (prefix << nb) | (uint64_t)d;
                shift -= nb;
                if (inbin <= (uint32_t)kSortCap || shift == 0) break;
            }
            // gather the elements of the final bin, sort, pick the rem-th
            if (threadIdx.x == 0) ncoll_s = 0;
            __syncthreads();
            for (int64_t i = threadIdx.x; i < src.n; i += blockDim.x) {
                uint64_t c;
                if (cand_at(a, r, src, i, c) && (c >> shift) == prefix) {
                    const uint32_t pos = atomicAdd(&ncoll_s, 1u);
                    if (pos < (uint32_t)kSortCap) sortbuf[pos] = c;
                }
            }
            __syncthreads();
            const int nc = (int)min(ncoll_s, (uint32_t)kSortCap);
            const int n2 = pow2_at_least(nc);
            for (int i = nc + threadIdx.x; i < n2; i += blockDim.x) sortbuf[i] = 0ull;
            __syncthreads();
            bitonic_desc_u64(sortbuf, n2);
            thresh = sortbuf[rem - 1];
            __syncthreads();
        }
        // every candidate composite >= thresh is chosen (exactly `need` of them)
        if (threadIdx.x == 0) nsel_s = 0;
        __syncthreads();
        if (small) {
            // already placed
        } else if (!src.from_row && ncand <= (uint32_t)kSortCap) {
            for (uint32_t i = threadIdx.x; i < need; i += blockDim.x)
                ids[nwin + i] = (int32_t)(~(uint32_t)(sortbuf[i] & 0xFFFFFFFFu));
        } else {
            for (int64_t i = threadIdx.x; i < src.n; i += blockDim.x) {
                uint64_t c;
                if (cand_at(a, r, src, i, c) && c >= thresh) {
                    const uint32_t pos = atomicAdd(&nsel_s, 1u);
                    if (pos < need) ids[nwin + pos] = (int32_t)(~(uint32_t)(c & 0xFFFFFFFFu));
                }
            }
        }
        __syncthreads();
        total = nwin + need;
    }
    __syncthreads();
    if (a.bitmap_words > 0) {
        // ascending order without sorting: mark the picks in a bitmap of ids, then each
        // thread emits the set bits of its word range at its exclusive-scan offset
        uint32_t* bm = reinterpret_cast<uint32_t*>(ids + kMaxK);
        const int nwords = a.bitmap_words;
        for (int i = threadIdx.x; i < nwords; i += blockDim.x) bm[i] = 0u;
        __syncthreads();
        for (int i = threadIdx.x; i < (int)total; i += blockDim.x) {
            const uint32_t v = (uint32_t)ids[i];
            if ((int)(v >> 5) < nwords) atomicOr(&bm[v >> 5], 1u << (v & 31));
        }
        __syncthreads();
        const int per = (nwords + blockDim.x - 1) / blockDim.x;
        const int w0 = threadIdx.x * per, w1 = min(nwords, w0 + per);
        uint32_t cntb = 0;
        for (int wi = w0; wi < w1; ++wi) cntb += __popc(bm[wi]);
        // block exclusive scan of cntb
        const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
        uint32_t incl = cntb;
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) red[wid] = incl;
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t acc = 0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
                const uint32_t t = red[w];
                red[w] = acc;
                acc += t;
            }
            ncoll_s = acc;  // distinct picks (equals `total` unless ids repeat)
        }
        __syncthreads();
        uint32_t off = red[wid] + incl - cntb;
        const int npick = (int)min(ncoll_s, (uint32_t)K);
        if (!a.expand8) {
            int32_t* o = a.out + (int64_t)r * K;
            for (int wi = w0; wi < w1; ++wi) {
                uint32_t m = bm[wi];
                while (m) {
                    const int b = __ffs(m) - 1;
                    m &= m - 1;
                    if (off < (uint32_t)K) o[off] = wi * 32 + b;
                    ++off;
                }
            }
            for (int i = npick + threadIdx.x; i < K; i += blockDim.x) o[i] = -1;
        } else {
            const int32_t lim = __ldg(a.expand_limit + r);
            int32_t* o = a.out + (int64_t)r * K * 8;
            for (int wi = w0; wi < w1; ++wi) {
                uint32_t m = bm[wi];
                while (m) {
                    const int b = __ffs(m) - 1;
                    m &= m - 1;
                    if (off < (uint32_t)K) {
                        const int64_t blk = (int64_t)wi * 32 + b;
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int64_t pos = blk * 8 + e;
                            o[off * 8 + e] = pos < lim ? (int32_t)pos : -1;
                        }
                    }
                    ++off;
                }
            }
            for (int i = npick * 8 + threadIdx.x; i < K * 8; i += blockDim.x) o[i] = -1;
        }
        return;
    }
    // order the chosen ids ascending: each id's rank among the (distinct) chosen ids
    int32_t* sorted = reinterpret_cast<int32_t*>(sortbuf);
    for (int i = threadIdx.x; i < (int)total; i += blockDim.x) {
        const int32_t v = ids[i];
        int rank = 0;
#pragma unroll 8
        for (int j = 0; j < (int)total; ++j) rank += (ids[j] < v) | ((ids[j] == v) & (j < i));
        sorted[rank] = v;
    }
    __syncthreads();
    ids = sorted;
    if (!a.expand8) {
        for (int i = threadIdx.x; i < K; i += blockDim.x)
            a.out[(int64_t)r * K + i] = (i < (int)total) ? ids[i] : -1;
    } else {
        const int32_t lim = __ldg(a.expand_limit + r);
        for (int i = threadIdx.x; i < K * 8; i += blockDim.x) {
            const int blk = i >> 3;
            int32_t v = -1;
            if (blk < (int)total) {
                const int64_t pos = (int64_t)ids[blk] * 8 + (i & 7);
                if (pos < lim) v = (int32_t)pos;
            }
            a.out[(int64_t)r * K * 8 + i] = v;
        }
    }
}

cudaError_t launch_topk(const TopkLaunch& l, cudaStream_t st) {
    if (l.K > kMaxK || l.K <= 0) return cudaErrorInvalidValue;
    TopkDev a;
    a.R = l.R;
    a.K = l.K;
    a.scores = l.scores;
    a.keys = l.keys;
    a.ld = l.ld;
    a.n_row = l.n_row;
    a.n_row_div = l.n_row_div > 0 ? l.n_row_div : 1;
    a.ids = l.ids;
    a.id_limit = l.id_limit;
    a.hist = l.hist;
    a.out = l.out;
    a.expand8 = l.expand8;
    a.expand_limit = l.expand_limit;
    a.counters = l.counters;
    a.winners = l.winners;
    a.cands = l.cands;
    a.ccap = l.ccap;
    a.status = l.status;
    const int64_t chunks = (l.max_n + kCollectChunk - 1) / kCollectChunk;
    if (chunks > 0) {
        dim3 grid((unsigned)chunks, (unsigned)l.R);
        topk_collect_kernel<<<grid, 256, 0, st>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // ids are < id_bound: a bitmap of that many bits orders the picks if it fits
    const int64_t words = (l.id_bound + 31) / 32;
    const size_t base = kSortCap * 8 + kBinsT * 4 + kMaxK * 4;
    a.bitmap_words = (l.id_bound > 0 && base + words * 4 <= 200 * 1024) ? (int)words : 0;
    const size_t smem = base + (size_t)a.bitmap_words * 4;
    cudaError_t e = cudaFuncSetAttribute(topk_finalize_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    topk_finalize_kernel<<<l.R, 512, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace csa2
