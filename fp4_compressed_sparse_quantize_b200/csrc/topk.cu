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
// 64-bit composite  (key << 32) | ~id  so that "larger composite" is the required order.
// One kernel, grid = chunks x rows:
//   1. the scan kernel already histogrammed the top 12 key bits of every row, which fixes
//      the threshold digit d0: fewer than K elements lie above it;
//   2. every CTA classifies its chunk: elements above d0 are sure winners, elements on d0
//      are candidates; both are appended to per-row lists (one atomic per list per CTA);
//   3. the last CTA of a row to finish (threadfence + counter, no waiting) finds the exact
//      `need`-th best candidate by 8-bit radix refinement over the candidate list (in shared
//      memory when it fits, else in global memory, else over the row itself when even the
//      list overflowed), marks the winners and chosen candidates in a shared bitmap of ids,
//      and emits the set bits in ascending order.
#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

constexpr int kBinsT = 4096;            // first radix digit (key >> 20), from the scan
constexpr int kCollectChunk = 8192;     // elements per CTA (32 per thread)
constexpr int kThreads = 256;
constexpr int kSmemCands = 4096;        // candidates refined in shared memory
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
    uint32_t* counters;      // [R][4]: winners, candidates, finished CTAs, spare
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

// Source of candidate composites for the refinement: a list (shared or global memory) or,
// after the candidate list overflowed, the whole row filtered to digit d0.
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

// Smallest composite T such that exactly `need` candidates are >= T (composites are
// unique). 8-bit radix refinement below the known top 12 bits; stops as soon as the chosen
// bin is taken whole.
__device__ uint64_t refine_threshold(const TopkDev& a, int r, const CandSource& src,
                                     uint32_t need, uint32_t* hist256, uint32_t* red) {
    uint64_t prefix = (uint64_t)src.d0;
    int shift = 52;
    uint32_t rem = need;
    while (shift > 0) {
        const int nb = shift < 8 ? shift : 8;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist256[i] = 0;
        __syncthreads();
        for (int64_t i = threadIdx.x; i < src.n; i += blockDim.x) {
            uint64_t c;
            if (cand_at(a, r, src, i, c) && (c >> shift) == prefix)
                atomicAdd(&hist256[(c >> (shift - nb)) & ((1u << nb) - 1u)], 1u);
        }
        __syncthreads();
        int d;
        uint32_t ab;
        if (!find_digit(hist256, 1 << nb, rem, d, ab, red)) {
            set_status(a.status, CSA2_DEV_BAD_COUNT);  // counts disagree: take everything
            return 0ull;
        }
        const uint32_t inbin = hist256[d];
        __syncthreads();
        rem -= ab;
        prefix = (prefix << nb) | (uint64_t)d;
        shift -= nb;
        if (inbin == rem) break;   // the whole bin is taken
    }
    return prefix << shift;
}

__global__ void __launch_bounds__(kThreads) topk_kernel(const TopkDev a) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ uint32_t red[40];
    __shared__ uint32_t hist256[256];
    __shared__ uint32_t wsum[2][32], wbase[2];
    __shared__ int last_s;
    __shared__ uint32_t npick_s;
    const int r = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t n = row_len(a, r);
    const int64_t start = (int64_t)blockIdx.x * kCollectChunk;
    const int64_t end = min(n, start + kCollectChunk);
    uint32_t* cnt = a.counters + (int64_t)r * 4;
    const int K = a.K;

    int d0;
    uint32_t above;
    // many == false: at most K valid elements in the row, all of them win
    const bool many = find_digit(a.hist + (int64_t)r * kBinsT, kBinsT, (uint32_t)K, d0, above, red);

    // ---- 1. classify this CTA's chunk and append winners / candidates -------------------
    if (start < end) {
        const unsigned lt = (1u << lane) - 1u;
        constexpr int kPer = kCollectChunk / kThreads;
        uint64_t comp[kPer];
        uint32_t valid = 0;
        if (a.scores && !a.ids) {
            float sv[kPer];
            const float* row = a.scores + (int64_t)r * a.ld;
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int64_t i = start + (int64_t)k * kThreads + tid;
                sv[k] = (i < end) ? __ldg(row + i) : 0.f;
            }
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int64_t i = start + (int64_t)k * kThreads + tid;
                comp[k] = ((uint64_t)score_key(sv[k]) << 32) | (uint64_t)(~(uint32_t)i);
                if (i < end) valid |= 1u << k;
            }
        } else {
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int64_t i = start + (int64_t)k * kThreads + tid;
                comp[k] = 0;
                if (i < end && load_elem(a, r, i, comp[k])) valid |= 1u << k;
            }
        }
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
        if (lane == 0) {
            wsum[0][wid] = cw;
            wsum[1][wid] = cc;
        }
        __syncthreads();
        if (tid == 0) {
            uint32_t tw = 0, tc = 0;
            for (int w = 0; w < kThreads / 32; ++w) {
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
        uint32_t pw = wbase[0] + wsum[0][wid], pc = wbase[1] + wsum[1][wid];
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            if ((mw[k] >> lane) & 1u) {
                const uint32_t pos = pw + __popc(mw[k] & lt);
                if (pos < (uint32_t)K) a.winners[(int64_t)r * K + pos] = comp[k];
            }
            if ((mc[k] >> lane) & 1u) {
                const uint32_t pos = pc + __popc(mc[k] & lt);
                if (pos < (uint32_t)a.ccap) a.cands[(int64_t)r * a.ccap + pos] = comp[k];
            }
            pw += __popc(mw[k]);
            pc += __popc(mc[k]);
        }
    }

    // ---- 2. the last CTA of the row finalises it ------------------------------------------
    __threadfence();
    __syncthreads();
    if (tid == 0) last_s = (atomicAdd(cnt + 2, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!last_s) return;
    __threadfence();

    uint64_t* cand_s = reinterpret_cast<uint64_t*>(dsm);                 // kSmemCands
    uint32_t* bm = reinterpret_cast<uint32_t*>(cand_s + kSmemCands);     // bitmap / id list
    const uint32_t nwin = min(__ldcg(cnt + 0), (uint32_t)K);
    const bool use_bm = a.bitmap_words > 0;
    const int nwords = a.bitmap_words;
    int32_t* picks = reinterpret_cast<int32_t*>(bm);                     // without a bitmap
    if (tid == 0) npick_s = 0;
    if (use_bm)
        for (int i = tid; i < nwords; i += kThreads) bm[i] = 0u;
    __syncthreads();
    auto pick = [&](uint64_t c) {
        const uint32_t id = ~(uint32_t)(c & 0xFFFFFFFFu);
        if (use_bm) {
            if ((int)(id >> 5) < nwords) atomicOr(&bm[id >> 5], 1u << (id & 31));
        } else {
            const uint32_t pos = atomicAdd(&npick_s, 1u);
            if (pos < (uint32_t)K) picks[pos] = (int32_t)id;
        }
    };
    for (uint32_t i = tid; i < nwin; i += kThreads) pick(__ldcg(a.winners + (int64_t)r * K + i));
    if (many) {
        const uint32_t need = (uint32_t)K - above;
        if (nwin != above) set_status(a.status, CSA2_DEV_BAD_COUNT);  // internal consistency
        const uint32_t ncand = __ldcg(cnt + 1);
        CandSource src;
        src.d0 = d0;
        src.from_row = ncand > (uint32_t)a.ccap;
        if (src.from_row) {
            src.list = nullptr;
            src.n = row_len(a, r);
        } else if (ncand <= (uint32_t)kSmemCands) {
            for (uint32_t i = tid; i < ncand; i += kThreads)
                cand_s[i] = __ldcg(a.cands + (int64_t)r * a.ccap + i);
            src.list = cand_s;
            src.n = ncand;
        } else {
            src.list = a.cands + (int64_t)r * a.ccap;
            src.n = ncand;
        }
        __syncthreads();
        const uint64_t T = refine_threshold(a, r, src, need, hist256, red);
        __syncthreads();
        for (int64_t i = tid; i < src.n; i += kThreads) {
            uint64_t c;
            if (cand_at(a, r, src, i, c) && c >= T) pick(c);
        }
    }
    __syncthreads();

    // ---- 3. emit the picks in ascending order ---------------------------------------------
    int npick;
    uint32_t off = 0;
    int w0 = 0, w1 = 0;
    if (use_bm) {
        const int per = (nwords + kThreads - 1) / kThreads;
        w0 = tid * per;
        w1 = min(nwords, w0 + per);
        uint32_t cntb = 0;
        for (int wi = w0; wi < w1; ++wi) cntb += __popc(bm[wi]);
        uint32_t incl = cntb;
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) red[wid] = incl;
        __syncthreads();
        if (tid == 0) {
            uint32_t acc = 0;
            for (int w = 0; w < kThreads / 32; ++w) {
                const uint32_t t = red[w];
                red[w] = acc;
                acc += t;
            }
            npick_s = acc;
        }
        __syncthreads();
        off = red[wid] + incl - cntb;
        npick = (int)min(npick_s, (uint32_t)K);
    } else {
        // rank each pick among the (distinct) picks
        npick = (int)min(npick_s, (uint32_t)K);
        int32_t* sorted = reinterpret_cast<int32_t*>(cand_s);
        for (int i = tid; i < npick; i += kThreads) {
            const int32_t v = picks[i];
            int rank = 0;
            for (int j = 0; j < npick; ++j) rank += (picks[j] < v) | ((picks[j] == v) & (j < i));
            sorted[rank] = v;
        }
        __syncthreads();
        picks = sorted;
    }
    const int32_t lim = a.expand8 ? __ldg(a.expand_limit + r) : 0;
    int32_t* o = a.out + (int64_t)r * K * (a.expand8 ? 8 : 1);
    auto emit = [&](uint32_t slot, int64_t id) {
        if (slot >= (uint32_t)K) return;
        if (!a.expand8) {
            o[slot] = (int32_t)id;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int64_t pos = id * 8 + e;
                o[slot * 8 + e] = pos < lim ? (int32_t)pos : -1;
            }
        }
    };
    if (use_bm) {
        for (int wi = w0; wi < w1; ++wi) {
            uint32_t m = bm[wi];
            while (m) {
                const int b = __ffs(m) - 1;
                m &= m - 1;
                emit(off++, (int64_t)wi * 32 + b);
            }
        }
    } else {
        for (int i = tid; i < npick; i += kThreads) emit((uint32_t)i, picks[i]);
    }
    const int mult = a.expand8 ? 8 : 1;
    for (int i = npick * mult + tid; i < K * mult; i += kThreads) o[i] = -1;
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
    // ids are < id_bound: a bitmap of that many bits orders the picks when it is small
    const int64_t words = (l.id_bound + 31) / 32;
    a.bitmap_words = (l.id_bound > 0 && words * 4 <= 64 * 1024) ? (int)words : 0;
    const size_t smem = (size_t)kSmemCands * 8 +
                        (a.bitmap_words > 0 ? (size_t)a.bitmap_words * 4 : (size_t)kMaxK * 4);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    int64_t chunks = (l.max_n + kCollectChunk - 1) / kCollectChunk;
    if (chunks < 1) chunks = 1;
    dim3 grid((unsigned)chunks, (unsigned)l.R);
    topk_kernel<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace csa2
