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
// The scan kernel already histogrammed the top 12 key bits of every row, which fixes the
// threshold digit d0: fewer than K elements lie above it. Elements above d0 are sure
// winners, elements on d0 are candidates, and the exact `need`-th best candidate is found
// by 8-bit radix refinement. Three kernels:
//   topk_bitmap_kernel  rows by position of up to 262,144 elements (Full layers, the pool's
//                       block maxima): one CTA, or a cluster of CTAs, per row; picks are
//                       marked in a bitmap of positions (see the kernel);
//   topk_gather_kernel  rows of gathered ids (Reindex over the pool): one 1024-thread CTA
//                       per row, winner and candidate lists in shared memory, picks ordered
//                       by a bitonic sort;
//   topk_kernel         longer rows (the 1M-entry Full layer), grid = chunks x rows: every
//                       CTA classifies its chunk into per-row lists (one atomic per list per
//                       CTA); the last CTA of a row to finish (threadfence + counter, no
//                       waiting) refines over the candidate list (in shared memory when it
//                       fits, else in global memory, else over the row itself when even the
//                       list overflowed) and emits the set bits of a bitmap of ids in
//                       ascending order.
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
    int ring;                // topk_bitmap_kernel: chunk buffers in flight
    int32_t* status;
};

__device__ __forceinline__ int64_t row_len(const TopkDev& a, int r) {
    if (a.ids) return a.ld;
    const int64_t n = ld_dep(a.n_row + r);
    return (n + a.n_row_div - 1) / a.n_row_div;
}

// element i of row r: returns false when it is not a valid candidate
__device__ __forceinline__ bool load_elem(const TopkDev& a, int r, int64_t i, uint64_t& comp) {
    uint32_t id = (uint32_t)i;
    if (a.ids) {
        const int32_t v = ld_dep(a.ids + (int64_t)r * a.ld + i);
        if (v < 0 || v >= ld_dep(a.id_limit + r)) return false;
        id = (uint32_t)v;
    }
    uint32_t key;
    if (a.scores)
        key = score_key(ld_dep(a.scores + (int64_t)r * a.ld + i));
    else
        key = ld_dep(a.keys + (int64_t)r * a.ld + i);
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

// Warp 0 only: over bins h[0..256) (counts), find d with above(d) < rem <= above(d) + h[d],
// above(d) = sum of h[e] for e > d. Writes d (or -1 when the total is < rem), above(d) and
// h[d] into out[0..3).
__device__ __forceinline__ void warp_find_digit256(const uint32_t* h, uint32_t rem, int* out) {
    const int lane = threadIdx.x & 31;
    uint32_t b[8], sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {   // lane 0 owns the 8 highest bins, highest first
        b[j] = h[255 - 8 * lane - j];
        sum += b[j];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    const uint32_t excl = incl - sum;
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    if (lane == 0 && total < rem) {
        out[0] = -1;
        out[1] = (int)total;
        out[2] = 0;
    }
    if (excl < rem && incl >= rem) {
        uint32_t acc = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (acc < rem && acc + b[j] >= rem) {
                out[0] = 255 - 8 * lane - j;
                out[1] = (int)acc;
                out[2] = (int)b[j];
            }
            acc += b[j];
        }
    }
}

// Emits the set bits of bm[0, nwords) in ascending order into output slots [0, K): the bit's
// index, or the 8 positions of that block (positions >= lim as -1) with expand8; pads the
// remaining slots with -1. Groups of 32 words are read by whole warps, one word per lane
// (conflict-free), and each warp owns a contiguous run of groups; a warp-level prefix sum
// gives every word its first slot. Block-wide (contains barriers); wsum takes 33 words.
template <int NT>
__device__ void emit_bitmap(const uint32_t* bm, int64_t nwords, int K, int32_t* o, bool expand8,
                            int32_t lim, uint32_t* wsum) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t ngroups = (nwords + 31) >> 5;
    const int64_t gpw = (ngroups + NW - 1) / NW;
    const int64_t g0 = warp * gpw, g1 = g0 + gpw < ngroups ? g0 + gpw : ngroups;
    auto word = [&](int64_t g) { const int64_t wi = g * 32 + lane; return wi < nwords ? bm[wi] : 0u; };
    uint32_t wtot = 0;
    for (int64_t g = g0; g < g1; ++g) wtot += __reduce_add_sync(0xffffffffu, (uint32_t)__popc(word(g)));
    if (lane == 0) wsum[warp] = wtot;
    __syncthreads();
    if (warp == 0) {
        const uint32_t x = lane < NW ? wsum[lane] : 0u;
        uint32_t xi = x;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t u = __shfl_up_sync(0xffffffffu, xi, d);
            if (lane >= d) xi += u;
        }
        if (lane < NW) wsum[lane] = xi - x;
        if (lane == 31) wsum[32] = xi;
    }
    __syncthreads();
    uint32_t base = wsum[warp];
    const uint32_t total = wsum[32];
    for (int64_t g = g0; g < g1 && base < (uint32_t)K; ++g) {
        uint32_t w = word(g);
        const uint32_t pc = (uint32_t)__popc(w);
        uint32_t incl = pc;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t u = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += u;
        }
        uint32_t slot = base + incl - pc;
        const int64_t wbase = (g * 32 + lane) * 32;
        while (w) {
            const int bit = __ffs(w) - 1;
            w &= w - 1;
            if (slot < (uint32_t)K) {
                const int64_t id = wbase + bit;
                if (!expand8) {
                    o[slot] = (int32_t)id;
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int64_t pos = id * 8 + e;
                        o[(int64_t)slot * 8 + e] = pos < lim ? (int32_t)pos : -1;
                    }
                }
            }
            ++slot;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    const int npick = (int)(total < (uint32_t)K ? total : (uint32_t)K);
    const int mult = expand8 ? 8 : 1;
    for (int i = npick * mult + (int)threadIdx.x; i < K * mult; i += NT) o[i] = -1;
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
        // one warp scans the (zero-padded) 256 bins
        int* dig = reinterpret_cast<int*>(red);
        if (threadIdx.x < 32) warp_find_digit256(hist256, rem, dig);
        __syncthreads();
        const int d = dig[0];
        const uint32_t ab = (uint32_t)dig[1], inbin = (uint32_t)dig[2];
        __syncthreads();
        if (d < 0) {
            set_status(a.status, CSA2_DEV_BAD_COUNT);  // counts disagree: take everything
            return 0ull;
        }
        rem -= ab;
        prefix = (prefix << nb) | (uint64_t)d;
        shift -= nb;
        if (inbin == rem) break;   // the whole bin is taken
    }
    return prefix << shift;
}

__global__ void __launch_bounds__(kThreads, 2) topk_kernel(const TopkDev a) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ uint32_t red[40];
    __shared__ uint32_t hist256[256];
    __shared__ uint32_t wsum[2][32], wbase[2];
    __shared__ int last_s;
    __shared__ uint32_t npick_s;
    const int r = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    grid_dep_launch();
    grid_dep_wait();
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
    // All of the chunk's scores are loaded first; they are then classified and appended in
    // batches of 8 per thread (one pair of list atomics per batch), which keeps the register
    // count low enough for several CTAs per SM.
    if (start < end) {
        const unsigned lt = (1u << lane) - 1u;
        constexpr int kPer = kCollectChunk / kThreads;
        constexpr int kB = 8;
        const bool plain = a.scores && !a.ids;
        float sv[kPer];
        if (plain) {
            const float* row = a.scores + (int64_t)r * a.ld;
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int64_t i = start + (int64_t)k * kThreads + tid;
                sv[k] = (i < end) ? ld_dep(row + i) : 0.f;
            }
        }
#pragma unroll
        for (int b0 = 0; b0 < kPer; b0 += kB) {
            uint64_t comp[kB];
            uint32_t valid = 0;
#pragma unroll
            for (int k = 0; k < kB; ++k) {
                const int64_t i = start + (int64_t)(b0 + k) * kThreads + tid;
                comp[k] = 0;
                if (plain) {
                    comp[k] = ((uint64_t)score_key(sv[b0 + k]) << 32) | (uint64_t)(~(uint32_t)i);
                    if (i < end) valid |= 1u << k;
                } else if (i < end && load_elem(a, r, i, comp[k])) {
                    valid |= 1u << k;
                }
            }
            uint32_t mw[kB], mc[kB];
            uint32_t cw = 0, cc = 0;
#pragma unroll
            for (int k = 0; k < kB; ++k) {
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
            for (int k = 0; k < kB; ++k) {
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
            __syncthreads();   // wsum and wbase are rewritten by the next batch
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
    const int32_t lim = a.expand8 ? ld_dep(a.expand_limit + r) : 0;
    int32_t* o = a.out + (int64_t)r * K * (a.expand8 ? 8 : 1);
    if (use_bm) {
        emit_bitmap<kThreads>(bm, nwords, K, o, a.expand8, lim, red);
        return;
    }
    // bitonic sort of the (distinct) picks, padded to a power of two (at most kMaxK)
    const int npick = (int)min(npick_s, (uint32_t)K);
    int p2 = 1;
    while (p2 < npick) p2 <<= 1;
    for (int i = npick + tid; i < p2; i += kThreads) picks[i] = INT32_MAX;
    __syncthreads();
    for (int k = 2; k <= p2; k <<= 1)
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < p2; i += kThreads) {
                const int l = i ^ j;
                if (l > i) {
                    const int32_t x = picks[i], y = picks[l];
                    if ((x > y) == ((i & k) == 0)) {
                        picks[i] = y;
                        picks[l] = x;
                    }
                }
            }
            __syncthreads();
        }
    for (int i = tid; i < npick; i += kThreads) {
        const int32_t id = picks[i];
        if (!a.expand8) {
            o[i] = id;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int64_t pos = (int64_t)id * 8 + e;
                o[(int64_t)i * 8 + e] = pos < lim ? (int32_t)pos : -1;
            }
        }
    }
    const int mult = a.expand8 ? 8 : 1;
    for (int i = npick * mult + tid; i < K * mult; i += kThreads) o[i] = -1;
}

// ---- one CTA per row ----------------------------------------------------------------------
// For rows of up to kRowMaxN elements a single 1024-thread CTA owns the row: the threshold
// digit, the winners, the candidates and the refinement all stay in shared memory, so
// there is no cross-CTA hand-off. Without ids the row's histogram and scores (or keys) are
// streamed into shared memory by bulk asynchronous copies (64 KiB chunks, two buffers): a
// single SM keeps far more bytes in flight that way than with per-thread loads. With ids
// (Reindex: short rows) the elements are read 8 per thread per batch.
constexpr int kRowThreads = 1024;
constexpr int kRowPerIds = 8;                // elements per thread per batch (ids)
constexpr int kRowCands = 4096;
constexpr int64_t kRowMaxN = 262144;
constexpr size_t kRowOffHist = 0;                                   // u32[4096]
constexpr size_t kRowOffCand = kRowOffHist + 4 * kBinsT;            // u64[kRowCands]
constexpr size_t kRowOffWin = kRowOffCand + 8 * kRowCands;          // u32[kMaxK]
constexpr size_t kRowOffBm = kRowOffWin + 4 * kMaxK;                // pick list

// Exclusive prefix sum of v over the 1024 threads (thread order); `total` gets the sum.
// Uses wsum[0..32); ends with a barrier, so wsum may be reused right away.
__device__ __forceinline__ uint32_t row_excl_scan(uint32_t v, uint32_t* wsum, uint32_t& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        uint32_t x = wsum[lane], xi = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(0xffffffffu, xi, o);
            if (lane >= o) xi += u;
        }
        wsum[lane] = xi - x;   // exclusive over warps
        if (lane == 31) wsum[32] = xi;
    }
    __syncthreads();
    const uint32_t r = wsum[warp] + incl - v;
    total = wsum[32];
    __syncthreads();
    return r;
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t elem_key(const TopkDev& a, int r, int64_t i) {
    return a.scores ? score_key(ld_dep(a.scores + (int64_t)r * a.ld + i))
                    : ld_dep(a.keys + (int64_t)r * a.ld + i);
}

// Shared-memory state of one row's selection.
struct RowState {
    uint32_t* hist;     // 4096 bins (the histogram, later 256-bin refinement counts)
    uint64_t* cand_s;   // candidates (composites), first kRowCands
    uint32_t* win_s;    // winner ids
    uint32_t* bm;       // the pick list (ids)
    uint32_t* wsum;
    int* dig_s;
    uint32_t* tot_s;    // running winner / candidate counts
};

// Classify PER elements per thread against d0 and append them to the winner / candidate
// lists. Element k has key[k] and id ID(k) and takes part when bit k of `valid` is set.
// Block-wide (contains barriers).
template <int PER, class IdOf>
__device__ __forceinline__ void row_classify(const TopkDev& a, const RowState& S, int r,
                                             const uint32_t (&key)[PER], IdOf ID,
                                             uint32_t valid, bool many, int d0, int ccap) {
    uint32_t wmask = 0, cmask = 0;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        const bool ok = (valid >> k) & 1u;
        const int dig = (int)(key[k] >> 20);
        if (ok && (!many || dig > d0)) wmask |= 1u << k;
        if (ok && many && dig == d0) cmask |= 1u << k;
    }
    const uint32_t cw = __popc(wmask), cc = __popc(cmask);
    uint32_t tot;
    const uint32_t ex = row_excl_scan(cw | (cc << 16), S.wsum, tot);
    uint32_t pw = S.tot_s[0] + (ex & 0xFFFFu), pc = S.tot_s[1] + (ex >> 16);
    uint64_t* gcand = a.cands + (int64_t)r * a.ccap;
    uint32_t wm = wmask, cm = cmask;
    // only the (few) selected elements are visited
    while (wm | cm) {
        const int k = __ffs(wm | cm) - 1;
        const uint32_t bit = 1u << k;
        uint32_t kk = 0;
#pragma unroll
        for (int j = 0; j < PER; ++j)
            if (j == k) kk = key[j];
        const uint32_t id = ID(k);
        if (wm & bit) {
            if (pw < (uint32_t)a.K) S.win_s[pw] = id;
            ++pw;
        } else {
            const uint64_t c = ((uint64_t)kk << 32) | (uint64_t)(~id);
            if (pc < (uint32_t)kRowCands) S.cand_s[pc] = c;
            else if (pc < (uint32_t)ccap) gcand[pc] = c;
            ++pc;
        }
        wm &= ~bit;
        cm &= ~bit;
    }
    __syncthreads();   // every thread has read tot_s
    if (threadIdx.x == 0) {
        S.tot_s[0] += tot & 0xFFFFu;
        S.tot_s[1] += tot >> 16;
    }
    __syncthreads();
}

// d0 (the digit holding the K-th best element) from this thread's four bins, highest first
// (thread 0 owns the top bins). Sets many / d0 / above for every thread.
__device__ __forceinline__ void row_threshold(const RowState& S, const uint32_t (&b4)[4], int K,
                                              bool& many, int& d0, uint32_t& above) {
    const int tid = threadIdx.x;
    const uint32_t local = b4[0] + b4[1] + b4[2] + b4[3];
    uint32_t total;
    const uint32_t excl = row_excl_scan(local, S.wsum, total);
    if (excl < (uint32_t)K && excl + local >= (uint32_t)K) {
        uint32_t acc = excl;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (acc < (uint32_t)K && acc + b4[j] >= (uint32_t)K) {
                S.dig_s[0] = 4 * (kRowThreads - 1 - tid) + 3 - j;
                S.dig_s[1] = (int)acc;
            }
            acc += b4[j];
        }
    }
    __syncthreads();
    many = total >= (uint32_t)K;
    d0 = many ? S.dig_s[0] : -1;
    above = many ? (uint32_t)S.dig_s[1] : total;
    __syncthreads();
}

// Refinement, picks and the ordered output of one gathered row, after every element was
// classified.
__device__ void row_finalize(const TopkDev& a, const RowState& S, int r, int64_t n,
                             uint32_t id_lim, bool many, int d0, uint32_t above, int ccap) {
    const int tid = threadIdx.x;
    const int K = a.K;
    const uint32_t nwin_all = S.tot_s[0], ncand = S.tot_s[1];
    const uint32_t nwin = min(nwin_all, (uint32_t)K);
    if (tid == 0 && (nwin_all > (uint32_t)K || (many && nwin_all != above)))
        set_status(a.status, CSA2_DEV_BAD_COUNT);
    __syncthreads();
    uint64_t* gcand = a.cands + (int64_t)r * a.ccap;

    if (many) {
        const uint32_t need = (uint32_t)K - above;
        const bool from_row = ncand > (uint32_t)max(ccap, kRowCands);
        const int64_t nsrc = from_row ? n : (int64_t)ncand;
        // candidate i of the source (false: not a candidate)
        auto cand = [&](int64_t i, uint64_t& c) -> bool {
            if (from_row) {
                const uint32_t kk = elem_key(a, r, i);
                const int32_t v = ld_dep(a.ids + (int64_t)r * a.ld + i);
                if (v < 0 || (uint32_t)v >= id_lim) return false;
                c = ((uint64_t)kk << 32) | (uint64_t)(~(uint32_t)v);
                return (int)(kk >> 20) == d0;
            }
            c = i < kRowCands ? S.cand_s[i] : __ldcg(gcand + i);
            return true;
        };
        uint64_t prefix = (uint64_t)d0;
        int shift = 52;
        uint32_t rem = need;
        while (shift > 0) {
            const int nb = shift < 8 ? shift : 8;
            if (tid < 256) S.hist[tid] = 0u;
            __syncthreads();
            for (int64_t i = tid; i < nsrc; i += kRowThreads) {
                uint64_t c;
                if (cand(i, c) && (c >> shift) == prefix)
                    atomicAdd(&S.hist[(c >> (shift - nb)) & ((1u << nb) - 1u)], 1u);
            }
            __syncthreads();
            if (tid < 32) warp_find_digit256(S.hist, rem, S.dig_s);
            __syncthreads();
            const int d = S.dig_s[0];
            const uint32_t ab = (uint32_t)S.dig_s[1], inbin = (uint32_t)S.dig_s[2];
            __syncthreads();   // dig_s is rewritten by the next pass
            if (d < 0) {
                if (tid == 0) set_status(a.status, CSA2_DEV_BAD_COUNT);
                prefix = 0;
                shift = 0;
                break;
            }
            rem -= ab;
            prefix = (prefix << nb) | (uint64_t)d;
            shift -= nb;
            if (inbin == rem) break;   // the whole bin is taken
        }
        const uint64_t T = prefix << shift;
        // mark the chosen candidates
        for (int64_t i = tid; i < nsrc; i += kRowThreads) {
            uint64_t c;
            if (cand(i, c) && c >= T) {
                const uint32_t id = ~(uint32_t)(c & 0xFFFFFFFFu);
                const uint32_t pos = atomicAdd(&S.tot_s[0], 1u);
                if (pos < (uint32_t)K) S.bm[pos] = id;
            }
        }
    }
    // winners
    for (uint32_t i = tid; i < nwin; i += kRowThreads)
        S.bm[i] = S.win_s[i];   // slots [0, nwin) of the pick list; candidates were appended after
    __syncthreads();

    // ---- emit in ascending id order ----------------------------------------------------------
    const int32_t lim = a.expand8 ? ld_dep(a.expand_limit + r) : 0;
    int32_t* o = a.out + (int64_t)r * K * (a.expand8 ? 8 : 1);
    auto emit = [&](uint32_t slot, int64_t id) {
        if (slot >= (uint32_t)K) return;
        if (!a.expand8) {
            o[slot] = (int32_t)id;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int64_t pos = id * 8 + e;
                o[(int64_t)slot * 8 + e] = pos < lim ? (int32_t)pos : -1;
            }
        }
    };
    // winners occupy [0, nwin), candidates were appended from tot_s[0] = nwin_all on: a
    // bitonic sort of the (distinct) picks, padded to a power of two (at most kMaxK)
    const int npick = (int)min(many ? S.tot_s[0] : nwin, (uint32_t)K);
    int p2 = 1;
    while (p2 < npick) p2 <<= 1;
    for (int i = npick + tid; i < p2; i += kRowThreads) S.bm[i] = 0xFFFFFFFFu;
    __syncthreads();
    for (int k = 2; k <= p2; k <<= 1)
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < p2; i += kRowThreads) {
                const int l = i ^ j;
                if (l > i) {
                    const uint32_t x = S.bm[i], y = S.bm[l];
                    if ((x > y) == ((i & k) == 0)) {
                        S.bm[i] = y;
                        S.bm[l] = x;
                    }
                }
            }
            __syncthreads();
        }
    for (int i = tid; i < npick; i += kRowThreads) emit((uint32_t)i, S.bm[i]);
    const int mult = a.expand8 ? 8 : 1;
    for (int i = npick * mult + tid; i < K * mult; i += kRowThreads) o[i] = -1;
}

// Rows of gathered ids (Reindex over the candidate pool): one CTA per row, elements read in
// batches of 8 per thread with plain loads, classified into winner and candidate lists.
__global__ void __launch_bounds__(kRowThreads, 1) topk_gather_kernel(const TopkDev a) {
    const int ccap = a.ccap;
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ uint32_t wsum[40];
    __shared__ int dig_s[4];
    __shared__ uint32_t tot_s[2];
    RowState S;
    S.hist = reinterpret_cast<uint32_t*>(dsm + kRowOffHist);
    S.cand_s = reinterpret_cast<uint64_t*>(dsm + kRowOffCand);
    S.win_s = reinterpret_cast<uint32_t*>(dsm + kRowOffWin);
    S.bm = reinterpret_cast<uint32_t*>(dsm + kRowOffBm);
    S.wsum = wsum;
    S.dig_s = dig_s;
    S.tot_s = tot_s;
    const int r = (int)blockIdx.x;
    const int tid = threadIdx.x;
    grid_dep_launch();
    grid_dep_wait();
    const int64_t n = row_len(a, r);
    const int K = a.K;
    const uint32_t id_lim = (uint32_t)max(0, ld_dep(a.id_limit + r));
    if (tid == 0) {
        tot_s[0] = tot_s[1] = 0u;
        dig_s[0] = -1;
        dig_s[1] = 0;
    }
    bool many;
    int d0;
    uint32_t above;
    constexpr int PER = kRowPerIds;
    constexpr int BATCH = kRowThreads * PER;
    uint32_t key[PER], id[PER];
    auto load = [&](int64_t base) {
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int64_t i = base + (int64_t)k * kRowThreads + tid;
            key[k] = i < n ? elem_key(a, r, i) : 0u;
            id[k] = i < n ? (uint32_t)ld_dep(a.ids + (int64_t)r * a.ld + i) : 0xFFFFFFFFu;
        }
    };
    load(0);
    const uint4 h4 = reinterpret_cast<const uint4*>(a.hist + (int64_t)r * kBinsT)[kRowThreads - 1 - tid];
    const uint32_t b4[4] = {h4.w, h4.z, h4.y, h4.x};
    row_threshold(S, b4, K, many, d0, above);
    for (int64_t base = 0; base < n; base += BATCH) {
        if (base > 0) load(base);
        uint32_t valid = 0;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int64_t i = base + (int64_t)k * kRowThreads + tid;
            if (i < n && (int32_t)id[k] >= 0 && id[k] < id_lim) valid |= 1u << k;
        }
        row_classify<PER>(a, S, r, key, [&](int k) {
            uint32_t v = 0;
#pragma unroll
            for (int j = 0; j < PER; ++j)
                if (j == k) v = id[j];
            return v;
        }, valid, many, d0, ccap);
    }
    row_finalize(a, S, r, n, id_lim, many, d0, above, ccap);
}

// ---- rows by position: picks marked in a bitmap of positions ---------------------------------
// One row per CTA, or per cluster of CL CTAs that split it into parts. Each CTA's part
// streams into shared memory by bulk copies (a ring of `ring` chunks of NT x 8 elements; a
// single SM keeps far more bytes in flight that way than with per-thread loads); the few
// elements before the first and after the last 16-byte unit are read directly. Winners
// (first digit above d0) are set in a bitmap of positions as they are read; candidates
// (first digit d0) go to a list through one warp-aggregated atomic per warp and chunk.
// Bitmap, list and counters live in the shared memory of the row's first CTA (the others
// write them through distributed shared memory); that CTA then finds the exact `need`-th
// best candidate by 8-bit radix refinement and emits the set bits in ascending order. No list
// of winners is kept, so the block-wide steps are d0, one barrier per chunk, the refinement
// passes and the final prefix sum.
constexpr int kBmPer = 8;                     // elements per thread per chunk
constexpr int kBmCands = 3968;                // candidates kept in shared memory
constexpr int64_t kBmMaxN = 262144;
constexpr size_t kBmOffHist = 0;                                   // u32[4096]
constexpr size_t kBmOffCand = kBmOffHist + 4 * kBinsT;             // u64[kBmCands]
constexpr size_t kBmOffH2 = kBmOffCand + 8 * (size_t)kBmCands;     // u32[256]
constexpr size_t kBmOffBm = kBmOffH2 + 4 * 256;                      // u32[bitmap words]
__host__ __device__ constexpr size_t bm_off_ring(int words) {
    return (kBmOffBm + 4 * (size_t)words + 127) & ~(size_t)127;
}
__host__ __device__ constexpr size_t bm_chunk_bytes(int nt) { return (size_t)nt * kBmPer * 4; }
__host__ __device__ constexpr size_t bm_off_bar(int words, int nt, int ring) {
    return bm_off_ring(words) + (size_t)ring * bm_chunk_bytes(nt);
}
__host__ __device__ constexpr size_t bm_smem(int words, int nt, int ring) {
    return bm_off_bar(words, nt, ring) + 8 * (size_t)(ring + 1);
}

template <int NT>
__device__ __forceinline__ uint32_t bm_excl_scan(uint32_t v, uint32_t* wsum, uint32_t& total) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t x = lane < NW ? wsum[lane] : 0u;
        uint32_t xi = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(0xffffffffu, xi, o);
            if (lane >= o) xi += u;
        }
        if (lane < NW) wsum[lane] = xi - x;
        if (lane == 31) wsum[32] = xi;
    }
    __syncthreads();
    const uint32_t res = wsum[warp] + incl - v;
    total = wsum[32];
    __syncthreads();
    return res;
}

template <int NT, int CL>
__global__ void __launch_bounds__(NT, 1024 / NT) topk_bitmap_kernel(const TopkDev a) {
    static_assert(NT % 32 == 0 && kBinsT % NT == 0, "block size");
    constexpr int BPT = kBinsT / NT;                    // first-digit bins per thread
    constexpr int CE = NT * kBmPer;                     // elements per chunk
    extern __shared__ __align__(16) uint8_t dsm[];
    const int words = a.bitmap_words, ring = a.ring;
    uint32_t* hist = reinterpret_cast<uint32_t*>(dsm + kBmOffHist);
    uint64_t* cand = reinterpret_cast<uint64_t*>(dsm + kBmOffCand);
    uint32_t* bm = reinterpret_cast<uint32_t*>(dsm + kBmOffBm);
    // the candidates' next 8 key bits, counted as they are found: the first refinement
    // pass's histogram
    uint32_t* h2 = reinterpret_cast<uint32_t*>(dsm + kBmOffH2);
    const uint32_t* buf = reinterpret_cast<const uint32_t*>(dsm + bm_off_ring(words));
    uint64_t* bar = reinterpret_cast<uint64_t*>(dsm + bm_off_bar(words, NT, ring));
    __shared__ uint32_t wsum[40];
    __shared__ int dig_s[4];
    __shared__ uint32_t cnt_s[2];   // this CTA's candidates and winners
    __shared__ uint32_t part_s[16]; // first CTA: every CTA's candidate, then winner count
    const int r = CL > 1 ? (int)blockIdx.y : (int)blockIdx.x;
    const uint32_t crank = CL > 1 ? cluster_rank() : 0u;
    const int tid = threadIdx.x, lane = tid & 31;
    const int K = a.K;
    grid_dep_launch();
    if (tid == 0) {
        for (int i = 0; i <= ring; ++i) mbar_init(&bar[i], 1);
        fence_mbar_init();
        cnt_s[0] = cnt_s[1] = 0u;
        dig_s[0] = -1;
        dig_s[1] = 0;
    }
    for (int i = tid; i < 256; i += NT) h2[i] = 0u;
    __syncthreads();
    // every CTA of the cluster has started before any writes another's shared memory (the
    // matching wait comes after the classification)
    if constexpr (CL > 1) cluster_arrive();
    grid_dep_wait();

    int64_t n = row_len(a, r);
    n = n < 0 ? 0 : (n > a.ld ? a.ld : n);
    n = n < (int64_t)words * 32 ? n : (int64_t)words * 32;
    // this CTA's part [p0, p1) of the row: whole bitmap words, so that every CTA builds its
    // own words in its own shared memory
    const int64_t part = CL > 1 ? ((((n + CL - 1) / CL) + 31) & ~(int64_t)31) : n;
    const int64_t p0 = (int64_t)crank * part < n ? (int64_t)crank * part : n;
    const int64_t p1 = p0 + part < n ? p0 + part : n;
    // this CTA's words [w0, w1): its part starts on a word boundary unless it is empty
    const int64_t pw0 = p0 >> 5, pw1 = p1 > p0 ? (p1 + 31) >> 5 : pw0;
    for (int64_t wi = pw0 + tid; wi < pw1; wi += NT) bm[wi] = 0u;
    const uint32_t* src = a.scores ? reinterpret_cast<const uint32_t*>(a.scores) : a.keys;
    const uint32_t* rowp = src + (int64_t)r * a.ld;
    // whole 16-byte units [b0, b1) by bulk copies; [p0, b0) and [b1, p1) read directly
    const int64_t lead = (int64_t)(((16u - (reinterpret_cast<uintptr_t>(rowp + p0) & 15u)) & 15u) >> 2);
    const int64_t b0 = p0 + lead < p1 ? p0 + lead : p1;
    const int64_t b1 = b0 + ((p1 - b0) & ~(int64_t)3);
    const int nch = (int)((b1 - b0 + CE - 1) / CE);
    auto issue = [&](int c) {
        const int64_t e0 = b0 + (int64_t)c * CE;
        const int64_t cnt = b1 - e0 < CE ? b1 - e0 : CE;
        const int slot = c % ring;
        mbar_arrive_expect_tx(&bar[1 + slot], (uint32_t)(cnt * 4));
        bulk_load(const_cast<uint32_t*>(buf) + (size_t)slot * CE, rowp + e0, (uint32_t)(cnt * 4), &bar[1 + slot]);
    };
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar[0], 4u * kBinsT);
        bulk_load(hist, a.hist + (int64_t)r * kBinsT, 4u * kBinsT, &bar[0]);
        for (int c = 0; c < nch && c < ring; ++c) issue(c);
    }
    // the stray elements: one per thread among the first few
    const int64_t xi = tid < b0 - p0 ? p0 + tid : (tid - (b0 - p0) < p1 - b1 ? b1 + (tid - (b0 - p0)) : -1);
    const uint32_t xraw = xi >= 0 ? ld_dep(rowp + xi) : 0u;
    auto key_of = [&](uint32_t v) { return a.scores ? score_key(__uint_as_float(v)) : v; };

    // ---- d0: the first digit that holds the K-th best element (every CTA) -------------------
    bool ok = mbar_wait(&bar[0], 0, a.status);
    uint32_t b[BPT], local = 0;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {   // thread 0 owns the highest bins, highest first
        b[j] = hist[kBinsT - 1 - BPT * tid - j];
        local += b[j];
    }
    uint32_t total;
    const uint32_t excl = bm_excl_scan<NT>(local, wsum, total);
    if (excl < (uint32_t)K && excl + local >= (uint32_t)K) {
        uint32_t acc = excl;
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
            if (acc < (uint32_t)K && acc + b[j] >= (uint32_t)K) {
                dig_s[0] = kBinsT - 1 - BPT * tid - j;
                dig_s[1] = (int)acc;
            }
            acc += b[j];
        }
    }
    __syncthreads();
    const bool many = total >= (uint32_t)K;
    const int d0 = many ? dig_s[0] : -1;
    const uint32_t above = many ? (uint32_t)dig_s[1] : total;

    // ---- classify: winners into the bitmap, candidates into the list ----------------------------
    // (addresses in the first CTA of the cluster; plain shared memory without a cluster)
    // Every CTA marks its own words of the bitmap and fills its own part of the candidate
    // list in its own shared memory, both at the places they take in the first CTA; the
    // others copy them there once classified.
    constexpr uint32_t RC = (uint32_t)(kBmCands / CL);
    auto set_bit = [&](int64_t pos) { atomicOr(&bm[pos >> 5], 1u << (pos & 31)); };
    auto put_cand = [&](uint32_t q, uint64_t c) {
        atomicAdd(&h2[(uint32_t)(c >> 44) & 0xFFu], 1u);
        if (q < RC) cand[crank * RC + q] = c;
    };
    auto reserve = [&](uint32_t cnt) -> uint32_t { return atomicAdd(&cnt_s[0], cnt); };
    uint32_t nwin_t = 0;   // this thread's winners
    if (xi >= 0) {
        const uint32_t kk = key_of(xraw);
        const int dig = (int)(kk >> 20);
        if (!many || dig > d0) {
            set_bit(xi);
            ++nwin_t;
        } else if (dig == d0) {
            put_cand(reserve(1u), ((uint64_t)kk << 32) | (uint64_t)(~(uint32_t)xi));
        }
    }
    for (int c = 0; c < nch; ++c) {
        const int slot = c % ring;
        if (!mbar_wait(&bar[1 + slot], (uint32_t)((c / ring) & 1), a.status)) ok = false;
        const int64_t e0 = b0 + (int64_t)c * CE;
        const int cnt = (int)(b1 - e0 < CE ? b1 - e0 : CE);
        const uint32_t* cb_ = buf + (size_t)slot * CE;
        uint32_t key[kBmPer];
        uint32_t nc_t = 0;   // this thread's candidates in the chunk
#pragma unroll
        for (int j = 0; j < kBmPer; ++j) {
            const int i = j * NT + tid;
            key[j] = i < cnt ? key_of(cb_[i]) : 0u;
            const int dig = (int)(key[j] >> 20);
            if (i < cnt && (!many || dig > d0)) {
                set_bit(e0 + i);
                ++nwin_t;
            }
            nc_t += (i < cnt && many && dig == d0) ? 1u : 0u;
        }
        const uint32_t ncw = __reduce_add_sync(0xffffffffu, nc_t);
        __syncthreads();   // every thread has read the slot: refill it
        if (tid == 0 && ok && c + ring < nch) issue(c + ring);
        if (ncw) {
            // one atomic per warp reserves its candidates' slots
            uint32_t q = 0;
            if (lane == 0) q = reserve(ncw);
            q = __shfl_sync(0xffffffffu, q, 0);
#pragma unroll
            for (int j = 0; j < kBmPer; ++j) {
                const int i = j * NT + tid;
                const bool isc = i < cnt && many && (int)(key[j] >> 20) == d0;
                const uint32_t cb = __ballot_sync(0xffffffffu, isc);
                if (isc)
                    put_cand(q + __popc(cb & ((1u << lane) - 1u)),
                             ((uint64_t)key[j] << 32) | (uint64_t)(~(uint32_t)(e0 + i)));
                q += (uint32_t)__popc(cb);
            }
        }
    }
    // this warp's winners
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nwin_t += __shfl_xor_sync(0xffffffffu, nwin_t, o);
    if (lane == 0 && nwin_t) atomicAdd(&cnt_s[1], nwin_t);
    __syncthreads();
    if constexpr (CL > 1) {
        cluster_wait();
        if (crank != 0) {
            // this CTA's words, candidates and counts into the first CTA
            const uint32_t bm0 = peer_addr(bm, 0), cand0 = peer_addr(cand, 0);
            for (int64_t wi = pw0 + tid; wi < pw1; wi += NT) st_peer_u32(bm0 + 4u * (uint32_t)wi, bm[wi]);
            const uint32_t nc = min(cnt_s[0], RC);
            for (uint32_t i = tid; i < nc; i += NT)
                st_peer_u64(cand0 + 8u * (crank * RC + i), cand[crank * RC + i]);
            const uint32_t h20 = peer_addr(h2, 0);
            for (int i = tid; i < 256; i += NT)
                if (h2[i]) red_add_peer_u32(h20 + 4u * i, h2[i]);
            if (tid == 0) {
                st_peer_u32(peer_addr(&part_s[crank], 0), cnt_s[0]);
                st_peer_u32(peer_addr(&part_s[CL + crank], 0), cnt_s[1]);
            }
        } else if (tid == 0) {
            part_s[0] = cnt_s[0];
            part_s[CL] = cnt_s[1];
        }
        // every part is in the first CTA's shared memory; the others are done
        cluster_arrive();
        cluster_wait();
        if (crank != 0) return;
    }
    auto part_cands = [&](int k) { return CL > 1 ? part_s[k] : cnt_s[0]; };
    uint32_t ncand = 0, nwin_all = 0;
    bool over = false;
#pragma unroll
    for (int k = 0; k < CL; ++k) {
        const uint32_t c = part_cands(k);
        ncand += c;
        over |= c > RC;
        nwin_all += CL > 1 ? part_s[CL + k] : cnt_s[1];
    }
    if (tid == 0 && (nwin_all > (uint32_t)K || (many && nwin_all != above)))
        set_status(a.status, CSA2_DEV_BAD_COUNT);

    // ---- the exact `need`-th best candidate -------------------------------------------------------
    if (many) {
        const uint32_t need = (uint32_t)K - above;
        const bool from_row = over;   // a part of the list overflowed: read the row again
        const int64_t nsrc = from_row ? n : (int64_t)ncand;
        // candidate i of the list: the parts follow one another
        uint32_t pc[CL];
#pragma unroll
        for (int k = 0; k < CL; ++k) pc[k] = part_cands(k);
        auto cnd = [&](int64_t i, uint64_t& c) -> bool {
            if (from_row) {
                const uint32_t kk = elem_key(a, r, i);
                c = ((uint64_t)kk << 32) | (uint64_t)(~(uint32_t)i);
                return (int)(kk >> 20) == d0;
            }
            uint32_t j = (uint32_t)i, slot = j;
#pragma unroll
            for (int k = 0; k < CL; ++k) {
                if (j < pc[k]) {
                    slot = (uint32_t)k * RC + j;
                    break;
                }
                j -= pc[k];
            }
            c = cand[slot];
            return true;
        };
        uint64_t prefix = (uint64_t)d0;
        int shift = 52;
        uint32_t rem = need;
        bool found = true;
        for (int pass = 0; shift > 0; ++pass) {
            const int nb = shift < 8 ? shift : 8;
            if (pass > 0) {   // the first pass's histogram is h2
                for (int i = tid; i < 256; i += NT) hist[i] = 0u;
                __syncthreads();
                for (int64_t i = tid; i < nsrc; i += NT) {
                    uint64_t c;
                    if (cnd(i, c) && (c >> shift) == prefix)
                        atomicAdd(&hist[(c >> (shift - nb)) & ((1u << nb) - 1u)], 1u);
                }
                __syncthreads();
            }
            if (tid < 32) warp_find_digit256(pass > 0 ? hist : h2, rem, dig_s);
            __syncthreads();
            const int d = dig_s[0];
            const uint32_t ab = (uint32_t)dig_s[1], inbin = (uint32_t)dig_s[2];
            __syncthreads();   // dig_s is rewritten by the next pass
            if (d < 0) {
                if (tid == 0) set_status(a.status, CSA2_DEV_BAD_COUNT);
                found = false;
                break;
            }
            rem -= ab;
            prefix = (prefix << nb) | (uint64_t)d;
            shift -= nb;
            if (inbin == rem) break;   // the whole bin is taken
        }
        if (found) {
            const uint64_t T = prefix << shift;
            for (int64_t i = tid; i < nsrc; i += NT) {
                uint64_t c;
                if (cnd(i, c) && c >= T) {
                    const uint32_t id = ~(uint32_t)(c & 0xFFFFFFFFu);
                    atomicOr(&bm[id >> 5], 1u << (id & 31));
                }
            }
        }
        __syncthreads();
    }

    // ---- emit the set bits in ascending position order -------------------------------------------
    const int32_t lim = a.expand8 ? ld_dep(a.expand_limit + r) : 0;
    emit_bitmap<NT>(bm, (n + 31) >> 5, K, a.out + (int64_t)r * K * (a.expand8 ? 8 : 1), a.expand8, lim,
                    wsum);
}

template <int NT, int CL>
static cudaError_t launch_bitmap(TopkDev a, int64_t max_n, int R, cudaStream_t st) {
    // bitmap words for the longest row; as many chunk buffers as fit beside it (two per SM
    // for 512-thread CTAs: at most 113 KiB each), between 2 and 4
    a.bitmap_words = (int)((max_n + 127) / 128 * 4);
    const size_t cap = NT == 512 ? 113 * 1024 : 227 * 1024;
    int ring = 4;
    while (ring > 2 && bm_smem(a.bitmap_words, NT, ring) > cap) --ring;
    a.ring = ring;
    const size_t smem = bm_smem(a.bitmap_words, NT, ring);
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    auto kern = topk_bitmap_kernel<NT, CL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (CL == 1) return launch_pdl(kern, dim3((unsigned)R), dim3(NT), smem, st, a);
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(CL, (unsigned)R);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, a);
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
    a.bitmap_words = 0;
    a.ring = 0;
    // ids are < id_bound: a bitmap of that many bits orders the picks when it fits
    const int64_t words = (l.id_bound + 31) / 32;
    cudaError_t e;
    if (!l.ids && l.max_n <= kBmMaxN) {
        // Few rows: a cluster per row spreads the reading over more SMs, within one wave:
        // eight 512-thread CTAs per row for rows of 64K elements or more (the pool's 131,072
        // block maxima at 1M context: 22.6 us against 26.3 us with four 1024-thread CTAs),
        // else 1024-thread CTAs (one per SM) while four per row fit, else 512-thread CTAs
        // (two per SM), with at least 4,096 elements per CTA.
        const int sms = device_sm_count();
        if (l.max_n >= 65536 && l.R * 8 <= sms) return launch_bitmap<512, 8>(a, l.max_n, l.R, st);
        if (l.max_n >= 4 * 8192 && l.R * 4 <= sms) return launch_bitmap<1024, 4>(a, l.max_n, l.R, st);
        if (l.max_n >= 8 * 4096 && l.R * 8 <= 2 * sms) return launch_bitmap<512, 8>(a, l.max_n, l.R, st);
        if (l.max_n >= 4 * 4096 && l.R * 4 <= 2 * sms) return launch_bitmap<512, 4>(a, l.max_n, l.R, st);
        if (l.max_n >= 2 * 4096 && l.R * 2 <= 2 * sms) return launch_bitmap<512, 2>(a, l.max_n, l.R, st);
        return launch_bitmap<512, 1>(a, l.max_n, l.R, st);
    }
    if (l.ids && l.max_n <= kRowMaxN) {
        // the picks (at most K) are ordered by a bitonic sort: a bitmap over every possible
        // id would be mostly empty, and zeroing and scanning it cost more than the sort
        const size_t rsmem = kRowOffBm + (size_t)kMaxK * 4;
        e = cudaFuncSetAttribute(topk_gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)rsmem);
        if (e != cudaSuccess) return e;
        return launch_pdl(topk_gather_kernel, dim3((unsigned)l.R), dim3(kRowThreads), rsmem, st, a);
    }
    a.bitmap_words = (l.id_bound > 0 && words * 4 <= 64 * 1024) ? (int)words : 0;
    const size_t smem = (size_t)kSmemCands * 8 +
                        (a.bitmap_words > 0 ? (size_t)a.bitmap_words * 4 : (size_t)kMaxK * 4);
    e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int64_t chunks = (l.max_n + kCollectChunk - 1) / kCollectChunk;
    if (chunks < 1) chunks = 1;
    dim3 grid((unsigned)chunks, (unsigned)l.R);
    return launch_pdl(topk_kernel, grid, dim3(kThreads), smem, st, a);
}

}  // namespace csa2
