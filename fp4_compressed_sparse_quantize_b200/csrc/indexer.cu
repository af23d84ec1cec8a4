// Indexer scoring on the 5th-generation tensor cores (tcgen05), fused with the first
// radix-select histogram of the exact Top-K and with the candidate-pool block maxima.
//
// "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (AI summary),
// Methodology in Plain English: Full layers score every causally visible compressed entry
// with their own indexer query; Reindex layers rescore the latest Full layer's indexer keys
// with their own query but only inside the candidate pool; the first decoder Full layer
// also keeps the blocks with the highest maximum score ("2,048 blocks of 8 positions").
// "DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale LLM Serving", Compressed
// Sparse Attention 2 (CSA2): Full / Reindex / Reuse modes, Top-512.
//
// Score (reading adopted; the pages print no formula):
//     s[r, j] = sum_{h < H_I} w[r, h] * max(0, <q_I[r, h, :], k_I[j, :]>)
//
// Design (one persistent CTA per SM):
//   warp 0      producer: TMA tiles of 128 (or 256) indexer keys (contiguous, 128-byte
//               swizzle) into an S-stage ring; in gather mode (Reindex) cp.async of the
//               pool's rows into the same swizzled layout; plus the query-group operand per
//               row group.
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M = 128 keys,
//               N = G queries x H_I heads, K = 128 channels) into a TMEM accumulator ring.
//   warp 2      does warp 1's mbarrier waits (a wait behind in-flight MMA commits is slow)
//               and posts a go / stop verdict per tile in a two-slot flag ring, up to two
//               tiles ahead of warp 1.
//   then EPI    epilogue groups of 4 warps: tcgen05.ld of one key row per thread,
//               ReLU-weighted head sum in fp32, coalesced score stores, shared-memory
//               histogram of the top 12 key bits per query row (first radix-select digit),
//               8-entry block maxima.
//               The histograms hold two 16-bit bins per word (half the shared memory, one
//               more stage in the ring) and are added to global memory before a bin could
//               pass 65,535.
// Every wait is bounded (2 s) and sets CSA2_DEV_TIMEOUT instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

constexpr int kTileRows = 128;  // keys per tile (MMA M, TMEM lanes)
constexpr int kBins = 4096;     // first radix digit: key >> 20
constexpr int kHW = kBins / 2;  // histogram words in shared memory (two 16-bit bins each)

struct ScanParams {
    int rows;               // query rows R (B*T)
    int G;                  // query rows per row group (they share a key tile)
    int T;                  // query rows per sequence
    int H_I;
    int64_t cap;            // key capacity per sequence
    const int32_t* n_row;   // [R] visible entries per query row (clamped)
    const int64_t* prefix;  // [R/G + 1] exclusive prefix of tiles per row group
    const float* w;         // [R][H_I]
    float* scores;          // [R][ld_scores]
    int64_t ld_scores;
    uint32_t* hist;         // [R][kBins]
    uint32_t* bkey;         // [R][ld_bkey] block-max keys, or null
    int64_t ld_bkey;
    uint32_t* bhist;        // [R][kBins] or null
    const int32_t* pool;    // gather mode: [R][P] positions, -1 = empty
    int P;
    const uint8_t* keys;    // gather mode: raw key base (row-major [B*cap][128*esize])
    const float* kscale;    // compact keys: fp32 scale per key [B*cap]
    int32_t* status;
};

// ---- shared memory plan ----------------------------------------------------------------
template <int NQ, int ESZ, int STAGES, int ACC, int G, int EPI, bool POOL, int TM>
struct ScanSmem {
    static constexpr int kRowsT = kTileRows * TM;         // keys per tile
    static constexpr int kTileBytes = kRowsT * 128 * ESZ;
    static constexpr int kQBytes = NQ * 128 * ESZ;
    static constexpr int kStageOff = 0;
    static constexpr int kQOff = kStageOff + STAGES * kTileBytes;
    // histograms: two 16-bit bins per 32-bit word (flushed before a bin can overflow)
    static constexpr int kHistOff = kQOff + 2 * kQBytes;
    static constexpr int kBHistOff = kHistOff + EPI * G * kBins * 2;
    static constexpr int kWOff = kBHistOff + (POOL ? EPI * kBins * 2 : 0);
    static constexpr int kBarOff = kWOff + EPI * 2 * NQ * 4;
    static constexpr int kNumBars = 2 * STAGES + 4 + 2 * ACC + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 64;
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1 KiB alignment
};

// named barrier of one 128-thread epilogue group (ids 1.. ; 0 is __syncthreads)
__device__ __forceinline__ void epi_bar_sync(int group) {
    asm volatile("bar.sync %0, 128;" ::"r"(group + 1) : "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Last row group g with prefix[g] <= t.
__device__ __forceinline__ int find_group(const int64_t* prefix, int ngroups, int64_t t) {
    int lo = 0, hi = ngroups - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Walks the tile sequence of one CTA and keeps the current row group and its tile range in
// registers (the prefix array is read only when the row group changes).
struct GroupCursor {
    int g;
    int64_t lo, hi;
    __device__ __forceinline__ void init(const int64_t* prefix, int ngroups, int64_t t) {
        g = find_group(prefix, ngroups, t);
        lo = ld_dep(prefix + g);
        hi = ld_dep(prefix + g + 1);
    }
    // returns true when t starts a new row group
    __device__ __forceinline__ bool advance(const int64_t* prefix, int64_t t) {
        bool moved = false;
        while (t >= hi) {
            ++g;
            lo = hi;
            hi = ld_dep(prefix + g + 1);
            moved = true;
        }
        return moved;
    }
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// 8 bytes (compact-key codes: one 16-code group per 16-byte slot)
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// NQ     = MMA N: G * H_I rounded up to a multiple of 16 (padding columns get weight 0)
// ESZ    = 1 (E4M3, kind::f8f6f4) or 2 (bf16, kind::f16)
// GATHER = Reindex: tile rows come from a pool list instead of a contiguous range
// TM     = 128-key halves per tile (one TMA box, TM MMA groups into adjacent TMEM columns)
// One thread issues every tcgen05.mma of the CTA (warp 1); warp 2 does its barrier waits.
// (Issuing from two warps on alternate tiles intermittently never completed an MMA commit
// on the 256K-context workload.)
constexpr int kEpiWarp0 = 3;                      // first epilogue warp

template <int NQ, int ESZ, int STAGES, int ACC, int G, bool GATHER, bool POOL, int EPI, int TM,
          bool KF4>
__global__ void __launch_bounds__(32 * kEpiWarp0 + 128 * EPI, 1)
    scan_kernel(const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_q, const ScanParams p) {
    using L = ScanSmem<NQ, ESZ, STAGES, ACC, G, EPI, POOL, TM>;
    static_assert(ACC % EPI == 0, "each epilogue group owns fixed accumulators");
    static_assert(!GATHER || TM == 1, "gathered tiles are 128 keys");
    static_assert(!KF4 || ESZ == 1, "compact keys take E4M3 queries");
    constexpr int kRowsT = L::kRowsT;
    constexpr int kKSteps = (128 * ESZ) / 32;         // 32 bytes of K per MMA instruction
    constexpr uint32_t kSlab = kRowsT * 128;          // bytes of one 128-byte-wide K slab
    constexpr uint32_t kQHalf = NQ * 128;
    constexpr uint32_t kAccCols = TM * NQ;
    constexpr uint32_t kTmemCols = (ACC * kAccCols <= 32) ? 32 : (ACC * kAccCols <= 64) ? 64
                                 : (ACC * kAccCols <= 128) ? 128 : (ACC * kAccCols <= 256) ? 256
                                 : 512;
    static_assert(ACC * kAccCols <= 512, "TMEM budget");
    // A = keys (compact keys: E2M1, format 5 of kind::f8f6f4; the tensor map unpacks each 16
    // codes into a 16-byte slot, so a key row is 128 bytes as with E4M3), B = queries
    constexpr uint32_t kIdesc =
        make_idesc(128, NQ, KF4 ? 5u : (ESZ == 2 ? 1u : 0u), ESZ == 2 ? 1u : 0u);
    constexpr int kCols = NQ / G;                     // accumulator columns per query row
    constexpr bool kWReg = (G == 1 && NQ <= 64);      // weights kept in registers

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* stage_base = smem + L::kStageOff;
    uint8_t* q_base = smem + L::kQOff;
    uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + L::kHistOff);
    uint32_t* bhist_s = reinterpret_cast<uint32_t*>(smem + L::kBHistOff);
    float* w_s = reinterpret_cast<float*>(smem + L::kWOff);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* qfull = bars + 2 * STAGES;
    uint64_t* qempty = qfull + 2;
    uint64_t* accfull = qempty + 2;
    uint64_t* accempty = accfull + ACC;
    uint64_t* done_bar = accempty + ACC;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8);
    // set when the wait for this CTA's last MMA commit gave up: MMAs may still be in flight,
    // so neither TMEM nor the shared-memory operands may be released or reused
    volatile int* mma_stuck = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 16);
    // the waiter's verdicts for the MMA issuer, two tiles deep: 0 = empty, 1 = go, 2 = stop
    int* go_ring = reinterpret_cast<int*>(smem + L::kMiscOff + 24);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ngroups = p.rows / G;
    grid_dep_launch();

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&qfull[s], 1);
            mbar_init(&qempty[s], 1);
        }
        for (int s = 0; s < ACC; ++s) {
            mbar_init(&accfull[s], 1);
            mbar_init(&accempty[s], 4);
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        *mma_stuck = 0;
        go_ring[0] = go_ring[1] = 0;
        fence_mbar_init();
    }
    if (warp >= kEpiWarp0) {
        for (int i = threadIdx.x - 32 * kEpiWarp0; i < EPI * G * kHW; i += 128 * EPI) hist_s[i] = 0;
        if (POOL)
            for (int i = threadIdx.x - 32 * kEpiWarp0; i < EPI * kHW; i += 128 * EPI) bhist_s[i] = 0;
    }
    if (warp == 1) tmem_alloc(tmem_holder, kTmemCols);
    if (warp == 0 && lane == 0 && !GATHER) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_q);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    // the tile prefix (and everything else in global memory) comes from earlier kernels
    grid_dep_wait();
    const int64_t total = ld_dep(p.prefix + ngroups);
    const int64_t t0 = total * blockIdx.x / gridDim.x;
    const int64_t t1 = total * (blockIdx.x + 1) / gridDim.x;

    if (t0 >= t1) {
        // no tiles for this CTA (uniform): release TMEM below
    } else if (warp == 0) {
        // ------------------------------------------------------------ producer
        GroupCursor cur;
        cur.init(p.prefix, ngroups, t0);
        int qg = -1, qcount = 0;
        int64_t it = 0;
        int gather_prev = -1;   // gather mode: the stage whose copies are still in flight
        const uint64_t policy = l2_policy_evict_first();
        for (int64_t t = t0; t < t1; ++t, ++it) {
            if (*abort_flag) break;
            cur.advance(p.prefix, t);
            const int64_t jt = t - cur.lo;
            const int r0 = cur.g * G;
            const int b = r0 / p.T;
            if (cur.g != qg) {
                const int qs = qcount & 1;
                bool ok = true;
                if (lane == 0) ok = mbar_wait(&qempty[qs], ((qcount >> 1) & 1) ^ 1, p.status);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) { if (lane == 0) *abort_flag = 1; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&qfull[qs], (uint32_t)L::kQBytes);
                    uint8_t* dst = q_base + qs * L::kQBytes;
                    for (int h = 0; h < ESZ; ++h)
                        tma_load_2d(dst + h * kQHalf, &tmap_q, &qfull[qs], h * 64 * (ESZ == 2),
                                    r0 * p.H_I);
                }
                qg = cur.g;
                ++qcount;
            }
            const int s = (int)(it % STAGES);
            const uint32_t round = (uint32_t)(it / STAGES);
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&empty[s], (round & 1) ^ 1, p.status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) { if (lane == 0) *abort_flag = 1; break; }
            uint8_t* dst = stage_base + s * L::kTileBytes;
            if (!GATHER) {
                if (lane == 0) {
                    // compact keys: the unpacking load counts the packed bytes it reads
                    // (64 per key), half of what it writes to shared memory
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(KF4 ? L::kTileBytes / 2
                                                                  : L::kTileBytes));
                    const int64_t row = (int64_t)b * p.cap + jt * kRowsT;
                    // one box of 128 rows per 128-key half (and per 64-channel half for bf16)
#pragma unroll
                    for (int hh = 0; hh < TM; ++hh)
                        for (int h = 0; h < ESZ; ++h)
                            tma_load_2d_hint(dst + h * kSlab + hh * kTileRows * 128, &tmap_k,
                                             &full[s], h * 64 * (ESZ == 2),
                                             (int32_t)(row + hh * kTileRows), policy);
                }
            } else {
                // pool rows of query row r0 (G == 1 in gather mode). The tile's 128 pool
                // positions are loaded first, four per lane, so that no copy waits for its
                // own index load; the rows then go 4 per pass, 8 lanes per row.
                static_assert(!GATHER || kRowsT == 128, "gathered tiles are 128 keys");
                const int32_t* pl = p.pool + (int64_t)r0 * p.P + jt * kRowsT;
                const int n_vis = ld_dep(p.n_row + r0);
                const uint32_t dst_u = smem_u32(dst);
                int pv[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int64_t slot = jt * kRowsT + 32 * k + lane;
                    const int v = (slot < p.P) ? ld_dep(pl + 32 * k + lane) : -1;
                    pv[k] = v >= n_vis ? -1 : v;
                }
#pragma unroll 4
                for (int rr = 0; rr < kRowsT; rr += 4) {
                    const int rl = rr + (lane >> 3);       // 4 rows per pass, 8 lanes per row
                    const int q = rr >> 5;                 // the same for every lane
                    const int pq = q == 0 ? pv[0] : q == 1 ? pv[1] : q == 2 ? pv[2] : pv[3];
                    const int pos = __shfl_sync(0xffffffffu, pq, rl & 31);
                    if (pos >= 0 && KF4) {
                        // compact key: 16 codes (8 bytes) per 16-byte slot, the layout the
                        // unpacking TMA load gives the contiguous tiles; the other half is 0
                        const uint8_t* src = p.keys + ((int64_t)b * p.cap + pos) * CSA2_FP4KEY_CODE_BYTES;
                        const int c = lane & 7;
                        const uint32_t off = rl * 128 + ((c ^ (rl & 7)) << 4);
                        cp_async8(dst_u + off, src + c * 8);
                        asm volatile("st.shared.v2.u32 [%0], {%1, %1};" ::"r"(dst_u + off + 8), "r"(0u)
                                     : "memory");
                    } else if (pos >= 0) {
                        const uint8_t* src = p.keys + ((int64_t)b * p.cap + pos) * (128 * ESZ);
                        for (int h = 0; h < ESZ; ++h) {
                            const int c = lane & 7;         // 16-byte chunk within 128 bytes
                            const uint32_t off = h * kSlab + rl * 128 + ((c ^ (rl & 7)) << 4);
                            cp_async16(dst_u + off, src + h * 128 + c * 16);
                        }
                    }
                }
                // two tiles in flight: the previous tile's copies are waited for (and made
                // visible to the tensor core) only now that this tile's are issued
                cp_async_commit();
                if (gather_prev >= 0) {
                    cp_async_wait<1>();
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[gather_prev]);
                }
                gather_prev = s;
            }
        }
        if (GATHER && gather_prev >= 0) {
            cp_async_wait<0>();
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[gather_prev]);
        }
        // Drain: every TMA issued into this CTA's shared memory must land before exit.
        if (!GATHER && lane == 0) {
            const int64_t n_issued = it;
            for (int64_t k = (n_issued > STAGES ? n_issued - STAGES : 0); k < n_issued; ++k)
                mbar_wait(&full[k % STAGES], (uint32_t)((k / STAGES) & 1), p.status);
            if (qcount > 0) mbar_wait(&qfull[(qcount - 1) & 1], ((qcount - 1) >> 1) & 1, p.status);
        }
    } else if (warp == 1 || warp == 2) {
        // ------------------------------------------------------------ MMA issue (warp 1)
        // and its barrier waits (warp 2). An mbarrier wait by the thread whose MMAs and
        // commits are still in flight costs a few hundred cycles even on a completed phase,
        // so the issuing thread never waits on an mbarrier: warp 2 waits for the key tile,
        // accumulator and query slot of each tile and posts its verdict (go / stop) in a
        // two-slot ring, up to two tiles ahead of warp 1, which reads the verdict with an
        // acquiring load and issues. Both walk the same tile sequence, and every wait on the
        // ring is bounded.
        const bool waiter = warp == 2;
        GroupCursor cur;
        cur.init(p.prefix, ngroups, t0);
        int qg = -1, qcount = 0, qs = 0;
        int64_t it = 0;
        const uint64_t a_desc0 = sw128_desc(smem_u32(stage_base), 16, 1024);
        const uint64_t b_desc0 = sw128_desc(smem_u32(q_base), 16, 1024);
        for (int64_t t = t0; t < t1; ++t, ++it) {
            cur.advance(p.prefix, t);
            const bool newgroup = cur.g != qg;
            const int qs_new = newgroup ? (qcount & 1) : qs;
            const int s = (int)(it % STAGES);
            const int a = (int)(it % ACC);
            int* slot = go_ring + (int)(it & 1);
            if (waiter) {
                bool ok = true;
                if (lane == 0) {
                    ok = !*abort_flag;
                    // the issuer has taken the verdict of tile it - 2
                    if (ok) ok = flag_wait(slot, false, abort_flag, p.status) == 0;
                    if (ok && newgroup)
                        ok = mbar_wait(&qfull[qs_new], (uint32_t)((qcount >> 1) & 1), p.status);
                    if (ok) ok = mbar_wait(&full[s], (uint32_t)((it / STAGES) & 1), p.status);
                    if (ok) ok = mbar_wait(&accempty[a], (uint32_t)(((it / ACC) & 1) ^ 1), p.status);
                    if (!ok) *abort_flag = 1;
                    st_release_cta(slot, ok ? 1 : 2);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            } else {
                // the previous row group's query slot is free once this thread's MMAs are done
                if (lane == 0 && newgroup && qg >= 0) mma_commit(&qempty[qs]);
                int v = 0;
                if (lane == 0) {
                    v = flag_wait(slot, true, abort_flag, p.status);
                    if (v != 1) *abort_flag = 1;
                    st_release_cta(slot, 0);
                }
                v = __shfl_sync(0xffffffffu, v, 0);
                if (v != 1) break;
                if (lane == 0) {
                    tc_fence_after();
                    // descriptor start addresses advance in 16-byte units
                    const uint64_t a_s = a_desc0 + ((uint64_t)(s * L::kTileBytes) >> 4);
                    const uint64_t b_s = b_desc0 + ((uint64_t)(qs_new * L::kQBytes) >> 4);
#pragma unroll
                    for (int hh = 0; hh < TM; ++hh) {
                        const uint32_t d = tmem_base + a * kAccCols + hh * NQ;
#pragma unroll
                        for (int kk = 0; kk < kKSteps; ++kk) {
                            const uint64_t ad = a_s + ((uint64_t)((kk >> 2) * kSlab + hh * 128 * 128 +
                                                                  (kk & 3) * 32) >> 4);
                            const uint64_t bd = b_s + ((uint64_t)((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4);
                            if (ESZ == 1)
                                mma_f8(d, ad, bd, kIdesc, kk > 0);
                            else
                                mma_f16(d, ad, bd, kIdesc, kk > 0);
                        }
                    }
                    mma_commit(&empty[s]);
                    mma_commit(&accfull[a]);
                }
                __syncwarp();
            }
            if (newgroup) {
                qs = qs_new;
                qg = cur.g;
                ++qcount;
            }
        }
        if (!waiter && lane == 0) {
            // all MMAs must complete before TMEM is released. If this wait gives up, the
            // commit never arrived and MMAs may still be reading the stage ring and writing
            // TMEM: the CTA then leaves its TMEM allocated (the status word carries TIMEOUT,
            // after which the caller must discard the context) rather than free columns that
            // the tensor core may still write.
            mma_commit(done_bar);
            if (!mbar_wait(done_bar, 0, p.status)) *mma_stuck = 1;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue groups
        // EPI groups of 4 warps take alternate tiles (group e owns iterations it = e mod
        // EPI and therefore TMEM accumulators a = it mod ACC of that residue), each with its
        // own histograms, weights and named barrier.
        const int e = (warp - kEpiWarp0) >> 2;
        const int et = threadIdx.x - 32 * kEpiWarp0 - 128 * e;  // 0..127 within the group
        const int row = 32 * (warp & 3) + lane;     // TMEM lane == key row within a half
        const uint32_t lane_addr = (uint32_t)(32 * (warp & 3)) << 16;
        uint32_t* hist_e = hist_s + e * G * kHW;
        uint32_t* bhist_e = bhist_s + e * kHW;
        // adds the group's shared histograms of row group g into global memory and clears them
        auto flush = [&](int g) {
            for (int gg = 0; gg < G; ++gg)
                for (int i = et; i < kHW; i += 128) {
                    const uint32_t v = hist_e[gg * kHW + i];
                    if (v) {
                        uint32_t* dst = p.hist + (int64_t)(g * G + gg) * kBins + 2 * i;
                        if (v & 0xFFFFu) atomicAdd(dst, v & 0xFFFFu);
                        if (v >> 16) atomicAdd(dst + 1, v >> 16);
                        hist_e[gg * kHW + i] = 0;
                    }
                }
            if (POOL)
                for (int i = et; i < kHW; i += 128) {
                    const uint32_t v = bhist_e[i];
                    if (v) {
                        uint32_t* dst = p.bhist + (int64_t)(g * G) * kBins + 2 * i;
                        if (v & 0xFFFFu) atomicAdd(dst, v & 0xFFFFu);
                        if (v >> 16) atomicAdd(dst + 1, v >> 16);
                        bhist_e[i] = 0;
                    }
                }
        };
        // a bin gains at most kRowsT per iteration: flush before 65,535 could be passed
        constexpr int kFlushEvery = 65535 / kRowsT;
        int since_flush = 0;
        float* w_e = w_s + e * 2 * NQ;
        GroupCursor cur;
        cur.init(p.prefix, ngroups, t0);
        int gcur = -1, wslot = 0;
        int nvis[G];
        float wr[kWReg ? NQ : 1];
        bool aborted = false;
        for (int64_t it = e; t0 + it < t1; it += EPI) {
            const int64_t t = t0 + it;
            cur.advance(p.prefix, t);
            const int64_t jt = t - cur.lo;
            const int r0 = cur.g * G;
            if (cur.g != gcur) {
                // flush the previous row group's histograms, then load the new weights
                epi_bar_sync(e);
                if (gcur >= 0) flush(gcur);
                since_flush = 0;
                wslot ^= 1;
                for (int i = et; i < NQ; i += 128)
                    w_e[wslot * NQ + i] = (i < G * p.H_I) ? ld_dep(p.w + (int64_t)r0 * p.H_I + i) : 0.f;
                epi_bar_sync(e);
                if (kWReg) {
#pragma unroll
                    for (int h = 0; h < (kWReg ? NQ : 1); ++h) wr[h] = w_e[wslot * NQ + h];
                }
#pragma unroll
                for (int gg = 0; gg < G; ++gg) nvis[gg] = ld_dep(p.n_row + r0 + gg);
                gcur = cur.g;
            }
            if (since_flush == kFlushEvery) {
                epi_bar_sync(e);
                flush(gcur);
                epi_bar_sync(e);
                since_flush = 0;
            }
            ++since_flush;
            const int a = (int)(it % ACC);
            // compact keys: this tile's key scales, loaded before the accumulator wait
            float ks[TM];
#pragma unroll
            for (int hh = 0; hh < TM; ++hh) {
                ks[hh] = 1.f;
                if (KF4) {
                    const int64_t j = jt * kRowsT + hh * 128 + row;
                    const int64_t kb = (int64_t)(r0 / p.T) * p.cap;
                    if (GATHER) {   // pool slot j of query row r0 holds the entry position
                        const int pos = (j < p.P) ? ld_dep(p.pool + (int64_t)r0 * p.P + j) : -1;
                        ks[hh] = (pos >= 0 && pos < p.cap) ? ld_dep(p.kscale + kb + pos) : 0.f;
                    } else {
                        ks[hh] = (j < p.cap) ? ld_dep(p.kscale + kb + j) : 0.f;
                    }
                }
            }
            aborted = aborted || *abort_flag;
            if (!aborted) {
                if (!mbar_wait(&accfull[a], (uint32_t)((it / ACC) & 1), p.status)) {
                    aborted = true;
                    *abort_flag = 1;
                }
            }
            if (aborted) continue;
            tc_fence_after();
            float sc[TM][G];
            const float* wv = w_e + wslot * NQ;
#pragma unroll
            for (int hh = 0; hh < TM; ++hh) {
#pragma unroll
                for (int gg = 0; gg < G; ++gg) {
                    // this query row's kCols columns of half hh; all loads before one wait
                    uint32_t v[kCols];
                    const uint32_t col = tmem_base + lane_addr + a * kAccCols + hh * NQ + gg * kCols;
#pragma unroll
                    for (int c = 0; c < kCols / 16; ++c) {
                        uint32_t (&vc)[16] = *reinterpret_cast<uint32_t(*)[16]>(v + 16 * c);
                        tmem_ld16(col + c * 16, vc);
                    }
                    tmem_ld_wait();
                    // four independent accumulation chains (heads h mod 4), two per packed
                    // f32x2 FMA; padding columns have weight 0
                    uint64_t c01 = 0ull, c23 = 0ull;
#pragma unroll
                    for (int h = 0; h < kCols; h += 4) {
                        auto wgt = [&](int x) { return kWReg ? wr[kWReg ? x : 0] : wv[gg * kCols + x]; };
                        auto pos = [&](int x) { return fmaxf(__uint_as_float(v[x]), 0.f); };
                        c01 = ffma2(f2pack(wgt(h), wgt(h + 1)), f2pack(pos(h), pos(h + 1)), c01);
                        c23 = ffma2(f2pack(wgt(h + 2), wgt(h + 3)), f2pack(pos(h + 2), pos(h + 3)), c23);
                    }
                    float s4[4];
                    f2unpack(c01, s4[0], s4[1]);
                    f2unpack(c23, s4[2], s4[3]);
                    float sv = (s4[0] + s4[1]) + (s4[2] + s4[3]);
                    if (KF4) sv *= ks[hh];   // the key's scale is >= 0: it leaves the ReLU
                    sc[hh][gg] = sv + 0.0f;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[a]);

#pragma unroll
            for (int hh = 0; hh < TM; ++hh) {
                const int64_t j = jt * kRowsT + hh * 128 + row;   // entry (or pool slot)
#pragma unroll
                for (int gg = 0; gg < G; ++gg) {
                    const int r = r0 + gg;
                    bool vis;
                    if (!GATHER) {
                        vis = j < nvis[gg];
                    } else {
                        int pos = (j < p.P) ? ld_dep(p.pool + (int64_t)r * p.P + j) : -1;
                        vis = pos >= 0 && pos < nvis[gg];
                    }
                    const float scv = sc[hh][gg];
                    const uint32_t key = score_key(scv);
                    if (vis) p.scores[(int64_t)r * p.ld_scores + j] = scv;
                    {
                        // scores cluster in a few bins: one shared atomic per distinct bin
                        const uint32_t bin = vis ? (key >> 20) : 0xFFFFFFFFu;
                        const uint32_t peers = __match_any_sync(0xffffffffu, bin);
                        if (vis && (lane == __ffs(peers) - 1))
                            atomicAdd(&hist_e[gg * kHW + (bin >> 1)],
                                      (uint32_t)__popc(peers) << (16 * (bin & 1)));
                    }
                    if (POOL) {
                        uint32_t bk = vis ? key : 0u;
                        bk = max(bk, __shfl_xor_sync(0xffffffffu, bk, 1));
                        bk = max(bk, __shfl_xor_sync(0xffffffffu, bk, 2));
                        bk = max(bk, __shfl_xor_sync(0xffffffffu, bk, 4));
                        const bool lead = (row & 7) == 0 && j < nvis[gg];
                        if (lead) p.bkey[(int64_t)r * p.ld_bkey + (j >> 3)] = bk;
                        const uint32_t bbin = lead ? (bk >> 20) : 0xFFFFFFFFu;
                        const uint32_t peers = __match_any_sync(0xffffffffu, bbin);
                        if (lead && (lane == __ffs(peers) - 1))
                            atomicAdd(&bhist_e[bbin >> 1], (uint32_t)__popc(peers) << (16 * (bbin & 1)));
                    }
                }
            }
        }
        // final flush
        epi_bar_sync(e);
        if (gcur >= 0) flush(gcur);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1 && !*mma_stuck) tmem_dealloc(tmem_base, kTmemCols);
}

// ---- per-row visible counts and tile prefix ---------------------------------------------
// decode: n_row[r] = n_vis0[r]; prefill: n_row[b*T+t] = floor((q_pos0[b]+t+1)/ratio).
// Counts are clamped to [0, cap] (CSA2_DEV_BAD_COUNT when clamping was needed); gather
// mode counts pool slots instead of entries for the tile prefix. Every CTA also clears its
// share of the histograms and counters that the scan and Top-K accumulate into; CTA 0
// computes the counts and the prefix.
__global__ void __launch_bounds__(1024) prep_rows_kernel(
    int rows, int T, int G, const int32_t* n_vis0, const int32_t* q_pos0, int ratio,
    int64_t cap, int P_gather, int tile_rows, int32_t* n_row, int64_t* prefix,
    int32_t* status, const ZeroList zero) {
    __shared__ int64_t warp_sums[32];
    __shared__ int64_t carry;
    grid_dep_launch();
    grid_dep_wait();
#pragma unroll
    for (int k = 0; k < 4; ++k)
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < zero.n16[k];
             i += (int64_t)gridDim.x * blockDim.x)
            zero.p[k][i] = make_uint4(0u, 0u, 0u, 0u);
    if (blockIdx.x != 0) return;
    if (threadIdx.x == 0) carry = 0;
    const int ngroups = rows / G;
    for (int base = 0; base < rows; base += blockDim.x) {
        const int r = base + threadIdx.x;
        if (r < rows) {
            int64_t n;
            if (q_pos0) {
                const int b = r / T, t = r - b * T;
                n = ((int64_t)ld_dep(q_pos0 + b) + t + 1) / ratio;
            } else {
                n = ld_dep(n_vis0 + r);
            }
            if (n < 0 || n > cap) {
                set_status(status, CSA2_DEV_BAD_COUNT);
                n = n < 0 ? 0 : cap;
            }
            n_row[r] = (int32_t)n;
        }
    }
    __syncthreads();
    for (int base = 0; base < ngroups; base += blockDim.x) {
        const int gi = base + threadIdx.x;
        int64_t tiles = 0;
        if (gi < ngroups) {
            const int64_t n = P_gather > 0 ? P_gather : n_row[gi * G + G - 1];
            tiles = (n + tile_rows - 1) / tile_rows;
        }
        // block-wide exclusive scan of `tiles`
        int64_t v = tiles;
        for (int o = 1; o < 32; o <<= 1) {
            int64_t u = __shfl_up_sync(0xffffffffu, v, o);
            if ((threadIdx.x & 31) >= o) v += u;
        }
        if ((threadIdx.x & 31) == 31) warp_sums[threadIdx.x >> 5] = v;
        __syncthreads();
        if (threadIdx.x < 32) {
            int64_t ws = warp_sums[threadIdx.x];
            for (int o = 1; o < 32; o <<= 1) {
                int64_t u = __shfl_up_sync(0xffffffffu, ws, o);
                if (threadIdx.x >= o) ws += u;
            }
            warp_sums[threadIdx.x] = ws;
        }
        __syncthreads();
        const int64_t before = carry + (threadIdx.x >= 32 ? warp_sums[(threadIdx.x >> 5) - 1] : 0) +
                               v - tiles;
        if (gi < ngroups) prefix[gi] = before;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = before + tiles;
        __syncthreads();
    }
    if (threadIdx.x == 0) prefix[ngroups] = carry;
}

// ---- host side -------------------------------------------------------------------------------

// 2-D map over a [rows][row_bytes] byte matrix, box = 128 bytes x box_rows, 128B swizzle.
static bool make_map(CUtensorMap* m, const void* base, int64_t rows, int esz, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const CUtensorMapDataType dt =
        esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    cuuint64_t dims[2] = {(cuuint64_t)128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(128 * esz)};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D map over compact keys: [rows] x 128 E2M1 codes packed 64 bytes per row; the load
// unpacks every 16 codes (8 bytes) into a 16-byte slot, giving 128-byte rows in shared
// memory (the operand layout of an E2M1 kind::f8f6f4 MMA), 128-byte swizzle.
static bool make_map_fp4(CUtensorMap* m, const void* base, int64_t rows, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)CSA2_FP4KEY_CODE_BYTES};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims,
                     strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// SM count of the current device (looked up per call: one process may drive GPUs of
// different sizes)
static int num_sms() { return device_sm_count(); }

// Largest stage count (<= 8) whose shared-memory plan fits in one SM.
template <int NQ, int ESZ, int ACC, int G, int EPI, bool POOL, int TM>
constexpr int pick_stages() {
    return ScanSmem<NQ, ESZ, 8, ACC, G, EPI, POOL, TM>::kAlloc <= 232448 ? 8
         : ScanSmem<NQ, ESZ, 7, ACC, G, EPI, POOL, TM>::kAlloc <= 232448 ? 7
         : ScanSmem<NQ, ESZ, 6, ACC, G, EPI, POOL, TM>::kAlloc <= 232448 ? 6
         : ScanSmem<NQ, ESZ, 5, ACC, G, EPI, POOL, TM>::kAlloc <= 232448 ? 5
         : ScanSmem<NQ, ESZ, 4, ACC, G, EPI, POOL, TM>::kAlloc <= 232448 ? 4
         : ScanSmem<NQ, ESZ, 3, ACC, G, EPI, POOL, TM>::kAlloc <= 232448 ? 3 : 2;
}

template <int NQ, int ESZ, int G, bool GATHER, bool POOL, bool KF4 = false>
static cudaError_t launch_scan_t(const CUtensorMap& mk, const CUtensorMap& mq,
                                 const ScanParams& p, cudaStream_t st) {
    // 384-key tiles for one FP8 query row per tile and 256-key tiles for two (prefill): the
    // per-tile hand-over (mbarrier waits behind in-flight commits, the verdict, the
    // commits) costs about the same whatever the tile holds, so the tiles are as large as
    // two accumulators allow; two epilogue groups whenever the TMEM accumulators split
    // evenly between them
    constexpr int TM = (G == 1 && !GATHER && ESZ == 1) ? 3 : (G == 2 && !GATHER && ESZ == 1) ? 2 : 1;
    constexpr int kAccCols = TM * NQ;
    constexpr int ACC = kAccCols <= 128 ? 4 : kAccCols <= 256 ? 2 : 1;
    constexpr int EPI = (ACC % 2 == 0 && G <= 2) ? 2 : 1;
    static_assert(ACC % EPI == 0, "accumulators per epilogue group");
    constexpr int STAGES = pick_stages<NQ, ESZ, ACC, G, EPI, POOL, TM>();
    using L = ScanSmem<NQ, ESZ, STAGES, ACC, G, EPI, POOL, TM>;
    static_assert(L::kAlloc <= 232448, "shared memory budget");
    auto kern = scan_kernel<NQ, ESZ, STAGES, ACC, G, GATHER, POOL, EPI, TM, KF4>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::kAlloc);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(num_sms()), dim3(32 * kEpiWarp0 + 128 * EPI), L::kAlloc, st,
                      mk, mq, p);
}

// Dispatch on (padded query columns, element size, group size, mode).
cudaError_t launch_index_scan(const ScanLaunch& a, cudaStream_t st) {
    const int esz = a.esz;
    const int NQreq = a.G * a.H_I;
    int NQ = (NQreq + 15) & ~15;
    CUtensorMap mk, mq;
    memset(&mk, 0, sizeof mk);
    memset(&mq, 0, sizeof mq);
    if (!make_map(&mq, a.q, (int64_t)a.rows * a.H_I, esz, NQ)) return cudaErrorInvalidValue;
    if (a.key_fp4 && esz != 1) return cudaErrorNotSupported;
    if (!a.gather && !a.key_fp4 &&
        !make_map(&mk, a.k, (int64_t)a.B * a.cap, esz, kTileRows))
        return cudaErrorInvalidValue;
    if (a.key_fp4 && !make_map_fp4(&mk, a.k, (int64_t)a.B * a.cap, kTileRows))
        return cudaErrorInvalidValue;
    ScanParams p;
    p.rows = a.rows;
    p.G = a.G;
    p.T = a.T;
    p.H_I = a.H_I;
    p.cap = a.cap;
    p.n_row = a.n_row;
    p.prefix = a.prefix;
    p.w = a.w;
    p.scores = a.scores;
    p.ld_scores = a.ld_scores;
    p.hist = a.hist;
    p.bkey = a.bkey;
    p.ld_bkey = a.ld_bkey;
    p.bhist = a.bhist;
    p.pool = a.pool;
    p.P = a.P;
    p.keys = reinterpret_cast<const uint8_t*>(a.k);
    p.kscale = a.kscale;
    p.status = a.status;

#define CSA2_SCAN(NQv, ESZv, Gv, GA, PO) return launch_scan_t<NQv, ESZv, Gv, GA, PO>(mk, mq, p, st)
#define CSA2_SCAN_NQ(ESZv, GA, PO)                    \
    do {                                              \
        if (NQ <= 16) CSA2_SCAN(16, ESZv, 1, GA, PO); \
        if (NQ <= 32) CSA2_SCAN(32, ESZv, 1, GA, PO); \
        if (NQ <= 64) CSA2_SCAN(64, ESZv, 1, GA, PO); \
        CSA2_SCAN(128, ESZv, 1, GA, PO);              \
    } while (0)

    if (a.key_fp4) {
#define CSA2_SCAN4(NQv, Gv, PO) return launch_scan_t<NQv, 1, Gv, false, PO, true>(mk, mq, p, st)
#define CSA2_SCAN4G(NQv) return launch_scan_t<NQv, 1, 1, true, false, true>(mk, mq, p, st)
        if (a.gather) {
            if (a.G != 1) return cudaErrorNotSupported;
            if (NQ <= 16) CSA2_SCAN4G(16);
            if (NQ <= 32) CSA2_SCAN4G(32);
            if (NQ <= 64) CSA2_SCAN4G(64);
            CSA2_SCAN4G(128);
        }
        if (a.G == 1) {
            if (a.pool_build) {
                if (NQ <= 16) CSA2_SCAN4(16, 1, true);
                if (NQ <= 32) CSA2_SCAN4(32, 1, true);
                if (NQ <= 64) CSA2_SCAN4(64, 1, true);
                CSA2_SCAN4(128, 1, true);
            }
            if (NQ <= 16) CSA2_SCAN4(16, 1, false);
            if (NQ <= 32) CSA2_SCAN4(32, 1, false);
            if (NQ <= 64) CSA2_SCAN4(64, 1, false);
            CSA2_SCAN4(128, 1, false);
        } else if (a.G == 2 && NQ <= 128 && !a.pool_build) {
            CSA2_SCAN4(128, 2, false);
        }
#undef CSA2_SCAN4G
#undef CSA2_SCAN4
        return cudaErrorNotSupported;
    }
    if (a.G == 1) {
        if (a.gather) {
            if (esz == 1) CSA2_SCAN_NQ(1, true, false);
            CSA2_SCAN_NQ(2, true, false);
        }
        if (esz == 1) {
            if (a.pool_build) CSA2_SCAN_NQ(1, false, true);
            CSA2_SCAN_NQ(1, false, false);
        }
        if (a.pool_build) CSA2_SCAN_NQ(2, false, true);
        CSA2_SCAN_NQ(2, false, false);
    } else if (a.G == 4 && NQ == 256 && esz == 1 && !a.gather && !a.pool_build) {
        CSA2_SCAN(256, 1, 4, false, false);
    } else if (a.G == 2 && NQ <= 128 && esz == 1 && !a.gather && !a.pool_build) {
        CSA2_SCAN(128, 1, 2, false, false);
    }
#undef CSA2_SCAN_NQ
#undef CSA2_SCAN
    return cudaErrorNotSupported;
}

int scan_tile_rows(int G, bool gather, int esz) {
    return (G == 1 && !gather && esz == 1) ? 3 * kTileRows
         : (G == 2 && !gather && esz == 1) ? 2 * kTileRows : kTileRows;
}

cudaError_t launch_prep_rows(int rows, int T, int G, const int32_t* n_vis0,
                             const int32_t* q_pos0, int ratio, int64_t cap, int P_gather,
                             int tile_rows, int32_t* n_row, int64_t* prefix, int32_t* status,
                             const ZeroList& zero, cudaStream_t st) {
    int64_t n16 = 0;
    for (int k = 0; k < 4; ++k) n16 += zero.n16[k];
    int64_t blocks = (n16 + 4 * 1024 - 1) / (4 * 1024);
    if (blocks < 1) blocks = 1;
    if (blocks > 64) blocks = 64;
    return launch_pdl(prep_rows_kernel, dim3((unsigned)blocks), dim3(1024), 0, st, rows, T, G,
                      n_vis0, q_pos0, ratio, cap, P_gather, tile_rows, n_row, prefix, status,
                      zero);
}

}  // namespace csa2
