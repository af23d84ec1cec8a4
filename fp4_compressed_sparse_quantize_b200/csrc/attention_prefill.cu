// Prefill sparse + sliding-window attention: every new token attends over its own selected
// FP4 main-KV entries and its causal window rows, on the 5th-generation tensor cores.
//
// "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (AI summary),
// Methodology in Plain English: a compressed global branch plus a sliding-window local
// branch; every layer computes its own query and keeps its own window KV. Main Findings:
// main KV is E2M1 with an E4M3 scale per 16 channels; the window KV stays FP8.
// "DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale LLM Serving", Causal
// Encoder-Decoder: a 128-token window in every layer, causal in prefill.
// Reading adopted (the pages do not spell out the join): one softmax over the token's
// selected entries and its window rows together; logits = scale * <q_h, x_i>; output
// sum_i p_i x_i (keys and values are the same 512-channel latent); no sink, no
// de-duplication; an empty row set gives a zero output.
//
// Numerics. A dequantised FP4 value (E2M1 x E4M3) has at most 6 significant bits and an
// E4M3 window value at most 4, inside fp16's normal range: the rows are EXACT in fp16. The
// query goes to fp16 after an exact per-head power-of-two rescale (largest |q| in
// [2^14, 2^15)), folded back into the logit factor. Probabilities enter P x V as an fp16
// (high, low) pair (~22 significant bits). All accumulation is fp32 in TMEM.
//
// One persistent CTA per SM walks a contiguous range of query tokens; the K + W rows of a
// token are processed in chunks of 128 with a single-pass online softmax:
//   dequant warps (8)  gather a chunk's rows (FP4 codes + scales, or E4M3 window rows)
//                      straight from global memory / L2 (an FP4 row's loads all issued before
//                      the first wait), dequantise them to fp16 and write the X tile
//                      [128 rows x 512 ch] as eight 128-byte-swizzled slabs; slab pair m of
//                      chunk c+1 is rewritten as soon as the P x V MMAs of chunk c that read it
//                      (output tile m) have completed. At a token's first chunk they also
//                      convert its query in place (bf16 -> fp16 with a per-head power-of-two
//                      rescale) once its TMA has landed.
//   waiter warp        does every mbarrier wait the MMA thread needs and hands over at a
//                      named barrier; loads each token's bf16 query [64 heads x 512] by TMA.
//   MMA thread         S^T = X Q^T (M = 128 rows, N = 64 heads, K = 512) into TMEM; then
//                      O^T += X^T P^T per 128-channel output tile (X read MN-major, P^T
//                      K-major [heads][rows]) as two N = 64 MMAs per k-step, the high and the
//                      low part of P, into one accumulator. TMEM: O^T tiles at columns 0, 64,
//                      128, 192 and S^T at 256 (each accumulator starts at a multiple of its
//                      width). (With the transposed X operand an N = 128 MMA over the stacked
//                      [P_hi | P_lo] rows did not produce that product on this part; two
//                      N = 64 MMAs do.)
//   softmax warps (8)  one chunk row per thread and half of the heads per warp: the logits
//                      come from TMEM; a head's running maximum is raised only when a logit
//                      exceeds it by more than 2^8 (then the accumulator columns of that
//                      head are rescaled in TMEM), so the common chunk needs no cross-thread
//                      maximum; every thread keeps its row's running per-head sums in its own
//                      TMEM lane (two buffers: a chunk reads one and writes old * rescale + p
//                      into the other, so a pass that is redone leaves no trace; reduced over
//                      the rows once per token, in a fixed order).
//                      P is computed against the running maxima in the same pass that checks
//                      them. At the end of a token they read O^T, divide by the sum and
//                      store the fp32 output.
// Every wait is bounded (2 s); a wait that gives up sets CSA2_DEV_TIMEOUT and the CTA runs
// out its loops without issuing further work.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {
namespace {

constexpr int kPR = 128;                       // rows per chunk
constexpr int kPD = 512;                       // latent channels
constexpr int kPH = 64;                        // heads (padded)
constexpr uint32_t kXSlab = kPR * 128;         // [128 rows][64 ch] fp16
constexpr uint32_t kQSlab = kPH * 128;         // [64 heads][64 ch] fp16 (bf16 on arrival)
constexpr uint32_t kPSlab = 2 * kPH * 128;     // [128 = hi|lo heads][64 rows] fp16, K-major
constexpr uint32_t kOffX = 0;
constexpr uint32_t kOffQ = 8 * kXSlab;
constexpr uint32_t kOffP = kOffQ + 8 * kQSlab;
constexpr uint32_t kOpBytes = kOffP + 2 * kPSlab;   // 229,376
constexpr uint32_t kDynBytes = kOpBytes + 1024;     // + alignment slack

constexpr uint32_t kColO = 0;                  // O^T tile m at column 64 m (hi and lo summed)
constexpr uint32_t kColS = 256;                // S^T: 64 columns
constexpr uint32_t kColL = 320;                // per-row running sums: 2 x 64 columns

constexpr int kWarpMma = 0, kWarpWait = 1;
constexpr int kSmWarp0 = 4, kSmWarps = 8;      // softmax warps 4..11
constexpr int kNumWarps = 18;                  // dequant warps: 2, 3, 12..17
constexpr int kThreads = 32 * kNumWarps;
constexpr float kLazy = 8.0f;                  // a head's maximum rises only past this (log2)

struct PrefillArgs {
    int Q, T, H, K, W;
    const uint8_t* codes;
    const uint8_t* scales;
    int64_t cap;
    const int32_t* idx;       // [Q][K]
    const uint8_t* swa;       // [B][W-1+T][512] E4M3
    const int32_t* q_pos0;    // [B] or null
    float qf;                 // scale * log2(e)
    float* out;               // [Q][H][512]
    int32_t* status;
};

__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(out)
        : "r"(byte));
    return out;
}

__device__ __forceinline__ void st_sh_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                         uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}
__device__ __forceinline__ void st_sh_u16(uint32_t addr, uint16_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
__device__ __forceinline__ uint4 ld_sh_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// 128-byte-swizzled 16-byte chunk c of row r of a [rows][128 B] tile
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,"
        "%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// named barrier 2: the 8 softmax warps; named barrier 1: the MMA warp and the waiter warp.
// OR of `pred` over the 256 softmax threads (they all execute it)
__device__ __forceinline__ bool sm_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 2, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void sm_sync() {
    asm volatile("bar.sync 2, 256;" ::: "memory");
}
__device__ __forceinline__ void hand_sync() {
    asm volatile("bar.sync 1, 64;" ::: "memory");
}

// exact split of p into p_hi + p_lo with p_hi representable in fp16: p_hi keeps 11
// significant bits (p in the fp16 normal range; below it the pair carries p to ~2^-25)
__device__ __forceinline__ float hi11f(float p) {
    return __uint_as_float((__float_as_uint(p) + 0x1000u) & 0xFFFFE000u);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q, const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bars[14];
    __shared__ __align__(16) float m_used_s[kPH];   // running maximum per head (base-2 logits)
    __shared__ __align__(16) float alpha_s[kPH];    // rescale factor of the current chunk
    __shared__ __align__(16) float inv_s[kPH];      // 1 / sum at the end of a token
    __shared__ __align__(16) float qf_s[kPH];       // logit factor per head of the token

    __shared__ uint32_t tmem_holder;
    __shared__ int flags[4];           // 0: abort, 1: go (hand-over), 2: MMA still in flight
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sX = smem_u32(sm + kOffX), sQ = smem_u32(sm + kOffQ), sP = smem_u32(sm + kOffP);
    float* scratch = reinterpret_cast<float*>(sm + kOffP);   // P region, between uses of P
    uint64_t* xfull = bars;            // [2] slabs 0-3 / 4-7 of the chunk written
    uint64_t* xempty = bars + 2;       // [4] slab pair m free (P x V tile m done)
    uint64_t* qfull = bars + 6;        // the query's bf16 bytes landed
    uint64_t* qempty = bars + 7;       // the token's last S^T completed
    uint64_t* sfull = bars + 8;
    uint64_t* pfull = bars + 9;
    uint64_t* ofull = bars + 10;
    uint64_t* oempty = bars + 11;
    uint64_t* done = bars + 12;        // teardown: every MMA of the CTA completed
    uint64_t* qready = bars + 13;      // the query is converted to fp16
    volatile int* abort_f = flags;
    volatile int* go_f = flags + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tk0 = (int)((int64_t)a.Q * blockIdx.x / gridDim.x);
    const int tk1 = (int)((int64_t)a.Q * (blockIdx.x + 1) / gridDim.x);
    const int rows = a.K + a.W;
    const int nch = rows > 0 ? (rows + kPR - 1) / kPR : 1;

    grid_dep_launch();
    if (threadIdx.x == 0) {
        mbar_init(&xfull[0], 8);
        mbar_init(&xfull[1], 8);
        for (int m = 0; m < 4; ++m) mbar_init(&xempty[m], 1);
        mbar_init(qfull, 1);
        mbar_init(qempty, 1);
        mbar_init(sfull, 1);
        mbar_init(pfull, kSmWarps);
        mbar_init(ofull, 1);
        mbar_init(oempty, kSmWarps);
        mbar_init(done, 1);
        mbar_init(qready, kSmWarps);
        flags[0] = flags[1] = flags[2] = flags[3] = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) tmem_alloc(&tmem_holder, 512);
    if (warp == kWarpWait && lane == 0) prefetch_tmap(&tmap_q);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_holder;
    grid_dep_wait();   // indices (Top-K) and the cache come from earlier kernels

    // bounded wait shared by all roles: once any wait gives up, every later wait is skipped
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (*abort_f) return false;
        if (mbar_wait(bar, parity, a.status)) return true;
        *abort_f = 1;
        return false;
    };

    // in-place conversion of the landed bf16 query into fp16 with a per-head power-of-two
    // rescale: 4 threads per head, each its head's row of two 64-channel slabs; a thread
    // starts at chunk (head mod 8) of the row so that the 8 heads of a warp touch 8
    // different bank groups (every 16-byte chunk converts in place, whatever its order)
    auto convert_q = [&](int ti_q, int st) {
        const bool ok = wait(qfull, ti_q & 1);
        const int h = st >> 2, qq = st & 3;
        float amax = 0.f;
        if (ok) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint4 v = ld_sh_v4(sQ + (2 * qq + (k >> 3)) * kQSlab + h * 128 + ((k + h) & 7) * 16);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w4[e] << 16)),
                                             fabsf(__uint_as_float(w4[e] & 0xFFFF0000u))));
            }
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        int shift = 0;
        if (amax > 0.f) {
            const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
            shift = min(126, max(-126, 14 - ex));
        }
        const float mul = __int_as_float((127 + shift) << 23);   // 2^shift, exact
        if (ok) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t ad = sQ + (2 * qq + (k >> 3)) * kQSlab + h * 128 + ((k + h) & 7) * 16;
                const uint4 v = ld_sh_v4(ad);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                uint32_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __half2 hv = __floats2half2_rn(__uint_as_float(w4[e] << 16) * mul,
                                                         __uint_as_float(w4[e] & 0xFFFF0000u) * mul);
                    o4[e] = *reinterpret_cast<const uint32_t*>(&hv);
                }
                st_sh_v4(ad, o4[0], o4[1], o4[2], o4[3]);
            }
        }
        if (qq == 0) qf_s[h] = a.qf * __int_as_float((127 - shift) << 23);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(qready);
    };

    if (warp == kWarpWait) {
        // ---------------------------------------------------------------- waiter
        int gc = 0, ti = 0;
        bool q_in_flight = false;
        if (tk0 < tk1) {
            if (lane == 0) {
                mbar_arrive_expect_tx(qfull, 8u * kQSlab);
                for (int j = 0; j < 8; ++j)
                    tma_load_2d(sm + kOffQ + j * kQSlab, &tmap_q, qfull, 64 * j, tk0 * a.H);
            }
            q_in_flight = true;
        }
        for (int tk = tk0; tk < tk1; ++tk, ++ti) {
            for (int c = 0; c < nch; ++c, ++gc) {
                bool ok = true;
                if (lane == 0) {
                    if (c == 0) ok = wait(qready, ti & 1);
                    ok = wait(&xfull[0], gc & 1) && ok;
                    *go_f = ok && !*abort_f;
                }
                if (c == 0) q_in_flight = false;   // the softmax warps consumed qfull
                hand_sync();                 // hand-over 1: slabs 0-3 (and the query)
                hand_sync();                 // the MMA thread has read the verdict
                if (lane == 0) *go_f = wait(&xfull[1], gc & 1);
                hand_sync();                 // hand-over 2: slabs 4-7
                hand_sync();
                if (c == nch - 1 && tk + 1 < tk1) {
                    // the query tile is free once this token's last S^T has completed
                    if (lane == 0 && wait(qempty, ti & 1)) {
                        mbar_arrive_expect_tx(qfull, 8u * kQSlab);
                        for (int j = 0; j < 8; ++j)
                            tma_load_2d(sm + kOffQ + j * kQSlab, &tmap_q, qfull, 64 * j,
                                        (tk + 1) * a.H);
                    }
                    q_in_flight = true;
                }
                if (lane == 0) {
                    ok = wait(pfull, gc & 1);
                    if (c == 0) ok = wait(oempty, (ti & 1) ^ 1) && ok;
                    *go_f = ok && !*abort_f;
                }
                hand_sync();                 // hand-over 3: P written (and O^T read out)
                hand_sync();
            }
        }
        // a query load whose bytes may still be landing must complete before the CTA exits
        if (q_in_flight && lane == 0) mbar_wait(qfull, ti & 1, a.status);
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------------- MMA issue
        constexpr uint32_t idS = make_idesc(128, 64, 0u, 0u);
        constexpr uint32_t idO = make_idesc(128, 64, 0u, 0u, /*a MN-major*/ 1u, 0u);
        for (int tk = tk0; tk < tk1; ++tk) {
            for (int c = 0; c < nch; ++c) {
                for (int half = 0; half < 2; ++half) {
                    hand_sync();
                    const bool go = *go_f;
                    hand_sync();
                    if (lane == 0 && go) {
                        tc_fence_after();
#pragma unroll 4
                        for (int kk = 16 * half; kk < 16 * half + 16; ++kk) {
                            const uint64_t ad = sw128_desc(sX + (kk >> 2) * kXSlab + (kk & 3) * 32, 16, 1024);
                            const uint64_t bd = sw128_desc(sQ + (kk >> 2) * kQSlab + (kk & 3) * 32, 16, 1024);
                            mma_f16(tmem + kColS, ad, bd, idS, kk > 0);
                        }
                        if (half == 1) {
                            mma_commit(sfull);
                            if (c == nch - 1) mma_commit(qempty);
                        }
                    }
                }
                hand_sync();
                const bool go = *go_f;
                hand_sync();
                if (lane == 0 && go) {
                    tc_fence_after();
#pragma unroll 1
                    for (int m = 0; m < 4; ++m) {
#pragma unroll
                        for (int kk = 0; kk < kPR / 16; ++kk) {
                            // A: channels [128 m, 128 m + 128) x rows [16 kk, +16), MN-major:
                            // the two 64-channel slabs apart by one slab, 8-row groups 1 KiB
                            const uint64_t ad = sw128_desc(sX + (2 * m) * kXSlab + kk * 2048, kXSlab, 1024);
                            // B: P^T K-major [hi heads | lo heads][rows], rows 16 kk .. +16
                            const uint32_t pb = sP + (kk >> 2) * kPSlab + (kk & 3) * 32;
                            const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
                            mma_f16(tmem + kColO + 64 * m, ad, sw128_desc(pb, 16, 1024), idO, acc);
                            mma_f16(tmem + kColO + 64 * m, ad, sw128_desc(pb + kPH * 128, 16, 1024), idO, 1u);
                        }
                        mma_commit(&xempty[m]);
                    }
                    if (c == nch - 1) mma_commit(ofull);
                }
            }
        }
    } else if (warp >= kSmWarp0 && warp < kSmWarp0 + kSmWarps) {
        // ---------------------------------------------------------------- softmax + epilogue
        const int sw = warp - kSmWarp0;
        const int quad = sw & 3, hh = sw >> 2;      // TMEM lane quadrant, head half
        const int rr = 32 * quad + lane;            // row of the chunk / channel of a tile
        const uint32_t tq = (uint32_t)(32 * quad) << 16;
        int gc = 0, ti = 0;
        for (int tk = tk0; tk < tk1; ++tk, ++ti) {
            const int b = tk / a.T, t = tk - b * a.T;
            const int64_t pos0 = a.q_pos0 ? (int64_t)ld_dep(a.q_pos0 + b) : (int64_t)(a.W - 1);
            for (int c = 0; c < nch; ++c, ++gc) {
                // validity of this thread's row (loaded before the wait)
                const int g = c * kPR + rr;
                bool valid = false;
                if (g < a.K) {
                    const int32_t e = ld_dep(a.idx + (int64_t)tk * a.K + g);
                    valid = e >= 0 && e < a.cap;
                } else if (g < rows) {
                    valid = pos0 + t + (g - a.K) - (a.W - 1) >= 0;
                }
                if (c == 0) wait(qready, ti & 1);   // this token's logit factors are in qf_s
                const bool ok = wait(sfull, gc & 1);
                tc_fence_after();
                // this thread's logits for 16 of its heads (base-2 units; -inf for empty rows)
                auto logits16 = [&](int q16, float (&x)[16]) {
                    uint32_t v[16];
                    tmem_ld16(tmem + tq + kColS + 32 * hh + 16 * q16, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        const float4 f = *reinterpret_cast<const float4*>(&qf_s[32 * hh + 16 * q16 + i]);
                        x[i] = valid ? __uint_as_float(v[i]) * f.x : -INFINITY;
                        x[i + 1] = valid ? __uint_as_float(v[i + 1]) * f.y : -INFINITY;
                        x[i + 2] = valid ? __uint_as_float(v[i + 2]) * f.z : -INFINITY;
                        x[i + 3] = valid ? __uint_as_float(v[i + 3]) * f.w : -INFINITY;
                    }
                };
                // probabilities of this row for the warp's 32 heads against the running maxima,
                // written as an fp16 (high, low) pair into P^T [hi heads | lo heads][rows]
                // (K-major: row rr is element rr % 64 of slab rr / 64 in each head's 128-byte
                // row), and the row's running sums (those of the previous chunk, times the
                // heads' rescale factors when `rescale`, plus p) into the other sum buffer;
                // returns whether a logit passed its head's maximum by more than 2^8
                const uint32_t prow = sP + (uint32_t)(rr >> 6) * kPSlab;
                const int rin = rr & 63;
                const uint32_t pcol = (uint32_t)(((rin >> 3) << 4) | ((rin & 7) << 1));
                const uint32_t lcur = tmem + tq + kColL + 64 * (gc & 1) + 32 * hh;
                const uint32_t lnext = tmem + tq + kColL + 64 * ((gc + 1) & 1) + 32 * hh;
                auto probs = [&](bool rescale) -> bool {
                    bool over = false;
#pragma unroll
                    for (int q16 = 0; q16 < 2; ++q16) {
                        float x[16];
                        logits16(q16, x);
                        uint32_t acc[16];
                        if (c > 0) {
                            tmem_ld16(lcur + 16 * q16, acc);
                            tmem_ld_wait();
                        }
#pragma unroll
                        for (int i = 0; i < 16; i += 4) {
                            const float4 m4 = *reinterpret_cast<const float4*>(&m_used_s[32 * hh + 16 * q16 + i]);
                            const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const int h = 32 * hh + 16 * q16 + i + j;
                                over |= x[i + j] > mv[j] + kLazy;
                                const float p = valid ? exp2f(x[i + j] - mv[j]) : 0.f;
                                const float old = c > 0 ? __uint_as_float(acc[i + j]) * (rescale ? alpha_s[h] : 1.f) : 0.f;
                                acc[i + j] = __float_as_uint(old + p);
                                const float ph = hi11f(p);
                                const __half hh16 = __float2half_rn(ph);
                                const __half hl16 = __float2half_rn(p - ph);
                                // the 16-byte chunk index (rin / 8) is XOR-swizzled by the row (h)
                                const uint32_t chi = (pcol ^ ((uint32_t)(h & 7) << 4));
                                st_sh_u16(prow + h * 128 + chi, *reinterpret_cast<const uint16_t*>(&hh16));
                                st_sh_u16(prow + (h + kPH) * 128 + chi, *reinterpret_cast<const uint16_t*>(&hl16));
                            }
                        }
                        tmem_st16(lnext + 16 * q16, acc);
                    }
                    return over;
                };
                // common case: the maxima hold, P is final after one pass; otherwise (always at
                // a token's first chunk) the per-head maxima are raised and P is written again
                bool need = (c == 0);
                if (!need) need = probs(false);
                need = sm_any(need);
                if (need) {
                    // per-head maximum over the chunk: the warp's [32 rows x 32 heads] logits
                    // go through the P region (free: the previous chunk's P x V has completed,
                    // and every speculative P write came before the barrier above),
                    // XOR-swizzled so that row-wise writes and head-wise reads are both
                    // conflict-free; lane L takes head 32 hh + L over the warp's rows, then the
                    // quadrant-0 warps take the maximum over the 4 quadrants
                    float* wsl = scratch + (sw * 32) * 32;
#pragma unroll
                    for (int q16 = 0; q16 < 2; ++q16) {
                        float x[16];
                        logits16(q16, x);
#pragma unroll
                        for (int i = 0; i < 16; ++i) wsl[lane * 32 + ((16 * q16 + i) ^ lane)] = x[i];
                    }
                    __syncwarp();
                    float wm = -INFINITY;
#pragma unroll 8
                    for (int lw = 0; lw < 32; ++lw) wm = fmaxf(wm, wsl[lw * 32 + (lane ^ lw)]);
                    sm_sync();   // every warp has read its block before the table overwrites it
                    scratch[quad * kPH + 32 * hh + lane] = wm;
                    sm_sync();
                    if (quad == 0) {
                        const int h = 32 * hh + lane;
                        const float cm = fmaxf(fmaxf(scratch[h], scratch[kPH + h]),
                                               fmaxf(scratch[2 * kPH + h], scratch[3 * kPH + h]));
                        const float mold = c == 0 ? -INFINITY : m_used_s[h];
                        const float mnew = cm > mold + kLazy ? cm : mold;
                        const float al = (mnew == mold) ? 1.f : exp2f(mold - mnew);
                        m_used_s[h] = mnew;
                        alpha_s[h] = al;
                    }
                    sm_sync();   // also: every read of the table is done before P overwrites it
                    if (c > 0) {
                        // rescale this thread's lanes of the accumulator columns of its heads
                        // (its running sums are rescaled by probs() below)
                        bool any = false;
#pragma unroll
                        for (int i = 0; i < 32; ++i) any |= alpha_s[32 * hh + i] != 1.f;
                        if (__any_sync(0xffffffffu, any) && ok) {
#pragma unroll 1
                            for (int m = 0; m < 4; ++m) {
                                const uint32_t col = kColO + 64 * m + 32 * hh;
#pragma unroll 1
                                for (int q16 = 0; q16 < 2; ++q16) {
                                    uint32_t r[16];
                                    tmem_ld16(tmem + tq + col + 16 * q16, r);
                                    tmem_ld_wait();
#pragma unroll
                                    for (int e = 0; e < 16; ++e)
                                        r[e] = __float_as_uint(__uint_as_float(r[e]) *
                                                               alpha_s[32 * hh + 16 * q16 + e]);
                                    tmem_st16(tmem + tq + col + 16 * q16, r);
                                }
                            }
                            tmem_st_wait();
                        }
                    }
                    probs(true);
                }
                tmem_st_wait();
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(pfull);
            }
            // ---- end of the token: normalise and store the output
            const bool ok = wait(ofull, ti & 1);
            tc_fence_after();
            // per-head sums over the 128 rows: each warp's [32 rows x 32 heads] running sums
            // go through the P region (consumed by now), XOR-swizzled so that row-wise writes
            // and head-wise reads are conflict-free; lane L adds head 32 hh + L over the warp's
            // rows, then the quadrant-0 warps add the 4 quadrants (a fixed order throughout)
            {
                float* wsl = scratch + (sw * 32) * 32;
#pragma unroll
                for (int q16 = 0; q16 < 2; ++q16) {
                    uint32_t v[16];
                    tmem_ld16(tmem + tq + kColL + 64 * (gc & 1) + 32 * hh + 16 * q16, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        wsl[lane * 32 + ((16 * q16 + i) ^ lane)] = __uint_as_float(v[i]);
                }
                __syncwarp();
                float acc = 0.f;
#pragma unroll 8
                for (int lw = 0; lw < 32; ++lw) acc += wsl[lw * 32 + (lane ^ lw)];
                sm_sync();   // every warp has read its block before the table overwrites it
                scratch[quad * kPH + 32 * hh + lane] = acc;
            }
            sm_sync();
            if (quad == 0) {
                const int h = 32 * hh + lane;
                const float l = (scratch[h] + scratch[kPH + h]) + (scratch[2 * kPH + h] + scratch[3 * kPH + h]);
                inv_s[h] = l > 0.f ? 1.f / l : 0.f;
            }
            sm_sync();
            if (ok) {
                float* orow = a.out + (int64_t)tk * a.H * kPD;
#pragma unroll 1
                for (int m = 0; m < 4; ++m) {
                    const int ch = 128 * m + rr;
#pragma unroll
                    for (int q16 = 0; q16 < 2; ++q16) {
                        uint32_t v[16];
                        tmem_ld16(tmem + tq + kColO + 64 * m + 32 * hh + 16 * q16, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int h = 32 * hh + 16 * q16 + e;
                            if (h < a.H) orow[(int64_t)h * kPD + ch] = __uint_as_float(v[e]) * inv_s[h];
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(oempty);
        }
    } else {
        // ---------------------------------------------------------------- dequant warps
        const int dq = warp < 4 ? warp - 2 : warp - 10;   // 0..7
        const int dt = 32 * dq + lane;
        const int rr = dt >> 1, part = dt & 1;             // row of the chunk, channel half
        int gc = 0, ti = 0;
        for (int tk = tk0; tk < tk1; ++tk, ++ti) {
            const int b = tk / a.T, t = tk - b * a.T;
            const int64_t pos0 = a.q_pos0 ? (int64_t)ld_dep(a.q_pos0 + b) : (int64_t)(a.W - 1);
            for (int c = 0; c < nch; ++c, ++gc) {
                const int g = c * kPR + rr;
                int kind = 0;                  // 0 empty, 1 FP4 entry, 2 window row
                const uint8_t* src = nullptr;
                const uint8_t* ssrc = nullptr;
                if (g < a.K) {
                    const int32_t e = ld_dep(a.idx + (int64_t)tk * a.K + g);
                    if (e >= 0 && e < a.cap) {
                        kind = 1;
                        const int64_t ent = (int64_t)b * a.cap + e;
                        src = a.codes + ent * CSA2_ENTRY_CODE_BYTES + 16 * part;
                        ssrc = a.scales + ent * CSA2_ENTRY_SCALE_BYTES;
                    } else if (e != -1 && part == 0) {
                        set_status(a.status, CSA2_DEV_BAD_INDEX);
                    }
                } else if (g < rows) {
                    const int v = g - a.K;
                    if (pos0 + t + v - (a.W - 1) >= 0) {
                        kind = 2;
                        src = a.swa + ((int64_t)b * (a.W - 1 + a.T) + t + v) * kPD + 32 * part;
                    }
                }
                // raw bytes for this thread's 32 channels of every slab: an FP4 row's code bytes
                // (16 per slab) and scales are all requested now, a window row's bytes (32 per
                // slab) half a row at a time
                uint4 raw[8];
                uint4 sc[2];
                if (kind == 1) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) raw[j] = ld_dep(reinterpret_cast<const uint4*>(src + 32 * j));
                    sc[0] = ld_dep(reinterpret_cast<const uint4*>(ssrc));
                    sc[1] = ld_dep(reinterpret_cast<const uint4*>(ssrc) + 1);
                } else if (kind == 2) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        raw[2 * j] = ld_dep(reinterpret_cast<const uint4*>(src + 64 * j));
                        raw[2 * j + 1] = ld_dep(reinterpret_cast<const uint4*>(src + 64 * j) + 1);
                    }
                }
                // the token's query: its TMA went out when the previous token's last S^T was done
                if (c == 0) convert_q(ti, dt);
#pragma unroll
                for (int half = 0; half < 2; ++half) {   // unrolled: raw[] is indexed by slab
                    if (kind == 2 && half == 1) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            raw[2 * j] = ld_dep(reinterpret_cast<const uint4*>(src + 64 * (4 + j)));
                            raw[2 * j + 1] = ld_dep(reinterpret_cast<const uint4*>(src + 64 * (4 + j)) + 1);
                        }
                    }
#pragma unroll
                    for (int mp = 0; mp < 2; ++mp) {
                        const int m = 2 * half + mp;     // slab pair
                        wait(&xempty[m], (uint32_t)((gc - 1) & 1));
#pragma unroll
                        for (int js = 0; js < 2; ++js) {
                            const int jl = 2 * mp + js;      // slab within the half
                            const int j = 4 * half + jl;     // slab 0..7
                            uint32_t o[16];
                            if (kind == 1) {
                                const uint4 cb = raw[j];
                                const uint32_t cw[4] = {cb.x, cb.y, cb.z, cb.w};
                                const int si = 4 * j + 2 * part;     // scale bytes si, si + 1
                                const uint32_t swd = (si < 16) ? ((si < 8) ? ((si < 4) ? sc[0].x : sc[0].y)
                                                                           : ((si < 12) ? sc[0].z : sc[0].w))
                                                               : ((si < 24) ? ((si < 20) ? sc[1].x : sc[1].y)
                                                                            : ((si < 28) ? sc[1].z : sc[1].w));
                                const uint32_t s01 = (swd >> (8 * (si & 3))) & 0xFFFFu;
                                const __half2 sp = e4m3x2_to_half2((uint16_t)s01);
                                const __half2 s0 = __half2half2(__low2half(sp));
                                const __half2 s1 = __half2half2(__high2half(sp));
#pragma unroll
                                for (int k = 0; k < 16; ++k) {
                                    const uint32_t byte = (cw[k >> 2] >> (8 * (k & 3))) & 0xFFu;
                                    uint32_t h2 = e2m1x2_to_h2(byte);
                                    const __half2 prod = __hmul2(*reinterpret_cast<__half2*>(&h2), k < 8 ? s0 : s1);
                                    o[k] = *reinterpret_cast<const uint32_t*>(&prod);
                                }
                            } else if (kind == 2) {
                                const uint4 e0 = raw[2 * jl], e1 = raw[2 * jl + 1];
                                const uint32_t ew[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
                                for (int k = 0; k < 16; ++k) {
                                    const __half2 hv = e4m3x2_to_half2((uint16_t)(ew[k >> 1] >> (16 * (k & 1))));
                                    o[k] = *reinterpret_cast<const uint32_t*>(&hv);
                                }
                            } else {
#pragma unroll
                                for (int k = 0; k < 16; ++k) o[k] = 0u;
                            }
                            const uint32_t base = sX + j * kXSlab;
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                st_sh_v4(base + sw_off(rr, 4 * part + k), o[4 * k], o[4 * k + 1],
                                         o[4 * k + 2], o[4 * k + 3]);
                        }
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&xfull[half]);
                }
            }
        }
    }

    // ---- teardown: every MMA must complete before TMEM is released; if this wait gives up,
    // TMEM stays allocated (the status word carries TIMEOUT and the context must be discarded)
    if (warp == kWarpMma && lane == 0) {
        mma_commit(done);
        if (!mbar_wait(done, 0, a.status)) flags[2] = 1;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma && !flags[2]) tmem_dealloc(tmem, 512);
}

}  // namespace

// Prefill attention of Q = B * T tokens (l.prefill): one persistent CTA per SM.
cudaError_t launch_attention_prefill(const AttnLaunch& l, cudaStream_t st) {
    if (l.Q < 1) return cudaSuccess;
    auto enc = tensor_map_encoder();
    if (!enc) return cudaErrorInvalidValue;
    CUtensorMap mq;
    memset(&mq, 0, sizeof mq);
    cuuint64_t dims[2] = {(cuuint64_t)kPD, (cuuint64_t)l.Q * l.H};
    cuuint64_t strides[1] = {(cuuint64_t)kPD * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)kPH};
    cuuint32_t es[2] = {1, 1};
    if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(l.q), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    PrefillArgs a;
    a.Q = l.Q;
    a.T = l.T;
    a.H = l.H;
    a.K = l.K;
    a.W = l.W;
    a.codes = l.codes;
    a.scales = l.scales;
    a.cap = l.cap;
    a.idx = l.idx;
    a.swa = l.swa;
    a.q_pos0 = l.q_pos0;
    a.qf = l.scale * 1.4426950408889634f;
    a.out = l.out;
    a.status = l.status;
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kDynBytes);
    if (e != cudaSuccess) return e;
    const int grid = l.Q < device_sm_count() ? l.Q : device_sm_count();
    return launch_pdl(attn_prefill_kernel, dim3((unsigned)grid), dim3(kThreads), kDynBytes, st,
                      mq, a);
}

}  // namespace csa2
