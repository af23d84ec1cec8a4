// Decode: gather + exact FP4 dequantisation + joint sparse / sliding-window attention on the
// 5th-generation tensor cores (tcgen05, TMEM accumulators).
//
// "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (AI summary),
// Methodology in Plain English: a compressed global branch plus a sliding-window local
// branch; every layer, Reuse included, computes its own query and keeps its own window KV.
// Main Findings: main KV is E2M1 with an E4M3 scale per 16 channels; the window KV stays
// FP8. "DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale LLM Serving", Causal
// Encoder-Decoder: a 128-token window in every layer.
//
// Reading adopted (the pages do not spell out the join): one softmax over the selected
// compressed entries and the window rows together; logits = scale * <q_h, x_i>; output
// sum_i p_i x_i (keys and values are the same 512-channel latent). No sink, no
// de-duplication. An empty row set gives a zero output.
//
// Numerics. FP4 x E4M3 and E4M3 values have at most 6 significant bits inside the fp16
// normal range, so the dequantised rows are EXACT in fp16. The query goes to fp16 after an
// exact per-head power-of-two rescale (largest |q| in [2^14, 2^15)), which keeps every
// element above 2^-28 of the head's largest exactly; the power of two is folded into the
// logit scale. Probabilities enter P x V as an fp16 (high, low) pair whose products are
// accumulated together (~22-bit probabilities: one fp16 rounding of P alone costs ~2e-3 of
// the output RMS on heavy-tailed channels). All accumulation is fp32 in TMEM.
//
// Kernels (prefill has its own kernel, attention_prefill.cu):
//   attn_stage_kernel   one warp per row: every selected FP4 row and window row of every
//                       query dequantised to fp16 rows [Q][K + W][512], and each query's
//                       heads rescaled to fp16 with their logit factors;
//   attn_decode_kernel  one CTA per (query, split of at most 160 rows): TMA loads of the
//                       staged rows and query, S = Q X^T with the 64 heads as M, softmax,
//                       [O_hi; O_lo] = [P_hi; P_lo] X, and either the splits' merge inside
//                       a thread-block cluster (distributed shared memory) or (max, sum,
//                       output) partials that attn_combine_kernel merges;
//   attn_empty_kernel   queries with no row at all (K + W == 0).
#include <cuda.h>
#include <algorithm>
#include <map>
#include <mutex>
#include <cudaTypedefs.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

constexpr int kD = 512;        // latent channels
constexpr int kHeads = 64;     // heads per CTA (MMA N), padded

struct TcAttnDev {
    int Q, T, H;
    const __nv_bfloat16* q;
    const uint8_t* codes;
    const uint8_t* scales;
    int64_t cap;
    const int32_t* idx;
    int K;
    const uint8_t* swa;
    int W;
    const int32_t* swa_valid;
    const int32_t* q_pos0;
    bool prefill;
    float scale;
    float* out;
    float* partial;          // O [Q * nsplit][H][512]
    float* partial_ml;       // (m, l) [Q * nsplit][2][H]
    int nsplit;
    bool part;               // decode: write (m, l, unnormalised O) partials even for one split
    int32_t* status;
    // staged decode: rows / query already dequantised by attn_stage_kernel
    const int32_t* st_valid;   // [Q][K + W] row kinds (0 = empty)
    const float* st_qf;        // [Q][64] logit factors
};

// one 64-channel slab of the query operand: [64 heads x 128 bytes]
struct TcSmem {
    static constexpr int kQSlab = kHeads * 128;           // 8 KiB
};

// byte offset of 16-byte chunk `c` (0..7) of row `r` inside one 128-byte-wide slab
__device__ __forceinline__ uint32_t slab_off(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ uint32_t e2m1x2_to_h2_tc(uint32_t byte) {
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(out)
        : "r"(byte));
    return out;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }


// Decode pre-pass: every selected main-KV row and window row of every query, dequantised to
// fp16 rows [Q][K + W][512] (exact), plus each query's heads rescaled to fp16 [Q][64][512] and
// their logit factors. One warp per row or head, 16 channels per lane, coalesced 1 KiB stores.
__global__ void __launch_bounds__(256) attn_stage_kernel(const TcAttnDev a, __half* __restrict__ xg,
                                                         __half* __restrict__ qg,
                                                         float* __restrict__ qfg,
                                                         int32_t* __restrict__ validg,
                                                         int row_blocks) {
    grid_dep_launch();
    grid_dep_wait();
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows = a.K + a.W;
    if ((int)blockIdx.y < row_blocks) {
        const int r = blockIdx.y * 8 + warp;
        if (r >= rows) return;
        int kind = 0;
        uint32_t hv[8];
        if (r < a.K) {
            const int32_t e = ld_dep(a.idx + (int64_t)b * a.K + r);
            if (e >= 0 && e < a.cap) {
                kind = 1;
                const int64_t ent = (int64_t)b * a.cap + e;
                const uint2 cb = ld_dep(reinterpret_cast<const uint2*>(a.codes + ent * CSA2_ENTRY_CODE_BYTES) + lane);
                const uint8_t sb = ld_dep(a.scales + ent * CSA2_ENTRY_SCALE_BYTES + lane);
                const __half2 s2 = __half2half2(__float2half_rn(e4m3_to_float(sb)));
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t byte = ((k < 4 ? cb.x : cb.y) >> (8 * (k & 3))) & 0xFFu;
                    uint32_t h2 = e2m1x2_to_h2_tc(byte);
                    hv[k] = h2_bits(__hmul2(*reinterpret_cast<__half2*>(&h2), s2));
                }
            } else if (e != -1 && lane == 0) {
                set_status(a.status, CSA2_DEV_BAD_INDEX);
            }
        } else {
            const int v = r - a.K;   // window row 0..W-1, oldest first
            const int nv = a.swa_valid ? ld_dep(a.swa_valid + b) : a.W;
            if (v >= a.W - nv) {
                kind = 2;
                const uint4 eb = ld_dep(reinterpret_cast<const uint4*>(a.swa + ((int64_t)b * a.W + v) * kD) + lane);
                const uint32_t ew[4] = {eb.x, eb.y, eb.z, eb.w};
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    hv[k] = h2_bits(e4m3x2_to_half2((uint16_t)(ew[k >> 1] >> (16 * (k & 1)))));
            }
        }
        if (kind == 0) {
#pragma unroll
            for (int k = 0; k < 8; ++k) hv[k] = 0u;
        }
        uint4* dst = reinterpret_cast<uint4*>(xg + ((int64_t)b * rows + r) * kD + lane * 16);
        dst[0] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        dst[1] = make_uint4(hv[4], hv[5], hv[6], hv[7]);
        if (lane == 0) validg[(int64_t)b * rows + r] = kind;
        return;
    }
    // heads: per-head power-of-two rescale into fp16
    const int h = ((int)blockIdx.y - row_blocks) * 8 + warp;
    if (h >= kHeads) return;
    float v[16];
    float amax = 0.f;
    if (h < a.H) {
        const uint4* src = reinterpret_cast<const uint4*>(a.q + ((int64_t)b * a.H + h) * kD + lane * 16);
        const uint4 u0 = ld_dep(src), u1 = ld_dep(src + 1);
        const uint32_t w8[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            v[2 * e] = __uint_as_float(w8[e] << 16);
            v[2 * e + 1] = __uint_as_float(w8[e] & 0xFFFF0000u);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(v[e]));
    } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = 0.f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int shift = 0;
    if (amax > 0.f) {
        const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
        shift = min(126, max(-126, 14 - ex));
    }
    const float mul = __int_as_float((127 + shift) << 23);   // 2^shift, exact
    uint32_t hw[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) hw[e] = h2_bits(__floats2half2_rn(v[2 * e] * mul, v[2 * e + 1] * mul));
    uint4* dst = reinterpret_cast<uint4*>(qg + ((int64_t)b * kHeads + h) * kD + lane * 16);
    dst[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    dst[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
    if (lane == 0) qfg[b * kHeads + h] = a.scale * 1.4426950408889634f * __int_as_float((127 - shift) << 23);
}


// ---- decode: one CTA per (query, split of at most 160 rows) ------------------------------
// The rows of a decode query are split evenly (a multiple of 32 per split, at most
// kDecRows) so that all splits of all queries fit in one wave of CTAs.
//
// Logits: S = Q X^T with the 64 heads as the MMA M dimension (M = 64) and rows as N, in two
// halves of the split's rows: half 0 into TMEM lanes 0-15 of every 32-lane subpartition,
// half 1 into lanes 16-31 (the M = 64 accumulator layout: head h in lane (h mod 16) +
// 32 (h / 16), row n in column n; a second accumulator may sit 16 lanes lower). The MMAs
// of each 64-channel slab start as soon as that slab of X and Q has landed.
// Softmax: thread (warp w, lane l) owns head 16 (w mod 4) + (l mod 16), row half l / 16 and
// column half w / 4 of it; maxima and sums are combined with one shuffle and one
// shared-memory exchange.
// Output: P is written as the stacked A operand [P_hi; P_lo] of [O_hi; O_lo] = P X with
// M = 128 rows ordered so that the high and low parts of head h are 16 TMEM lanes apart in
// the same subpartition (row 32 (h / 16) + (h mod 16) high, +16 low); X is the MN-major B
// operand (N = 256 channels, two halves). The epilogue adds the two parts with one shuffle.
constexpr int kDecRows = kAttnDecodeRows;

struct DecSmem {
    int xslab;   // bytes per X slab: rows x 128 B
    __device__ __host__ explicit DecSmem(int rps) : xslab(rps * 128) {}
    // the X region also takes the 128 KiB output tile of the epilogue
    __device__ __host__ int q() const { return 8 * xslab > 131072 ? 8 * xslab : 131072; }
    // after S: P (3 slabs of [128 stacked heads x 64 rows], 16 KiB each) and the tail
    __device__ __host__ int phi() const { return q(); }
    __device__ __host__ int tail() const { return q() + 6 * TcSmem::kQSlab; }   // 16 KiB
    __device__ __host__ int bytes() const { return q() + 8 * TcSmem::kQSlab; }
};

// exact split of p into p_hi + p_lo with p_hi representable in fp16 (p in the fp16 normal
// range; below it the pair carries p to within 2^-25): p_hi keeps 11 significant bits
__device__ __forceinline__ float hi11(float p) {
    return __uint_as_float((__float_as_uint(p) + 0x1000u) & 0xFFFFE000u);
}

// CL: the nsplit CTAs of one query form a thread-block cluster and merge their partial
// results through distributed shared memory (no partials in global memory, no merge kernel).
template <bool CL>
__global__ void __launch_bounds__(256, 1) attn_decode_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                             const __grid_constant__ CUtensorMap tmap_q,
                                                             const __grid_constant__ CUtensorMap tmap_o,
                                                             const TcAttnDev a, int rps) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar[10];   // 0-7: slab j of X and Q landed; 8: S done; 9: P X done
    __shared__ uint32_t tmem_holder;
    __shared__ int mma_stuck;      // a wait for the last MMA commit gave up: keep TMEM
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const DecSmem L(rps);
    const uint32_t sX = smem_u32(sm), sQ = smem_u32(sm + L.q()), sP = smem_u32(sm + L.phi());
    float* tail = reinterpret_cast<float*>(sm + L.tail());
    float* qf = tail;              // [64]
    float* m_s = tail + 64;        // [64]
    float* l_s = tail + 128;       // [64]
    float* inv_s = tail + 192;     // [64]
    float* redm = tail + 256;      // [2][64]
    float* redl = tail + 384;      // [2][64]
    uint32_t* vmask = reinterpret_cast<uint32_t*>(tail + 512);   // row validity bits [8]

    const int qrow = blockIdx.x, split = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rows = a.K + a.W;
    const int r0 = split * rps;    // first row of this split
    const int half_rows = rps >> 1;

    grid_dep_launch();
    if (tid == 0) {
#pragma unroll
        for (int j = 0; j < 10; ++j) mbar_init(&bar[j], 1);
        mma_stuck = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&tmem_holder, 512);
    grid_dep_wait();   // the staged rows and query come from the pre-pass
    if (tid == 0) {
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
            mbar_arrive_expect_tx(&bar[j], (uint32_t)L.xslab + TcSmem::kQSlab);
            tma_load_2d(sm + j * L.xslab, &tmap_x, &bar[j], 64 * j, qrow * rows + r0);
            tma_load_2d(sm + L.q() + j * TcSmem::kQSlab, &tmap_q, &bar[j], 64 * j, qrow * kHeads);
        }
    }
    // row kinds and logit factors, held in registers until the Q tile is dead
    int pre_valid = 0;
    float pre_qf = 0.f;
    if (tid < rps && r0 + tid < rows) pre_valid = ld_dep(a.st_valid + (int64_t)qrow * rows + r0 + tid);
    if (tid < kHeads) pre_qf = ld_dep(a.st_qf + qrow * kHeads + tid);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_holder;
    bool ok = true;
    bool loads_ok = true;

    // ---- S = Q X^T, M = 64, N = rps / 2 per half, K = 512: slab by slab as it lands ------------
    if (tid == 0) {
        const uint32_t idesc = make_idesc(64, half_rows, 0u, 0u);
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
            if (!mbar_wait(&bar[j], 0, a.status)) ok = loads_ok = false;
            tc_fence_after();
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int kk = 4 * j + k4;
                const uint64_t ad = sw128_desc(sQ + j * TcSmem::kQSlab + k4 * 32, 16, 1024);
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint64_t bd = sw128_desc(sX + j * L.xslab + part * half_rows * 128 + k4 * 32, 16, 1024);
                    mma_f16(tmem + ((uint32_t)(16 * part) << 16) + 256u, ad, bd, idesc, kk > 0);
                }
            }
        }
        mma_commit(&bar[8]);
    }
    if (!mbar_wait(&bar[8], 0, a.status)) ok = false;
    tc_fence_after();
    // the Q tile is dead: its tail takes the row validity bits and the logit factors
    {
        const uint32_t vb = __ballot_sync(0xffffffffu, pre_valid != 0);
        if (lane == 0) vmask[warp] = vb;   // rows 32 warp .. +31 (rows >= rps are 0)
    }
    if (tid < kHeads) qf[tid] = pre_qf;
    __syncthreads();

    // ---- softmax over this split's rows ------------------------------------------------------
    const int quad = warp & 3, wh = warp >> 2;
    const int hl = lane & 15, rh = lane >> 4;
    const int h = 16 * quad + hl;                    // head of this thread
    const int ncol = rps >> 2;                       // columns per thread: multiple of 8, <= 40
    const int cstart = rh * half_rows + wh * ncol;   // first row (of the split) of the thread
    const uint32_t sbase = tmem + ((uint32_t)(32 * quad) << 16) + 256u + (uint32_t)(wh * ncol);
    const float f = qf[h];
    uint32_t sv[kDecRows / 4];
#pragma unroll
    for (int g = 0; g < kDecRows / 32; ++g)
        if (8 * g < ncol) tmem_ld8(sbase + 8 * g, *reinterpret_cast<uint32_t(*)[8]>(sv + 8 * g));
    uint32_t vm[2];                                  // validity bits of rows cstart .. +63
    {
        const int wi = cstart >> 5, sh = cstart & 31;
        vm[0] = __funnelshift_r(vmask[wi], vmask[wi + 1], sh);
        vm[1] = __funnelshift_r(vmask[wi + 1], vmask[wi + 2], sh);
    }
    tmem_ld_wait();
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < kDecRows / 4; ++j) {
        const float x = __uint_as_float(sv[j]) * f;
        sv[j] = __float_as_uint(x);
        if (j < ncol && ((vm[j >> 5] >> (j & 31)) & 1u)) mx = fmaxf(mx, x);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (rh == 0) redm[wh * 64 + h] = mx;
    __syncthreads();
    const float m = fmaxf(redm[h], redm[64 + h]);
    const float base = (m == -INFINITY) ? 0.f : m;
    float ls = 0.f;
    const int prow = 32 * quad + hl;                 // stacked P row of the high part
#pragma unroll
    for (int g = 0; g < kDecRows / 32; ++g) {
        if (8 * g < ncol) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = 8 * g + 2 * e;
                const float p0 = ((vm[j >> 5] >> (j & 31)) & 1u) ? exp2f(__uint_as_float(sv[j]) - base) : 0.f;
                const float p1 = ((vm[(j + 1) >> 5] >> ((j + 1) & 31)) & 1u) ? exp2f(__uint_as_float(sv[j + 1]) - base) : 0.f;
                ls += p0 + p1;
                const float h0 = hi11(p0), h1 = hi11(p1);
                hi[e] = h2_bits(__floats2half2_rn(h0, h1));
                lo[e] = h2_bits(__floats2half2_rn(p0 - h0, p1 - h1));
            }
            const int c = cstart + 8 * g;            // 8 rows: one 16-byte chunk per part
            const uint32_t sl = sP + (uint32_t)((c >> 6) * 2 * TcSmem::kQSlab);
            st_shared_v4(sl + slab_off(prow, (c & 63) >> 3), hi[0], hi[1], hi[2], hi[3]);
            st_shared_v4(sl + slab_off(prow + 16, (c & 63) >> 3), lo[0], lo[1], lo[2], lo[3]);
        }
    }
    ls += __shfl_xor_sync(0xffffffffu, ls, 16);
    if (rh == 0) redl[wh * 64 + h] = ls;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    if (rh == 0 && wh == 0) {
        const float l = redl[h] + redl[64 + h];
        m_s[h] = m;
        l_s[h] = l;
        inv_s[h] = l > 0.f ? 1.f / l : 0.f;
    }

    // ---- [O_hi; O_lo] = P X: M = 128, N = 256 channels (two halves), K = rps rows ------------
    // X (rows x channels, channels contiguous) is the MN-major B operand: 64-channel slabs
    // apart by one X slab (LBO), 8-row groups 1 KiB apart (SBO). D fills TMEM columns
    // [0, 512); the logits there were all read above.
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = make_idesc(128, 256, 0u, 0u, 0u, /*b MN-major*/ 1u);
        const int nk = rps >> 4;
#pragma unroll 1
        for (int nh = 0; nh < 2; ++nh)
#pragma unroll 1
            for (int kk = 0; kk < nk; ++kk) {
                const uint64_t ad =
                    sw128_desc(sP + (kk >> 2) * 2 * TcSmem::kQSlab + (kk & 3) * 32, 16, 1024);
                const uint64_t bd = sw128_desc(sX + (4 * nh) * L.xslab + kk * 16 * 128,
                                               (uint32_t)L.xslab, 1024);
                mma_f16(tmem + 256 * nh, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
        mma_commit(&bar[9]);
    }
    if (!mbar_wait(&bar[9], 0, a.status)) {
        ok = false;
        mma_stuck = 1;   // MMAs may still write TMEM: it is not released below
    }
    tc_fence_after();
    __syncthreads();

    // ---- epilogue: O = O_hi + O_lo (lanes l and l ^ 16) into shared memory as 16 boxes of
    // [64 heads][32 channels] (128-byte rows, 16-byte chunks XOR-swizzled by head), then one
    // bulk tensor store per box
    float* osm = reinterpret_cast<float*>(sm);
    const int oblk = a.nsplit == 1 ? qrow : qrow * a.nsplit + split;
    const uint32_t tq = (uint32_t)(32 * quad) << 16;
    const int cbase = 256 * wh;                // channels of this warp
    const float oscale = (a.nsplit == 1 && !a.part) ? inv_s[h] : 1.f;
    if (ok) {
#pragma unroll 1
        for (int cc = 0; cc < 256; cc += 64) {
            uint32_t v[4][16];
#pragma unroll
            for (int k = 0; k < 4; ++k) tmem_ld16(tmem + tq + cbase + cc + 16 * k, v[k]);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float o[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float x = __uint_as_float(v[k][e]);
                    o[e] = (x + __shfl_xor_sync(0xffffffffu, x, 16)) * oscale;
                }
                // lanes 0-15 store channels +0..7, lanes 16-31 channels +8..15
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int c = cbase + cc + 16 * k + 8 * rh + 4 * j;
                    float* dst = osm + (c >> 5) * (kHeads * 32) + h * 32 + ((((c & 31) >> 2) ^ (h & 7)) << 2);
                    const int e0 = 4 * j;   // of this lane's half: o[e0 + 8 rh ..]
                    *reinterpret_cast<float4*>(dst) =
                        rh ? make_float4(o[e0 + 8], o[e0 + 9], o[e0 + 10], o[e0 + 11])
                           : make_float4(o[e0], o[e0 + 1], o[e0 + 2], o[e0 + 3]);
                }
            }
        }
    }
    if constexpr (CL) {
        // every split of this query has its (max, sum) and unnormalised output tile in shared
        // memory; CTA k of the cluster finishes the 32-channel boxes b = k (mod nsplit): it
        // reads box b of every split, weights them by 2^(m_s - M) and divides by the merged
        // sum. Box b of this CTA is read by this CTA only, so it is overwritten in place.
        const uint32_t ns = (uint32_t)a.nsplit, k = cluster_rank();
        float* wgt = tail + 1024;    // [8 splits][64 heads]
        float* ginv = tail + 1536;   // [64 heads]
        cluster_sync_all();
        if (tid < kHeads) {
            float mv[8], lv[8], M = -INFINITY;
#pragma unroll
            for (uint32_t sp = 0; sp < 8; ++sp) {
                mv[sp] = -INFINITY;
                lv[sp] = 0.f;
                if (sp < ns) {
                    mv[sp] = __uint_as_float(ld_peer_u32(peer_addr(&m_s[tid], sp)));
                    lv[sp] = __uint_as_float(ld_peer_u32(peer_addr(&l_s[tid], sp)));
                    M = fmaxf(M, mv[sp]);
                }
            }
            const float Mb = (M == -INFINITY) ? 0.f : M;
            float L = 0.f;
#pragma unroll
            for (uint32_t sp = 0; sp < 8; ++sp) {
                if (sp < ns) {
                    const float wv = exp2f(mv[sp] - Mb);
                    L += wv * lv[sp];
                    wgt[sp * kHeads + tid] = wv;
                }
            }
            ginv[tid] = L > 0.f ? 1.f / L : 0.f;
        }
        __syncthreads();
        // items of this thread: (box k + ns i / 2, half i mod 2 of its 512 16-byte chunks)
        const int nitems = 2 * (int)((16 - k + ns - 1) / ns);
        auto item_off = [&](int i) {
            const int bx = (int)k + (int)ns * (i >> 1);
            const int u = (i & 1) * 256 + tid, hh = u >> 3, ch = u & 7;
            return bx * (kHeads * 32) + hh * 32 + ((ch ^ (hh & 7)) << 2);
        };
        if (ns <= 4) {
            // four items at a time, every split's chunk of all four loads in flight at once
#pragma unroll 1
            for (int i0 = 0; i0 < nitems; i0 += 4) {
                float4 v[4][4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (uint32_t sp = 0; sp < 4; ++sp)
                        if (i0 + j < nitems && sp < ns) {
                            const int off = item_off(i0 + j);
                            v[j][sp] = sp == k ? *reinterpret_cast<const float4*>(osm + off)
                                               : ld_peer_f4(peer_addr(osm + off, sp));
                        }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (i0 + j < nitems) {
                        const int off = item_off(i0 + j);
                        const int hh = ((((i0 + j) & 1) * 256 + tid) >> 3);
                        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                        for (uint32_t sp = 0; sp < 4; ++sp)
                            if (sp < ns) {
                                const float wv = wgt[sp * kHeads + hh];
                                acc.x += wv * v[j][sp].x;
                                acc.y += wv * v[j][sp].y;
                                acc.z += wv * v[j][sp].z;
                                acc.w += wv * v[j][sp].w;
                            }
                        const float iv = ginv[hh];
                        *reinterpret_cast<float4*>(osm + off) =
                            make_float4(acc.x * iv, acc.y * iv, acc.z * iv, acc.w * iv);
                    }
                }
            }
        } else {
#pragma unroll 1
            for (int i = 0; i < nitems; ++i) {
                const int off = item_off(i);
                const int hh = (((i & 1) * 256 + tid) >> 3);
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (uint32_t sp = 0; sp < 8; ++sp) {
                    if (sp < ns) {
                        const float4 v = sp == k ? *reinterpret_cast<const float4*>(osm + off)
                                                 : ld_peer_f4(peer_addr(osm + off, sp));
                        const float wv = wgt[sp * kHeads + hh];
                        acc.x += wv * v.x;
                        acc.y += wv * v.y;
                        acc.z += wv * v.z;
                        acc.w += wv * v.w;
                    }
                }
                const float iv = ginv[hh];
                *reinterpret_cast<float4*>(osm + off) =
                    make_float4(acc.x * iv, acc.y * iv, acc.z * iv, acc.w * iv);
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && ok) {
#pragma unroll 1
            for (uint32_t bx = k; bx < 16; bx += ns)
                tma_store_3d(&tmap_o, osm + bx * (kHeads * 32), 32 * (int)bx, 0, qrow);
            bulk_commit();
            bulk_wait_all();
        }
        cluster_sync_all();   // the other splits have finished reading this CTA's tiles
    } else {
        if (ok && (a.nsplit > 1 || a.part) && warp == 0) {
            float* ml = a.partial_ml + (int64_t)oblk * 2 * a.H;
            for (int x = lane; x < a.H; x += 32) {
                ml[x] = m_s[x];
                ml[a.H + x] = l_s[x];
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && ok) {
#pragma unroll 1
            for (int b = 0; b < 16; ++b)
                tma_store_3d(&tmap_o, osm + b * (kHeads * 32), 32 * b, 0, oblk);
            bulk_commit();
            bulk_wait_all();
        }
    }
    if (tid == 0 && !loads_ok)   // a load that timed out may still be in flight: bounded
        for (int j = 0; j < 8; ++j) mbar_wait(&bar[j], 0, a.status);
    tc_fence_after();
    if (warp == 0 && !mma_stuck) tmem_dealloc(tmem, 512);
}

// Queries with no row at all (K + W == 0): the softmax of an empty set contributes nothing,
// so the output is zero; a partial result is (maximum -inf, sum 0, output 0), which the
// partial merge weighs by zero.
__global__ void __launch_bounds__(256) attn_empty_kernel(float* o, float* ml, int Q, int H) {
    grid_dep_launch();
    grid_dep_wait();
    const int64_t n4 = (int64_t)Q * H * kD / 4;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x)
        reinterpret_cast<float4*>(o)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ml)
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)Q * H;
             i += (int64_t)gridDim.x * blockDim.x) {
            const int64_t q = i / H, h = i - q * H;
            ml[q * 2 * H + h] = -INFINITY;
            ml[q * 2 * H + H + h] = 0.f;
        }
}

// [rows][512] fp16 matrix, box = 64 channels x box_rows, 128-byte swizzle
static bool fp16_rows_map(CUtensorMap* m, const void* base, int64_t rows, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(kD * 2)};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// [blocks][H][512] fp32, box = 32 channels x H heads x 1 block, 128-byte swizzle
static bool out_map_sw(CUtensorMap* m, void* base, int H, int64_t blocks) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)blocks};
    cuuint64_t strides[2] = {(cuuint64_t)(kD * 4), (cuuint64_t)H * kD * 4};
    cuuint32_t box[3] = {32u, (cuuint32_t)H, 1u};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t attention_stage_bytes(int Q, int rows) {
    return (size_t)Q * rows * kD * 2 + (size_t)Q * kHeads * kD * 2 + (size_t)Q * kHeads * 4 +
           (size_t)Q * rows * 4 + 4 * 256;
}

// Whether the decode splits of a query can run as one thread-block cluster (the merge then
// happens in distributed shared memory, with no partials in global memory and no merge
// kernel). More queries than the clusters resident at once simply take several waves: at
// 64 queries (two waves) this is 1% faster per step than partials plus the merge kernel.
// Looked up once per (splits, shared memory) shape.
static bool cluster_merge_fits(int Q, int nsplit, int dsmem) {
    if (nsplit < 2 || nsplit > 8) return false;
    static std::mutex mu;
    static std::map<std::pair<int, int>, int> cache;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(nsplit, dsmem);
    auto it = cache.find(key);
    if (it == cache.end()) {
        int n = 0;
        if (cudaFuncSetAttribute(attn_decode_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, dsmem) == cudaSuccess) {
            cudaLaunchConfig_t cfg;
            memset(&cfg, 0, sizeof cfg);
            cfg.gridDim = dim3(1, (unsigned)nsplit);
            cfg.blockDim = dim3(256);
            cfg.dynamicSmemBytes = dsmem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 1;
            attr[0].val.clusterDim.y = (unsigned)nsplit;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, attn_decode_kernel<true>, &cfg) != cudaSuccess) n = 0;
        }
        cudaGetLastError();   // a refused query leaves no sticky error
        it = cache.emplace(key, n).first;
    }
    return Q >= 1 && it->second >= 1;
}

int attention_decode_launches(int Q, int K, int W) {
    const int rows = K + W;
    if (rows <= 0) return 1;
    const int nsplit = attention_splits(Q, K, W, false);
    if (nsplit == 1) return 2;   // stage + attention
    const int rps = attention_rows_per_split(rows, nsplit);
    return cluster_merge_fits(Q, nsplit, DecSmem(rps).bytes() + 1024) ? 2 : 3;
}

cudaError_t launch_attention_tc(const AttnLaunch& l, cudaStream_t st, bool* merged) {
    *merged = false;
    TcAttnDev a;
    memset(&a, 0, sizeof a);
    a.Q = l.Q;
    a.T = l.T;
    a.H = l.H;
    a.q = reinterpret_cast<const __nv_bfloat16*>(l.q);
    a.codes = l.codes;
    a.scales = l.scales;
    a.cap = l.cap;
    a.idx = l.idx;
    a.K = l.K;
    a.swa = l.swa;
    a.W = l.W;
    a.swa_valid = l.swa_valid;
    a.q_pos0 = l.q_pos0;
    a.prefill = l.prefill;
    a.scale = l.scale;
    a.out = l.out;
    a.partial = l.partial;
    a.part = l.o_part != nullptr;
    a.partial_ml = (l.nsplit > 1 || a.part) ? l.partial + (int64_t)l.Q * l.nsplit * l.H * kD
                                            : nullptr;
    a.nsplit = l.nsplit;
    a.status = l.status;
    dim3 grid((unsigned)l.Q, (unsigned)l.nsplit);
    CUtensorMap mx, mq;
    memset(&mx, 0, sizeof mx);
    memset(&mq, 0, sizeof mq);
    if (l.K + l.W == 0) {
        // no row at all: the output (or partial) of an empty softmax, final as written
        *merged = true;
        const int64_t n = (int64_t)l.Q * l.H;
        const int blocks = (int)std::min<int64_t>((n * kD / 4 + 255) / 256, 4096);
        return launch_pdl(attn_empty_kernel, dim3((unsigned)std::max(blocks, 1)), dim3(256), 0, st,
                          a.part ? l.o_part : l.out, a.part ? l.ml_part : nullptr, l.Q, l.H);
    }
    if (!l.prefill && l.stage) {
        // staged decode: pre-pass, then one CTA per (query, split)
        const int rows = l.K + l.W;
        const int rps = attention_rows_per_split(rows, l.nsplit);
        if (rps > kDecRows || (int64_t)rps * l.nsplit < rows) return cudaErrorInvalidValue;
        uint8_t* base = reinterpret_cast<uint8_t*>(l.stage);
        __half* xg = reinterpret_cast<__half*>(base);
        base += (size_t)l.Q * rows * kD * 2;
        base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(base) + 255) & ~(uintptr_t)255);
        __half* qg = reinterpret_cast<__half*>(base);
        base += (size_t)l.Q * kHeads * kD * 2;
        float* qfg = reinterpret_cast<float*>(base);
        base += (size_t)l.Q * kHeads * 4;
        base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(base) + 255) & ~(uintptr_t)255);
        int32_t* validg = reinterpret_cast<int32_t*>(base);
        if (!fp16_rows_map(&mx, xg, (int64_t)l.Q * rows, rps)) return cudaErrorInvalidValue;
        if (!fp16_rows_map(&mq, qg, (int64_t)l.Q * kHeads, kHeads)) return cudaErrorInvalidValue;
        a.st_valid = validg;
        a.st_qf = qfg;
        const int row_blocks = (rows + 7) / 8;
        cudaError_t e = launch_pdl(attn_stage_kernel,
                                   dim3((unsigned)l.Q, (unsigned)(row_blocks + kHeads / 8)),
                                   dim3(256), 0, st, a, xg, qg, qfg, validg, row_blocks);
        if (e != cudaSuccess) return e;
        const int dsmem = DecSmem(rps).bytes() + 1024;
        CUtensorMap mos;
        memset(&mos, 0, sizeof mos);
        if (l.nsplit > 1 && !a.part && cluster_merge_fits(l.Q, l.nsplit, dsmem)) {
            // the splits of a query form one cluster and write the final output themselves
            if (!out_map_sw(&mos, l.out, l.H, l.Q)) return cudaErrorInvalidValue;
            e = cudaFuncSetAttribute(attn_decode_kernel<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, dsmem);
            if (e != cudaSuccess) return e;
            cudaLaunchConfig_t cfg;
            memset(&cfg, 0, sizeof cfg);
            cfg.gridDim = grid;
            cfg.blockDim = dim3(256);
            cfg.dynamicSmemBytes = dsmem;
            cfg.stream = st;
            cudaLaunchAttribute attr[2];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 1;
            attr[0].val.clusterDim.y = (unsigned)l.nsplit;
            attr[0].val.clusterDim.z = 1;
            attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[1].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 2;
            e = cudaLaunchKernelEx(&cfg, attn_decode_kernel<true>, mx, mq, mos, a, rps);
            if (e == cudaSuccess) *merged = true;
            return e;
        }
        if ((l.nsplit > 1 || a.part) ? !out_map_sw(&mos, l.partial, l.H, (int64_t)l.Q * l.nsplit)
                                     : !out_map_sw(&mos, l.out, l.H, l.Q))
            return cudaErrorInvalidValue;
        e = cudaFuncSetAttribute(attn_decode_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, dsmem);
        if (e != cudaSuccess) return e;
        return launch_pdl(attn_decode_kernel<false>, grid, dim3(256), (size_t)dsmem, st, mx, mq,
                          mos, a, rps);
    }
    return cudaErrorInvalidValue;   // decode always has a staging area (api.cu)
}

}  // namespace csa2
