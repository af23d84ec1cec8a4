// KV compressor + indexer-K projection, fused with FP4 quantize-on-write.
//
// "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (AI summary),
// Methodology in Plain English: the compressor no longer uses overlapping source entries
// or absolute positional embeddings, and the indexer K is derived by projecting the main
// KV entries. "DeepSeek V4.1 Flash: smaller KV cache, same post-training", How did
// DeepSeek V4.1 reduce the KV cache?, names the compressed entries (C_l) and compression
// weights (Z_l); its equation is lost. Reading taken (the plainest those support):
//   entry j of a sequence pools source tokens r*j .. r*j + r - 1; per channel d,
//     x[j][d] = bf16( sum_t softmax_t(Z[t][d]) * C[t][d] )
//   codes, scales = FP4 quantize-on-write of x[j] (as csa2_quantize_kv)
//   k[j][e] = sum_d W[e][d] * x[j][d], stored as E4M3 (RNE, saturating) or bf16.
//
// One CTA per E entries, E = 8, 16 or 32: the fewest that still fill the SMs (the MMA's M is
// 128; rows E.. are computed and discarded, the projection being tiny next to the pooling's
// loads), 16 warps (128 registers a thread; each warp's entries are pooled one after the
// other, so more warps mean shorter chains of dependent loads):
//  1. pooling: warp w takes entries w, w+16, ...; lane l owns channels [16l, 16l+16), i.e.
//     one FP4 scale block. Per token the warp reads the 1 KiB latent and logit rows in one
//     coalesced sweep (up to 2 tokens: all of an entry's rows in one batch of loads, issued
//     before the entry's cache offset is known; more tokens: a pass for the maxima, then one
//     for the sums); the softmax (max, then exp-weighted sums) runs in fp32 per channel.
//     (Two entries' rows per batch was slower after an L2 flush.)
//     The bf16 latent goes to the global FP4 cache (codes + scale, this lane's block) and
//     into shared memory as the MMA's A operand (K-major, 128-byte swizzle, 8 slabs of
//     64 channels);
//  2. projection: one thread issues tcgen05.mma kind::f16 (bf16 x bf16 -> fp32 in TMEM),
//     M = 128 entries, N = 64 key channels, K = 512, twice. Both halves of W are TMA-loaded
//     at the start: the first into rows 64-127 of the A operand's slabs, which hold no
//     entry (the MMA reads them as discarded rows), the second into its own 64 KiB;
//  3. epilogue: warp 0 reads TMEM lanes 0-31 (one entry per thread), converts and stores
//     the 128-channel key row.
#include "csa2_common.cuh"
#include "csa2_internal.h"
#include "fp4_block.cuh"

namespace csa2 {
namespace {

constexpr int kM = 128;                    // MMA rows (A operand rows in shared memory)
constexpr int kMaxE = 32;                  // entries per CTA at most (rows E.. of the MMA unused)
constexpr int kD = 512;                    // latent channels
constexpr int kDi = 128;                   // indexer-key channels
constexpr int kThreads = 512;
constexpr int kESlab = kM * 128;           // 128 entries x 64 bf16 channels = 16 KiB
constexpr int kWSlab = 64 * 128;           // 64 key channels x 64 bf16 channels = 8 KiB
constexpr int kOffE = 0;                   // 8 slabs: 128 KiB
constexpr int kWInE = 64 * 128;            // W's first half: rows 64.. of each A slab (8 KiB)
constexpr int kOffW = 8 * kESlab;          // 8 slabs of W's second half: 64 KiB
static_assert(kMaxE <= 64, "W's first half shares the A slabs above the entries' rows");
constexpr int kOffRow = kOffW + 8 * kWSlab;   // int64 per entry: cache row or -1
constexpr int kOffBar = kOffRow + kM * 8;
constexpr int kDynBytes = kOffBar + 64 + 1024;   // + alignment slack

struct CompressDev {
    int B, n_new, r;
    int64_t ld, bstride;          // elements between tokens / sequences of C and Z
    const __nv_bfloat16* C;
    const __nv_bfloat16* Z;
    const int32_t* dst_off;
    uint8_t* codes;
    uint8_t* scales;
    uint8_t* keys;                // [B][cap][128] E4M3 or bf16, or compact-key codes [B][cap][64]
    float* key_scales;            // compact keys: fp32 scale per key [B][cap]
    int key_bf16;
    int key_fp4;
    int epc;                      // entries per CTA (8, 16 or 32)
    int64_t cap;
    __nv_bfloat16* latent;        // [B * n_new][512] or null
    int32_t* status;
};

__device__ __forceinline__ void bf16x16_to_float(const uint4& a, const uint4& b, float (&x)[16]) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        x[2 * k] = __uint_as_float(w[k] << 16);
        x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
}

// Per channel, the softmax over the entry's nt <= NT tokens of the logits zr weighting the
// latents cr (rows already in registers), rounded to bf16: the maximum first, then the
// exp-weighted sums in token order.
template <int NT>
__device__ __forceinline__ void pool_rows(const uint4 (&zr)[NT][2], const uint4 (&cr)[NT][2],
                                          int nt, float (&x)[16]) {
    float zmax[16], den[16], num[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        zmax[k] = -INFINITY;
        den[k] = num[k] = 0.f;
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (t < nt) {
            float z[16];
            bf16x16_to_float(zr[t][0], zr[t][1], z);
#pragma unroll
            for (int k = 0; k < 16; ++k) zmax[k] = fmaxf(zmax[k], z[k]);
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (t < nt) {
            float z[16], c[16];
            bf16x16_to_float(zr[t][0], zr[t][1], z);
            bf16x16_to_float(cr[t][0], cr[t][1], c);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float e = expf(z[k] - zmax[k]);
                den[k] += e;
                num[k] = fmaf(e, c[k], num[k]);
            }
        }
    }
#pragma unroll
    for (int k = 0; k < 16; ++k)
        x[k] = __bfloat162float(__float2bfloat16_rn(__fdiv_rn(num[k], den[k])));
}

__global__ void __launch_bounds__(kThreads, 1)
    compress_kv_kernel(const __grid_constant__ CUtensorMap tmap_w, const CompressDev a) {
    extern __shared__ uint8_t dsm_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                             ~(uintptr_t)1023);
    int64_t* row_dst = reinterpret_cast<int64_t*>(sm + kOffRow);
    uint64_t* wfull = reinterpret_cast<uint64_t*>(sm + kOffBar);
    uint64_t* mdone = wfull + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(wfull + 3);
    volatile int* stuck = reinterpret_cast<volatile int*>(wfull + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sE = smem_u32(sm + kOffE), sW = smem_u32(sm + kOffW);

    grid_dep_launch();
    if (threadIdx.x == 0) {
        mbar_init(wfull, 1);
        mbar_init(mdone, 1);
        *stuck = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_w);
    }
    if (warp == 1) tmem_alloc(tmem_holder, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    grid_dep_wait();   // C, Z, W and the offsets come from earlier work on the stream

    if (threadIdx.x == 0) {   // W: key channels 0..63 into the A slabs, 64..127 apart
        mbar_arrive_expect_tx(wfull, 16 * kWSlab);
        for (int s = 0; s < 8; ++s) {
            tma_load_2d(sm + kOffE + s * kESlab + kWInE, &tmap_w, wfull, 64 * s, 0);
            tma_load_2d(sm + kOffW + s * kWSlab, &tmap_w, wfull, 64 * s, 64);
        }
    }

    // ---- 1. pooling, FP4 write and the A operand ----------------------------------------
    const int64_t total = (int64_t)a.B * a.n_new;
    const int epc = a.epc;
    if (threadIdx.x >= epc && threadIdx.x < kM) row_dst[threadIdx.x] = -1;
    // entry m of this CTA: its sequence b, index j and cache offset (the offset is used only
    // by the writes, so the entry's rows are requested without waiting for it)
    auto locate = [&](int m, int& b, int& j, int64_t& dst) -> bool {
        const int64_t g = (int64_t)blockIdx.x * epc + m;
        b = 0;
        j = 0;
        dst = -1;
        if (m >= epc || g >= total) return false;
        b = (int)(g / a.n_new);
        j = (int)(g - (int64_t)b * a.n_new);
        dst = (int64_t)ld_dep(a.dst_off + b) + j;
        return true;
    };
    // this lane's 16 channels of token t of entry (b, j): logits and latents
    auto zrow = [&](int b, int j, int t) {
        return reinterpret_cast<const uint4*>(a.Z + (int64_t)b * a.bstride +
                                              ((int64_t)j * a.r + t) * a.ld + lane * 16);
    };
    auto crow_src = [&](int b, int j, int t) {
        return reinterpret_cast<const uint4*>(a.C + (int64_t)b * a.bstride +
                                              ((int64_t)j * a.r + t) * a.ld + lane * 16);
    };
    // the writes of entry m: its bf16 latent into the A operand (and the optional latent
    // output), its FP4 codes and scale into the cache
    auto finish = [&](int m, bool have, int b, int64_t dst, const float (&x)[16]) {
        int64_t crow = -1;
        if (have) {
            if (dst >= 0 && dst < a.cap)
                crow = (int64_t)b * a.cap + dst;
            else if (lane == 0)
                set_status(a.status, CSA2_DEV_BAD_INDEX);
        }
        // bf16 latent: 16 channels = two 16-byte chunks of row m in slab lane/4
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            pk[k] = (__float_as_uint(x[2 * k]) >> 16) | (__float_as_uint(x[2 * k + 1]) & 0xFFFF0000u);
        {
            uint8_t* row = sm + kOffE + (lane >> 2) * kESlab + m * 128;
            const int c0 = (lane & 3) * 2;
            *reinterpret_cast<uint4*>(row + (((c0) ^ (m & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(row + (((c0 + 1) ^ (m & 7)) << 4)) =
                make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        if (lane == 0) row_dst[m] = crow;
        if (crow >= 0) {
            uint2 packed;
            uint8_t sc;
            fp4_quantize_block16(x, packed, sc);
            reinterpret_cast<uint2*>(a.codes + crow * CSA2_ENTRY_CODE_BYTES)[lane] = packed;
            a.scales[crow * CSA2_ENTRY_SCALE_BYTES + lane] = sc;
            if (a.latent) {
                const int64_t g = (int64_t)blockIdx.x * epc + m;
                uint4* lp = reinterpret_cast<uint4*>(a.latent + g * kD + lane * 16);
                lp[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                lp[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
    };

    for (int m = warp; m < epc; m += kThreads / 32) {
        int b, j;
        int64_t dst;
        const bool have = locate(m, b, j, dst);
        float x[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) x[k] = 0.f;
        if (have && a.r <= 2) {
            // up to 2 tokens: every latent and logit row of the entry in one batch of loads
            // (a batch of 4 spilled registers at 512 threads)
            uint4 zr[2][2], cr[2][2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (t < a.r) {
                    zr[t][0] = ld_dep(zrow(b, j, t));
                    zr[t][1] = ld_dep(zrow(b, j, t) + 1);
                    cr[t][0] = ld_dep(crow_src(b, j, t));
                    cr[t][1] = ld_dep(crow_src(b, j, t) + 1);
                }
            }
            pool_rows<2>(zr, cr, a.r, x);
        } else if (have) {
            float zmax[16], den[16], num[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                zmax[k] = -INFINITY;
                den[k] = num[k] = 0.f;
            }
            for (int t = 0; t < a.r; ++t) {
                float z[16];
                bf16x16_to_float(ld_dep(zrow(b, j, t)), ld_dep(zrow(b, j, t) + 1), z);
#pragma unroll
                for (int k = 0; k < 16; ++k) zmax[k] = fmaxf(zmax[k], z[k]);
            }
            for (int t = 0; t < a.r; ++t) {
                float z[16], c[16];
                bf16x16_to_float(ld_dep(zrow(b, j, t)), ld_dep(zrow(b, j, t) + 1), z);
                bf16x16_to_float(ld_dep(crow_src(b, j, t)), ld_dep(crow_src(b, j, t) + 1), c);
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const float e = expf(z[k] - zmax[k]);
                    den[k] += e;
                    num[k] = fmaf(e, c[k], num[k]);
                }
            }
#pragma unroll
            for (int k = 0; k < 16; ++k)
                x[k] = __bfloat162float(__float2bfloat16_rn(__fdiv_rn(num[k], den[k])));
        }
        finish(m, have, b, dst, x);
    }
    // the A operand was written by plain stores: make it visible to the tensor core
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- 2. projection ------------------------------------------------------------------
    if (threadIdx.x == 0) {
        constexpr uint32_t idesc = make_idesc(128, 64, 1u, 1u);   // bf16 x bf16 -> fp32
        const bool ok = mbar_wait(wfull, 0, a.status);
        if (ok) {
            tc_fence_after();
            // fully unrolled: each descriptor is a base plus a constant (the start-address
            // field counts 16-byte units and no address reaches 256 KiB), so the issuing
            // thread spends a few instructions per MMA
            const uint64_t a0 = sw128_desc(sE, 16, 1024);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const uint64_t b0 = sw128_desc(half == 0 ? sE + kWInE : sW, 16, 1024);
                const uint32_t wstride = half == 0 ? (uint32_t)kESlab : (uint32_t)kWSlab;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t ad = a0 + (uint64_t)(((kk >> 2) * kESlab + (kk & 3) * 32) >> 4);
                    const uint64_t bd = b0 + (uint64_t)(((kk >> 2) * wstride + (kk & 3) * 32) >> 4);
                    mma_f16(tmem + 64 * half, ad, bd, idesc, kk > 0);
                }
            }
            mma_commit(mdone);
        }
        if (!ok) *stuck = 1;   // an MMA or a load may still be in flight
    }
    __syncwarp();

    // ---- 3. epilogue: one entry per thread of warps 0-3 ------------------------------------
    if (warp < (epc + 31) / 32) {
        bool ok = !*stuck && mbar_wait(mdone, 0, a.status);
        ok = __all_sync(0xffffffffu, ok);   // tcgen05.ld below is warp-collective
        if (!ok) *stuck = 1;
        tc_fence_after();
        const int m = warp * 32 + lane;
        const int64_t crow = row_dst[m];
        if (ok && a.key_fp4) {
            // compact key of the bf16-rounded projection (csa2_quantize_keys_fp4's decisions):
            // pass 1 its amax, pass 2 the E2M1 codes under s = amax / 6
            const uint32_t row_t = tmem + ((uint32_t)(warp * 32) << 16);
            auto rounded = [](uint32_t u) { return __bfloat162float(__float2bfloat16_rn(__uint_as_float(u))); };
            float amax = 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < kDi; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(row_t + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(rounded(v[k])));
            }
            const float s = __fdiv_rn(amax, 6.0f);
#pragma unroll 1
            for (int c0 = 0; c0 < kDi; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(row_t + c0, v);
                tmem_ld_wait();
                uint32_t w[2] = {0u, 0u};
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float x0 = rounded(v[2 * k]), x1 = rounded(v[2 * k + 1]);
                    const float q0 = (s > 0.f) ? __fdiv_rn(fabsf(x0), s) : 0.f;
                    const float q1 = (s > 0.f) ? __fdiv_rn(fabsf(x1), s) : 0.f;
                    uint16_t byte;
                    asm("{\n\t.reg .b8 t;\n\t"
                        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
                        "cvt.u16.u8 %0, t;\n\t}"
                        : "=h"(byte)
                        : "f"(q1), "f"(q0));
                    uint32_t bb = byte & 0x77u;
                    bb |= (__float_as_uint(x0) >> 31) << 3;
                    bb |= (__float_as_uint(x1) >> 31) << 7;
                    w[k >> 2] |= bb << (8 * (k & 3));
                }
                if (crow >= 0)
                    *reinterpret_cast<uint2*>(a.keys + crow * (kDi / 2) + c0 / 2) = make_uint2(w[0], w[1]);
            }
            if (crow >= 0) a.key_scales[crow] = s;
        } else if (ok) {
#pragma unroll 1
            for (int c0 = 0; c0 < kDi; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
                tmem_ld_wait();
                if (crow < 0) continue;
                if (a.key_bf16) {
                    uint32_t o[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * k]),
                                                                       __uint_as_float(v[2 * k + 1]));
                        o[k] = *reinterpret_cast<const uint32_t*>(&h);
                    }
                    uint4* kp = reinterpret_cast<uint4*>(a.keys + (crow * kDi + c0) * 2);
                    kp[0] = make_uint4(o[0], o[1], o[2], o[3]);
                    kp[1] = make_uint4(o[4], o[5], o[6], o[7]);
                } else {
                    uint32_t o[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint16_t lo, hi;
                        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
                            : "=h"(lo) : "f"(__uint_as_float(v[4 * k + 1])), "f"(__uint_as_float(v[4 * k])));
                        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
                            : "=h"(hi) : "f"(__uint_as_float(v[4 * k + 3])), "f"(__uint_as_float(v[4 * k + 2])));
                        o[k] = (uint32_t)lo | ((uint32_t)hi << 16);
                    }
                    *reinterpret_cast<uint4*>(a.keys + crow * kDi + c0) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1 && !*stuck) tmem_dealloc(tmem, 128);
}

}  // namespace

cudaError_t launch_compress_kv(const CompressLaunch& l, cudaStream_t st) {
    const int64_t entries = (int64_t)l.B * l.n_new;
    if (entries == 0) return cudaSuccess;
    auto enc = tensor_map_encoder();
    if (!enc) return cudaErrorInvalidValue;
    // W: [128 key channels][512] bf16, box = 64 channels x 64 key channels, 128-byte swizzle
    CUtensorMap mw;
    memset(&mw, 0, sizeof mw);
    cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)kDi};
    cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t es[2] = {1, 1};
    if (enc(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(l.w_proj), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    CompressDev a;
    memset(&a, 0, sizeof a);
    a.B = l.B;
    a.n_new = l.n_new;
    a.r = l.r;
    a.ld = l.ld;
    a.bstride = l.bstride;
    a.C = reinterpret_cast<const __nv_bfloat16*>(l.C);
    a.Z = reinterpret_cast<const __nv_bfloat16*>(l.Z);
    a.dst_off = l.dst_off;
    a.codes = l.codes;
    a.scales = l.scales;
    a.keys = reinterpret_cast<uint8_t*>(l.keys);
    a.key_bf16 = l.key_bf16;
    a.key_fp4 = l.key_fp4;
    if (l.key_fp4)
        a.key_scales = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(l.keys) +
                                                (size_t)l.B * l.cap * CSA2_FP4KEY_CODE_BYTES);
    a.cap = l.cap;
    a.latent = reinterpret_cast<__nv_bfloat16*>(l.latent);
    a.status = l.status;
    cudaError_t e = cudaFuncSetAttribute(compress_kv_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kDynBytes);
    if (e != cudaSuccess) return e;
    // the fewest entries per CTA (8, 16, 32) whose grid still fits on the SMs: few entries
    // (a decode step) spread over several CTAs, each with one short chain of loads per warp
    const int sms = device_sm_count();
    a.epc = kMaxE;
    for (int e8 = 8; e8 < kMaxE; e8 *= 2)
        if ((entries + e8 - 1) / e8 <= sms) {
            a.epc = e8;
            break;
        }
    const int64_t grid = (entries + a.epc - 1) / a.epc;
    return launch_pdl(compress_kv_kernel, dim3((unsigned)grid), dim3(kThreads), (size_t)kDynBytes,
                      st, mw, a);
}

}  // namespace csa2
