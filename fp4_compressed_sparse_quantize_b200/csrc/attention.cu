// Fused gather + exact FP4 dequantisation + joint sparse / sliding-window attention.
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
// Numerics: FP4 x E4M3 and E4M3 values have at most 6 significant bits and lie inside the
// fp16 normal range, so the dequantised rows are EXACT in fp16. The query goes to fp16 after
// an exact per-head power-of-two rescaling (largest |q| in [2^14, 2^15)), which keeps every
// element above 2^-28 of the head's largest exactly; the power of two is folded back into
// the logit scale. Probabilities enter the P x V product as fp16 (bf16 would cost
// ~8x the error) and, because a single fp16 rounding of P already costs ~2e-3 of the output
// RMS on heavy-tailed channels, P is carried as an fp16 (high, low) pair whose two products
// are accumulated together (~22-bit probabilities). Accumulation is fp32.
//
// Structure: a CTA owns one query row (all heads) and a range of 64-row chunks of the
// concatenated [selected entries | window rows] list. Per chunk: cp.async gather of the raw
// rows, dequantisation into a swizzled fp16 tile, S = Q X^T and O += P X on the tensor
// cores (mma.sync m16n8k16), online softmax across chunks. Decode splits the rows of a
// query over several CTAs and merges the partial (max, sum, output) triples afterwards.
#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

constexpr int kR = 64;        // rows per chunk
constexpr int kDm = 512;      // latent channels
constexpr int kHP = 64;       // heads per CTA (padded)

struct AttnDev {
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
    float* partial;
    int nsplit, nchunks, chunks_per_split;
    int32_t* status;
};

struct AttnSmem {
    static constexpr int kQ = 0;                        // 64 x 1024 B (fp16, swizzled)
    static constexpr int kX = kQ + kHP * 1024;          // 64 x 1024 B
    static constexpr int kP = kX + kR * 1024;           // 64 x 128 B  (P, fp16 high part)
    static constexpr int kPlo = kP + kHP * 128;         // 64 x 128 B  (P - high, fp16)
    static constexpr int kRaw = kPlo + kHP * 128;       // 64 x 512 B
    static constexpr int kQf = kRaw + kR * 512;         // 64 floats
    static constexpr int kRedM = kQf + kHP * 4;         // 2 x 64 floats
    static constexpr int kRedS = kRedM + 2 * kHP * 4;   // 2 x 64 floats
    static constexpr int kValid = kRedS + 2 * kHP * 4;  // 64 ints (0 invalid, 1 fp4, 2 e4m3)
    static constexpr int kBytes = kValid + kR * 4;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// byte offset of 16-byte chunk `c` of row `r` in a tile with `rowbytes`-byte rows
__device__ __forceinline__ uint32_t swz(int r, int c, int rowbytes) {
    return (uint32_t)(r * rowbytes + ((c ^ (r & 7)) << 4));
}

// two E2M1 codes (one byte: low nibble first) -> fp16x2, exactly
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(out)
        : "r"(byte));
    return out;
}

__global__ void __launch_bounds__(256, 1) attn_kernel(const AttnDev a) {
    extern __shared__ __align__(1024) uint8_t sm[];
    using L = AttnSmem;
    const uint32_t sQ = smem_u32(sm + L::kQ), sX = smem_u32(sm + L::kX),
                   sP = smem_u32(sm + L::kP), sPlo = smem_u32(sm + L::kPlo),
                   sRaw = smem_u32(sm + L::kRaw);
    float* qf = reinterpret_cast<float*>(sm + L::kQf);
    float* redm = reinterpret_cast<float*>(sm + L::kRedM);
    float* reds = reinterpret_cast<float*>(sm + L::kRedS);
    int* rvalid = reinterpret_cast<int*>(sm + L::kValid);

    const int qrow = blockIdx.x;
    const int split = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = qrow / a.T, t = qrow - b * a.T;
    const int c_begin = split * a.chunks_per_split;
    const int c_end = min(a.nchunks, c_begin + a.chunks_per_split);

    // ---- query: per-head power-of-two rescale into fp16 ---------------------------------
    {
        uint4 raw[8][2];   // the warp's 8 heads, all loads in flight before use
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int h = warp + 8 * k;
            if (h < a.H) {
                const uint4* src = reinterpret_cast<const uint4*>(
                    a.q + ((int64_t)qrow * a.H + h) * kDm + lane * 16);
                raw[k][0] = __ldg(src);
                raw[k][1] = __ldg(src + 1);
            } else {
                raw[k][0] = raw[k][1] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int h = warp + 8 * k;
            float v[16];
            const uint32_t w8[8] = {raw[k][0].x, raw[k][0].y, raw[k][0].z, raw[k][0].w,
                                    raw[k][1].x, raw[k][1].y, raw[k][1].z, raw[k][1].w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                v[2 * e] = __uint_as_float(w8[e] << 16);
                v[2 * e + 1] = __uint_as_float(w8[e] & 0xFFFF0000u);
            }
            float amax = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(v[e]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            int shift = 0;
            if (amax > 0.f) {
                const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
                shift = min(126, max(-126, 14 - ex));
            }
            const float mul = ldexpf(1.0f, shift);
            uint32_t hw[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                __half2 h2 = __floats2half2_rn(v[2 * e] * mul, v[2 * e + 1] * mul);
                hw[e] = *reinterpret_cast<uint32_t*>(&h2);
            }
            // lane owns channels [16 lane, 16 lane + 16) = chunks 2 lane, 2 lane + 1
            const uint32_t d0 = sQ + swz(h, 2 * lane, 1024), d1 = sQ + swz(h, 2 * lane + 1, 1024);
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(d0), "r"(hw[0]),
                         "r"(hw[1]), "r"(hw[2]), "r"(hw[3]));
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(d1), "r"(hw[4]),
                         "r"(hw[5]), "r"(hw[6]), "r"(hw[7]));
            if (lane == 0) qf[h] = a.scale * 1.4426950408889634f * ldexpf(1.0f, -shift);
        }
    }

    const int hg = warp & 3;       // head group: heads [16 hg, 16 hg + 16)
    const int half = warp >> 2;    // S: rows [32 half, +32); PV: channels [256 half, +256)
    const int hA = 16 * hg + (lane >> 2), hB = hA + 8;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float o[32][4];
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    const int rows_total = a.K + a.W;
    for (int ch = c_begin; ch < c_end; ++ch) {
        // ---- gather raw rows ------------------------------------------------------------
        {
            const int i = tid >> 2, part = tid & 3;  // 4 threads per row
            const int g = ch * kR + i;
            int kind = 0;
            const uint8_t* src = nullptr;
            if (g < a.K) {
                const int32_t e = __ldg(a.idx + (int64_t)qrow * a.K + g);
                if (e >= 0 && e < a.cap) {
                    kind = 1;
                } else if (e != -1) {
                    if (part == 0) set_status(a.status, CSA2_DEV_BAD_INDEX);
                }
                if (kind == 1) {
                    const int64_t ent = (int64_t)b * a.cap + e;
                    // chunks 0..15 codes, 16..17 scales
                    for (int c = part; c < 18; c += 4) {
                        const uint8_t* s = c < 16 ? a.codes + ent * CSA2_ENTRY_CODE_BYTES + c * 16
                                                  : a.scales + ent * CSA2_ENTRY_SCALE_BYTES +
                                                        (c - 16) * 16;
                        cp16(sRaw + i * 512 + c * 16, s);
                    }
                }
            } else if (g < rows_total) {
                const int v = g - a.K;  // window row 0..W-1 (oldest first)
                int64_t srow;
                bool ok;
                if (!a.prefill) {
                    const int nv = a.swa_valid ? __ldg(a.swa_valid + b) : a.W;
                    ok = v >= a.W - nv;
                    srow = (int64_t)b * a.W + v;
                } else {
                    const int64_t rw = t + v;  // buffer row of token t's window row v
                    const int64_t pos =
                        (a.q_pos0 ? (int64_t)__ldg(a.q_pos0 + b) : (int64_t)(a.W - 1)) - (a.W - 1) + rw;
                    ok = pos >= 0;
                    srow = (int64_t)b * (a.W - 1 + a.T) + rw;
                }
                if (ok) {
                    kind = 2;
                    src = a.swa + srow * kDm;
                    for (int c = part; c < 32; c += 4) cp16(sRaw + i * 512 + c * 16, src + c * 16);
                }
            }
            if (part == 0) rvalid[i] = kind;
            asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        // ---- dequantise into the fp16 X tile -------------------------------------------------
        {
            const int i = tid >> 2, part = tid & 3;
            const int kind = rvalid[i];
            const uint8_t* raw = sm + L::kRaw + i * 512;
#pragma unroll 2
            for (int gi = 0; gi < 8; ++gi) {
                const int grp = part * 8 + gi;  // 16-channel group 0..31
                uint32_t hv[8];
                if (kind == 1) {
                    const uint2 cb = *reinterpret_cast<const uint2*>(raw + grp * 8);
                    const __half2 s2 = __half2half2(__float2half_rn(e4m3_to_float(raw[256 + grp])));
                    const uint32_t cw[2] = {cb.x, cb.y};
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        uint32_t h2 = e2m1x2_to_h2((cw[k >> 2] >> (8 * (k & 3))) & 0xFFu);
                        __half2 x = __hmul2(*reinterpret_cast<__half2*>(&h2), s2);
                        hv[k] = *reinterpret_cast<uint32_t*>(&x);
                    }
                } else if (kind == 2) {
                    const uint4 eb = *reinterpret_cast<const uint4*>(raw + grp * 16);
                    const uint32_t ew[4] = {eb.x, eb.y, eb.z, eb.w};
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        __half2 x = e4m3x2_to_half2((uint16_t)(ew[k >> 1] >> (16 * (k & 1))));
                        hv[k] = *reinterpret_cast<uint32_t*>(&x);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) hv[k] = 0u;
                }
                const uint32_t d0 = sX + swz(i, 2 * grp, 1024), d1 = sX + swz(i, 2 * grp + 1, 1024);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(d0), "r"(hv[0]),
                             "r"(hv[1]), "r"(hv[2]), "r"(hv[3]));
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(d1), "r"(hv[4]),
                             "r"(hv[5]), "r"(hv[6]), "r"(hv[7]));
            }
        }
        __syncthreads();
        // ---- S = Q X^T for heads [16 hg, +16) x rows [32 half, +32) ---------------------------
        float s[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll 4
        for (int ks = 0; ks < 32; ++ks) {
            uint32_t a0, a1, a2, a3;
            const int qr = 16 * hg + (lane & 15);
            ldsm_x4(sQ + swz(qr, 2 * ks + (lane >> 4), 1024), a0, a1, a2, a3);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b0, b1, b2, b3;
                const int xr = 32 * half + 16 * np + (lane & 7) + ((lane >> 4) << 3);
                ldsm_x4(sX + swz(xr, 2 * ks + ((lane >> 3) & 1), 1024), b0, b1, b2, b3);
                mma16816(s[2 * np], a0, a1, a2, a3, b0, b1);
                mma16816(s[2 * np + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        // ---- online softmax ---------------------------------------------------------------------
        const float fA = qf[hA], fB = qf[hB];
        float mA = -INFINITY, mB = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int rr = 32 * half + 8 * nt + 2 * (lane & 3) + e;
                const bool ok = rvalid[rr] != 0;
                s[nt][e] = ok ? s[nt][e] * fA : -INFINITY;
                s[nt][2 + e] = ok ? s[nt][2 + e] * fB : -INFINITY;
                mA = fmaxf(mA, s[nt][e]);
                mB = fmaxf(mB, s[nt][2 + e]);
            }
#pragma unroll
        for (int o2 = 1; o2 <= 2; o2 <<= 1) {
            mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, o2));
            mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, o2));
        }
        if ((lane & 3) == 0) {
            redm[half * kHP + hA] = mA;
            redm[half * kHP + hB] = mB;
        }
        __syncthreads();
        const float mcA = fmaxf(redm[hA], redm[kHP + hA]);
        const float mcB = fmaxf(redm[hB], redm[kHP + hB]);
        const float mnA = fmaxf(m_run[0], mcA), mnB = fmaxf(m_run[1], mcB);
        const float baseA = (mnA == -INFINITY) ? 0.f : mnA;
        const float baseB = (mnB == -INFINITY) ? 0.f : mnB;
        const float alA = exp2f(m_run[0] - baseA), alB = exp2f(m_run[1] - baseB);
        // P = exp2(logit - max) in fp32, stored as an fp16 pair (high, low) so that the
        // P x V product keeps ~22 bits of every probability.
        float sumA = 0.f, sumB = 0.f;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const float p0 = exp2f(s[nt][0] - baseA), p1 = exp2f(s[nt][1] - baseA);
            const float p2 = exp2f(s[nt][2] - baseB), p3 = exp2f(s[nt][3] - baseB);
            sumA += p0 + p1;
            sumB += p2 + p3;
            const __half2 pa = __floats2half2_rn(p0, p1);
            const __half2 pb = __floats2half2_rn(p2, p3);
            const __half2 la = __floats2half2_rn(p0 - __low2float(pa), p1 - __high2float(pa));
            const __half2 lb = __floats2half2_rn(p2 - __low2float(pb), p3 - __high2float(pb));
            const int rr = 32 * half + 8 * nt + 2 * (lane & 3);  // P column (row of X)
            const uint32_t offA = swz(hA, rr >> 3, 128) + (rr & 7) * 2;
            const uint32_t offB = swz(hB, rr >> 3, 128) + (rr & 7) * 2;
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(sP + offA), "r"(*reinterpret_cast<const uint32_t*>(&pa)));
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(sP + offB), "r"(*reinterpret_cast<const uint32_t*>(&pb)));
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(sPlo + offA), "r"(*reinterpret_cast<const uint32_t*>(&la)));
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(sPlo + offB), "r"(*reinterpret_cast<const uint32_t*>(&lb)));
        }
#pragma unroll
        for (int o2 = 1; o2 <= 2; o2 <<= 1) {
            sumA += __shfl_xor_sync(0xffffffffu, sumA, o2);
            sumB += __shfl_xor_sync(0xffffffffu, sumB, o2);
        }
        if ((lane & 3) == 0) {
            reds[half * kHP + hA] = sumA;
            reds[half * kHP + hB] = sumB;
        }
        __syncthreads();
        l_run[0] = l_run[0] * alA + reds[hA] + reds[kHP + hA];
        l_run[1] = l_run[1] * alB + reds[hB] + reds[kHP + hB];
        m_run[0] = mnA;
        m_run[1] = mnB;
#pragma unroll
        for (int nt = 0; nt < 32; ++nt) {
            o[nt][0] *= alA;
            o[nt][1] *= alA;
            o[nt][2] *= alB;
            o[nt][3] *= alB;
        }
        // ---- O += P X for heads [16 hg, +16) x channels [256 half, +256) ------------------------
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
            const int pr = 16 * hg + (lane & 15);
            ldsm_x4(sP + swz(pr, 2 * ks + (lane >> 4), 128), a0, a1, a2, a3);
            ldsm_x4(sPlo + swz(pr, 2 * ks + (lane >> 4), 128), c0, c1, c2, c3);
            const int xr = 16 * ks + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int np = 0; np < 16; ++np) {
                uint32_t b0, b1, b2, b3;
                const int chk = (256 * half + 16 * np) / 8 + (lane >> 4);
                ldsm_x4_t(sX + swz(xr, chk, 1024), b0, b1, b2, b3);
                mma16816(o[2 * np], a0, a1, a2, a3, b0, b1);
                mma16816(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
                mma16816(o[2 * np], c0, c1, c2, c3, b0, b1);
                mma16816(o[2 * np + 1], c0, c1, c2, c3, b2, b3);
            }
        }
        __syncthreads();  // X, P, reductions are rewritten by the next chunk
    }

    // ---- write ----------------------------------------------------------------------------------
    if (a.nsplit == 1) {
        const float invA = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
        const float invB = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
#pragma unroll
        for (int nt = 0; nt < 32; ++nt) {
            const int c = 256 * half + 8 * nt + 2 * (lane & 3);
            if (hA < a.H)
                *reinterpret_cast<float2*>(a.out + ((int64_t)qrow * a.H + hA) * kDm + c) =
                    make_float2(o[nt][0] * invA, o[nt][1] * invA);
            if (hB < a.H)
                *reinterpret_cast<float2*>(a.out + ((int64_t)qrow * a.H + hB) * kDm + c) =
                    make_float2(o[nt][2] * invB, o[nt][3] * invB);
        }
    } else {
        // partial layout per (qrow, split): O [H][512], m [H], l [H]
        float* base = a.partial + ((int64_t)qrow * a.nsplit + split) * ((int64_t)a.H * (kDm + 2));
#pragma unroll
        for (int nt = 0; nt < 32; ++nt) {
            const int c = 256 * half + 8 * nt + 2 * (lane & 3);
            if (hA < a.H)
                *reinterpret_cast<float2*>(base + (int64_t)hA * kDm + c) = make_float2(o[nt][0], o[nt][1]);
            if (hB < a.H)
                *reinterpret_cast<float2*>(base + (int64_t)hB * kDm + c) = make_float2(o[nt][2], o[nt][3]);
        }
        if (half == 0 && (lane & 3) == 0) {
            float* ml = base + (int64_t)a.H * kDm;
            if (hA < a.H) { ml[hA] = m_run[0]; ml[a.H + hA] = l_run[0]; }
            if (hB < a.H) { ml[hB] = m_run[1]; ml[a.H + hB] = l_run[1]; }
        }
    }
}

// Merge the per-split partial results of one (query row, head): out = sum_s 2^(m_s - M)
// O_s / sum_s 2^(m_s - M) l_s (base-2 logits). One CTA per (row, head), 4 channels/thread.
__global__ void __launch_bounds__(128) attn_combine_kernel(const float* __restrict__ partial,
                                                           int nsplit, int H,
                                                           float* __restrict__ out) {
    __shared__ float wgt[64];
    __shared__ float inv_s;
    const int qrow = blockIdx.x, h = blockIdx.y;
    const int64_t stride = (int64_t)H * (kDm + 2);
    const float* base = partial + (int64_t)qrow * nsplit * stride;
    if (threadIdx.x < 32) {
        const int s = threadIdx.x;
        float m = -INFINITY, l = 0.f;
        if (s < nsplit) {
            m = base[s * stride + (int64_t)H * kDm + h];
            l = base[s * stride + (int64_t)H * kDm + H + h];
        }
        float M = m;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float Mb = (M == -INFINITY) ? 0.f : M;
        const float wv = (s < nsplit) ? exp2f(m - Mb) : 0.f;
        float L = wv * l;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (s < nsplit) wgt[s] = wv;
        if (s == 0) inv_s = L > 0.f ? 1.f / L : 0.f;
    }
    __syncthreads();
    const int c = threadIdx.x * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < nsplit; ++s) {
        const float4 v = *reinterpret_cast<const float4*>(base + s * stride + (int64_t)h * kDm + c);
        const float wv = wgt[s];
        acc.x += wv * v.x;
        acc.y += wv * v.y;
        acc.z += wv * v.z;
        acc.w += wv * v.w;
    }
    const float inv = inv_s;
    *reinterpret_cast<float4*>(out + ((int64_t)qrow * H + h) * kDm + c) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

int attention_splits(int Q, int K, int W, bool prefill) {
    const int nchunks = (K + W + 127) / 128;     // 128-row chunks of the tensor-core kernel
    if (prefill || nchunks <= 1) return 1;
    const int sms = device_sm_count();
    int ns = (2 * sms + Q - 1) / Q;
    if (ns > nchunks) ns = nchunks;
    if (ns > 32) ns = 32;
    if (ns < 1) ns = 1;
    // equalise chunks per split
    const int cps = (nchunks + ns - 1) / ns;
    return (nchunks + cps - 1) / cps;
}

cudaError_t launch_attention_tc(const AttnLaunch& l, cudaStream_t st);

cudaError_t launch_attention(const AttnLaunch& l, cudaStream_t st) {
    cudaError_t e = launch_attention_tc(l, st);
    if (e != cudaSuccess || l.nsplit == 1) return e;
    attn_combine_kernel<<<dim3((unsigned)l.Q, (unsigned)l.H), 128, 0, st>>>(l.partial, l.nsplit,
                                                                          l.H, l.out);
    return cudaGetLastError();
}

}  // namespace csa2
