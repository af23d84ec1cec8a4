// Split bookkeeping of the sparse attention: how many CTAs share the rows of one decode
// query, and the merge of their partial results.
//
// "DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale LLM Serving", Compressed Sparse
// Attention 2 (CSA2): one softmax over the selected compressed entries and the window rows.
// When the rows of a query are split over several CTAs, each CTA leaves its unnormalised
// output O_s with its per-head maximum m_s and sum l_s (base-2 logits); merging them is the
// usual exact log-sum-exp combination.
//
// Partial layout (workspace): O [Q * nsplit][H][512] fp32, then (m, l) [Q * nsplit][2][H].
#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

constexpr int kDm = 512;      // latent channels

// Merge the per-split partial results of one (query row, head): out = sum_s 2^(m_s - M)
// O_s / sum_s 2^(m_s - M) l_s (base-2 logits). One CTA per (row, head), 4 channels/thread.
// Every thread issues its partial-output loads (eight splits at a time) before it reads the
// per-split (max, sum) pairs, so the two load latencies overlap.
__global__ void __launch_bounds__(128) attn_combine_kernel(const float* __restrict__ partial,
                                                           int nsplit, int H,
                                                           float* __restrict__ out) {
    grid_dep_launch();
    grid_dep_wait();
    const int qrow = blockIdx.x, h = blockIdx.y;
    const int64_t stride = (int64_t)H * kDm;            // between splits of one row
    const float* base = partial + (int64_t)qrow * nsplit * stride;
    const int c = threadIdx.x * 4;
    // m of split s at mls[s * mstride], l at mls[s * mstride + H]
    const int64_t mstride = 2 * (int64_t)H;
    const float* mls = partial + (int64_t)gridDim.x * nsplit * stride +
                       (int64_t)qrow * nsplit * mstride + h;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
    float4 v[8];
    auto load8 = [&](int s0) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = s0 + j < nsplit
                       ? __ldg(reinterpret_cast<const float4*>(base + (s0 + j) * stride +
                                                               (int64_t)h * kDm + c))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    load8(0);
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) M = fmaxf(M, __ldg(mls + s * mstride));
    const float Mb = (M == -INFINITY) ? 0.f : M;
    for (int s0 = 0; s0 < nsplit; s0 += 8) {
        if (s0 > 0) load8(s0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (s0 + j < nsplit) {
                const float wv = exp2f(__ldg(mls + (s0 + j) * mstride) - Mb);
                L += wv * __ldg(mls + (s0 + j) * mstride + H);
                acc.x += wv * v[j].x;
                acc.y += wv * v[j].y;
                acc.z += wv * v[j].z;
                acc.w += wv * v[j].w;
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    *reinterpret_cast<float4*>(out + ((int64_t)qrow * H + h) * kDm + c) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

int attention_rows_per_split(int rows, int nsplit) {
    const int r = (rows + nsplit - 1) / nsplit;
    return (r + 31) & ~31;
}

int attention_splits(int Q, int K, int W, bool prefill) {
    const int rows = K + W;
    if (prefill || rows <= 0) return 1;
    const int sms = device_sm_count();
    const int need = (rows + kAttnDecodeRows - 1) / kAttnDecodeRows;   // rows per split cap
    const int most = (rows + 31) / 32;                                // 32 rows at least
    int ns = sms / (Q > 0 ? Q : 1);                                   // one wave of CTAs
    if (ns < need) ns = need;
    if (ns > most) ns = most;
    if (ns < 1) ns = 1;
    const int rps = attention_rows_per_split(rows, ns);
    return (rows + rps - 1) / rps;
}

cudaError_t launch_attention_tc(const AttnLaunch& l, cudaStream_t st, bool* merged);

cudaError_t launch_attention(const AttnLaunch& l, cudaStream_t st) {
    bool merged = false;
    cudaError_t e = launch_attention_tc(l, st, &merged);
    if (e != cudaSuccess || l.nsplit == 1 || merged) return e;
    return launch_pdl(attn_combine_kernel, dim3((unsigned)l.Q, (unsigned)l.H), dim3(128), 0, st,
                      (const float*)l.partial, l.nsplit, l.H, l.out);
}

}  // namespace csa2
