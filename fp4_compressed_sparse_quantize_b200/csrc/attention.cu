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
// per-split (max, sum) pairs, so the two load latencies overlap. With o_part set, the merge
// is itself left as a partial result: O = sum_s 2^(m_s - M) O_s with (M, L) into ml_part.
__global__ void __launch_bounds__(128) attn_combine_kernel(const CombineArgs a) {
    grid_dep_launch();
    grid_dep_wait();
    const int qrow = blockIdx.x, h = blockIdx.y, H = a.H, nsplit = a.nsplit;
    const float* base = a.o + (int64_t)qrow * a.o_q;
    const int c = threadIdx.x * 4;
    // m of split s at mls[s * ml_s], l at mls[s * ml_s + H]
    const float* mls = a.ml + (int64_t)qrow * a.ml_q + h;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
    float4 v[8];
    auto load8 = [&](int s0) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = s0 + j < nsplit
                       ? ld_dep(reinterpret_cast<const float4*>(base + (s0 + j) * a.o_s +
                                                               (int64_t)h * kDm + c))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    load8(0);
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) M = fmaxf(M, ld_dep(mls + s * a.ml_s));
    const float Mb = (M == -INFINITY) ? 0.f : M;
    for (int s0 = 0; s0 < nsplit; s0 += 8) {
        if (s0 > 0) load8(s0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (s0 + j < nsplit) {
                const float wv = exp2f(ld_dep(mls + (s0 + j) * a.ml_s) - Mb);
                L += wv * ld_dep(mls + (s0 + j) * a.ml_s + H);
                acc.x += wv * v[j].x;
                acc.y += wv * v[j].y;
                acc.z += wv * v[j].z;
                acc.w += wv * v[j].w;
            }
        }
    }
    const int64_t oi = ((int64_t)qrow * H + h) * kDm + c;
    if (a.o_part) {
        *reinterpret_cast<float4*>(a.o_part + oi) = acc;
        if (threadIdx.x == 0) {
            a.ml_part[(int64_t)qrow * 2 * H + h] = M;
            a.ml_part[(int64_t)qrow * 2 * H + H + h] = L;
        }
        return;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    *reinterpret_cast<float4*>(a.out + oi) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

cudaError_t launch_combine(const CombineArgs& a, int Q, cudaStream_t st) {
    return launch_pdl(attn_combine_kernel, dim3((unsigned)Q, (unsigned)a.H), dim3(128), 0, st, a);
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
    // few queries: at most 8 splits whenever the row cap allows, so that a query's splits
    // merge inside one cluster instead of through partials and the merge kernel (1M-context
    // batch 4: 52.5 us against 57.7 us for two layers' attention)
    if (ns > 8 && need <= 8) ns = 8;
    if (ns < 1) ns = 1;
    const int rps = attention_rows_per_split(rows, ns);
    return (rows + rps - 1) / rps;
}

cudaError_t launch_attention_tc(const AttnLaunch& l, cudaStream_t st, bool* merged);
cudaError_t launch_attention_prefill(const AttnLaunch& l, cudaStream_t st);

cudaError_t launch_attention(const AttnLaunch& l, cudaStream_t st) {
    if (l.prefill) return launch_attention_prefill(l, st);
    bool merged = false;
    cudaError_t e = launch_attention_tc(l, st, &merged);
    const bool part = l.o_part != nullptr;
    if (e != cudaSuccess || merged || (l.nsplit == 1 && !part)) return e;
    // split partials in the workspace: O [Q * nsplit][H][512], then (m, l) [Q * nsplit][2][H]
    CombineArgs c;
    c.o = l.partial;
    c.ml = l.partial + (int64_t)l.Q * l.nsplit * l.H * kDm;
    c.o_s = (int64_t)l.H * kDm;
    c.o_q = (int64_t)l.nsplit * c.o_s;
    c.ml_s = 2 * (int64_t)l.H;
    c.ml_q = (int64_t)l.nsplit * c.ml_s;
    c.nsplit = l.nsplit;
    c.H = l.H;
    c.out = l.out;
    c.o_part = l.o_part;
    c.ml_part = l.ml_part;
    return launch_combine(c, l.Q, st);
}

}  // namespace csa2
