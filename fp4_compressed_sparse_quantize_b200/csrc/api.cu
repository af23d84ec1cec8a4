// C ABI of libcsa2: argument validation, workspace layout and kernel dispatch.
// Every entry point validates on the host before launching anything and never aborts.
#include <stdio.h>

#include <algorithm>

#include "csa2.h"
#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

static inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kStatusBytes = 256;
constexpr int kBins = 4096;

// Workspace plan of csa2_index_score_topk. Every buffer is 256-byte aligned.
struct TopkPlan {
    int R, G;
    int64_t row_len;    // scores per row (cap for Full, P_in for Reindex)
    int64_t ld_scores;
    int ccap;
    int64_t nblk;       // pool blocks per row (0: no pool)
    int pccap;
    size_t off_nrow, off_prefix, off_scores, off_hist, off_cnt, off_win, off_cand;
    size_t off_bkey, off_bhist, off_pcnt, off_pwin, off_pcand;
    size_t total;
};

// Query rows sharing one key tile in prefill: two rows of 64 heads fill an N = 128 MMA
// (full tensor rate) and leave the epilogue two groups of warps.
static int choose_group(int T, int H_I, int esz, bool prefill, bool pool) {
    if (!prefill || pool || esz != 1) return 1;
    if (2 * H_I <= 128 && H_I % 16 == 0 && T % 2 == 0) return 2;
    return 1;
}

static TopkPlan plan_topk(int B, int T, int H_I, int esz, int64_t row_len, int K,
                          int pool_blocks, bool prefill, bool own_scores) {
    TopkPlan p;
    memset(&p, 0, sizeof p);
    p.R = B * T;
    p.G = choose_group(T, H_I, esz, prefill, pool_blocks > 0);
    p.row_len = row_len;
    p.ld_scores = row_len;
    const int64_t ccap_max = p.R <= 256 ? 65536 : 8192;
    p.ccap = (int)std::min<int64_t>(std::max<int64_t>(row_len, 1), ccap_max);
    size_t o = kStatusBytes;
    p.off_nrow = o;
    o = align_up(o + sizeof(int32_t) * p.R, 256);
    p.off_prefix = o;
    o = align_up(o + sizeof(int64_t) * (p.R + 1), 256);
    p.off_scores = o;
    if (own_scores) o = align_up(o + sizeof(float) * (size_t)p.R * p.ld_scores, 256);
    p.off_hist = o;
    o = align_up(o + sizeof(uint32_t) * (size_t)p.R * kBins, 256);
    p.off_cnt = o;
    o = align_up(o + sizeof(uint32_t) * 4 * (size_t)p.R, 256);
    p.off_win = o;
    o = align_up(o + sizeof(uint64_t) * (size_t)p.R * K, 256);
    p.off_cand = o;
    o = align_up(o + sizeof(uint64_t) * (size_t)p.R * p.ccap, 256);
    if (pool_blocks > 0) {
        p.nblk = (row_len + CSA2_POOL_BLOCK - 1) / CSA2_POOL_BLOCK;
        p.pccap = (int)std::min<int64_t>(std::max<int64_t>(p.nblk, 1), ccap_max);
        p.off_bkey = o;
        o = align_up(o + sizeof(uint32_t) * (size_t)p.R * p.nblk, 256);
        p.off_bhist = o;
        o = align_up(o + sizeof(uint32_t) * (size_t)p.R * kBins, 256);
        p.off_pcnt = o;
        o = align_up(o + sizeof(uint32_t) * 4 * (size_t)p.R, 256);
        p.off_pwin = o;
        o = align_up(o + sizeof(uint64_t) * (size_t)p.R * pool_blocks, 256);
        p.off_pcand = o;
        o = align_up(o + sizeof(uint64_t) * (size_t)p.R * p.pccap, 256);
    }
    p.total = o;
    return p;
}

// Attention workspace: status word, split partials, and for decode the staging area of the
// dequantised rows (`rows` = K + W per query). Partials (np splits; 0 = none) are needed when
// a decode query's rows are split or the call leaves a partial result.
static size_t attn_partial_bytes(int Q, int H, int np) {
    return np > 0 ? align_up(sizeof(float) * (size_t)Q * np * H * (CSA2_D_MAIN + 2), 256) : 0;
}
static size_t attn_ws_bytes(int Q, int H, int np, int stage_rows) {
    size_t b = kStatusBytes + attn_partial_bytes(Q, H, np);
    if (stage_rows > 0) b += attention_stage_bytes(Q, stage_rows);
    return b;
}

// Upper bound of attention_splits() over every window size the API accepts (W <= 1024):
// its unrounded split count, which grows with the row count.
static int attn_split_bound(int Q, int K) {
    const int sms = device_sm_count();
    const int rows = K + 1024;
    int ns = sms / std::max(Q, 1);
    ns = std::max(ns, (rows + kAttnDecodeRows - 1) / kAttnDecodeRows);
    ns = std::min(ns, (rows + 31) / 32);
    return std::max(1, ns);
}

__global__ void bounded_wait_probe_kernel(int32_t* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        // nobody arrives: the wait must give up and report, not hang
        mbar_wait(&bar, 0, status, limit_ns);
        // complete the phase so the barrier is left consistent
        mbar_arrive(&bar);
    }
}

}  // namespace csa2

using namespace csa2;

static csa2_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

// Per-host-thread benchmark events for the next indexer scan (see csa2_set_stage_events).
static thread_local cudaEvent_t g_stage_ev[2] = {nullptr, nullptr};

extern "C" {

int csa2_version(void) { return 100; }

const char* csa2_status_string(csa2_status_t s) {
    switch (s) {
        case CSA2_OK: return "ok";
        case CSA2_ERR_ARG: return "invalid argument";
        case CSA2_ERR_UNSUPPORTED: return "unsupported geometry or dtype";
        case CSA2_ERR_CUDA: return "CUDA error";
        case CSA2_ERR_WORKSPACE: return "workspace missing or too small";
        case CSA2_ERR_DEVICE: return "device status word is non-zero";
    }
    return "unknown status";
}

csa2_status_t csa2_read_device_status(const void* ws, int32_t* out, void* stream) {
    if (!ws || !out) return CSA2_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return CSA2_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return CSA2_ERR_CUDA;
    *out = v;
    return v ? CSA2_ERR_DEVICE : CSA2_OK;
}

csa2_status_t csa2_set_stage_events(void* ev_start, void* ev_stop) {
    if ((ev_start == nullptr) != (ev_stop == nullptr)) return CSA2_ERR_ARG;
    g_stage_ev[0] = reinterpret_cast<cudaEvent_t>(ev_start);
    g_stage_ev[1] = reinterpret_cast<cudaEvent_t>(ev_stop);
    return CSA2_OK;
}

csa2_status_t csa2_record_event(void* ev, void* stream) {
    if (!ev) return CSA2_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus capst = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &capst) != cudaSuccess) return CSA2_ERR_CUDA;
    const unsigned flags =
        capst == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
    return cuda_status(cudaEventRecordWithFlags(reinterpret_cast<cudaEvent_t>(ev), st, flags));
}

csa2_status_t csa2_reset_device_status(void* ws, void* stream) {
    if (!ws) return CSA2_ERR_ARG;
    return cuda_status(
        cudaMemsetAsync(ws, 0, sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream)));
}

csa2_status_t csa2_debug_bounded_wait(int32_t* status, uint64_t timeout_ns, void* stream) {
    if (!status || timeout_ns == 0 || timeout_ns > 10000000000ull) return CSA2_ERR_ARG;
    bounded_wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status,
                                                                                    timeout_ns);
    return cuda_status(cudaGetLastError());
}

csa2_status_t csa2_quantize_kv(const void* kv, int B, int n_new, int64_t ld_kv,
                               int64_t bstride_kv, const int32_t* dst_off, uint8_t* codes,
                               uint8_t* scales, int64_t cap, int32_t* status, void* stream) {
    if (B < 0 || n_new < 0 || cap < 1) return CSA2_ERR_ARG;
    if ((int64_t)B * n_new == 0) return CSA2_OK;
    if (!kv || !dst_off || !codes || !scales) return CSA2_ERR_ARG;
    if (ld_kv < CSA2_D_MAIN || ld_kv % 8 != 0 || bstride_kv % 8 != 0) return CSA2_ERR_ARG;
    if (bstride_kv < (int64_t)(n_new - 1) * ld_kv + CSA2_D_MAIN && B > 1) return CSA2_ERR_ARG;
    if (!aligned16(kv) || !aligned16(codes) || !aligned16(scales)) return CSA2_ERR_ARG;
    if ((int64_t)B * n_new > (int64_t)1 << 40) return CSA2_ERR_ARG;
    return cuda_status(launch_quantize_kv(kv, B, n_new, ld_kv, bstride_kv, dst_off, codes, scales,
                                          cap, status, reinterpret_cast<cudaStream_t>(stream)));
}

csa2_status_t csa2_compress_kv(int B, int n_new, int r, const void* C, const void* Z, int64_t ld,
                               int64_t bstride, const void* w_proj, csa2_dtype_t key_dtype,
                               const int32_t* dst_off, uint8_t* codes, uint8_t* scales,
                               void* k_I, int64_t cap, void* latent_out, int32_t* status,
                               void* stream) {
    if (B < 0 || n_new < 0 || cap < 1 || r < 1 || r > 64) return CSA2_ERR_ARG;
    if ((int64_t)B * n_new == 0) return CSA2_OK;
    if (key_dtype != CSA2_DTYPE_E4M3 && key_dtype != CSA2_DTYPE_BF16 &&
        key_dtype != CSA2_DTYPE_E4M3_FP4KEY)
        return CSA2_ERR_ARG;
    if (key_dtype == CSA2_DTYPE_E4M3_FP4KEY && (reinterpret_cast<uintptr_t>(k_I) & 31u) != 0)
        return CSA2_ERR_ARG;
    if (!C || !Z || !w_proj || !dst_off || !codes || !scales || !k_I) return CSA2_ERR_ARG;
    if (ld < CSA2_D_MAIN || ld % 8 != 0 || bstride % 8 != 0 || bstride < 0) return CSA2_ERR_ARG;
    if (B > 1 && bstride < ((int64_t)r * n_new - 1) * ld + CSA2_D_MAIN) return CSA2_ERR_ARG;
    if (!aligned16(C) || !aligned16(Z) || !aligned16(w_proj) || !aligned16(codes) ||
        !aligned16(scales) || !aligned16(k_I) || !aligned16(latent_out))
        return CSA2_ERR_ARG;
    if ((int64_t)B * n_new > (int64_t)1 << 31) return CSA2_ERR_ARG;
    CompressLaunch l;
    memset(&l, 0, sizeof l);
    l.B = B;
    l.n_new = n_new;
    l.r = r;
    l.ld = ld;
    l.bstride = bstride;
    l.C = C;
    l.Z = Z;
    l.w_proj = w_proj;
    l.key_bf16 = key_dtype == CSA2_DTYPE_BF16;
    l.key_fp4 = key_dtype == CSA2_DTYPE_E4M3_FP4KEY;
    l.dst_off = dst_off;
    l.codes = codes;
    l.scales = scales;
    l.keys = k_I;
    l.cap = cap;
    l.latent = latent_out;
    l.status = status;
    return cuda_status(launch_compress_kv(l, reinterpret_cast<cudaStream_t>(stream)));
}

csa2_status_t csa2_quantize_keys_fp4(const void* k, int B, int n_new, int64_t ld, int64_t bstride,
                                     const int32_t* dst_off, void* keys, int64_t cap,
                                     int32_t* status, void* stream) {
    if (B < 0 || n_new < 0 || cap < 1) return CSA2_ERR_ARG;
    if ((int64_t)B * n_new == 0) return CSA2_OK;
    if (!k || !dst_off || !keys) return CSA2_ERR_ARG;
    if (ld < CSA2_D_INDEX || ld % 8 != 0 || bstride % 8 != 0 || bstride < 0) return CSA2_ERR_ARG;
    if (B > 1 && bstride < (int64_t)(n_new - 1) * ld + CSA2_D_INDEX) return CSA2_ERR_ARG;
    if (!aligned16(k) || (reinterpret_cast<uintptr_t>(keys) & 31u) != 0) return CSA2_ERR_ARG;
    if ((int64_t)B * n_new > (int64_t)1 << 40 || (int64_t)B * cap > ((int64_t)1 << 40))
        return CSA2_ERR_ARG;
    uint8_t* codes = reinterpret_cast<uint8_t*>(keys);
    float* scales = reinterpret_cast<float*>(codes + (size_t)B * cap * CSA2_FP4KEY_CODE_BYTES);
    return cuda_status(launch_quantize_keys_fp4(k, B, n_new, ld, bstride, dst_off, codes, scales,
                                                cap, status,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

int csa2_sparse_attn_decode_launches(int B, int K, int W) {
    if (B < 1 || K < 0 || W < 0 || W > 1024 || K > 65536) return -1;
    return attention_decode_launches(B, K, W);
}

size_t csa2_workspace_bytes(csa2_op_t op, int B, int T, int H, int64_t cap, int K,
                            int pool_blocks) {
    if (B < 1 || T < 1 || H < 1 || cap < 1 || K < 0) return 0;
    switch (op) {
        case CSA2_OP_INDEX_SCORE_TOPK: {
            if (K < 1) return 0;
            TopkPlan p = plan_topk(B, T, H, 1, cap, K, pool_blocks, T > 1, true);
            TopkPlan p2 = plan_topk(B, T, H, 2, cap, K, pool_blocks, T > 1, true);
            return std::max(p.total, p2.total);
        }
        case CSA2_OP_SPARSE_ATTN_DECODE:
            // sized for windows of up to 1024 rows
            return attn_ws_bytes(B, H, attn_split_bound(B, K), K + 1024);
        case CSA2_OP_SPARSE_ATTN_PREFILL:
            return attn_ws_bytes(B * T, H, 0, 0);
    }
    return 0;
}

csa2_status_t csa2_index_score_topk(csa2_mode_t mode, int B, int T, int H_I,
                                    csa2_dtype_t qk_dtype, const void* q_I, const float* w,
                                    const void* k_I, int64_t cap, const int32_t* n_vis0,
                                    int ratio, const int32_t* q_pos0, int K,
                                    const int32_t* pool_in, int P_in, int32_t* pool_out,
                                    int pool_blocks, int32_t* idx_out, float* scores_out,
                                    void* ws, size_t ws_bytes, void* stream) {
    if (mode != CSA2_MODE_FULL && mode != CSA2_MODE_REINDEX && mode != CSA2_MODE_REUSE)
        return CSA2_ERR_ARG;
    if (B < 1 || T < 1 || cap < 1 || K < 1) return CSA2_ERR_ARG;
    if ((int64_t)B * T > 65535) return CSA2_ERR_UNSUPPORTED;
    if (K > 2048) return CSA2_ERR_UNSUPPORTED;
    if (!idx_out) return CSA2_ERR_ARG;
    if (mode == CSA2_MODE_REUSE) {
        // Reuse layers skip indexing: the earlier layer's indices are used as they are.
        if (pool_in || pool_out) return CSA2_ERR_ARG;
        return CSA2_OK;
    }
    if (qk_dtype != CSA2_DTYPE_BF16 && qk_dtype != CSA2_DTYPE_E4M3 &&
        qk_dtype != CSA2_DTYPE_E4M3_FP4KEY)
        return CSA2_ERR_ARG;
    const bool key_fp4 = qk_dtype == CSA2_DTYPE_E4M3_FP4KEY;
    if (key_fp4 && (reinterpret_cast<uintptr_t>(k_I) & 31u) != 0) return CSA2_ERR_ARG;
    if (H_I < 1 || H_I > 128) return CSA2_ERR_UNSUPPORTED;
    if (!q_I || !w || !k_I) return CSA2_ERR_ARG;
    if (!aligned16(q_I) || !aligned16(k_I) || !aligned16(w)) return CSA2_ERR_ARG;
    const bool prefill = q_pos0 != nullptr;
    if (!prefill && (T != 1 || !n_vis0)) return CSA2_ERR_ARG;
    if (prefill && ratio < 1) return CSA2_ERR_ARG;
    if (cap > (int64_t)1 << 30 || (int64_t)B * cap > ((int64_t)1 << 31) - 1)
        return CSA2_ERR_UNSUPPORTED;
    const int esz = qk_dtype == CSA2_DTYPE_BF16 ? 2 : 1;
    if (mode == CSA2_MODE_FULL) {
        if (pool_in) return CSA2_ERR_ARG;
        if (pool_out && (pool_blocks < 1 || pool_blocks > 2048)) return CSA2_ERR_ARG;
        if (!pool_out) pool_blocks = 0;
    } else {  // REINDEX
        if (!pool_in || P_in < 1 || pool_out) return CSA2_ERR_ARG;
        pool_blocks = 0;
    }
    if (scores_out && !aligned16(scores_out)) return CSA2_ERR_ARG;
    const bool reindex = mode == CSA2_MODE_REINDEX;
    const int64_t row_len = reindex ? P_in : cap;
    TopkPlan pl = plan_topk(B, T, H_I, esz, row_len, K, pool_blocks, prefill, scores_out == nullptr);
    if (!ws) return CSA2_ERR_WORKSPACE;
    if (ws_bytes < pl.total || !aligned16(ws)) return CSA2_ERR_WORKSPACE;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* wb = reinterpret_cast<uint8_t*>(ws);
    int32_t* status = reinterpret_cast<int32_t*>(wb);
    int32_t* n_row = reinterpret_cast<int32_t*>(wb + pl.off_nrow);
    int64_t* prefix = reinterpret_cast<int64_t*>(wb + pl.off_prefix);
    float* scores = scores_out ? scores_out : reinterpret_cast<float*>(wb + pl.off_scores);
    uint32_t* hist = reinterpret_cast<uint32_t*>(wb + pl.off_hist);
    uint32_t* cnt = reinterpret_cast<uint32_t*>(wb + pl.off_cnt);
    const int R = pl.R;

    cudaError_t e;
    // histograms and counters start at zero: cleared by the prep kernel
    ZeroList zl;
    memset(&zl, 0, sizeof zl);
    zl.p[0] = reinterpret_cast<uint4*>(hist);
    zl.n16[0] = (int64_t)R * kBins * 4 / 16;
    zl.p[1] = reinterpret_cast<uint4*>(cnt);
    zl.n16[1] = (int64_t)R * 4 * 4 / 16;
    if (pool_blocks > 0) {
        zl.p[2] = reinterpret_cast<uint4*>(wb + pl.off_bhist);
        zl.n16[2] = (int64_t)R * kBins * 4 / 16;
        zl.p[3] = reinterpret_cast<uint4*>(wb + pl.off_pcnt);
        zl.n16[3] = (int64_t)R * 4 * 4 / 16;
    }
    e = launch_prep_rows(R, T, pl.G, n_vis0, q_pos0, ratio, cap, reindex ? P_in : 0,
                         scan_tile_rows(pl.G, reindex, esz), n_row, prefix, status, zl, st);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;

    ScanLaunch sl;
    memset(&sl, 0, sizeof sl);
    sl.B = B;
    sl.T = T;
    sl.rows = R;
    sl.G = pl.G;
    sl.H_I = H_I;
    sl.esz = esz;
    sl.cap = cap;
    sl.q = q_I;
    sl.k = k_I;
    sl.w = w;
    sl.n_row = n_row;
    sl.prefix = prefix;
    sl.scores = scores;
    sl.ld_scores = pl.ld_scores;
    sl.hist = hist;
    sl.pool_build = pool_blocks > 0;
    sl.bkey = pool_blocks > 0 ? reinterpret_cast<uint32_t*>(wb + pl.off_bkey) : nullptr;
    sl.ld_bkey = pl.nblk;
    sl.bhist = pool_blocks > 0 ? reinterpret_cast<uint32_t*>(wb + pl.off_bhist) : nullptr;
    sl.gather = reindex;
    sl.pool = pool_in;
    sl.P = P_in;
    sl.status = status;
    sl.key_fp4 = key_fp4;
    sl.kscale = key_fp4 ? reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(k_I) +
                                                         (size_t)B * cap * CSA2_FP4KEY_CODE_BYTES)
                        : nullptr;
    const cudaEvent_t ev0 = g_stage_ev[0], ev1 = g_stage_ev[1];
    g_stage_ev[0] = g_stage_ev[1] = nullptr;
    // inside a stream capture the events become external record nodes (usable for timing)
    cudaStreamCaptureStatus capst = cudaStreamCaptureStatusNone;
    if ((ev0 || ev1) && cudaStreamIsCapturing(st, &capst) != cudaSuccess) return CSA2_ERR_CUDA;
    const unsigned ev_flags =
        capst == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
    if (ev0 && cudaEventRecordWithFlags(ev0, st, ev_flags) != cudaSuccess) return CSA2_ERR_CUDA;
    e = launch_index_scan(sl, st);
    if (ev1 && e == cudaSuccess) e = cudaEventRecordWithFlags(ev1, st, ev_flags);
    if (e == cudaErrorNotSupported) return CSA2_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return CSA2_ERR_CUDA;

    TopkLaunch tl;
    memset(&tl, 0, sizeof tl);
    tl.R = R;
    tl.K = K;
    tl.scores = scores;
    tl.ld = pl.ld_scores;
    tl.max_n = row_len;
    tl.n_row = n_row;
    tl.n_row_div = 1;
    tl.ids = reindex ? pool_in : nullptr;
    tl.id_limit = reindex ? n_row : nullptr;
    tl.hist = hist;
    tl.out = idx_out;
    tl.counters = cnt;
    tl.winners = reinterpret_cast<uint64_t*>(wb + pl.off_win);
    tl.cands = reinterpret_cast<uint64_t*>(wb + pl.off_cand);
    tl.ccap = pl.ccap;
    tl.id_bound = cap;
    tl.status = status;
    e = launch_topk(tl, st);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;

    if (pool_blocks > 0) {
        TopkLaunch pt;
        memset(&pt, 0, sizeof pt);
        pt.R = R;
        pt.K = pool_blocks;
        pt.keys = sl.bkey;
        pt.ld = pl.nblk;
        pt.max_n = pl.nblk;
        pt.n_row = n_row;
        pt.n_row_div = CSA2_POOL_BLOCK;
        pt.hist = sl.bhist;
        pt.out = pool_out;
        pt.expand8 = true;
        pt.expand_limit = n_row;
        pt.counters = reinterpret_cast<uint32_t*>(wb + pl.off_pcnt);
        pt.winners = reinterpret_cast<uint64_t*>(wb + pl.off_pwin);
        pt.cands = reinterpret_cast<uint64_t*>(wb + pl.off_pcand);
        pt.ccap = pl.pccap;
        pt.id_bound = pl.nblk;
        pt.status = status;
        e = launch_topk(pt, st);
        if (e != cudaSuccess) return CSA2_ERR_CUDA;
    }
    return CSA2_OK;
}

static csa2_status_t attn_common(bool prefill, int B, int T, int H, const void* q,
                                 const uint8_t* codes, const uint8_t* scales, int64_t cap,
                                 const int32_t* idx, int K, const uint8_t* swa, int W,
                                 const int32_t* swa_valid, const int32_t* q_pos0, float scale,
                                 float* out, void* ws, size_t ws_bytes, void* stream,
                                 float* o_part = nullptr, float* ml_part = nullptr) {
    if (B < 1 || T < 1 || cap < 1 || K < 0 || W < 0) return CSA2_ERR_ARG;
    if (H < 1) return CSA2_ERR_ARG;
    if (H > 64 || W > 1024 || K > 65536) return CSA2_ERR_UNSUPPORTED;
    const bool part = o_part != nullptr;
    if (part) {
        if (!ml_part || !aligned16(o_part) || prefill) return CSA2_ERR_ARG;
        out = o_part;   // only checked for alignment below; the result goes to o_part/ml_part
    }
    if (!q || !out || !ws) return !ws ? CSA2_ERR_WORKSPACE : CSA2_ERR_ARG;
    if (K > 0 && (!codes || !scales || !idx)) return CSA2_ERR_ARG;
    if (W > 0 && !swa) return CSA2_ERR_ARG;
    if (!(scale == scale)) return CSA2_ERR_ARG;
    if (!aligned16(q) || !aligned16(out) || !aligned16(ws) || (codes && !aligned16(codes)) ||
        (scales && !aligned16(scales)) || (swa && !aligned16(swa)))
        return CSA2_ERR_ARG;
    const int64_t Q = (int64_t)B * T;
    if (Q > 2147483647) return CSA2_ERR_UNSUPPORTED;
    const int nsplit = attention_splits((int)Q, K, W, prefill);
    const int stage_rows = prefill ? 0 : K + W;
    const int np = (nsplit > 1 || part) ? nsplit : 0;   // partial splits in the workspace
    if (ws_bytes < attn_ws_bytes((int)Q, H, np, stage_rows)) return CSA2_ERR_WORKSPACE;
    AttnLaunch l;
    memset(&l, 0, sizeof l);
    l.Q = (int)Q;
    l.T = T;
    l.H = H;
    l.q = q;
    l.codes = codes;
    l.scales = scales;
    l.cap = cap;
    l.idx = idx;
    l.K = K;
    l.swa = swa;
    l.W = W;
    l.swa_valid = swa_valid;
    l.q_pos0 = q_pos0;
    l.prefill = prefill;
    l.scale = scale;
    l.out = part ? nullptr : out;
    l.o_part = part ? o_part : nullptr;
    l.ml_part = part ? ml_part : nullptr;
    l.nsplit = nsplit;
    l.partial = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + kStatusBytes);
    l.stage = stage_rows > 0 ? reinterpret_cast<uint8_t*>(ws) + kStatusBytes +
                                   attn_partial_bytes((int)Q, H, np)
                             : nullptr;
    l.status = reinterpret_cast<int32_t*>(ws);
    return cuda_status(launch_attention(l, reinterpret_cast<cudaStream_t>(stream)));
}

csa2_status_t csa2_sparse_attn_decode(csa2_mode_t mode, int B, int H, const void* q,
                                      const uint8_t* codes, const uint8_t* scales,
                                      int64_t cap, const int32_t* idx, int K,
                                      const uint8_t* swa, int W, const int32_t* swa_valid,
                                      float scale, float* out, void* ws, size_t ws_bytes,
                                      void* stream) {
    if (mode != CSA2_MODE_FULL && mode != CSA2_MODE_REINDEX && mode != CSA2_MODE_REUSE)
        return CSA2_ERR_ARG;
    return attn_common(false, B, 1, H, q, codes, scales, cap, idx, K, swa, W, swa_valid,
                       nullptr, scale, out, ws, ws_bytes, stream);
}

csa2_status_t csa2_sparse_attn_prefill(int B, int T, int H, const void* q,
                                       const uint8_t* codes, const uint8_t* scales,
                                       int64_t cap, const int32_t* idx, int K,
                                       const uint8_t* swa, int W, const int32_t* q_pos0,
                                       float scale, float* out, void* ws, size_t ws_bytes,
                                       void* stream) {
    return attn_common(true, B, T, H, q, codes, scales, cap, idx, K, swa, W, nullptr, q_pos0,
                       scale, out, ws, ws_bytes, stream);
}

csa2_status_t csa2_sparse_attn_decode_partial(csa2_mode_t mode, int B, int H, const void* q,
                                              const uint8_t* codes, const uint8_t* scales,
                                              int64_t cap, const int32_t* idx, int K,
                                              const uint8_t* swa, int W,
                                              const int32_t* swa_valid, float scale,
                                              float* o_part, float* ml_part, void* ws,
                                              size_t ws_bytes, void* stream) {
    if (mode != CSA2_MODE_FULL && mode != CSA2_MODE_REINDEX && mode != CSA2_MODE_REUSE)
        return CSA2_ERR_ARG;
    if (!o_part || !ml_part) return CSA2_ERR_ARG;
    return attn_common(false, B, 1, H, q, codes, scales, cap, idx, K, swa, W, swa_valid,
                       nullptr, scale, nullptr, ws, ws_bytes, stream, o_part, ml_part);
}

csa2_status_t csa2_attn_merge_partials(int B, int H, int G, const float* o_parts,
                                       const float* ml_parts, float* out, void* stream) {
    if (B < 1 || H < 1 || H > 64 || G < 1 || !o_parts || !ml_parts || !out) return CSA2_ERR_ARG;
    if (!aligned16(o_parts) || !aligned16(out)) return CSA2_ERR_ARG;
    CombineArgs c;
    c.o = o_parts;
    c.ml = ml_parts;
    c.o_q = (int64_t)H * CSA2_D_MAIN;
    c.o_s = (int64_t)B * c.o_q;
    c.ml_q = 2 * (int64_t)H;
    c.ml_s = (int64_t)B * c.ml_q;
    c.nsplit = G;
    c.H = H;
    c.out = out;
    c.o_part = nullptr;
    c.ml_part = nullptr;
    return cuda_status(launch_combine(c, B, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
