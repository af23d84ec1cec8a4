// Internal launch interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <utility>

namespace csa2 {

// The driver's tensor-map encoder, looked up once per process (null if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Launch with programmatic stream serialisation (see grid_dep_wait / grid_dep_launch).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct ScanLaunch {
    int B, T, rows, G, H_I, esz;
    int64_t cap;
    const void* q;          // [rows][H_I][128]
    const void* k;          // [B][cap][128]
    const float* w;         // [rows][H_I]
    const int32_t* n_row;   // [rows]
    const int64_t* prefix;  // [rows/G + 1]
    float* scores;
    int64_t ld_scores;
    uint32_t* hist;
    bool pool_build;
    uint32_t* bkey;
    int64_t ld_bkey;
    uint32_t* bhist;
    bool gather;
    const int32_t* pool;
    int P;
    int32_t* status;
    bool key_fp4;           // compact keys: E2M1 codes (TMA-unpacked) + fp32 scale per key
    const float* kscale;    // [B][cap] scales of compact keys
};

cudaError_t launch_quantize_kv(const void* kv, int B, int n_new, int64_t ld_kv,
                               int64_t bstride_kv, const int32_t* dst_off, uint8_t* codes,
                               uint8_t* scales, int64_t cap, int32_t* status,
                               cudaStream_t stream);

cudaError_t launch_quantize_keys_fp4(const void* k, int B, int n_new, int64_t ld,
                                     int64_t bstride, const int32_t* dst_off, uint8_t* codes,
                                     float* scales, int64_t cap, int32_t* status,
                                     cudaStream_t stream);

// Compressor + indexer-K projection + FP4 write (csa2_compress_kv).
struct CompressLaunch {
    int B, n_new, r;
    int64_t ld, bstride;
    const void* C;
    const void* Z;
    const void* w_proj;
    int key_bf16;
    int key_fp4;            // compact 68-byte keys (two-plane buffer in keys)
    const int32_t* dst_off;
    uint8_t* codes;
    uint8_t* scales;
    void* keys;
    int64_t cap;
    void* latent;
    int32_t* status;
};

cudaError_t launch_compress_kv(const CompressLaunch& l, cudaStream_t st);

// Up to four workspace buffers that the prep kernel clears (16-byte units).
struct ZeroList {
    uint4* p[4];
    int64_t n16[4];
};

cudaError_t launch_prep_rows(int rows, int T, int G, const int32_t* n_vis0,
                             const int32_t* q_pos0, int ratio, int64_t cap, int P_gather,
                             int tile_rows, int32_t* n_row, int64_t* prefix, int32_t* status,
                             const ZeroList& zero, cudaStream_t st);

// keys per scan tile for a query-group size and mode
int scan_tile_rows(int G, bool gather, int esz);

cudaError_t launch_index_scan(const ScanLaunch& a, cudaStream_t st);

// Exact Top-K over rows of fp32 scores or u32 keys.
struct TopkLaunch {
    int R;                   // rows
    int K;                   // picks per row
    const float* scores;     // [R][ld] or null (then keys)
    const uint32_t* keys;    // [R][ld] order-preserving keys
    int64_t ld;
    int64_t max_n;           // largest row length (grid sizing)
    const int32_t* n_row;    // [R] candidate count per row (prefix [0, n))
    int n_row_div;           // n_row[r] is divided by this (rounded up): 8 for pool blocks
    const int32_t* ids;      // [R][ld] ids (gather mode), or null: id = position
    const int32_t* id_limit; // [R] ids must be < id_limit[r] (gather mode)
    const uint32_t* hist;    // [R][4096] histogram of key >> 20
    int32_t* out;            // [R][K] (or [R][K*8] with expand8)
    bool expand8;            // output = 8 positions per picked block, < n_row[r]
    const int32_t* expand_limit; // [R] visible positions for expand8
    uint32_t* counters;      // [R][4]
    uint64_t* winners;       // [R][K]
    uint64_t* cands;         // [R][ccap]
    int ccap;
    int64_t id_bound;        // every id is below this (0: unknown)
    int32_t* status;
};

cudaError_t launch_topk(const TopkLaunch& a, cudaStream_t st);

struct AttnLaunch {
    int Q;                   // query rows (B for decode, B*T for prefill)
    int T;                   // tokens per sequence (1 for decode)
    int H;
    const void* q;           // bf16 [Q][H][512]
    const uint8_t* codes;    // [B][cap][256]
    const uint8_t* scales;   // [B][cap][32]
    int64_t cap;
    const int32_t* idx;      // [Q][K]
    int K;
    const uint8_t* swa;      // decode [B][W][512]; prefill [B][W-1+T][512]
    int W;
    const int32_t* swa_valid;  // decode, nullable
    const int32_t* q_pos0;     // prefill, nullable
    bool prefill;
    float scale;
    float* out;              // [Q][H][512]
    float* partial;          // workspace for split rows
    float* o_part;           // non-null: leave the result as a partial (unnormalised O [Q][H][512]
    float* ml_part;          //   and (M, L) [Q][2][H], base-2 logits) instead of writing out
    int nsplit;
    void* stage;             // decode staging area (attention_stage_bytes), or null
    int32_t* status;
};

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t st);
// Merge of partial attention results: split s of row q at o + s*o_s + q*o_q ([H][512]) and
// (m, l) at ml + s*ml_s + q*ml_q ([2][H]); into out [Q][H][512], or (o_part, ml_part) when set.
struct CombineArgs {
    const float* o;
    const float* ml;
    int64_t o_s, o_q, ml_s, ml_q;
    int nsplit, H;
    float* out;
    float* o_part;
    float* ml_part;
};
cudaError_t launch_combine(const CombineArgs& a, int Q, cudaStream_t st);
size_t attention_stage_bytes(int Q, int rows);
// Decode splits the K + W rows of a query into equal runs of at most kAttnDecodeRows rows
// (a multiple of 32), as many as fill one wave of CTAs; prefill never splits.
constexpr int kAttnDecodeRows = 160;
int attention_splits(int Q, int K, int W, bool prefill);
// kernels one decode attention call launches for Q queries (stage, attention, merge or not)
int attention_decode_launches(int Q, int K, int W);
int attention_rows_per_split(int rows, int nsplit);

int device_sm_count();

}  // namespace csa2
