/*
 * csa2.h — C ABI of libcsa2: CSA2 compressed sparse attention over an FP4 main-KV cache,
 * hand-written for NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources are web pages about the DeepSeek-V4.1-Flash
 * report; each entry point cites the passage that defines its operation):
 *   [AIS] "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (ai.info
 *         AI summary): "Main Findings" (FP4 format choice), "Methodology in Plain
 *         English" (CSA2 modes, Hierarchical Sparse Indexer, indexer K).
 *   [TDG] "DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale LLM Serving":
 *         "Compressed Sparse Attention 2 (CSA2)", "Quantization and Memory
 *         Management", "Causal Encoder-Decoder" (128-token SWA in every layer).
 *   [TLB] "DeepSeek V4.1 Flash: smaller KV cache, same post-training": "How did
 *         DeepSeek V4.1 reduce the KV cache?" (three modes, FP4 KV cache, SWA).
 *
 * Conventions for every entry point
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise. The caller
 *     owns all memory; the library never allocates device memory. Scratch space comes
 *     from a caller-supplied workspace sized by csa2_workspace_bytes().
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream) and returns before the device work finishes.
 *   - Row-major layouts, last dimension contiguous. Pointers to codes, scales, keys,
 *     queries, window rows and outputs must be 16-byte aligned.
 *   - Argument errors are reported as CSA2_ERR_ARG / CSA2_ERR_UNSUPPORTED /
 *     CSA2_ERR_WORKSPACE before anything is launched. Launch failures return
 *     CSA2_ERR_CUDA. Errors found on the device (an index outside its buffer, a
 *     visible count above the capacity, a bounded wait that ran out) never fault: the
 *     offending item is skipped and a bit is OR-ed into the device status word that
 *     lives in the first 4 bytes of the workspace; read it with
 *     csa2_read_device_status(). The status word is sticky until
 *     csa2_reset_device_status() clears it. A workspace must be zero-filled (or reset)
 *     once before first use.
 *   - Calls on different streams with different workspaces may run concurrently; calls
 *     that share a workspace must be ordered (same stream). The library's only global
 *     state is: lookups of immutable facts, made once and shared by all threads under a
 *     lock or as a benign race of identical values (the driver's tensor-map encoder entry
 *     point; per decode-attention shape, whether its split clusters fit one wave of the
 *     current device); the per-host-thread benchmark events of csa2_set_stage_events();
 *     and the fixed device array of csa2_index_score_topk_noalloc() (see there).
 *   - Fixed geometry: main-KV latent D = 512 channels, indexer dimension 128, candidate
 *     pool blocks of 8 positions. Other sizes return CSA2_ERR_UNSUPPORTED.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum csa2_status {
    CSA2_OK = 0,
    CSA2_ERR_ARG = 1,          /* null pointer, bad size, misalignment, mode/pool mismatch */
    CSA2_ERR_UNSUPPORTED = 2,  /* geometry or dtype not built */
    CSA2_ERR_CUDA = 3,         /* a CUDA call or kernel launch failed */
    CSA2_ERR_WORKSPACE = 4,    /* workspace missing or smaller than csa2_workspace_bytes() */
    CSA2_ERR_DEVICE = 5        /* csa2_read_device_status() found a non-zero status word */
} csa2_status_t;

/* Per-layer CSA2 mode [AIS Methodology], [TDG CSA2], [TLB three modes]. */
typedef enum csa2_mode {
    CSA2_MODE_FULL = 0,    /* score every visible entry, pick fresh Top-K (and the pool) */
    CSA2_MODE_REINDEX = 1, /* rescore only the candidate pool of the latest Full layer   */
    CSA2_MODE_REUSE = 2    /* no indexer work: the earlier layer's indices are reused     */
} csa2_mode_t;

/* Storage type of the indexer query and key. */
typedef enum csa2_dtype {
    CSA2_DTYPE_BF16 = 0,
    CSA2_DTYPE_E4M3 = 1,   /* OCP FP8 E4M3 ("fn": no infinities, max 448) */
    /* E4M3 query with compact 68-byte keys (csa2_quantize_keys_fp4): the key buffer holds
     * two planes, E2M1 codes [B][cap][64] and then fp32 scales [B][cap] starting at byte
     * B*cap*64; its start must be 32-byte aligned. Full and Reindex modes. */
    CSA2_DTYPE_E4M3_FP4KEY = 2
} csa2_dtype_t;

/* Operations that need a workspace. */
typedef enum csa2_op {
    CSA2_OP_INDEX_SCORE_TOPK = 0,
    CSA2_OP_SPARSE_ATTN_DECODE = 1,
    CSA2_OP_SPARSE_ATTN_PREFILL = 2
} csa2_op_t;

/* Bits of the device status word. */
#define CSA2_DEV_BAD_INDEX   0x1  /* an index / offset pointed outside its buffer       */
#define CSA2_DEV_BAD_COUNT   0x2  /* a visible count was negative or above capacity     */
#define CSA2_DEV_TIMEOUT     0x4  /* a bounded wait inside a kernel gave up             */

#define CSA2_D_MAIN 512           /* main-KV latent channels                            */
#define CSA2_D_INDEX 128          /* indexer query / key channels                       */
#define CSA2_SCALE_GROUP 16       /* channels per E4M3 scale                            */
#define CSA2_ENTRY_CODE_BYTES 256 /* packed E2M1 bytes per main-KV entry (512 / 2)      */
#define CSA2_ENTRY_SCALE_BYTES 32 /* E4M3 scale bytes per main-KV entry (512 / 16)      */
#define CSA2_POOL_BLOCK 8         /* positions per candidate-pool block                 */
#define CSA2_FP4KEY_CODE_BYTES 64 /* E2M1 code bytes of a compact indexer key (128 / 2)  */

/*
 * csa2_quantize_kv — FP4 quantize-on-write of new main-KV entries.
 * [AIS Main Findings, FP4 format choice], [TDG Quantization and Memory Management],
 * [TLB FP4 KV cache]: E2M1 elements with one E4M3 scale per 16 channels (NVFP4 without
 * its second-level global scale). Per 16-channel block: amax = max|x|; scale =
 * E4M3(amax / 6) rounded to nearest-even and saturated at 448; each element code =
 * E2M1(|x| / scale) rounded to nearest-even, saturated at 6, with the sign bit of x
 * (a zero scale gives zero magnitudes). Quotients are IEEE-rounded fp32 divisions.
 *
 *   kv       bf16 [B][n_new][512]: element (b,i,c) at kv[b*bstride_kv + i*ld_kv + c]
 *            (strides in elements; ld_kv >= 512, multiples of 8). Must be finite:
 *            non-finite input gives unspecified codes.
 *   dst_off  int32 [B]: entry index where sequence b's first new entry is written.
 *   codes    uint8 [B][cap][256]: channel 2k in the low nibble of byte k.
 *   scales   uint8 [B][cap][32]: E4M3 bit patterns, one per 16 channels.
 * Entries outside [0, cap) are skipped and set CSA2_DEV_BAD_INDEX; with no workspace
 * argument that bit goes to `status` (nullable int32 device word).
 */
CSA2_API csa2_status_t csa2_quantize_kv(const void* kv, int B, int n_new, int64_t ld_kv,
                               int64_t bstride_kv, const int32_t* dst_off, uint8_t* codes,
                               uint8_t* scales, int64_t cap, int32_t* status, void* stream);

/*
 * csa2_compress_kv — KV compressor and indexer-K projection, fused with FP4
 * quantize-on-write: n_new new entries per sequence from r*n_new source tokens.
 * [AIS Methodology in Plain English]: no overlapping source entries and no absolute
 * positional embedding in the compressor; the indexer K is a projection of the main KV
 * entries. [TLB How did DeepSeek V4.1 reduce the KV cache?] names the compressed entries
 * (C_l) and compression weights (Z_l); the equation itself is lost, so this is a reading:
 *   entry j pools tokens r*j .. r*j+r-1; per channel d
 *     x[j][d] = bf16_RNE( sum_t softmax_t(Z[t][d]) * C[t][d] )   (fp32 arithmetic)
 *   codes, scales = csa2_quantize_kv's FP4 encoding of x[j], at entry dst_off[b] + j;
 *   k_I[j][e] = sum_d w_proj[e][d] * x[j][d]  (tensor cores, fp32 accumulation),
 *     stored as E4M3 (RNE, saturating at 448) or bf16 (RNE).
 *
 *   C, Z     bf16 latents and compression logits of the source tokens: element
 *            (b, token i, channel c) at C[b*bstride + i*ld + c] (same for Z; token i of
 *            sequence b is source token r*j + t of entry j). ld >= 512, ld and bstride
 *            multiples of 8; 16-byte aligned; finite values.
 *   r        tokens per entry, 1..64.
 *   w_proj   bf16 [128][512], row e = the weights of key channel e; 16-byte aligned.
 *   key_dtype  CSA2_DTYPE_E4M3 or CSA2_DTYPE_BF16: the storage type of k_I; or
 *            CSA2_DTYPE_E4M3_FP4KEY: k_I is the two-plane compact-key buffer and each key
 *            is csa2_quantize_keys_fp4's encoding of the bf16-rounded projection.
 *   dst_off  int32 [B]: entry index of sequence b's first new entry.
 *   codes, scales  the FP4 cache as in csa2_quantize_kv.
 *   k_I      [B][cap][128] in key_dtype: the indexer-key cache (compact keys: 32-byte
 *            aligned two-plane buffer).
 *   latent_out  nullable bf16 [B][n_new][512]: the pooled bf16 latents x.
 *   status   nullable int32 device word: CSA2_DEV_BAD_INDEX for an entry outside
 *            [0, cap) (that entry is skipped), CSA2_DEV_TIMEOUT for a bounded wait that
 *            gave up.
 * The caller owns every buffer; nothing is allocated. Host-side validation returns
 * CSA2_ERR_ARG before anything is launched.
 */
CSA2_API csa2_status_t csa2_compress_kv(int B, int n_new, int r, const void* C, const void* Z,
                                        int64_t ld, int64_t bstride, const void* w_proj,
                                        csa2_dtype_t key_dtype, const int32_t* dst_off,
                                        uint8_t* codes, uint8_t* scales, void* k_I,
                                        int64_t cap, void* latent_out, int32_t* status,
                                        void* stream);

/*
 * csa2_quantize_keys_fp4 — compact 68-byte indexer keys.
 * [AIS Main Findings], [TLB How is DeepSeek V4.1 Flash different] (Figure 1): 890 bytes of
 * global KV per token; with 2.5 stored entry-sets per token and 288-byte FP4 main entries
 * that leaves 68 bytes per indexer key. The pages give no key format; reading: E2M1 codes
 * of the 128 channels (64 bytes, channel 2k in the low nibble of byte k) times one fp32
 * scale per key. Decisions in IEEE fp32: s = amax / 6; magnitude = E2M1(|x| / s) rounded
 * to nearest-even and saturated at 6, sign copied from x; s == 0 gives zero magnitudes.
 *
 *   k        bf16 [B][n_new][128]: element (b,i,c) at k[b*bstride + i*ld + c]; ld >= 128,
 *            ld and bstride multiples of 8; 16-byte aligned; finite values.
 *   dst_off  int32 [B]: entry index of sequence b's first new key.
 *   keys     the two-plane compact key buffer of CSA2_DTYPE_E4M3_FP4KEY (codes
 *            [B][cap][64], then fp32 scales [B][cap] at byte B*cap*64); 32-byte aligned.
 *   status   nullable int32 device word: CSA2_DEV_BAD_INDEX for a key outside [0, cap).
 */
CSA2_API csa2_status_t csa2_quantize_keys_fp4(const void* k, int B, int n_new, int64_t ld,
                                              int64_t bstride, const int32_t* dst_off,
                                              void* keys, int64_t cap, int32_t* status,
                                              void* stream);

/*
 * csa2_index_score_topk — indexer scoring + exact Top-K selection, per layer mode.
 * [AIS Methodology]: each layer has its own indexer query; Full layers score, Reindex
 * layers rescore the latest Full layer's keys, Reuse layers skip indexing; the first
 * decoder Full layer scores the whole causally visible range and also keeps the blocks
 * with the highest maximum score (e.g. 2,048 blocks of 8 = 16,384 positions) as a
 * candidate pool that later Reindex layers search. [TDG CSA2]: Top-512.
 * Score (the pages print no formula; reading adopted):
 *     s[t,j] = sum_{h<H_I} w[t,h] * max(0, <q_I[t,h,:], k_I[j,:]>)
 * computed with fp32 accumulation. Top-K key: (score descending, position ascending).
 *
 *   mode      FULL / REINDEX / REUSE. REUSE validates arguments and launches nothing.
 *   B, T      sequences and query tokens per sequence (T = 1 for decode).
 *   H_I       indexer heads, 1..128.
 *   qk_dtype  storage type of q_I and k_I; CSA2_DTYPE_E4M3_FP4KEY: E4M3 q_I and compact
 *             68-byte keys (the score is the same formula over the keys' decoded values
 *             e2m1(code) * scale).
 *   q_I       [B][T][H_I][128];  w  fp32 [B][T][H_I];  k_I  [B][cap][128] (compact keys:
 *             the two-plane buffer described at CSA2_DTYPE_E4M3_FP4KEY).
 *   n_vis0    int32 [B]: visible entries per sequence (decode, q_pos0 == NULL).
 *   ratio, q_pos0
 *             prefill visibility (q_pos0 != NULL): token t of sequence b sits at
 *             position p = q_pos0[b] + t and sees entries j with (j+1)*ratio <= p+1,
 *             i.e. N(t) = floor((p + 1) / ratio). Ignored when q_pos0 == NULL.
 *   K         entries to select (1..2048).
 *   pool_in   REINDEX only: int32 [B][T][P_in] candidate positions (-1 = empty slot);
 *             must be non-NULL for REINDEX and NULL otherwise.
 *   pool_out  FULL only, nullable: int32 [B][T][pool_blocks*8]: visible positions of the
 *             pool_blocks blocks with the highest block maximum (ties: lower block),
 *             ascending, padded with -1.
 *   idx_out   int32 [B][T][K]: chosen positions in ascending order, padded with -1 when
 *             fewer than K are visible.
 *   scores_out nullable fp32 [B][T][cap] (FULL) or [B][T][P_in] (REINDEX): the scores;
 *             entries not visible are left untouched.
 *   ws, ws_bytes  workspace of at least csa2_workspace_bytes(CSA2_OP_INDEX_SCORE_TOPK,..).
 */
CSA2_API csa2_status_t csa2_index_score_topk(csa2_mode_t mode, int B, int T, int H_I,
                                    csa2_dtype_t qk_dtype, const void* q_I, const float* w,
                                    const void* k_I, int64_t cap, const int32_t* n_vis0,
                                    int ratio, const int32_t* q_pos0, int K,
                                    const int32_t* pool_in, int P_in, int32_t* pool_out,
                                    int pool_blocks, int32_t* idx_out, float* scores_out,
                                    void* ws, size_t ws_bytes, void* stream);

/*
 * csa2_sparse_attn_decode — gather + dequantise the selected FP4 main-KV rows and
 * attend over them together with the sliding-window rows.
 * [AIS Methodology]: a compressed global branch plus a sliding-window local branch;
 * every layer has its own query and window KV. [TDG Causal Encoder-Decoder, CSA2]:
 * 128-token window in every layer. [AIS Main Findings]: window KV stays FP8.
 * Reading adopted (pages silent): one softmax over the union of the K selected entries
 * and the window rows, logits = scale * <q_h, x_i>, output sum_i p_i x_i (keys and values
 * are the same latent row), no de-duplication and no sink; an empty row set gives 0.
 *
 *   mode      recorded and validated only: Full, Reindex and Reuse layers run the same
 *             kernel (a Reuse layer passes the earlier layer's idx).
 *   q         bf16 [B][H][512], H in 1..64 (more heads: CSA2_ERR_UNSUPPORTED).
 *   codes, scales  main-KV cache as written by csa2_quantize_kv, capacity cap.
 *   idx       int32 [B][K]; -1 entries are skipped; other entries outside [0, cap) are
 *             skipped and set CSA2_DEV_BAD_INDEX.
 *   swa       E4M3 [B][W][512]: the last W window rows, oldest first; W in 0..1024.
 *   swa_valid nullable int32 [B]: only the last swa_valid[b] rows are used.
 *   scale     logit multiplier (e.g. 1/sqrt(512)).
 *   out       fp32 [B][H][512].
 */
CSA2_API csa2_status_t csa2_sparse_attn_decode(csa2_mode_t mode, int B, int H, const void* q,
                                      const uint8_t* codes, const uint8_t* scales,
                                      int64_t cap, const int32_t* idx, int K,
                                      const uint8_t* swa, int W, const int32_t* swa_valid,
                                      float scale, float* out, void* ws, size_t ws_bytes,
                                      void* stream);

/*
 * csa2_sparse_attn_prefill — csa2_sparse_attn_decode for T new tokens per sequence,
 * each with its own indices and a causal window ([TDG Causal Encoder-Decoder]).
 *   q         bf16 [B][T][H][512];  idx  int32 [B][T][K].
 *   swa       E4M3 [B][W-1+T][512]: row r holds position q_pos0[b] - (W-1) + r; token t
 *             uses rows t .. t+W-1 (the last one is itself); rows whose position is
 *             negative are skipped.
 *   q_pos0    nullable int32 [B] (NULL: every row is valid).
 *   out       fp32 [B][T][H][512].
 */
CSA2_API csa2_status_t csa2_sparse_attn_prefill(int B, int T, int H, const void* q,
                                       const uint8_t* codes, const uint8_t* scales,
                                       int64_t cap, const int32_t* idx, int K,
                                       const uint8_t* swa, int W, const int32_t* q_pos0,
                                       float scale, float* out, void* ws, size_t ws_bytes,
                                       void* stream);

/*
 * csa2_index_score_topk_noalloc — csa2_index_score_topk for callers that cannot allocate
 * device memory. (This entry point has no counterpart on the source pages; it is a
 * deployment convenience.) Callers such as plugins inside an inference engine that owns
 * every device allocation, or latency-critical loops where an allocation may synchronise
 * the device, cannot provide a workspace. This variant takes the same arguments minus the
 * workspace and uses a fixed 16 MiB device array inside the library instead (held on every
 * GPU that loads the library until the process exits).
 *   status   nullable int32 device word: the call's device status bits are OR-ed into it.
 * Returns CSA2_ERR_WORKSPACE when csa2_workspace_bytes() for the call exceeds 16 MiB. The
 * first call on a device looks up the array's address with that device current; make it
 * before any stream capture. All calls share the array, which keeps the previous call's
 * contents (the call clears what must start at zero): calls that overlap on the GPU race,
 * so order them on one stream. It allocates nothing.
 */
CSA2_API csa2_status_t csa2_index_score_topk_noalloc(
    csa2_mode_t mode, int B, int T, int H_I, csa2_dtype_t qk_dtype, const void* q_I,
    const float* w, const void* k_I, int64_t cap, const int32_t* n_vis0, int ratio,
    const int32_t* q_pos0, int K, const int32_t* pool_in, int P_in, int32_t* pool_out,
    int pool_blocks, int32_t* idx_out, float* scores_out, int32_t* status, void* stream);

/* Workspace bytes an operation needs (0 on invalid arguments).
 *   CSA2_OP_INDEX_SCORE_TOPK: H = H_I; cap = cache capacity (Full) or P_in (Reindex);
 *                             pool_blocks = 0 when no pool is built.
 *   CSA2_OP_SPARSE_ATTN_*:    H = query heads; cap and pool_blocks are ignored.
 * The size depends on the device's SM count for the decode attention (query rows are split
 * across SMs), so query it on the device that will run the call. */
CSA2_API size_t csa2_workspace_bytes(csa2_op_t op, int B, int T, int H, int64_t cap, int K,
                            int pool_blocks);

/* Number of kernels one csa2_sparse_attn_decode call launches for B queries with K selected
 * entries and W window rows on the current device: 1 with no rows, 2 (row staging +
 * attention) when a query's rows are not split or when its splits merge inside the
 * attention kernel (a thread-block cluster per query, when the device can hold all of them
 * at once), 3 when a separate merge kernel combines the splits. For launch accounting and
 * graph planning; -1 on invalid arguments. */
CSA2_API int csa2_sparse_attn_decode_launches(int B, int K, int W);

/*
 * Context parallelism: G GPUs each own a contiguous shard [lo, hi) of every sequence's
 * compressed entries (lo a multiple of 8), run csa2_index_score_topk(FULL) on it with
 * scores_out (and pool_out), turn the selections into candidate lists with the calls below,
 * all-gather the lists (e.g. NCCL) and merge them. The merged Top-K and pool equal the
 * single-GPU ones exactly. [TDG Compressed Sparse Attention 2 (CSA2)]: the Full layer
 * keeps the 512 highest-scoring entries and the 2,048 blocks of 8 with the highest block
 * maxima; both selections decompose over shards because the order (score descending, index
 * ascending) is total and a score depends only on its own entry. (The pages describe one
 * GPU; sharding is this library's extension for million-entry contexts.) All pointers are
 * device pointers, all calls asynchronous on `stream`; CSA2_ERR_ARG on bad sizes or null
 * pointers.
 *
 * csa2_cp_topk_candidates — a shard's Top-K as (score, global index) pairs.
 *   scores     fp32 [rows][ld_scores]: the shard's scores_out.
 *   idx        int32 [rows][K]: the shard's idx_out (shard-local, -1 padded).
 *   offset     global index of the shard's first entry (offset + ld_scores < 2^31).
 *   cand_score fp32 [rows][K], cand_idx int32 [rows][K]: (score, offset + idx), or (0, -1).
 */
CSA2_API csa2_status_t csa2_cp_topk_candidates(int rows, const float* scores, int64_t ld_scores,
                                               const int32_t* idx, int K, int64_t offset,
                                               float* cand_score, int32_t* cand_idx,
                                               void* stream);

/*
 * csa2_cp_pool_candidates — a shard's candidate pool as (block maximum, global block) pairs.
 *   pool       int32 [rows][P]: the shard's pool_out (ascending shard-local positions).
 *   max_blocks pairs per row written to cand_bmax fp32 / cand_block int32 [rows][max_blocks],
 *              block = (offset + position) / 8, padded with (0, -1). offset % 8 == 0.
 */
CSA2_API csa2_status_t csa2_cp_pool_candidates(int rows, const float* scores, int64_t ld_scores,
                                               const int32_t* pool, int P, int max_blocks,
                                               int64_t offset, float* cand_bmax,
                                               int32_t* cand_block, void* stream);

/*
 * csa2_cp_merge — the K best of every row's n_cand candidates by (score descending, index
 * ascending), written to idx_out int32 [rows][K] in ascending index order, -1 padded.
 * Candidates with index -1 are ignored; indices must be distinct. n_cand <= 16384
 * (CSA2_ERR_UNSUPPORTED above: 8 shards of 2,048 pool blocks, or 32 shards of K = 512),
 * K <= n_cand. Used for entries (scores) and for pool blocks (block maxima) alike.
 */
CSA2_API csa2_status_t csa2_cp_merge(int rows, int n_cand, const float* cand_score,
                                     const int32_t* cand_idx, int K, int32_t* idx_out,
                                     void* stream);

/*
 * csa2_cp_pool_expand — merged pool blocks int32 [rows][nb] (ascending, -1 padded) to the
 * pool's entry positions int32 [rows][P] (ascending, -1 padded): block b contributes the
 * positions 8b .. 8b+7 below n_row[r] (nullable int32 [rows]: NULL = all).
 */
CSA2_API csa2_status_t csa2_cp_pool_expand(int rows, const int32_t* blocks, int nb,
                                           const int32_t* n_row, int P, int32_t* pool_out,
                                           void* stream);

/*
 * csa2_cp_local_idx — this shard's view of the merged selection: idx_local[i] = idx[i] - lo
 * for lo <= idx[i] < hi, else -1 (n elements, any row layout).
 */
CSA2_API csa2_status_t csa2_cp_local_idx(int64_t n, const int32_t* idx, int64_t lo, int64_t hi,
                                         int32_t* idx_local, void* stream);

/*
 * csa2_sparse_attn_decode_partial — csa2_sparse_attn_decode over the rows this caller holds
 * (its shard's selected entries, and the window rows on one shard only), left as a partial
 * result for csa2_attn_merge_partials: o_part fp32 [B][H][512] = sum_i 2^(l_i - m) x_i and
 * ml_part fp32 [B][2][H] = (m, sum_i 2^(l_i - m)), with l_i the logits in base-2 units
 * (scale * log2(e) * <q_h, x_i>); a head with no rows (all indices -1, or K = W = 0 for a
 * shard that holds nothing) gives (-inf, 0) and a zero o_part, which the merge weighs 0.
 * Same arguments and checks as csa2_sparse_attn_decode, the same workspace.
 * [TDG Compressed Sparse Attention 2 (CSA2)]: one softmax over the selected entries and the
 * window rows; splitting the rows and merging partials is the exact log-sum-exp identity.
 *
 * csa2_attn_merge_partials — out fp32 [B][H][512] = sum_g 2^(m_g - M) o_g / sum_g 2^(m_g - M)
 * l_g over G partials laid out rank-major (o_parts [G][B][H][512], ml_parts [G][B][2][H], as
 * an all-gather along a new leading dimension leaves them). H <= 64.
 */
CSA2_API csa2_status_t csa2_sparse_attn_decode_partial(csa2_mode_t mode, int B, int H,
                                                       const void* q, const uint8_t* codes,
                                                       const uint8_t* scales, int64_t cap,
                                                       const int32_t* idx, int K,
                                                       const uint8_t* swa, int W,
                                                       const int32_t* swa_valid, float scale,
                                                       float* o_part, float* ml_part, void* ws,
                                                       size_t ws_bytes, void* stream);
CSA2_API csa2_status_t csa2_attn_merge_partials(int B, int H, int G, const float* o_parts,
                                                const float* ml_parts, float* out, void* stream);

/*
 * Persistent-cache records: one sequence's entries [lo, lo + n) copied between the device
 * caches and a host buffer in a fixed byte format. [AIS Main Findings]: the global KV cache
 * is held in HBM and a persistent KV cache exists besides it; [TDG The KV Cache Revolution]:
 * the cache is accounted in bytes per token. The byte format and the copies only (no storage
 * tier). Record: a 64-byte header (magic "CSA2", version 1, D = 512, D_I = 128, lo, n,
 * key_bytes, bytes per entry) | codes [n][256] | scales [n][32] | indexer keys [n][key_bytes]
 * (key_bytes 0 = none, 128 = E4M3 keys, 256 = bf16 keys). Host buffers may be pageable or
 * pinned (pinned: the copies are asynchronous on `stream`).
 *
 * csa2_cache_record_bytes — bytes of a record of n entries (0 on bad arguments).
 * csa2_cache_export — writes the header at once and enqueues one device-to-host copy per
 *   array; the record is complete when `stream` reaches that point. codes/scales/k_I are the
 *   caches ([B][cap][256], [B][cap][32], [B][cap][key_bytes]); k_I NULL iff key_bytes = 0.
 *   CSA2_ERR_ARG when lo + n > cap, host_bytes is too small, or arguments are inconsistent.
 * csa2_cache_import — validates the (complete) record's header on the host and enqueues
 *   host-to-device copies to the header's lo of sequence b. CSA2_ERR_ARG on a bad magic,
 *   version, size or range, or when the record's keys and k_I disagree;
 *   CSA2_ERR_UNSUPPORTED for other channel counts.
 */
CSA2_API size_t csa2_cache_record_bytes(int64_t n, int key_bytes);
CSA2_API csa2_status_t csa2_cache_export(const uint8_t* codes, const uint8_t* scales,
                                         const void* k_I, int key_bytes, int64_t cap, int b,
                                         int64_t lo, int64_t n, void* host, size_t host_bytes,
                                         void* stream);
CSA2_API csa2_status_t csa2_cache_import(const void* host, size_t host_bytes, uint8_t* codes,
                                         uint8_t* scales, void* k_I, int64_t cap, int b,
                                         void* stream);

/* Static text for a status code. Never NULL. */
CSA2_API const char* csa2_status_string(csa2_status_t status);

/* Copy the device status word (first 4 bytes of `ws`, a device pointer) to *out (host)
 * after synchronising `stream`. Returns CSA2_ERR_DEVICE when the word is non-zero. */
CSA2_API csa2_status_t csa2_read_device_status(const void* ws, int32_t* out, void* stream);

/* Clear the device status word (asynchronous on `stream`). */
CSA2_API csa2_status_t csa2_reset_device_status(void* ws, void* stream);

/* Library version: major * 10000 + minor * 100 + patch. */
CSA2_API int csa2_version(void);

/* Benchmark hook: when set, the next csa2_index_score_topk() issued from the calling host
 * thread records `ev_start` (a cudaEvent_t passed as void*) on its stream right before
 * its indexer-scan kernel launch and `ev_stop` right after it, then forgets both. The
 * setting is per host thread and consumed by one call; NULL, NULL clears it. During a stream
 * capture the two records become external event nodes of the graph, so replays of the graph
 * can be timed with them. */
CSA2_API csa2_status_t csa2_set_stage_events(void* ev_start, void* ev_stop);

/* Benchmark hook: records `ev` (a cudaEvent_t passed as void*) on `stream`; during a stream
 * capture the record becomes an external event node of the graph, so replays of the graph
 * can be timed between two such events (a plain cudaEventRecord inside a capture only adds a
 * dependency). Outside a capture it is an ordinary record. */
CSA2_API csa2_status_t csa2_record_event(void* ev, void* stream);

/* Test hook for the bounded waits: launches one block that waits on an mbarrier that is
 * never signalled, gives up after timeout_ns and sets CSA2_DEV_TIMEOUT in `status`
 * (device int32). Never faults or hangs. */
CSA2_API csa2_status_t csa2_debug_bounded_wait(int32_t* status, uint64_t timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA2_H */
