/*
 * CSA2 oracle: a plain, slow CPU restatement of what the CSA2 hot path computes.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path (the CUDA library and its
 * Python binding) links, imports or calls this file. Only the tests, the smoke check
 * and the CPU-baseline leg of the benchmark use it. It shares no code, header, table
 * or constant generator with the CUDA kernels.
 *
 * Arithmetic is done in double precision on the exact input values (bf16, E4M3 and
 * E2M1 all decode exactly into a double). Loops run in the order the definitions are
 * written; the only parallelism (OpenMP) is over independent outputs, which does not
 * change any result.
 *
 * Sources (web pages about the DeepSeek-V4.1-Flash report):
 *  [AIS]  "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (ai.info
 *         AI summary), sections "Main Findings" and "Methodology in Plain English".
 *  [TDG]  "DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale LLM Serving"
 *         (technologiesdigest.com), sections "Compressed Sparse Attention 2 (CSA2)"
 *         and "Quantization and Memory Management".
 *  [TLB]  "DeepSeek V4.1 Flash: smaller KV cache, same post-training" (traillabs.ai),
 *         section "How did DeepSeek V4.1 reduce the KV cache?".
 *
 * Pinning status (what each function is checked against, in tests/test_oracle_*.py):
 *  - codecs: exhaustive tables, torch's float8_e4m3fn cast, an exact-rational
 *    threshold formulation, the 448 x 6 = 2688 saturation point [AIS Main Findings];
 *  - index score: brute force on tiny inputs against a library contraction;
 *  - Top-K / pool: against Python's sorted() on tiny inputs with planted ties and
 *    against the Top-K-inside-pool invariant;
 *  - attention: K = all entries against torch's scaled_dot_product_attention in fp64,
 *    one-key and q = 0 closed forms;
 *  - prefill visibility and window rows: a token-by-token simulation of the compressor
 *    and of the window buffer, for ratios 1-3 and windows clipped at position 0; the
 *    composed prefill query with every visible entry selected against dense attention.
 *  - bf16 encoder: torch's float32 -> bfloat16 cast on float32 inputs, hand-placed
 *    midpoints and subnormals;
 *  - compressor: r = 1 is the identity, equal logits give the mean, a dominant logit
 *    (chosen per channel) selects its token, shifting a channel's logits or permuting
 *    the tokens of a group changes nothing, every output lies inside its tokens' range,
 *    and a hand-worked two-token case;
 *  - projection: one-hot latents give W's columns, an identity W copies the first Di
 *    channels, and random inputs match a float64 matrix-vector product.
 *  - compact 68-byte keys: keys whose scale is a power of two round-trip exactly,
 *    the largest magnitude takes code 6, negation flips only sign bits, midpoints
 *    round to even, an independent nearest-grid search agrees on random keys, the
 *    68-byte record gives 890 bytes per token, and scores against compact keys equal
 *    the bf16-key scores of the same values;
 *  The compressor and projection follow a READING (the pages lose the equation):
 *  parity with the pages' own compressor is unpinned.
 *  The index-score FORMULA itself (sum over heads of w_h * ReLU(q_h . k)) is not
 *  printed on the pages: parity with the pages' own scorer is unpinned; the reading is
 *  stated where it is used.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_EXPORT __attribute__((visibility("default")))

#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads for the oracle's parallel loops from now on (n >= 1). */
ORC_EXPORT void orc_set_num_threads(int n) {
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Threads the oracle's parallel loops use (for reporting a CPU baseline's core count). */
ORC_EXPORT int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------------ */
/* Number formats                                                                  */
/* ------------------------------------------------------------------------------ */

/* bf16: the upper 16 bits of an IEEE binary32. */
ORC_EXPORT double orc_bf16_value(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* E2M1 (the FP4 element format named in [AIS Main Findings], [TDG Quantization]):
 * 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no Inf/NaN.
 * Exponent field 0 is subnormal: 0.5 * m. Otherwise (1 + m/2) * 2^(e-1).
 * The eight magnitudes are therefore 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
ORC_EXPORT double orc_e2m1_value(unsigned code) {
    unsigned sign = (code >> 3) & 1u;
    unsigned e = (code >> 1) & 3u;
    unsigned m = code & 1u;
    double mag;
    if (e == 0)
        mag = 0.5 * (double)m;
    else
        mag = (1.0 + 0.5 * (double)m) * ldexp(1.0, (int)e - 1);
    return sign ? -mag : mag;
}

/* E4M3 "FN" (the scale format named in [AIS Main Findings]): 1 sign bit, 4 exponent
 * bits (bias 7), 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); the all-ones
 * pattern S.1111.111 is NaN; there is no infinity. Largest finite value 1.75*2^8 = 448. */
ORC_EXPORT double orc_e4m3_value(uint8_t code) {
    unsigned sign = (code >> 7) & 1u;
    unsigned e = (code >> 3) & 15u;
    unsigned m = code & 7u;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = ((double)m / 8.0) * ldexp(1.0, -6);
    else
        mag = (1.0 + (double)m / 8.0) * ldexp(1.0, (int)e - 7);
    return sign ? -mag : mag;
}

/* Round-to-nearest-even onto a sorted list of non-negative magnitudes whose codes are
 * 0..n-1 (code parity = mantissa LSB), saturating anything above the last one.
 * Returns the magnitude code. Brute force: look at every candidate. */
static unsigned rne_onto_grid(double v, const double* grid, unsigned n) {
    unsigned best = 0;
    double best_d = fabs(v - grid[0]);
    for (unsigned c = 1; c < n; ++c) {
        double d = fabs(v - grid[c]);
        if (d < best_d || (d == best_d && (c & 1u) == 0 && (best & 1u) == 1)) {
            best = c;
            best_d = d;
        }
    }
    if (v > grid[n - 1]) best = n - 1; /* saturate finite overflow */
    return best;
}

/* E4M3 encoder: round to nearest, ties to even, finite overflow saturates to +-448. */
ORC_EXPORT uint8_t orc_e4m3_encode(double v) {
    double grid[127];
    for (unsigned c = 0; c < 127; ++c) grid[c] = orc_e4m3_value((uint8_t)c);
    unsigned sign = signbit(v) ? 1u : 0u;
    unsigned mag = rne_onto_grid(fabs(v), grid, 127);
    return (uint8_t)((sign << 7) | mag);
}

/* E2M1 encoder: round to nearest, ties to even, saturating at 6; the sign bit is
 * copied from the input (so -0 and negative values that round to zero give 0x8). */
ORC_EXPORT unsigned orc_e2m1_encode(double v) {
    double grid[8];
    for (unsigned c = 0; c < 8; ++c) grid[c] = orc_e2m1_value(c);
    unsigned sign = signbit(v) ? 1u : 0u;
    unsigned mag = rne_onto_grid(fabs(v), grid, 8);
    return (sign << 3) | mag;
}

/* ------------------------------------------------------------------------------ */
/* FP4 main-KV quantize-on-write                                                   */
/* [AIS Main Findings "FP4 format choice"], [TDG Quantization and Memory           */
/* Management], [TLB "FP4 KV cache"]: E2M1 elements with one E4M3 scale per 16     */
/* channels, NVFP4 without its second-level global scale.                          */
/* ------------------------------------------------------------------------------ */

/* One 16-channel block. Reading adopted where the pages are silent (NVFP4 practice):
 *  1. amax = max |x_i| over the block;
 *  2. scale code = E4M3_RNE_sat(amax / 6)  (6 = largest E2M1 magnitude), s = its value;
 *  3. if s == 0 every magnitude code is 0; else magnitude_i = E2M1_RNE_sat(|x_i| / s);
 *  4. the sign bit of each code is the sign bit of x_i.
 * amax/6 and |x_i|/s are formed in double; neither quotient can fall on a rounding
 * midpoint unless the exact quotient does (a bf16 numerator over 6 or over a
 * 4-significant-bit scale is either dyadic and exact, or far from every dyadic
 * midpoint), so the double rounding is harmless. */
/* step 2: the block's scale code from its largest magnitude */
ORC_EXPORT uint8_t orc_fp4_scale_code(double amax) { return orc_e4m3_encode(amax / 6.0); }

/* steps 3-4: the element code of x under a decoded scale value s */
ORC_EXPORT unsigned orc_fp4_code(double x, double s) {
    unsigned sign = signbit(x) ? 8u : 0u;
    unsigned mag = 0;
    if (s > 0.0) mag = orc_e2m1_encode(fabs(x) / s) & 7u;
    return sign | mag;
}

ORC_EXPORT void orc_quantize_block16(const double* x, uint8_t* codes4 /*16 nibbles*/,
                                     uint8_t* scale_code) {
    double amax = 0.0;
    for (int i = 0; i < 16; ++i)
        if (fabs(x[i]) > amax) amax = fabs(x[i]);
    uint8_t sc = orc_fp4_scale_code(amax);
    double s = orc_e4m3_value(sc);
    for (int i = 0; i < 16; ++i) codes4[i] = (uint8_t)orc_fp4_code(x[i], s);
    *scale_code = sc;
}

/* Batched forms of the two steps above (plain loops, for exhaustive tests). */
ORC_EXPORT void orc_fp4_scale_codes_many(const double* amax, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_fp4_scale_code(amax[i]);
}

ORC_EXPORT void orc_fp4_codes_many(const double* x, const double* s, int64_t n,
                                   uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)orc_fp4_code(x[i], s[i]);
}

ORC_EXPORT void orc_e4m3_encode_many(const double* v, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

/* Quantize n entries of D channels (D a multiple of 16) given as bf16 bit patterns,
 * row i at kv + i*ld. Output layout: codes row i = D/2 bytes, channel 2k in the low
 * nibble of byte k and channel 2k+1 in the high nibble; scales row i = D/16 bytes. */
ORC_EXPORT void orc_quantize_entries(const uint16_t* kv, int64_t n, int64_t ld, int D,
                                     uint8_t* codes, uint8_t* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        for (int blk = 0; blk < D / 16; ++blk) {
            double x[16];
            uint8_t c[16];
            for (int t = 0; t < 16; ++t) x[t] = orc_bf16_value(kv[i * ld + blk * 16 + t]);
            orc_quantize_block16(x, c, &scales[i * (D / 16) + blk]);
            for (int t = 0; t < 8; ++t)
                codes[i * (D / 2) + blk * 8 + t] = (uint8_t)(c[2 * t] | (c[2 * t + 1] << 4));
        }
    }
}

/* Value of channel c of one stored entry: E2M1 code value times its block's scale. */
ORC_EXPORT void orc_dequant_entry(const uint8_t* codes, const uint8_t* scales, int D,
                                  double* x) {
    for (int c = 0; c < D; ++c) {
        uint8_t byte = codes[c / 2];
        unsigned nib = (c % 2 == 0) ? (byte & 15u) : (byte >> 4);
        x[c] = orc_e2m1_value(nib) * orc_e4m3_value(scales[c / 16]);
    }
}

/* ------------------------------------------------------------------------------ */
/* Indexer score                                                                   */
/* [AIS Methodology] (indexer K, "index scores", own indexer query per layer),      */
/* [TDG CSA2] (Full / Reindex rescoring). The pages print no formula. Reading:      */
/*   s_j = sum_{h<H} w_h * max(0, sum_{d<Di} q[h,d] * k_j[d])                       */
/* with q, k decoded exactly from their storage type, summed in double, then +0.0   */
/* (so that a zero score is +0).                                                   */
/* ------------------------------------------------------------------------------ */

enum { ORC_BF16 = 0, ORC_E4M3 = 1 };

static double load_elem(const void* base, int dtype, int64_t i) {
    if (dtype == ORC_BF16) return orc_bf16_value(((const uint16_t*)base)[i]);
    return orc_e4m3_value(((const uint8_t*)base)[i]);
}

/* scores for entries rows[0..n) (rows == NULL means rows 0..n-1) of k [*, Di] */
ORC_EXPORT void orc_index_scores(int H, int Di, int dtype, const void* q /*[H,Di]*/,
                                 const float* w /*[H]*/, const void* k /*[*,Di]*/,
                                 const int32_t* rows, int64_t n, double* s) {
    double* qd = (double*)malloc(sizeof(double) * (size_t)H * Di);
    for (int64_t i = 0; i < (int64_t)H * Di; ++i) qd[i] = load_elem(q, dtype, i);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        int64_t r = rows ? rows[j] : j;
        double kd[1024];
        for (int d = 0; d < Di; ++d) kd[d] = load_elem(k, dtype, r * Di + d);
        double acc = 0.0;
        for (int h = 0; h < H; ++h) {
            double dot = 0.0;
            for (int d = 0; d < Di; ++d) dot += qd[(int64_t)h * Di + d] * kd[d];
            double relu = dot > 0.0 ? dot : 0.0;
            acc += (double)w[h] * relu;
        }
        s[j] = acc + 0.0;
    }
    free(qd);
}

/* ------------------------------------------------------------------------------ */
/* Compact indexer keys: 68 bytes per entry                                        */
/* [AIS Main Findings] and [TLB "How is DeepSeek V4.1 Flash different"] (Figure 1): */
/* 890 bytes of global KV per token. With 2.5 stored entry-sets per token (byte     */
/* accounting below) and 288-byte FP4 main entries, 890 leaves 68 bytes for an      */
/* indexer key. Reading (the pages give no key format): a 128-channel key as E2M1   */
/* codes (64 bytes, channel 2k in the low nibble of byte k) times one fp32 scale    */
/* (4 bytes) per key, scale = amax / 6 so that the largest magnitude maps to 6.      */
/* The quantizer's decisions are taken in IEEE fp32, the precision of the key       */
/* format's own scale: s = fl32(amax / 6), code = E2M1_RNE_sat(fl32(|x| / s)), the   */
/* sign bit copied from x; s == 0 gives zero magnitudes.                            */
/* ------------------------------------------------------------------------------ */

ORC_EXPORT void orc_quantize_key_fp4(const uint16_t* k /*bf16 [Di]*/, int Di, uint8_t* codes,
                                     float* scale) {
    float amax = 0.0f;
    for (int d = 0; d < Di; ++d) {
        float a = fabsf((float)orc_bf16_value(k[d]));
        if (a > amax) amax = a;
    }
    volatile float six = 6.0f;
    float sc = amax / six;                       /* one IEEE fp32 division */
    for (int d = 0; d < Di; d += 2) {
        unsigned nib[2];
        for (int t = 0; t < 2; ++t) {
            float x = (float)orc_bf16_value(k[d + t]);
            unsigned sign = signbit(x) ? 8u : 0u;
            unsigned mag = 0;
            if (sc > 0.0f) {
                float qv = fabsf(x) / sc;        /* one IEEE fp32 division */
                mag = orc_e2m1_encode((double)qv) & 7u;
            }
            nib[t] = sign | mag;
        }
        codes[d / 2] = (uint8_t)(nib[0] | (nib[1] << 4));
    }
    *scale = sc;
}

ORC_EXPORT void orc_quantize_keys_fp4(const uint16_t* k, int64_t n, int Di, uint8_t* codes,
                                      float* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        orc_quantize_key_fp4(k + i * Di, Di, codes + i * (Di / 2), &scales[i]);
}

/* Value of channel d of a compact key: E2M1 code value times the key's scale. */
ORC_EXPORT void orc_dequant_key_fp4(const uint8_t* codes, float scale, int Di, double* x) {
    for (int d = 0; d < Di; ++d) {
        uint8_t byte = codes[d / 2];
        unsigned nib = (d % 2 == 0) ? (byte & 15u) : (byte >> 4);
        x[d] = orc_e2m1_value(nib) * (double)scale;
    }
}

/* Index scores (the formula above) against compact keys, q as E4M3 [H][Di]. */
ORC_EXPORT void orc_index_scores_fp4key(int H, int Di, const uint8_t* q, const float* w,
                                        const uint8_t* codes /*[*][Di/2]*/,
                                        const float* scales /*[*]*/, const int32_t* rows,
                                        int64_t n, double* s) {
    double* qd = (double*)malloc(sizeof(double) * (size_t)H * Di);
    for (int64_t i = 0; i < (int64_t)H * Di; ++i) qd[i] = orc_e4m3_value(q[i]);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        int64_t r = rows ? rows[j] : j;
        double kd[1024];
        orc_dequant_key_fp4(codes + r * (Di / 2), scales[r], Di, kd);
        double acc = 0.0;
        for (int h = 0; h < H; ++h) {
            double dot = 0.0;
            for (int d = 0; d < Di; ++d) dot += qd[(int64_t)h * Di + d] * kd[d];
            double relu = dot > 0.0 ? dot : 0.0;
            acc += (double)w[h] * relu;
        }
        s[j] = acc + 0.0;
    }
    free(qd);
}

/* ------------------------------------------------------------------------------ */
/* Exact Top-K [TDG CSA2] ("Top-512"), [AIS Key Contributions] (Top-K indices).     */
/* Keys (score descending, id ascending) — the lower id wins an exact tie.          */
/* Output: the chosen ids in ascending order, padded with -1 up to K.               */
/* ------------------------------------------------------------------------------ */

typedef struct {
    double s;
    int64_t id;
} orc_pair;

static int cmp_score_desc_id_asc(const void* a, const void* b) {
    const orc_pair* x = (const orc_pair*)a;
    const orc_pair* y = (const orc_pair*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id);
}

static int cmp_i64(const void* a, const void* b) {
    int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
    return (x < y) ? -1 : (x > y);
}

/* s[0..n) with ids[i] (ids == NULL: id = i). Returns the number chosen, min(K, n). */
ORC_EXPORT int64_t orc_topk(const double* s, const int32_t* ids, int64_t n, int64_t K,
                            int32_t* out) {
    orc_pair* p = (orc_pair*)malloc(sizeof(orc_pair) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) {
        p[i].s = s[i];
        p[i].id = ids ? ids[i] : i;
    }
    qsort(p, (size_t)n, sizeof(orc_pair), cmp_score_desc_id_asc);
    int64_t m = n < K ? n : K;
    int64_t* sel = (int64_t*)malloc(sizeof(int64_t) * (size_t)(m > 0 ? m : 1));
    for (int64_t i = 0; i < m; ++i) sel[i] = p[i].id;
    qsort(sel, (size_t)m, sizeof(int64_t), cmp_i64);
    for (int64_t i = 0; i < K; ++i) out[i] = (i < m) ? (int32_t)sel[i] : -1;
    free(sel);
    free(p);
    return m;
}

/* ------------------------------------------------------------------------------ */
/* Hierarchical Sparse Indexer candidate pool                                      */
/* [AIS Methodology]: the first Full layer keeps the blocks with the highest        */
/* maximum index score, e.g. 2,048 blocks of 8 positions = 16,384 candidates;       */
/* [TDG CSA2], [TLB]: later Reindex layers search only inside it.                  */
/* Reading: blocks are aligned at multiples of `blk`; block c covers positions      */
/* [c*blk, c*blk+blk) intersected with [0, n); bmax_c = max score over that range;  */
/* the top `nblk` blocks by (bmax desc, c asc) are kept; the pool is their visible  */
/* positions in ascending order, padded with -1 up to nblk*blk.                     */
/* ------------------------------------------------------------------------------ */

ORC_EXPORT int64_t orc_pool(const double* s, int64_t n, int64_t nblk, int blk,
                            int32_t* pool_out) {
    int64_t nb = (n + blk - 1) / blk;
    double* bmax = (double*)malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
    for (int64_t c = 0; c < nb; ++c) {
        double m = -INFINITY;
        for (int64_t j = c * blk; j < c * blk + blk && j < n; ++j)
            if (s[j] > m) m = s[j];
        bmax[c] = m;
    }
    int32_t* chosen = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nblk > 0 ? nblk : 1));
    int64_t m = orc_topk(bmax, NULL, nb, nblk, chosen);
    int64_t w = 0;
    for (int64_t i = 0; i < m; ++i) {
        int64_t c = chosen[i];
        for (int64_t j = c * blk; j < c * blk + blk && j < n; ++j) pool_out[w++] = (int32_t)j;
    }
    for (int64_t i = w; i < nblk * blk; ++i) pool_out[i] = -1;
    free(chosen);
    free(bmax);
    return w;
}

/* ------------------------------------------------------------------------------ */
/* Sparse + sliding-window attention                                               */
/* [AIS Methodology]: a sliding-window local branch plus a compressed global branch;*/
/* [TDG CED, CSA2]: 128-token SWA in every layer, every layer has its own query.    */
/* Reading (pages silent on the join): one softmax over the concatenation of the    */
/* selected compressed entries and the window rows (no de-duplication, no sink),    */
/* logits tau * <q_h, x_i>, output sum_i softmax_i * x_i (keys and values are the   */
/* same latent row x_i). An empty row set gives a zero output.                      */
/* ------------------------------------------------------------------------------ */

/* q: H x D doubles; rows: nrows x D doubles; out: H x D doubles. */
ORC_EXPORT void orc_attention(int H, int D, const double* q, const double* rows,
                              int64_t nrows, double tau, double* out) {
#pragma omp parallel for schedule(static)
    for (int h = 0; h < H; ++h) {
        double* o = out + (int64_t)h * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (nrows == 0) continue;
        double* logit = (double*)malloc(sizeof(double) * (size_t)nrows);
        double mx = -INFINITY;
        for (int64_t i = 0; i < nrows; ++i) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += q[(int64_t)h * D + d] * rows[i * D + d];
            logit[i] = tau * dot;
            if (logit[i] > mx) mx = logit[i];
        }
        double den = 0.0;
        for (int64_t i = 0; i < nrows; ++i) den += exp(logit[i] - mx);
        for (int64_t i = 0; i < nrows; ++i) {
            double p = exp(logit[i] - mx) / den;
            for (int d = 0; d < D; ++d) o[d] += p * rows[i * D + d];
        }
        free(logit);
    }
}

/* ------------------------------------------------------------------------------ */
/* Prefill visibility and the causal window                                        */
/* [TDG Causal Encoder-Decoder]: every layer attends over a 128-token sliding       */
/* window; [TDG CSA2] and [AIS Methodology]: the Full layer scores the causally     */
/* visible compressed entries; [TDG CSA2]: the encoder compresses at ratio 2, the   */
/* decoder at ratio 1. Reading (the pages do not spell the rule out): a compressed  */
/* entry at ratio r summarises r consecutive tokens, entry j covering positions     */
/* r*j .. r*j + r - 1, and a token at position p may read entry j only once every   */
/* token the entry covers is at or before p. The window of the token at position p  */
/* is the positions p-W+1 .. p that exist (>= 0).                                  */
/* ------------------------------------------------------------------------------ */

/* Number of compressed entries visible to the token at position p (they are the
 * prefix 0 .. n-1): count the entries whose last covered position is <= p. */
ORC_EXPORT int64_t orc_prefill_visible(int64_t p, int ratio) {
    int64_t n = 0;
    while ((int64_t)ratio * n + ratio - 1 <= p) ++n;
    return n;
}

/* Window rows of query token t of a prefill chunk whose first token sits at position
 * q_pos0. The chunk's window buffer holds W-1+T rows, row i holding position
 * q_pos0 - (W-1) + i (the W-1 positions before the chunk, then the chunk's own). Writes
 * the buffer rows of the positions p-W+1 .. p (p = q_pos0 + t) that are >= 0, ascending,
 * and returns their number. */
ORC_EXPORT int orc_prefill_window_rows(int64_t q_pos0, int W, int64_t t, int32_t* rows_out) {
    const int64_t p = q_pos0 + t;
    const int64_t first_buffer_pos = q_pos0 - (W - 1);
    int n = 0;
    for (int64_t pos = p - W + 1; pos <= p; ++pos) {
        if (pos < 0) continue;
        rows_out[n++] = (int32_t)(pos - first_buffer_pos);
    }
    return n;
}

/* ------------------------------------------------------------------------------ */
/* KV compressor and indexer-K projection                                          */
/* [AIS Methodology in Plain English]: the V4.1 compressor no longer uses           */
/* overlapping source entries or absolute positional embeddings, and the indexer K  */
/* is derived by projecting the main KV entries. [TLB "How did DeepSeek V4.1 reduce */
/* the KV cache?"] names the compressed entries C_l and the compression weights     */
/* Z_l but its equation is lost. Reading (the plainest one these support):          */
/*  - entry j pools source tokens r*j .. r*j + r - 1 (no overlap, nothing added for  */
/*    position): per channel d, a softmax over those r tokens of the logits Z[t][d]  */
/*    weights their latents C[t][d];                                              */
/*  - the pooled latent is rounded to bf16 (the input format of quantize-on-write),  */
/*    quantized to FP4 as above, and projected by a [Di][D] matrix W to the indexer  */
/*    key k[e] = sum_d W[e][d] * x[d], which is then stored in the indexer format.    */
/* ------------------------------------------------------------------------------ */

/* bf16 encoder: round to nearest, ties to even, onto the binary format with 8
 * significant bits (exponent range of binary32; subnormal quantum 2^-133). Written from
 * that definition: scale the magnitude so that its 8 significant bits are the integer
 * part, round that to the nearest integer with ties to even, scale back. */
static double round_half_even(double v) {
    double f = floor(v);
    double d = v - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

ORC_EXPORT uint16_t orc_bf16_encode(double v) {
    const int sign = signbit(v) ? 1 : 0;
    double a = fabs(v);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else {
        int e;
        frexp(a, &e);                  /* a = f * 2^e, 0.5 <= f < 1 */
        int q = e - 8;                 /* quantum of an 8-significant-bit number */
        if (q < -133) q = -133;        /* subnormal range */
        r = round_half_even(ldexp(a, -q));
        r = ldexp(r, q);
    }
    float f = (float)r;                /* exact: r has at most 8 significant bits */
    if (sign) f = -f;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

ORC_EXPORT void orc_bf16_encode_many(const double* v, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_encode(v[i]);
}

/* Pooled latents of n_entries entries of D channels. Source token t of the entry group
 * has latent row C + t*ld and logit row Z + t*ld (bf16 bit patterns); entry j reads tokens
 * r*j .. r*j + r - 1. out[j*D + d] = sum_t softmax_t(Z[t][d]) * C[t][d], in double (the
 * largest logit is subtracted before exp, which leaves the softmax unchanged). */
ORC_EXPORT void orc_compress_entries(const uint16_t* Cs, const uint16_t* Zs, int64_t n_entries,
                                     int r, int D, int64_t ld, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n_entries; ++j) {
        for (int d = 0; d < D; ++d) {
            double zmax = -INFINITY;
            for (int t = 0; t < r; ++t) {
                double z = orc_bf16_value(Zs[(j * r + t) * ld + d]);
                if (z > zmax) zmax = z;
            }
            double den = 0.0, num = 0.0;
            for (int t = 0; t < r; ++t) {
                double a = exp(orc_bf16_value(Zs[(j * r + t) * ld + d]) - zmax);
                den += a;
                num += a * orc_bf16_value(Cs[(j * r + t) * ld + d]);
            }
            out[j * D + d] = num / den;
        }
    }
}

/* Indexer keys of n entries: out[i*Di + e] = sum_d W[e][d] * x[i*D + d], W as bf16 bit
 * patterns [Di][D] (row e = the weights of key channel e), in double. */
ORC_EXPORT void orc_project_keys(const double* x, int64_t n, int D, const uint16_t* W, int Di,
                                 double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        for (int e = 0; e < Di; ++e) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += orc_bf16_value(W[(int64_t)e * D + d]) * x[i * D + d];
            out[i * Di + e] = acc;
        }
    }
}

/* ------------------------------------------------------------------------------ */
/* Byte accounting                                                                 */
/* [AIS Main Findings], [TLB] Figure 1: 890 bytes of global KV per token.           */
/* [TDG CSA2]: encoder = 3 groups (1 Full + 5 Reuse) at ratio 2; decoder = 5 groups */
/* of 4 at ratio 1 whose first Full layer owns the only decoder KV (Reindex and     */
/* Reuse layers borrow it) [TLB "Three modes of CSA2"].                             */
/* Stored entry-sets per token = 3 * (1/2) + 1 * (1/1) = 2.5.                       */
/* ------------------------------------------------------------------------------ */

ORC_EXPORT int orc_main_entry_bytes(int D) { return D / 2 + D / 16; }

ORC_EXPORT double orc_kv_bytes_per_token(int D, double indexer_entry_bytes,
                                         int enc_full_layers, int enc_ratio,
                                         int dec_full_layers, int dec_ratio) {
    double sets = (double)enc_full_layers / enc_ratio + (double)dec_full_layers / dec_ratio;
    return sets * ((double)orc_main_entry_bytes(D) + indexer_entry_bytes);
}
