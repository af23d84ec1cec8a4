// Persistent-cache records: one sequence's range of compressed entries moved between the
// device cache and a host buffer (pinned host memory, or bytes bound for a file), in a fixed
// byte format. "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression", Main
// Findings: the global KV cache is held in HBM, and a persistent KV cache (with its own
// footprint) exists besides it; the main-KV entry is E2M1 with an E4M3 scale per 16
// channels, i.e. 256 code bytes + 32 scale bytes = 288 B for 512 channels.
// "DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale LLM Serving", The KV Cache
// Revolution: the cache is accounted in bytes per token. This is the byte format and the
// copies only: no storage tier, eviction or time-to-live policy.
//
// Record = header (64 B) | codes [n][256] | scales [n][32] | (optional) indexer keys
// [n][key_bytes] (128 for E4M3 keys, 256 for bf16).
// The copies are plain cudaMemcpyAsync calls on the caller's stream, one per array.
#include <cstdint>
#include <cstring>

#include "csa2.h"
#include "csa2_internal.h"

namespace {

constexpr uint32_t kMagic = 0x32415343u;   // "CSA2" little-endian
constexpr uint32_t kVersion = 1u;

struct Header {
    uint32_t magic, version;
    int32_t d_main, d_index;
    int64_t lo, n;
    uint32_t key_bytes, entry_bytes;   // indexer-key bytes per entry (0: none), record bytes per entry
    uint8_t reserved[24];
};
static_assert(sizeof(Header) == 64, "record header is 64 bytes");

bool key_bytes_ok(int kb) { return kb == 0 || kb == CSA2_D_INDEX || kb == 2 * CSA2_D_INDEX; }

size_t entry_bytes(int kb) {
    return (size_t)CSA2_ENTRY_CODE_BYTES + CSA2_ENTRY_SCALE_BYTES + (size_t)kb;
}

// [lo, lo + n) inside [0, cap), tested without forming lo + n (a record's header is
// untrusted input and may hold values whose sum overflows)
bool range_ok(int64_t lo, int64_t n, int64_t cap) {
    return cap >= 1 && lo >= 0 && n >= 0 && n <= cap && lo <= cap - n;
}

// the byte offsets of sequence b's entries, (b * cap + cap) * (288 + key bytes), fit int64
bool offsets_ok(int b, int64_t cap, int kb) {
    const int64_t per = (int64_t)entry_bytes(kb);
    return b >= 0 && cap >= 1 && cap <= INT64_MAX / per / ((int64_t)b + 1);
}

}  // namespace

extern "C" {

CSA2_API size_t csa2_cache_record_bytes(int64_t n, int key_bytes) {
    if (n < 0 || !key_bytes_ok(key_bytes)) return 0;
    if ((uint64_t)n > (SIZE_MAX - sizeof(Header)) / entry_bytes(key_bytes)) return 0;
    return sizeof(Header) + (size_t)n * entry_bytes(key_bytes);
}

CSA2_API csa2_status_t csa2_cache_export(const uint8_t* codes, const uint8_t* scales,
                                         const void* k_I, int key_bytes, int64_t cap, int b,
                                         int64_t lo, int64_t n, void* host, size_t host_bytes,
                                         void* stream) {
    if (!codes || !scales || !host || !range_ok(lo, n, cap)) return CSA2_ERR_ARG;
    if (!key_bytes_ok(key_bytes) || (key_bytes > 0) != (k_I != nullptr)) return CSA2_ERR_ARG;
    if (!offsets_ok(b, cap, key_bytes)) return CSA2_ERR_ARG;
    const size_t need = csa2_cache_record_bytes(n, key_bytes);
    if (need == 0 || host_bytes < need) return CSA2_ERR_ARG;
    Header h;
    memset(&h, 0, sizeof h);
    h.magic = kMagic;
    h.version = kVersion;
    h.d_main = CSA2_D_MAIN;
    h.d_index = CSA2_D_INDEX;
    h.lo = lo;
    h.n = n;
    h.key_bytes = (uint32_t)key_bytes;
    h.entry_bytes = (uint32_t)entry_bytes(key_bytes);
    uint8_t* dst = static_cast<uint8_t*>(host);
    memcpy(dst, &h, sizeof h);
    if (n == 0) return CSA2_OK;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t e0 = (int64_t)b * cap + lo;
    size_t off = sizeof h;
    cudaError_t e = cudaMemcpyAsync(dst + off, codes + e0 * CSA2_ENTRY_CODE_BYTES,
                                    (size_t)n * CSA2_ENTRY_CODE_BYTES, cudaMemcpyDeviceToHost, st);
    off += (size_t)n * CSA2_ENTRY_CODE_BYTES;
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(dst + off, scales + e0 * CSA2_ENTRY_SCALE_BYTES,
                            (size_t)n * CSA2_ENTRY_SCALE_BYTES, cudaMemcpyDeviceToHost, st);
    off += (size_t)n * CSA2_ENTRY_SCALE_BYTES;
    if (e == cudaSuccess && key_bytes > 0)
        e = cudaMemcpyAsync(dst + off, static_cast<const uint8_t*>(k_I) + e0 * key_bytes,
                            (size_t)n * key_bytes, cudaMemcpyDeviceToHost, st);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

CSA2_API csa2_status_t csa2_cache_import(const void* host, size_t host_bytes, uint8_t* codes,
                                         uint8_t* scales, void* k_I, int64_t cap, int b,
                                         void* stream) {
    if (!host || !codes || !scales || cap < 1 || b < 0 || host_bytes < sizeof(Header))
        return CSA2_ERR_ARG;
    Header h;
    memcpy(&h, host, sizeof h);
    if (h.magic != kMagic || h.version != kVersion) return CSA2_ERR_ARG;
    if (h.d_main != CSA2_D_MAIN || h.d_index != CSA2_D_INDEX) return CSA2_ERR_UNSUPPORTED;
    // every header field is validated before any arithmetic on it
    if (h.key_bytes > 2u * CSA2_D_INDEX) return CSA2_ERR_ARG;
    const int kb = (int)h.key_bytes;
    if (!key_bytes_ok(kb) || !range_ok(h.lo, h.n, cap) || h.entry_bytes != entry_bytes(kb))
        return CSA2_ERR_ARG;
    if (!offsets_ok(b, cap, kb)) return CSA2_ERR_ARG;
    const size_t need = csa2_cache_record_bytes(h.n, kb);
    if (need == 0 || host_bytes < need) return CSA2_ERR_ARG;
    if ((kb > 0) != (k_I != nullptr)) return CSA2_ERR_ARG;   // keys in the record <=> a key cache
    if (h.n == 0) return CSA2_OK;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint8_t* src = static_cast<const uint8_t*>(host);
    const int64_t e0 = (int64_t)b * cap + h.lo;
    size_t off = sizeof h;
    cudaError_t e = cudaMemcpyAsync(codes + e0 * CSA2_ENTRY_CODE_BYTES, src + off,
                                    (size_t)h.n * CSA2_ENTRY_CODE_BYTES, cudaMemcpyHostToDevice, st);
    off += (size_t)h.n * CSA2_ENTRY_CODE_BYTES;
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(scales + e0 * CSA2_ENTRY_SCALE_BYTES, src + off,
                            (size_t)h.n * CSA2_ENTRY_SCALE_BYTES, cudaMemcpyHostToDevice, st);
    off += (size_t)h.n * CSA2_ENTRY_SCALE_BYTES;
    if (e == cudaSuccess && kb > 0)
        e = cudaMemcpyAsync(static_cast<uint8_t*>(k_I) + e0 * kb, src + off, (size_t)h.n * kb,
                            cudaMemcpyHostToDevice, st);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

}  // extern "C"
