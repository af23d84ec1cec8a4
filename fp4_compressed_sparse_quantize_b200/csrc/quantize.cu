// FP4 quantize-on-write of main-KV entries.
//
// "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (AI summary), Main
// Findings, FP4 format choice; "DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale
// LLM Serving", Quantization and Memory Management: E2M1 elements, one E4M3 scale per
// 16 channels, NVFP4 without the second-level global scale.
//
// One warp per 512-channel entry: lane l owns channels [16l, 16l+16), i.e. exactly one
// scale block. Loads are two 16-byte vectors per lane (a warp reads the 1 KiB row in one
// coalesced sweep); stores are 8 code bytes and 1 scale byte per lane (256 + 32 B per
// warp, contiguous). The work is trivially HBM-bound (1 KiB in, 288 B out per entry).
//
// Rounding: fp4_quantize_block16 (fp4_block.cuh).
#include "csa2_common.cuh"
#include "csa2_internal.h"
#include "fp4_block.cuh"

namespace csa2 {

__global__ void __launch_bounds__(256) quantize_kv_kernel(
    const __nv_bfloat16* kv, int B, int n_new, int64_t ld_kv, int64_t bstride_kv,
    const int32_t* dst_off, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, int64_t cap, int32_t* status) {
    grid_dep_launch();
    grid_dep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t entry = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (entry >= (int64_t)B * n_new) return;
    const int b = (int)(entry / n_new);
    const int i = (int)(entry - (int64_t)b * n_new);
    const int64_t dst = (int64_t)ld_dep(dst_off + b) + i;
    if (dst < 0 || dst >= cap) {
        if (lane == 0) set_status(status, CSA2_DEV_BAD_INDEX);
        return;
    }
    const __nv_bfloat16* row = kv + (int64_t)b * bstride_kv + (int64_t)i * ld_kv + lane * 16;
    uint4 v0 = ld_dep(reinterpret_cast<const uint4*>(row));
    uint4 v1 = ld_dep(reinterpret_cast<const uint4*>(row) + 1);
    uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float x[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        x[2 * k] = __uint_as_float(w[k] << 16);
        x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
    uint2 packed;
    uint8_t sc;
    fp4_quantize_block16(x, packed, sc);
    const int64_t e = (int64_t)b * cap + dst;
    reinterpret_cast<uint2*>(codes + e * CSA2_ENTRY_CODE_BYTES)[lane] = packed;
    scales[e * CSA2_ENTRY_SCALE_BYTES + lane] = sc;
}

cudaError_t launch_quantize_kv(const void* kv, int B, int n_new, int64_t ld_kv,
                               int64_t bstride_kv, const int32_t* dst_off, uint8_t* codes,
                               uint8_t* scales, int64_t cap, int32_t* status,
                               cudaStream_t stream) {
    const int64_t entries = (int64_t)B * n_new;
    if (entries == 0) return cudaSuccess;
    const int warps = 8;
    const int64_t grid = (entries + warps - 1) / warps;
    return launch_pdl(quantize_kv_kernel, dim3((unsigned)grid), dim3(warps * 32), 0, stream,
                      reinterpret_cast<const __nv_bfloat16*>(kv), B, n_new, ld_kv, bstride_kv,
                      dst_off, codes, scales, cap, status);
}

}  // namespace csa2
