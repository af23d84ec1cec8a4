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

// Compact 68-byte indexer keys: E2M1 codes of a 128-channel key (64 bytes, channel 2k in
// the low nibble of byte k) and one fp32 scale = amax / 6. "DeepSeek-V4.1-Flash: Pushing
// the Limits of KV Cache Compression" (AI summary), Main Findings: 890 bytes of global KV
// per token, i.e. 68 bytes per indexer key next to the 288-byte FP4 main entry. Decisions in
// IEEE fp32: s = amax / 6 (div.rn), magnitude = E2M1_RNE_sat(|x| / s) (div.rn, then
// cvt.rn.satfinite), sign copied from x. One warp per key, lane l owns channels [4l, 4l+4).
__global__ void __launch_bounds__(256) quantize_keys_fp4_kernel(
    const __nv_bfloat16* k, int B, int n_new, int64_t ld, int64_t bstride,
    const int32_t* dst_off, uint8_t* __restrict__ codes, float* __restrict__ scales,
    int64_t cap, int32_t* status) {
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
    const uint2 v = ld_dep(reinterpret_cast<const uint2*>(k + (int64_t)b * bstride +
                                                          (int64_t)i * ld + lane * 4));
    const float x[4] = {__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                        __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u)};
    float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = __fdiv_rn(amax, 6.0f);
    uint32_t two = 0;
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
        const float a = (s > 0.f) ? __fdiv_rn(fabsf(x[2 * k2]), s) : 0.f;
        const float c = (s > 0.f) ? __fdiv_rn(fabsf(x[2 * k2 + 1]), s) : 0.f;
        uint16_t byte;
        asm("{\n\t.reg .b8 t;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
            "cvt.u16.u8 %0, t;\n\t}"
            : "=h"(byte)
            : "f"(c), "f"(a));
        uint32_t bb = byte & 0x77u;
        bb |= (__float_as_uint(x[2 * k2]) >> 31) << 3;
        bb |= (__float_as_uint(x[2 * k2 + 1]) >> 31) << 7;
        two |= bb << (8 * k2);
    }
    const int64_t e = (int64_t)b * cap + dst;
    reinterpret_cast<uint16_t*>(codes + e * CSA2_FP4KEY_CODE_BYTES)[lane] = (uint16_t)two;
    if (lane == 0) scales[e] = s;
}

cudaError_t launch_quantize_keys_fp4(const void* k, int B, int n_new, int64_t ld,
                                     int64_t bstride, const int32_t* dst_off, uint8_t* codes,
                                     float* scales, int64_t cap, int32_t* status,
                                     cudaStream_t stream) {
    const int64_t entries = (int64_t)B * n_new;
    if (entries == 0) return cudaSuccess;
    const int warps = 8;
    const int64_t grid = (entries + warps - 1) / warps;
    return launch_pdl(quantize_keys_fp4_kernel, dim3((unsigned)grid), dim3(warps * 32), 0, stream,
                      reinterpret_cast<const __nv_bfloat16*>(k), B, n_new, ld, bstride, dst_off,
                      codes, scales, cap, status);
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
