// FP4 block quantizer shared by quantize-on-write and the compressor.
//
// "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (AI summary), Main
// Findings, FP4 format choice: E2M1 elements with one E4M3 scale per 16 channels, NVFP4
// without the second-level global scale.
//
// Rounding: the scale is E4M3(amax / 6) and each magnitude is E2M1(|x| / s), both with
// round-to-nearest-even and saturation (cvt.rn.satfinite), where the quotients are IEEE
// fp32 divisions. Neither quotient can land on a rounding midpoint unless the exact
// quotient does: the numerator has 8 significant bits (x is a bf16 value) and the divisor
// (6, or an E4M3 value with at most 4) leaves a non-dyadic quotient far from every dyadic
// midpoint, and a dyadic quotient is exact in fp32. A reciprocal-multiply would not have
// that property.
#pragma once

#include "csa2_common.cuh"

namespace csa2 {

// One 16-channel block of bf16 values (held as floats). codes: 8 bytes, channel 2k in the
// low nibble of byte k; the sign bit of each code is the sign bit of its value.
__device__ __forceinline__ void fp4_quantize_block16(const float (&x)[16], uint2& codes,
                                                     uint8_t& scale) {
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(x[k]));
    const float q = __fdiv_rn(amax, 6.0f);
    uint16_t sc2;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(sc2) : "f"(0.0f), "f"(q));
    scale = (uint8_t)(sc2 & 0xFF);
    const float s = e4m3_to_float(scale);
    uint32_t packed_lo = 0, packed_hi = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float a = (s > 0.f) ? __fdiv_rn(fabsf(x[2 * k]), s) : 0.f;
        const float c = (s > 0.f) ? __fdiv_rn(fabsf(x[2 * k + 1]), s) : 0.f;
        uint16_t byte;
        asm("{\n\t.reg .b8 t;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
            "cvt.u16.u8 %0, t;\n\t}"
            : "=h"(byte)
            : "f"(c), "f"(a));
        uint32_t bb = byte & 0x77u;  // magnitudes only
        bb |= (__float_as_uint(x[2 * k]) >> 31) << 3;
        bb |= (__float_as_uint(x[2 * k + 1]) >> 31) << 7;
        if (k < 4)
            packed_lo |= bb << (8 * k);
        else
            packed_hi |= bb << (8 * (k - 4));
    }
    codes = make_uint2(packed_lo, packed_hi);
}

}  // namespace csa2
