// FP4 (E2M1) quantisation of one group of 16 values with an E4M3 scale, shared by
// the bulk quantiser (fp4_quant.cu) and the decode-step cache append
// (cache_append.cu), so both write the same bytes.
//
// Format: "DeepSeek-V4.1 Flash Pushes KV Cache Compression for Agent Workloads",
// section "Ana Gelisme" (E2M1 values, E4M3 scale per 16 channels). Rounding
// rules fixed by this library: scale = E4M3 nearest amax/6 (ties to even,
// saturating at 448); code = E2M1 nearest x/scale (ties to even, saturating
// at +-6); zero scale -> zero codes; no -0.
// The E2M1 decision compares |x| with the seven midpoints times the scale; each
// product has at most 7 significant bits and is exact in fp32, so the decision
// is the one the exact quotient gives. Strict and non-strict comparisons
// alternate so that ties go to the even code.
#pragma once

#include <cstdint>

namespace csa2 {

__device__ __forceinline__ uint32_t e4m3_from_f32_rne_sat(float v) {
    // Hardware conversion: round to nearest even, clamp to the largest finite
    // value (448). The value is non-negative here.
    uint16_t packed;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(packed) : "f"(0.0f), "f"(v));
    return packed & 0xFFu;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    float v = (e == 0) ? (float)m * 0.001953125f                        // m * 2^-9
                       : __uint_as_float(((e + 120u) << 23) | (m << 20)); // 2^(e-7) * (1 + m/8)
    return (b & 0x80u) ? -v : v;
}

// Codes of 16 values (element i in nibble i: packed[i / 8] bits 4 (i % 8)..) and the
// scale byte.
__device__ __forceinline__ uint32_t fp4_quantize_group16(const float (&v)[16], uint32_t (&packed)[2]) {
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const uint32_t sc = e4m3_from_f32_rne_sat(__fdiv_rn(amax, 6.0f));
    const float s = e4m3_to_f32(sc);
    packed[0] = packed[1] = 0u;
    if (s > 0.f) {
        const float t1 = 0.25f * s, t2 = 0.75f * s, t3 = 1.25f * s, t4 = 1.75f * s;
        const float t5 = 2.5f * s, t6 = 3.5f * s, t7 = 5.0f * s;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float a = fabsf(v[i]);
            uint32_t c = (uint32_t)(a > t1) + (uint32_t)(a >= t2) + (uint32_t)(a > t3) + (uint32_t)(a >= t4) +
                         (uint32_t)(a > t5) + (uint32_t)(a >= t6) + (uint32_t)(a > t7);
            if (v[i] < 0.f && c != 0u) c |= 8u;
            packed[i >> 3] |= c << (4 * (i & 7));
        }
    }
    return sc;
}

}  // namespace csa2
