// fp4_cvt.cuh -- exact FP4 E2M1 -> f16 decode and exact power-of-two
// prescaling of bf16 activations into f16, for the f16 tcgen05 path.
//
// Storage format (10100.com article 151357339, section "moe专家的容量瓶颈"):
// FP4 E2M1 codes, two per byte (low nibble = even K index), and one UE8M0
// scale s per 32 consecutive K of a weight row, W = E2M1(code) * 2^(s-127).
//
// Decode.  sm_100a converts a byte of two E2M1 codes to an f16x2 pair in one
// instruction (cvt.rn.f16x2.e2m1x2; low nibble -> low half).  Every E2M1
// value (0, +-0.5 .. +-6) is an f16 number, so the conversion is exact; the
// f16 path then multiplies a block by 2^(s - s_ref) of its row (exact while
// the row's scales span at most 23 binades) and the fp32 result by
// 2^(s_ref - 127).
//
// Activations.  The tensor-core operands are f16, the activations bf16.  A
// bf16 value has 8 significant bits and f16 11, so v * 2^sigma is exactly an
// f16 number whenever it lies in [2^-17, 2^16): sigma is chosen per row from
// the largest magnitude m as sigma = 14 - floor(log2 m), putting m in
// [2^14, 2^15).  Only entries below m * 2^-31 lose bits (they round to the
// f16 subnormal grid), an error below 2^-25 of m.  The product is scaled
// back by 2^-sigma in fp32, again a power of two.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace moe {

// Eight E2M1 codes (one 32-bit word, byte b = codes 2b, 2b+1) -> four f16x2.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t o[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
        : "r"(w));
}

// sigma for a row (or block) whose largest |bf16| has the bit pattern
// `maxbits` (sign cleared).  Zero rows and rows holding inf/NaN get sigma 0
// (nothing to scale; inf/NaN propagate); sigma is clamped to [-113, 126] so
// that 2^sigma and 2^-sigma are normal fp32 numbers.
__device__ __forceinline__ int prescale_sigma(uint32_t maxbits) {
    const int field = static_cast<int>(maxbits >> 7);
    if (maxbits == 0 || field >= 255) return 0;
    const int s = 141 - (field == 0 ? 1 : field);   // 14 - (field - 127); bf16 subnormals as 2^-126
    return s > 126 ? 126 : s;
}
__device__ __forceinline__ float pow2i(int e) {     // 2^e, -126 <= e <= 127
    return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

// Two fp32 values -> f16x2 (round to nearest even), lower K in the low half.
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// A bf16x2 word scaled by `mult` (a power of two) -> f16x2.
__device__ __forceinline__ uint32_t bf16x2_scaled_to_f16x2(uint32_t v, float mult) {
    const float lo = __uint_as_float(v << 16) * mult;
    const float hi = __uint_as_float(v & 0xFFFF0000u) * mult;
    return f32x2_to_f16x2(lo, hi);
}

__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t v) {
    const uint32_t a = v & 0x7FFFu, b = (v >> 16) & 0x7FFFu;
    return a > b ? a : b;
}

}  // namespace moe
