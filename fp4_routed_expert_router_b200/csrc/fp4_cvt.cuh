// fp4_cvt.cuh -- exact FP4 E2M1 -> f16 decode, UE8M0 block scales and exact
// power-of-two prescaling of bf16 activations into f16.
//
// Storage format (10100.com article 151357339, section "moe专家的容量瓶颈"):
// FP4 E2M1 codes, two per byte (low nibble = even K index), and one UE8M0
// scale s per 32 consecutive K of a weight row, W = E2M1(code) * 2^(s-127).
//
// Decode.  sm_100a converts a byte of two E2M1 codes to an f16x2 pair in one
// instruction (cvt.rn.f16x2.e2m1x2; low nibble -> low half).  Every E2M1
// value (0, +-0.5 .. +-6) is an f16 number, so the conversion is exact.  The
// scale is not applied to the f16 weights: an MMA covers 16 K of a single
// 32-K block, and the fp32 block result is multiplied by 2^(s-127) (a normal
// fp32 power of two for 2 <= s <= 252), which is exact.
//
// Activations.  The tensor-core operands are f16, the activations bf16.  A
// bf16 value has 8 significant bits and f16 11, so v * 2^sigma is exactly an
// f16 number whenever it lies in [2^-17, 2^16): sigma is chosen per row (or
// per 32-K block) from the largest magnitude m as sigma = 14 - floor(log2 m),
// putting m in [2^14, 2^15).  Only entries below m * 2^-31 lose bits (they
// round to the f16 subnormal grid), an error below 2^-25 of m.  The product
// is scaled back by 2^-sigma in fp32, again a power of two.
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

// 2^(s-127) for the scale byte j (0..3) of a little-endian word of scales.
__device__ __forceinline__ float ue8m0_mult(uint32_t word, int j) {
    return __uint_as_float(__byte_perm(word, 0u, 0x4440u | static_cast<uint32_t>(j)) << 23);
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

// mma.sync m16n8k16, f16 x f16 -> fp32.  Accumulate into d, or start from 0.
__device__ __forceinline__ void mma_f16_acc(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16_zero(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

}  // namespace moe
