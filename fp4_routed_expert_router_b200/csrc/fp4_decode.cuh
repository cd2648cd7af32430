// fp4_decode.cuh -- exact E2M1 x 2^(s-127) -> bf16 decode in registers.
//
// Storage format (10100.com article 151357339, section "moe专家的容量瓶颈"):
// FP4 E2M1 codes two per byte (low nibble = even K index) and one UE8M0
// scale s per 32 consecutive K values of a row.  A code c has sign bit 3 and
// magnitude index m = c & 7 with E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}.
// Every product E2M1 * 2^(s-127) has at most two significant bits, so it is
// an exact bf16 number; for 2 <= s <= 252 it is a *normal* bf16 number with
//   bits(m) = 0                                   for m = 0
//           = (s-1) << 7                          for m = 1  (0.5 * 2^(s-127))
//           = ((s-1) << 7) + m * 64               for m >= 2
// (exponent field s-1 .. s+2 and mantissa 0 or 0x40), plus the sign at bit 15.
//
// The decoder turns one 32-bit word (8 codes) into four bf16x2 words with
// byte permutes: a per-scale table of the 8 low bytes (l0:l1) and 8 high bytes
// (h0:h1) is indexed by the magnitudes with PRMT, the sign bits are OR-ed
// into the high bytes, and two more PRMTs interleave low and high bytes.
// To let one AND place four sign bits at once, the slot stores every code
// word re-encoded: nibble j keeps magnitude m_j in bits 0..2, and bit 3 of
// nibble 2j+1 / 2j carries the sign of code j / code 4+j (j = 0..3).  Cost:
// 13 integer instructions per 8 weights, no branches, exact.
#pragma once
#include <cstdint>

#ifndef __CUDACC__   // plain C++ host build (CPU tests of the decoder)
#define __host__
#define __device__
#define __forceinline__ inline
#endif

namespace moe {

// Per-scale byte tables, packed for PRMT: entries 0..3 in l0/h0, 4..7 in l1/h1.
struct Fp4Lut {
    uint32_t l0, l1, h0, h1;
};

__host__ __device__ inline Fp4Lut make_fp4_lut(uint32_t s) {
    uint32_t bits[8];
    uint32_t base = (s - 1u) << 7;
    bits[0] = 0;
    bits[1] = base;
    for (uint32_t m = 2; m < 8; ++m) bits[m] = base + m * 64u;
    Fp4Lut t;
    t.l0 = (bits[0] & 0xFF) | (bits[1] & 0xFF) << 8 | (bits[2] & 0xFF) << 16 | (bits[3] & 0xFF) << 24;
    t.l1 = (bits[4] & 0xFF) | (bits[5] & 0xFF) << 8 | (bits[6] & 0xFF) << 16 | (bits[7] & 0xFF) << 24;
    t.h0 = (bits[0] >> 8) | (bits[1] >> 8) << 8 | (bits[2] >> 8) << 16 | (bits[3] >> 8) << 24;
    t.h1 = (bits[4] >> 8) | (bits[5] >> 8) << 8 | (bits[6] >> 8) << 16 | (bits[7] >> 8) << 24;
    return t;
}

// Checkpoint code word -> slot code word (sign bits moved, magnitudes kept).
__host__ __device__ inline uint32_t fp4_reencode_word(uint32_t v) {
    uint32_t w = v & 0x77777777u;
    for (int j = 0; j < 4; ++j) {
        w |= ((v >> (4 * j + 3)) & 1u) << (8 * j + 7);        // sign of code j
        w |= ((v >> (16 + 4 * j + 3)) & 1u) << (8 * j + 3);   // sign of code 4+j
    }
    return w;
}

// PRMT in its default mode: result byte n = byte (s >> 4n) & 7 of {y:x}
// (selector values 0..7; the selectors used here never set bit 3).
__host__ __device__ __forceinline__ uint32_t byte_perm(uint32_t x, uint32_t y, uint32_t s) {
#ifdef __CUDA_ARCH__
    return __byte_perm(x, y, s);
#else
    uint64_t v = (static_cast<uint64_t>(y) << 32) | x;
    uint32_t r = 0;
    for (int n = 0; n < 4; ++n) r |= static_cast<uint32_t>((v >> (8 * ((s >> (4 * n)) & 7))) & 0xFF) << (8 * n);
    return r;
#endif
}

// Slot code word (8 codes k0..k7) -> four bf16x2 words (k0,k1) (k2,k3) (k4,k5)
// (k6,k7), lower K index in the low half.
__host__ __device__ __forceinline__ void fp4_decode8(uint32_t w, const Fp4Lut& t, uint32_t out[4]) {
    uint32_t m = w & 0x77777777u;
#ifdef __CUDA_ARCH__
    uint32_t mb = __umulhi(m, 0x10000u);     // m >> 16 on the multiply pipe
#else
    uint32_t mb = m >> 16;
#endif
    uint32_t loA = byte_perm(t.l0, t.l1, m);
    uint32_t hiA = byte_perm(t.h0, t.h1, m) | (w & 0x80808080u);
    uint32_t loB = byte_perm(t.l0, t.l1, mb);
    uint32_t hiB = byte_perm(t.h0, t.h1, mb) | ((w * 16u) & 0x80808080u);
    out[0] = byte_perm(loA, hiA, 0x5140);
    out[1] = byte_perm(loA, hiA, 0x7362);
    out[2] = byte_perm(loB, hiB, 0x5140);
    out[3] = byte_perm(loB, hiB, 0x7362);
}

}  // namespace moe
