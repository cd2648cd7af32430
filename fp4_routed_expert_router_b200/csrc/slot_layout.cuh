// slot_layout.cuh -- byte layout of one expert inside its arena slot.
//
// The expert object of the checkpoint (10100.com article 151357339, sections
// "moe专家的容量瓶颈" and "SSD读取性能") holds w1, w3 codes [I, H/2], w2 codes
// [H, I/2] (two FP4 E2M1 codes per byte, low nibble = even K) and UE8M0
// scales s1, s3 [I, H/32], s2 [H, I/32] (one per 32 K), 18,800,640 bytes for
// the V4.1 shape.  The arena stores the same bytes, rearranged so that every
// unit of work the decode kernels stream is one contiguous, 16-byte aligned
// range (a single bulk copy), codes and scales together:
//
//  up blocks    for rt in [0, I/16), f in [0, H/KBu):         UB bytes each
//               [w1 16 rows x KBu/2][w3 16 rows x KBu/2][s1 16 x KBu/32][s3 16 x KBu/32]
//  down blocks  for nt in [0, H/16), f in [0, I/KBd), after all up blocks:  DB each
//               [w2 16 rows x KBd/2][s2 16 x KBd/32]
//
// KBu (K extent of an up block) is the largest of 512, 256, 128 dividing H;
// KBd is I/2 when that is a multiple of 128, else I.  Inside a block, code
// rows whose length is a multiple of 128 bytes are swizzled: in odd rows the
// two 64-byte halves of every 128-byte group are swapped, so that the 16-byte
// fragment loads of rows g and g+1 (one quarter-warp phase) use disjoint
// shared-memory banks without padding (rows of 64 mod 128 bytes alternate
// bank halves by themselves).  Each 32-bit word of codes is also re-encoded:
// magnitudes stay in place, the eight sign bits move (see fp4_decode.cuh).
// Scale bytes are stored as they are.
#pragma once
#include <cstddef>
#include <cstdint>

namespace moe {

struct SlotLayout {
    int H, I;
    int KBu, nfu;     // K extent of an up block, up blocks per 16-row tile (H / KBu)
    int KBd, nfd;     // same for down blocks (I / KBd)
    size_t UB, DB;    // bytes of one up block / one down block
    size_t up_bytes;  // all up blocks (= 2 * I * (H/2 + H/32))
    size_t bytes;     // whole slot
};

__host__ __device__ inline SlotLayout make_slot_layout(int H, int I) {
    SlotLayout L;
    L.H = H;
    L.I = I;
    L.KBu = (H % 512 == 0) ? 512 : (H % 256 == 0) ? 256 : 128;
    L.nfu = H / L.KBu;
    L.KBd = ((I / 2) % 128 == 0) ? I / 2 : I;
    L.nfd = I / L.KBd;
    L.UB = static_cast<size_t>(32) * (L.KBu / 2 + L.KBu / 32);
    L.DB = static_cast<size_t>(16) * (L.KBd / 2 + L.KBd / 32);
    L.up_bytes = static_cast<size_t>(I / 16) * L.nfu * L.UB;
    L.bytes = L.up_bytes + static_cast<size_t>(H / 16) * L.nfd * L.DB;
    return L;
}

// Swizzled position of 16-byte chunk q of code row r (row length rowbytes).
__host__ __device__ inline int swizzle_chunk(int q, int r, int rowbytes) {
    return (rowbytes % 128 == 0 && (r & 1)) ? (q ^ 4) : q;
}

}  // namespace moe
