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
// KBu (KBd), the K extent of an up (down) block, is 256 when it divides H
// (I), else 128: a block row is then 128 (64) bytes, and a 128-row tile of
// one block is exactly four (two) 64-wide K steps of the tensor-core path.
// Inside a block, code rows whose length is a multiple of 128 bytes are
// swizzled: 16-byte chunk q of row r sits at q ^ ((r & 7) ^ ((r & 1) << 2)).
// Eight consecutive rows then hold any given chunk in eight different bank
// groups (conflict-free 16-byte loads when each lane reads one row), and rows
// 2m, 2m+1 hold any aligned group of four chunks in opposite halves of the
// 128 bytes (conflict-free mma fragment loads: lanes read rows g, g+1 x four
// chunks).  Rows of 64 bytes are not swizzled (they alternate bank halves by
// themselves).  Each 32-bit word of codes is also re-encoded: magnitudes stay
// in place, the eight sign bits move (see fp4_decode.cuh).  Scale bytes are
// stored as they are.
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
    L.KBu = (H % 256 == 0) ? 256 : 128;
    L.nfu = H / L.KBu;
    L.KBd = (I % 256 == 0) ? 256 : 128;
    L.nfd = I / L.KBd;
    L.UB = static_cast<size_t>(32) * (L.KBu / 2 + L.KBu / 32);
    L.DB = static_cast<size_t>(16) * (L.KBd / 2 + L.KBd / 32);
    L.up_bytes = static_cast<size_t>(I / 16) * L.nfu * L.UB;
    L.bytes = L.up_bytes + static_cast<size_t>(H / 16) * L.nfd * L.DB;
    return L;
}

// Swizzled position of 16-byte chunk q of code row r (row length rowbytes).
__host__ __device__ inline int swizzle_chunk(int q, int r, int rowbytes) {
    return (rowbytes % 128 == 0) ? (q ^ ((r & 7) ^ ((r & 1) << 2))) : q;
}

}  // namespace moe
