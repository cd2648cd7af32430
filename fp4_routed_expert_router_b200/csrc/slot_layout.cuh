// slot_layout.cuh -- byte layout of one expert inside its arena slot.
//
// The expert object of the checkpoint (10100.com article 151357339, sections
// "moe专家的容量瓶颈" and "SSD读取性能") holds w1, w3 codes [I, H/2], w2 codes
// [H, I/2] (two FP4 E2M1 codes per byte, low nibble = even K) and UE8M0
// scales s1, s3 [I, H/32], s2 [H, I/32] (one per 32 K), 18,800,640 bytes for
// the V4.1 shape.  The arena stores the same bytes, rearranged so that every
// unit of work the kernels stream is one contiguous, 16-byte aligned range
// (a single bulk copy), codes and scales together:
//
//  up blocks    for rt in [0, I/16), f in [0, H/KBu):         UB bytes each
//               [w1 16 rows x KBu/2][w3 16 rows x KBu/2][s1 16 x KBu/32][s3 16 x KBu/32]
//  down blocks  for nt in [0, H/16), f in [0, I/KBd), after all up blocks:  DB each
//               [w2 16 rows x KBd/2][s2 16 x KBd/32]
//
// KBu (KBd), the K extent of an up (down) block, is 256 when it divides H
// (I), else 128: a block row is 128 (64) bytes, i.e. two (one) groups of
// 128 K.  Scale bytes are stored as they are, row-major inside the block.
//
// Code bytes keep the checkpoint's nibbles (E2M1, sign in bit 3, low nibble
// = even K), but inside each 64-byte group of a row (128 K = four 32-K scale
// blocks) the sixteen 32-bit words are transposed: 16-byte chunk c of the
// group holds, as its words j = 0..3, the codes K = 32j + 8c .. 32j + 8c + 7
// of the group.  A lane that reads chunk c therefore gets eight consecutive
// codes of each of the four scale blocks -- exactly the K slice that lane
// column c of an mma.sync m16n8k16 fragment owns when one MMA covers 16 K of
// a single scale block (decode_fused.cuh), and four 16-byte loads give one
// row all 128 codes in K order (tcgen05 path).
//
// Rows whose length is a multiple of 128 bytes are swizzled: chunk q of code
// row r sits at q ^ ((r & 7) ^ ((r & 1) << 2)).  Eight consecutive rows then
// hold any given chunk in eight different 16-byte bank groups (conflict-free
// when each lane reads one row), and rows 2m, 2m+1 hold any aligned group of
// four chunks in opposite halves of the 128 bytes (conflict-free fragment
// loads: lanes read rows g, g+1 x four chunks).  64-byte rows are not
// swizzled (consecutive rows alternate bank halves by themselves).
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

// Byte offset, inside a block's code rows (row length rowbytes), of the
// 32-bit word holding codes K = 128 q + 32 j + 8 c .. +7 of row r.
__host__ __device__ inline int code_word_offset(int r, int q, int j, int c, int rowbytes) {
    return r * rowbytes + swizzle_chunk(4 * q + c, r, rowbytes) * 16 + 4 * j;
}

// Loader mapping, thread i of the relayout (moe_fp4_api.cu load_slot_kernel)
// for i < 3 * I * H / 32: the 16-byte code chunk it writes.  The checkpoint
// object holds w1, w3 codes [I, H/2], then w2 codes [H, I/2].  Returns the
// offset in the object of the chunk's word 0 (words j = 0..3 are 16 bytes
// apart there: codes K = 128 q + 32 j + 8 c .. +7 of a 64-byte row group) and
// the chunk's offset in the slot.
__host__ __device__ inline void slot_code_chunk(const SlotLayout& L, size_t i, size_t* src, size_t* dst) {
    const size_t H = L.H, I = L.I;
    const size_t n13 = I * H / 32;
    size_t r, qq, KB, nf, srow, base;
    if (i < 2 * n13) {                                       // w1 / w3 chunk
        const size_t mat = i / n13, rem = i - mat * n13;
        r = rem / (H / 32);
        qq = rem - r * (H / 32);
        KB = L.KBu;
        nf = L.nfu;
        srow = mat * (I * H / 2) + r * (H / 2);
        base = mat * 16 * (KB / 2);
    } else {                                                 // w2 chunk
        const size_t rem = i - 2 * n13;
        r = rem / (I / 32);
        qq = rem - r * (I / 32);
        KB = L.KBd;
        nf = L.nfd;
        srow = I * H + r * (I / 2);
        base = 0;
    }
    const size_t f = qq / (KB / 32), qi = qq - f * (KB / 32);
    const int q = static_cast<int>(qi / 4), c = static_cast<int>(qi % 4);
    *src = srow + f * (KB / 2) + 64 * q + 4 * c;
    const size_t block = (i < 2 * n13) ? ((r / 16) * nf + f) * L.UB : L.up_bytes + ((r / 16) * nf + f) * L.DB;
    *dst = block + base + code_word_offset(static_cast<int>(r % 16), q, 0, c, static_cast<int>(KB / 2));
}

// Loader mapping for scale byte b < 3 * I * H / 32 (object order s1, s3, s2,
// each row-major): its offset in the slot.
__host__ __device__ inline size_t slot_scale_byte(const SlotLayout& L, size_t b) {
    const size_t H = L.H, I = L.I;
    const size_t s13 = I * H / 32;
    if (b < 2 * s13) {
        const size_t mat = b / s13, rem = b - mat * s13;
        const size_t r = rem / (H / 32), q = rem - r * (H / 32);
        const size_t f = q / (L.KBu / 32), qi = q - f * (L.KBu / 32);
        return ((r / 16) * L.nfu + f) * L.UB + 32 * (L.KBu / 2) + mat * 16 * (L.KBu / 32) + (r % 16) * (L.KBu / 32) + qi;
    }
    const size_t rem = b - 2 * s13;
    const size_t r = rem / (I / 32), q = rem - r * (I / 32);
    const size_t f = q / (L.KBd / 32), qi = q - f * (L.KBd / 32);
    return L.up_bytes + ((r / 16) * L.nfd + f) * L.DB + 16 * (L.KBd / 2) + (r % 16) * (L.KBd / 32) + qi;
}

}  // namespace moe
