// slot_layout.cuh -- byte layout of one expert inside its arena slot.
//
// The expert object of the checkpoint (10100.com article 151357339, sections
// "moe专家的容量瓶颈" and "SSD读取性能") holds w1, w3 codes [I, H/2], w2 codes
// [H, I/2] (two FP4 E2M1 codes per byte, low nibble = even K) and UE8M0
// scales s1, s3 [I, H/32], s2 [H, I/32] (one per 32 K), 18,800,640 bytes for
// the V4.1 shape.  The arena holds the same bytes regrouped into units: a
// unit is one 128-row x 128-K tile of one matrix, codes and scales together,
// 8,704 contiguous bytes that one bulk copy moves into shared memory:
//
//  up units     for mat in {w1, w3}, rt in [0, I/128), ku in [0, H/128)
//  down units   for nt in [0, H/128), ku in [0, I/128), after all up units
//
//  unit bytes   [codes 8192][scale atom 512]
//    codes      row r, K k (0..127): byte (r/8)*512 + (k/32)*128 + (r%8)*16 + (k%32)/2,
//               nibble k & 1 (low = even K, as in the checkpoint)
//    scales     row r, 32-K block b (0..3): byte 8192 + (r%32)*16 + (r/32)*4 + b
//
// The codes are the K-major, no-swizzle canonical operand layout of the
// 5th-generation tensor cores for 4-bit types: a core matrix is 8 rows x 16
// bytes (32 codes = one scale block) stored as 128 contiguous bytes; core
// matrices adjacent in K are 128 bytes apart (leading byte offset) and those
// adjacent in M 512 bytes apart (stride byte offset).  A tcgen05.mma
// kind::mxf4 with K = 64 reads two core-matrix columns: unit bytes +256 j for
// step j.  The scale atom is the 32-row x 16-byte tile that tcgen05.cp
// .32x128b.warpx4 copies into tensor memory, where TMEM lane r%32 (in every
// lane quadrant) column r/32 then holds row r's four scale bytes -- the
// arrangement the block-scaled MMA reads (byte 2j, 2j+1 for step j).  The
// f16 dequantising path of prefill reads the same units: a thread takes one
// row's 16-byte chunk of one scale block and the block's scale byte.
#pragma once
#include <cstddef>
#include <cstdint>

namespace moe {

constexpr int kUnitRows = 128;
constexpr int kUnitK = 128;
constexpr int kUnitCodeBytes = kUnitRows * kUnitK / 2;                 // 8192
constexpr int kUnitScaleBytes = kUnitRows * kUnitK / 32;               // 512
constexpr int kUnitBytes = kUnitCodeBytes + kUnitScaleBytes;           // 8704

struct SlotLayout {
    int H, I;
    int KU;           // up units along K (H / 128)
    int RT;           // up row tiles (I / 128)
    int KD;           // down units along K (I / 128)
    int NT;           // down row tiles (H / 128)
    size_t up_bytes;  // all up units
    size_t bytes;     // whole slot
};

__host__ __device__ inline SlotLayout make_slot_layout(int H, int I) {
    SlotLayout L;
    L.H = H;
    L.I = I;
    L.KU = H / kUnitK;
    L.RT = I / kUnitRows;
    L.KD = I / kUnitK;
    L.NT = H / kUnitRows;
    L.up_bytes = static_cast<size_t>(2) * L.RT * L.KU * kUnitBytes;
    L.bytes = L.up_bytes + static_cast<size_t>(L.NT) * L.KD * kUnitBytes;
    return L;
}

// Offset of up unit (mat 0 = w1 / 1 = w3, row tile rt, K unit ku) in the slot.
__host__ __device__ inline size_t up_unit_offset(const SlotLayout& L, int mat, int rt, int ku) {
    return (static_cast<size_t>(mat * L.RT + rt) * L.KU + ku) * kUnitBytes;
}
// Offset of down unit (row tile nt, K unit ku) in the slot.
__host__ __device__ inline size_t down_unit_offset(const SlotLayout& L, int nt, int ku) {
    return L.up_bytes + (static_cast<size_t>(nt) * L.KD + ku) * kUnitBytes;
}
// Byte of a unit holding codes K = 32 c .. 32 c + 31 of row r (16 bytes from there).
__host__ __device__ inline int unit_code_chunk(int r, int c) { return (r >> 3) * 512 + c * 128 + (r & 7) * 16; }
// Byte of a unit holding the scale of row r, 32-K block b.
__host__ __device__ inline int unit_scale_byte(int r, int b) {
    return kUnitCodeBytes + (r & 31) * 16 + (r >> 5) * 4 + b;
}

// Loader mapping, thread i < 3 * I * H / 32 of the relayout: the 16-byte
// code chunk it moves (32 codes of one row and one scale block, contiguous
// in both places).  The checkpoint object holds w1, w3 codes [I, H/2], then
// w2 codes [H, I/2].  Returns the chunk's offset in the object and in the slot.
__host__ __device__ inline void slot_code_chunk(const SlotLayout& L, size_t i, size_t* src, size_t* dst) {
    const size_t H = L.H, I = L.I;
    const size_t n13 = I * H / 32;
    if (i < 2 * n13) {                                       // w1 / w3 chunk
        const size_t mat = i / n13, rem = i - mat * n13;
        const size_t r = rem / (H / 32), c = rem - r * (H / 32);
        *src = mat * (I * H / 2) + r * (H / 2) + 16 * c;
        *dst = up_unit_offset(L, static_cast<int>(mat), static_cast<int>(r / 128), static_cast<int>(c / 4)) +
               unit_code_chunk(static_cast<int>(r % 128), static_cast<int>(c % 4));
    } else {                                                 // w2 chunk
        const size_t rem = i - 2 * n13;
        const size_t r = rem / (I / 32), c = rem - r * (I / 32);
        *src = I * H + r * (I / 2) + 16 * c;
        *dst = down_unit_offset(L, static_cast<int>(r / 128), static_cast<int>(c / 4)) +
               unit_code_chunk(static_cast<int>(r % 128), static_cast<int>(c % 4));
    }
}

// Loader mapping for scale byte b < 3 * I * H / 32 (object order s1, s3, s2,
// each row-major): its offset in the slot.
__host__ __device__ inline size_t slot_scale_byte(const SlotLayout& L, size_t b) {
    const size_t H = L.H, I = L.I;
    const size_t s13 = I * H / 32;
    if (b < 2 * s13) {
        const size_t mat = b / s13, rem = b - mat * s13;
        const size_t r = rem / (H / 32), q = rem - r * (H / 32);
        return up_unit_offset(L, static_cast<int>(mat), static_cast<int>(r / 128), static_cast<int>(q / 4)) +
               unit_scale_byte(static_cast<int>(r % 128), static_cast<int>(q % 4));
    }
    const size_t rem = b - 2 * s13;
    const size_t r = rem / (I / 32), q = rem - r * (I / 32);
    return down_unit_offset(L, static_cast<int>(r / 128), static_cast<int>(q / 4)) +
           unit_scale_byte(static_cast<int>(r % 128), static_cast<int>(q % 4));
}

}  // namespace moe
