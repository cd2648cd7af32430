"""The slot layout (csrc/slot_layout.cuh) on CPU: sizes of the V4.1 and tiny
shapes; the relayout (the loader's per-thread mapping) writes every slot byte
exactly once, and reading a slot the way the kernels address it (code word
of (row, 128-K group, 32-K block, lane column), scale byte of (row, block))
gives back every checkpoint nibble and scale; the row swizzle is a
permutation inside every 128-byte group, and the two read patterns the
kernels use hit eight different 16-byte bank groups per 128-byte
shared-memory wavefront (no bank conflicts):
  decode fragments: a quarter warp reads rows g, g+1 (g even) x the four lane
                    columns of one 128-K group;
  tcgen05 dequant: eight consecutive rows read the same logical chunk."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_DRIVER = r"""
#define __host__
#define __device__
#include "slot_layout.cuh"
#include <cstdio>
#include <initializer_list>
using namespace moe;
int main() {
    int H, I;
    while (std::scanf("%d %d", &H, &I) == 2) {
        SlotLayout L = make_slot_layout(H, I);
        std::printf("%d %d %d %d %zu %zu %zu %zu\n", L.KBu, L.nfu, L.KBd, L.nfd, L.UB, L.DB, L.up_bytes, L.bytes);
    }
    // swizzle table for 128-byte rows and 64-byte rows
    for (int rowbytes : {128, 256, 64})
        for (int r = 0; r < 16; ++r) {
            for (int q = 0; q < rowbytes / 16; ++q) std::printf("%d ", swizzle_chunk(q, r, rowbytes));
            std::printf("\n");
        }
    return 0;
}
"""


_ROUNDTRIP = r"""
#define __host__
#define __device__
#include "slot_layout.cuh"
#include <cstdio>
#include <cstdint>
#include <vector>
using namespace moe;
// stdin: "H I" lines.  For a pseudo-random checkpoint object: build the slot
// with the loader's mapping, then read every (matrix, row, K) code and every
// scale back with the kernels' addressing.  stdout: slot bytes, bytes not
// written exactly once, wrong codes, wrong scales.
int main() {
    int H, I;
    while (std::scanf("%d %d", &H, &I) == 2) {
        const SlotLayout L = make_slot_layout(H, I);
        const size_t IH = static_cast<size_t>(I) * H;
        std::vector<uint8_t> ck(3 * IH / 2 + 3 * IH / 32), slot(L.bytes, 0), hit(L.bytes, 0);
        uint64_t st = 0x9E3779B97F4A7C15ull;
        for (auto& v : ck) { st = st * 6364136223846793005ull + 1442695040888963407ull; v = uint8_t(st >> 56); }
        for (size_t i = 0; i < 3 * IH / 32; ++i) {
            size_t s, d;
            slot_code_chunk(L, i, &s, &d);
            for (int j = 0; j < 4; ++j)
                for (int b = 0; b < 4; ++b) { slot[d + 4 * j + b] = ck[s + 16 * j + b]; hit[d + 4 * j + b]++; }
        }
        for (size_t b = 0; b < 3 * IH / 32; ++b) {
            const size_t d = slot_scale_byte(L, b);
            slot[d] = ck[3 * IH / 2 + b];
            hit[d]++;
        }
        size_t cover = 0, bad_code = 0, bad_scale = 0;
        for (uint8_t h : hit) cover += (h != 1);
        for (int mat = 0; mat < 3; ++mat) {
            const int rows = mat < 2 ? I : H, K = mat < 2 ? H : I;
            const int KB = mat < 2 ? L.KBu : L.KBd, nf = mat < 2 ? L.nfu : L.nfd;
            const int rowbytes = KB / 2, sb = KB / 32;
            for (int r = 0; r < rows; ++r)
                for (int k = 0; k < K; ++k) {
                    const int f = k / KB, kk = k % KB, q = kk / 128, j = (kk % 128) / 32, c = (kk % 32) / 8;
                    const int e = kk % 8;
                    const size_t blk = mat < 2 ? (size_t(r / 16) * nf + f) * L.UB
                                               : L.up_bytes + (size_t(r / 16) * nf + f) * L.DB;
                    const size_t codes = blk + (mat == 1 ? 16 * rowbytes : 0);
                    const uint8_t byte = slot[codes + code_word_offset(r % 16, q, j, c, rowbytes) + e / 2];
                    const size_t co = (mat < 2 ? size_t(mat) * IH / 2 + size_t(r) * (H / 2)
                                               : IH + size_t(r) * (I / 2)) + k / 2;
                    bad_code += ((byte >> (4 * (e & 1))) & 15) != ((ck[co] >> (4 * (k & 1))) & 15);
                    if (k % 32 == 0) {
                        const size_t scl = mat < 2 ? blk + 32 * rowbytes + mat * 16 * sb : blk + 16 * rowbytes;
                        const size_t so = 3 * IH / 2 + (mat < 2 ? size_t(mat) * IH / 32 + size_t(r) * (H / 32)
                                                                : 2 * IH / 32 + size_t(r) * (I / 32)) + k / 32;
                        bad_scale += slot[scl + (r % 16) * sb + kk / 32] != ck[so];
                    }
                }
        }
        std::printf("%zu %zu %zu %zu\n", L.bytes, cover, bad_code, bad_scale);
    }
    return 0;
}
"""


def test_relayout_roundtrip_reads_back_every_code_and_scale(tmp_path):
    src, exe = tmp_path / "rt.cpp", tmp_path / "rt"
    src.write_text(_ROUNDTRIP)
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I",
                           os.path.join(ROOT, "fp4_routed_expert_router_b200", "csrc"), str(src), "-o", str(exe)])
    out = subprocess.run([str(exe)], input="5120 2304\n256 128\n384 256\n", capture_output=True, text=True,
                         check=True).stdout.splitlines()
    rows = [list(map(int, l.split())) for l in out]
    assert rows[0][0] == 18_800_640
    for nbytes, cover, bad_code, bad_scale in rows:
        assert (cover, bad_code, bad_scale) == (0, 0, 0), (nbytes, cover, bad_code, bad_scale)


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    d = tmp_path_factory.mktemp("layout")
    src, exe = d / "d.cpp", d / "d"
    src.write_text(_DRIVER)
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I",
                           os.path.join(ROOT, "fp4_routed_expert_router_b200", "csrc"), str(src), "-o", str(exe)])
    out = subprocess.run([str(exe)], input="5120 2304\n256 128\n", capture_output=True, text=True,
                         check=True).stdout.splitlines()
    sizes = [list(map(int, l.split())) for l in out[:2]]
    rows = [list(map(int, l.split())) for l in out[2:]]
    return sizes, {128: rows[0:16], 256: rows[16:32], 64: rows[32:48]}


def test_sizes(driver):
    sizes, _ = driver
    v41, tiny = sizes
    assert v41 == [256, 20, 256, 9, 4352, 2176, 2304 // 16 * 20 * 4352, 18_800_640]
    assert v41[6] + 5120 // 16 * 9 * 2176 == 18_800_640
    H, I = 256, 128
    assert tiny[0] == 256 and tiny[2] == 128           # K blocks: 256 when it divides, else 128
    assert tiny[7] == 2 * (I * H // 2 + I * H // 32) + (H * I // 2 + H * I // 32)


def test_swizzle_is_a_permutation_per_128_byte_group(driver):
    _, sw = driver
    for rowbytes in (128, 256):
        for r, row in enumerate(sw[rowbytes]):
            for g0 in range(0, rowbytes // 16, 8):
                assert sorted(row[g0:g0 + 8]) == list(range(g0, g0 + 8)), (rowbytes, r)
    for row in sw[64]:                                  # 64-byte rows are not swizzled
        assert row == [0, 1, 2, 3]


def _bank_group(row_offset_bytes, chunk):
    return ((row_offset_bytes + 16 * chunk) // 16) % 8


@pytest.mark.parametrize("rowbytes", [128, 256])
def test_gemv_fragment_phase_is_conflict_free(driver, rowbytes):
    _, sw = driver
    for g in range(0, 16, 2):                           # a quarter warp: rows g, g+1, lanes c = 0..3
        for jj in range(rowbytes // 64):                # aligned group of four chunks
            groups = [_bank_group(rr * rowbytes, sw[rowbytes][rr][4 * jj + c]) for rr in (g, g + 1)
                      for c in range(4)]
            assert len(set(groups)) == 8, (g, jj, groups)


@pytest.mark.parametrize("rowbytes", [128, 256])
def test_dequant_rows_are_conflict_free(driver, rowbytes):
    _, sw = driver
    for r0 in (0, 8):                                   # eight consecutive rows of a 16-row block
        for q in range(rowbytes // 16):
            groups = [_bank_group(r * rowbytes, sw[rowbytes][r][q]) for r in range(r0, r0 + 8)]
            assert len(set(groups)) == 8, (r0, q, groups)
