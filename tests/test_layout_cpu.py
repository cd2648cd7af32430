"""The slot layout (csrc/slot_layout.cuh) on CPU: sizes of the V4.1 and tiny
shapes, the row swizzle is a permutation inside every 128-byte group, and the
two read patterns the kernels use hit eight different 16-byte bank groups per
128-byte shared-memory wavefront (no bank conflicts):
  GEMV fragments: a quarter warp reads rows g, g+1 (g even) x four chunks of
                  one aligned group of four;
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
