"""The slot layout (csrc/slot_layout.cuh) on CPU: unit counts and sizes of
the V4.1 and tiny shapes; the relayout (the loader's per-thread mapping)
writes every slot byte exactly once, and reading a slot the way the kernels
address it (unit of (matrix, row tile, K unit), 16-byte code chunk of (row,
32-K block), scale byte of (row, block)) gives back every checkpoint nibble
and scale; and the code chunks sit where the tensor-core operand descriptor
of the decode kernel expects them (core matrices of 8 rows x 16 bytes,
128 bytes apart along K, 512 bytes apart along M, +256 bytes per K = 64
step) and the scale bytes where the 32 x 128-bit TMEM copy puts row r's
four scales in lane r % 32, column r / 32."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "fp4_routed_expert_router_b200", "csrc")

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
// scale back with the kernels' addressing.  stdout: slot bytes, units, bytes
// not written exactly once, wrong codes, wrong scales.
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
            for (int b = 0; b < 16; ++b) { slot[d + b] = ck[s + b]; hit[d + b]++; }
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
            for (int r = 0; r < rows; ++r)
                for (int k = 0; k < K; ++k) {
                    const size_t unit = mat < 2 ? up_unit_offset(L, mat, r / 128, k / 128)
                                                : down_unit_offset(L, r / 128, k / 128);
                    const int rr = r % 128, kk = k % 128;
                    const uint8_t byte = slot[unit + unit_code_chunk(rr, kk / 32) + (kk % 32) / 2];
                    const size_t co = (mat < 2 ? size_t(mat) * IH / 2 + size_t(r) * (H / 2)
                                               : IH + size_t(r) * (I / 2)) + k / 2;
                    bad_code += ((byte >> (4 * (kk & 1))) & 15) != ((ck[co] >> (4 * (k & 1))) & 15);
                    if (k % 32 == 0) {
                        const size_t so = 3 * IH / 2 + (mat < 2 ? size_t(mat) * IH / 32 + size_t(r) * (H / 32)
                                                                : 2 * IH / 32 + size_t(r) * (I / 32)) + k / 32;
                        bad_scale += slot[unit + unit_scale_byte(rr, kk / 32)] != ck[so];
                    }
                }
        }
        const size_t units = 2 * size_t(L.RT) * L.KU + size_t(L.NT) * L.KD;
        std::printf("%zu %zu %zu %zu %zu\n", L.bytes, units, cover, bad_code, bad_scale);
    }
    // descriptor geometry: chunk (r, c) = K-step (c / 2) * 256 + M group (r / 8) * 512 + K core (c % 2) * 128
    // + (r % 8) * 16; scale (r, b) = 8192 + lane (r % 32) * 16 + column (r / 32) * 4 + b
    int bad_geom = 0;
    for (int r = 0; r < 128; ++r)
        for (int c = 0; c < 4; ++c) {
            bad_geom += unit_code_chunk(r, c) != (c / 2) * 256 + (r / 8) * 512 + (c % 2) * 128 + (r % 8) * 16;
            bad_geom += unit_scale_byte(r, c) != kUnitCodeBytes + (r % 32) * 16 + (r / 32) * 4 + c;
        }
    std::printf("geom %d %d %d\n", bad_geom, kUnitBytes, kUnitCodeBytes);
    return 0;
}
"""


@pytest.fixture(scope="module")
def roundtrip(tmp_path_factory):
    d = tmp_path_factory.mktemp("layout")
    src, exe = d / "rt.cpp", d / "rt"
    src.write_text(_ROUNDTRIP)
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I", CSRC, str(src), "-o", str(exe)])
    out = subprocess.run([str(exe)], input="5120 2304\n256 128\n384 256\n", capture_output=True, text=True,
                         check=True).stdout.splitlines()
    rows = [list(map(int, l.split())) for l in out[:-1]]
    geom = list(map(int, out[-1].split()[1:]))
    return rows, geom


def test_v41_slot_is_2160_units_of_8704_bytes(roundtrip):
    rows, _ = roundtrip
    nbytes, units = rows[0][:2]
    assert nbytes == 18_800_640                       # the page's expert object size
    assert units == 2 * 18 * 40 + 40 * 18 == 2160
    assert units * 8704 == nbytes


def test_relayout_roundtrip_reads_back_every_code_and_scale(roundtrip):
    rows, _ = roundtrip
    for nbytes, units, cover, bad_code, bad_scale in rows:
        assert (cover, bad_code, bad_scale) == (0, 0, 0), (nbytes, cover, bad_code, bad_scale)
    H, I = 256, 128                                     # tiny: 2 (w1/w3) x 1 x 2 + 2 x 1 units
    assert rows[1][0] == 2 * (I * H // 2 + I * H // 32) + (H * I // 2 + H * I // 32)
    assert rows[1][1] == 6


def test_units_match_the_tensor_core_operand_geometry(roundtrip):
    _, geom = roundtrip
    bad, unit_bytes, code_bytes = geom
    assert bad == 0
    assert (unit_bytes, code_bytes) == (8704, 8192)
