"""Host-side checks of the C ABI and of the in-register FP4 decoder (no GPU):
the libraries load and export every declared symbol, argument checks reject
bad configs, the slot size matches the page's byte count, and the decoder's
integer arithmetic (compiled for the host with g++) is exact."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from fp4_routed_expert_router_b200 import build as pkg_build
from fp4_routed_expert_router_b200 import moe
from tests import helpers

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    pkg_build.build()
    return moe.load()


def _declared(header: str) -> list[str]:
    src = open(os.path.join(ROOT, "include", header)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_fp4_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared("moe_fp4.h")
    assert names, "no declarations found"
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(moe.EXPORTS)


def test_synth_library_exports():
    S = moe.load_synth()
    assert S.moe_synth_expert_bytes(5120, 2304) == 18_800_640


def test_slot_bytes_matches_printed_expert_size(lib):
    g = helpers.golden_kv("expert_bytes.txt")
    c = moe.Config(g["hidden"], g["inter"], g["experts_per_layer"], g["top_k"], 1, 1, 1)
    assert lib.moe_fp4_slot_bytes(ctypes.byref(c)) == g["expert_bytes"]


@pytest.mark.parametrize("bad", [
    (5000, 2304, 384, 6, 1, 1, 1),      # hidden not a multiple of 128
    (5120, 2300, 384, 6, 1, 1, 1),      # inter not a multiple of 128
    (5120, 2304, 2048, 6, 1, 1, 1),     # too many experts
    (5120, 2304, 384, 0, 1, 1, 1),      # k = 0
    (5120, 2304, 4, 6, 1, 1, 1),        # k > E
    (5120, 2304, 384, 6, 0, 1, 1),      # no layers
    (5120, 2304, 384, 6, 1, 0, 1),      # no slots
    (5120, 2304, 384, 6, 1, 1, 0),      # no tokens
])
def test_bad_configs_rejected_before_any_cuda_call(lib, bad):
    c = moe.Config(*bad)
    assert lib.moe_fp4_slot_bytes(ctypes.byref(c)) == 0
    h = ctypes.c_void_p()
    assert lib.moe_fp4_create(ctypes.byref(c), 0, None, 0, ctypes.byref(h)) == moe.EINVAL
    assert not h.value


def test_null_context_rejected(lib):
    assert lib.moe_fp4_route(None, 0, None, None, 0, None, None, None, None, None, None) == moe.EINVAL
    assert lib.moe_fp4_forward(None, 0, None, 0, None, None, None, None, None, None, None, None) == moe.EINVAL
    assert lib.moe_fp4_last_error(None, None, 0) == moe.EINVAL
    assert lib.moe_fp4_saliency(None, 0, None, None, None, None, None) == moe.EINVAL
    assert lib.moe_fp4_stream_experts(None, 0, None, 0, None, None, None) == moe.EINVAL
    assert lib.moe_fp4_residency_stats(None, None) == moe.EINVAL
    assert lib.moe_fp4_expert_outputs(None, 0, None, 0, None, None, None) == moe.EINVAL
    assert lib.moe_fp4_combine(None, 0, None, None, None, None, None, None) == moe.EINVAL
    lib.moe_fp4_destroy(None)


_HARNESS = r"""
#include "fp4_decode.cuh"
#include <cstdio>
#include <cstdint>
using namespace moe;
// stdin: lines "scale word"; stdout: the four decoded bf16x2 words
int main() {
    unsigned s; unsigned long long v;
    while (std::scanf("%u %llx", &s, &v) == 2) {
        uint32_t o[4];
        fp4_decode8(fp4_reencode_word((uint32_t)v), make_fp4_lut(s), o);
        std::printf("%08x %08x %08x %08x\n", o[0], o[1], o[2], o[3]);
    }
    return 0;
}
"""


def test_register_decoder_is_exact(tmp_path):
    """Slot re-encoding + PRMT decode == table value * 2^(s-127), for every
    supported scale byte and random code words."""
    src = tmp_path / "h.cpp"
    exe = tmp_path / "h"
    src.write_text(_HARNESS)
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-x", "c++",
                           "-I", os.path.join(ROOT, "fp4_routed_expert_router_b200", "csrc"),
                           str(src), "-o", str(exe)])
    rng = np.random.default_rng(0)
    scales = np.repeat(np.arange(2, 253), 40)
    words = rng.integers(0, 2 ** 32, size=scales.size, dtype=np.uint64)
    words[:16] = np.array([0x76543210, 0xFEDCBA98] * 8, dtype=np.uint64)
    inp = "".join(f"{s} {w:x}\n" for s, w in zip(scales, words))
    out = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, check=True).stdout.split()
    dec = np.array([int(v, 16) for v in out], dtype=np.uint64).reshape(-1, 4)
    tab = helpers.e2m1_table()
    for n in range(8):
        bits = ((dec[:, n // 2] >> np.uint64(16 * (n % 2))) & np.uint64(0xFFFF)).astype(np.uint16)
        got = helpers.bf16_bits_to_f64(bits)
        codes = ((words >> np.uint64(4 * n)) & np.uint64(15)).astype(np.int64)
        want = tab[codes] * np.exp2(scales.astype(np.float64) - 127)
        assert np.array_equal(got, want)
        assert np.array_equal(np.signbit(got), np.signbit(want))
