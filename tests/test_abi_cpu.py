"""Host-side checks of the C ABI (no GPU): the libraries load and export
every declared symbol, argument checks reject bad configs, and the slot size
matches the page's byte count."""
import ctypes
import os
import re

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
    assert lib.moe_fp4_route_forward(None, 0, None, None, None, 0, None, None, None, None, None, None, None,
                                     None) == moe.EINVAL
    assert lib.moe_fp4_set_option(None, moe.OPT_WAIT_LIMIT_US, 10) == moe.EINVAL
    lib.moe_fp4_destroy(None)
