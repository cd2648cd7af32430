"""Launch plans of the two GEMM paths, computed on the CPU by the library's own
host code (csrc/decode_mx.cuh make_mx_plan, csrc/tc_prefill.cuh tc_args),
against the B200 limits the kernels are launched under: 232,448 bytes of
opt-in shared memory per block (the library keeps 1,024 of them for static
shared memory) and 512 TMEM columns.

- decode kernel: every batch it takes (T*k <= 768, routed inside the kernel
  for T*k <= 64) gets a plan whose ring slots are a multiple of the six MMA
  issuers, at most 24, whose ring starts 1,024-byte aligned with 16-byte
  aligned slots (bulk-copy destinations), and whose shared memory fits; one
  token of the V4.1 layer gets the full 24-slot ring;
- tcgen05 path: for both tile shapes (64-token items with six stages for
  batches of at most 64 tokens, else 128-token items with four) the two
  accumulators and the A stages fill exactly the 512 TMEM columns, the B ring
  starts 1,024-byte aligned (128-byte swizzle atoms), at least two code-ring
  entries fit, and the kernel's dynamic shared memory fits.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "fp4_routed_expert_router_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
OPTIN = 232448
LIMIT = OPTIN - 1024
SHAPES = [(5120, 2304, 384, 6), (256, 128, 16, 2), (5120, 2304, 128, 3)]
TOKENS = [1, 2, 3, 4, 8, 16, 17, 32, 64, 65, 128, 130, 256, 2048]

_HARNESS = r"""
#include "decode_mx.cuh"
#include "tc_prefill.cuh"
#include <cstdio>
using namespace moe;
int main() {
    const int limit = %(limit)d;
    const int shapes[][4] = {%(shapes)s};
    const int tokens[] = {%(tokens)s};
    for (const auto& sh : shapes) {
        const int H = sh[0], I = sh[1], E = sh[2], k = sh[3];
        const SlotLayout L = make_slot_layout(H, I);
        for (int T : tokens) {
            for (int routed = 0; routed < 2; ++routed) {
                const MxPlan p = make_mx_plan(L, T, k, E, routed != 0, limit);
                std::printf("mx %%d %%d %%d %%d %%d %%d %%d %%d %%d %%d %%d\n", H, I, E, k, T, routed, p.ok, p.slots,
                            p.slot_bytes, p.off_ring, p.smem_bytes);
            }
            TcPlan tp{};
            tp.smem_limit = limit;
            tp.sm_count = 148;
            ExpertArgs g{};
            g.E = E;
            g.k = k;
            g.H = H;
            g.I = I;
            const int nmax = tc_nmax_for(T);
            for (int up = 0; up < 2; ++up) {
                const TcArgs t = tc_args(tp, g, L, T, up != 0, nullptr, nmax);
                std::printf("tc %%d %%d %%d %%d %%d %%d %%d %%d %%d %%d %%d %%d %%zu\n", H, I, E, k, T, up, nmax,
                            tc_stages(nmax), t.centries, t.off_b, t.off_code, t.entry_bytes, tc_smem_bytes(t));
            }
        }
    }
    return 0;
}
"""


@pytest.fixture(scope="module")
def plans(tmp_path_factory):
    if not shutil.which(NVCC) and not os.path.exists(NVCC):
        pytest.skip("nvcc not found")
    d = tmp_path_factory.mktemp("plans")
    src = d / "plans.cu"
    src.write_text(_HARNESS % {
        "limit": LIMIT,
        "shapes": ", ".join("{%d, %d, %d, %d}" % s for s in SHAPES),
        "tokens": ", ".join(str(t) for t in TOKENS),
    })
    exe = d / "plans"
    res = subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-I", CSRC,
                          str(src), "-o", str(exe), "-lcuda"], capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    mx, tc = [], []
    for line in out.splitlines():
        f = line.split()
        (mx if f[0] == "mx" else tc).append([int(v) for v in f[1:]])
    return mx, tc


def test_decode_kernel_plans_fit(plans):
    mx, _ = plans
    assert len(mx) == 2 * len(SHAPES) * len(TOKENS)
    for H, I, E, k, T, routed, ok, slots, slot_bytes, off_ring, smem in mx:
        takes = T * k <= 768 and (not routed or (T * k <= 64 and E <= 384))
        if not takes:
            continue
        assert ok == 1, (H, E, k, T, routed)
        assert slots % 6 == 0 and 6 <= slots <= 24, slots
        assert off_ring % 1024 == 0 and slot_bytes % 16 == 0
        assert smem <= LIMIT, (T, smem)
        if (H, I, E, k, T) == (5120, 2304, 384, 6, 1):
            assert slots == 24


def test_tcgen05_plans_fit(plans):
    _, tc = plans
    assert len(tc) == 2 * len(SHAPES) * len(TOKENS)
    for H, I, E, k, T, up, nmax, stages, centries, off_b, off_code, entry_bytes, smem in tc:
        assert nmax == (64 if T <= 64 else 128)
        assert 2 * nmax + 64 * stages == 512                  # accumulators + A stages = all of TMEM
        assert off_b % 1024 == 0                              # 128-byte swizzle atoms
        assert off_code - off_b == stages * 2 * nmax * 128    # B ring: stages x 2 atoms x nmax rows
        assert entry_bytes % 16 == 0 and off_code % 16 == 0
        assert centries >= 2, (H, E, T, up)
        assert smem <= LIMIT, (H, E, T, up, smem)
