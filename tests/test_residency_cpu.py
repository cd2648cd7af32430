"""The expert-streaming slot policy (csrc/residency.h, host C++) against an
independent Python model of least-recently-used replacement.  CPU only: the
header is compiled with g++ into a small driver."""
import os
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_DRIVER = r"""
#include "residency.h"
#include <cstdio>
#include <vector>
using namespace moe;
// stdin: n_slots n_keys, then requests "n k0 k1 ..."; stdout per key: "slot hit evicted"
int main() {
    int n_slots, n_keys;
    if (std::scanf("%d %d", &n_slots, &n_keys) != 2) return 1;
    std::vector<int64_t> owner(n_slots, -1);
    std::vector<int32_t> where(n_keys, -1);
    std::vector<uint64_t> last(n_slots, 0);
    uint64_t clock = 0;
    int n;
    while (std::scanf("%d", &n) == 1) {
        std::vector<int64_t> keys(n);
        for (auto& k : keys) { long long v; std::scanf("%lld", &v); k = v; }
        std::vector<int32_t> slot(n); std::vector<uint8_t> hit(n); std::vector<int64_t> ev(n);
        const bool ok = lru_plan(owner.data(), where.data(), last.data(), n_slots, ++clock, keys.data(), n,
                                 slot.data(), hit.data(), ev.data());
        if (!ok) { std::printf("refused\n"); continue; }
        for (int i = 0; i < n; ++i) std::printf("%d %d %lld\n", slot[i], hit[i], (long long)ev[i]);
    }
    return 0;
}
"""


def _model(n_slots, requests):
    """Least recently used, written from its definition: resident keys are
    hits; a miss takes the lowest free slot, else the slot whose key was
    requested longest ago among those not requested now (lowest slot on a
    tie)."""
    owner = [None] * n_slots
    last = [0] * n_slots
    out = []
    for clock, req in enumerate(requests, start=1):
        if len(req) > n_slots:
            out.append("refused")
            continue
        where = {k: s for s, k in enumerate(owner) if k is not None}
        for k in req:
            if k in where:
                last[where[k]] = clock
        rows = []
        for k in req:
            if k in where:
                rows.append((where[k], 1, -1))
                continue
            free = [s for s in range(n_slots) if owner[s] is None]
            if free:
                v = free[0]
            else:
                cand = [s for s in range(n_slots) if last[s] < clock]
                v = min(cand, key=lambda s: (last[s], s))
            ev = owner[v] if owner[v] is not None else -1
            owner[v] = k
            where[k] = v
            if ev != -1:
                del where[ev]
            last[v] = clock
            rows.append((v, 0, ev))
        out.extend(f"{a} {b} {c}" for a, b, c in rows)
    return out


@pytest.mark.parametrize("n_slots,n_keys,seed", [(5, 16, 0), (12, 40, 1), (3, 3, 2), (64, 384, 3)])
def test_lru_plan_matches_model(tmp_path, n_slots, n_keys, seed):
    src = tmp_path / "d.cpp"
    exe = tmp_path / "d"
    src.write_text(_DRIVER)
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I",
                           os.path.join(ROOT, "fp4_routed_expert_router_b200", "csrc"), str(src), "-o", str(exe)])
    rng = np.random.default_rng(seed)
    # Zipf-like popularity so that hits, misses and evictions all occur
    p = 1.0 / np.arange(1, n_keys + 1) ** 1.1
    p /= p.sum()
    requests = []
    for _ in range(300):
        n = int(rng.integers(1, min(n_slots, 8) + 1))
        requests.append([int(k) for k in rng.choice(n_keys, n, replace=False, p=p)])
    requests.append(list(range(min(n_keys, n_slots + 1))))      # larger than the arena when n_keys > n_slots
    inp = f"{n_slots} {n_keys}\n" + "".join(f"{len(r)} {' '.join(map(str, r))}\n" for r in requests)
    got = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, check=True).stdout.splitlines()
    assert got == _model(n_slots, requests)
