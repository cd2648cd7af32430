"""The f16 operands of the prefill tensor-core GEMM, on the CPU.

The prefill path multiplies on the f16 tensor cores (kind::f16, fp32
accumulate).  Its two conversions are design readings -- the pages fix only
the FP4 E2M1 + UE8M0 weights and bf16 activations (10100.com article
151357339, section "moe专家的容量瓶颈") -- and these tests pin what they
keep, restated from their definitions with numpy's float16 rounding (round to
nearest even) as the reference step:

- weights: each E2M1 value times 2^(s - s_ref), s_ref the row's largest
  block-scale byte, is exact in f16 while s_ref - s <= 23, and the first
  span that is not exact is 24 (the row scale 2^(s_ref - 127) is applied
  later in fp32);
- activations: a bf16 row is multiplied by 2^sigma with sigma = 14 - e_max
  (e_max the exponent of the row's largest magnitude, capped at 126), which
  puts the maximum in [2^14, 2^15), well below the f16 limit 65504; every
  element with |v| >= max * 2^-31 converts exactly, the rest are off by at
  most max * 2^-39.
"""
from __future__ import annotations

import numpy as np
import pytest

from fp4_routed_expert_router_b200 import synth
from tests.helpers import e2m1_table


def sigma_of(row_max: float) -> int:
    """The per-row prescale exponent: 14 - e_max, bf16 subnormals as 2^-126, at most 126."""
    if row_max == 0.0:
        return 0
    e = int(np.frexp(np.float64(row_max))[1]) - 1     # 2^e <= row_max < 2^(e + 1)
    return min(14 - max(e, -126), 126)


@pytest.mark.parametrize("span", range(0, 24))
def test_weight_times_scale_ratio_is_exact_in_f16(span):
    vals = e2m1_table()
    exact = vals * 2.0 ** -span
    assert np.array_equal(exact.astype(np.float16).astype(np.float64), exact)


def test_weight_span_24_is_the_first_inexact_one():
    vals = e2m1_table()
    exact = vals * 2.0 ** -24
    assert not np.array_equal(exact.astype(np.float16).astype(np.float64), exact)


def _rows(n: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((n, 256)).astype(np.float32)
    z *= np.exp2(-rng.uniform(0, 40, size=(n, 256))).astype(np.float32)   # up to 40 binades below the max
    z *= np.exp2(rng.integers(-100, 100, size=(n, 1))).astype(np.float32)
    z[rng.random((n, 256)) < 0.03] = 0.0
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(z)).reshape(n, 256)


def test_prescaled_activation_rows_fit_f16_and_keep_bf16_values():
    for v in _rows(300, 20260917):
        m = float(np.max(np.abs(v)))
        if m == 0.0:
            continue
        sg = sigma_of(m)
        scaled = v.astype(np.float64) * 2.0 ** sg
        assert float(np.max(np.abs(scaled))) < 65504.0
        if m >= 2.0 ** -112:                              # sigma not capped: max lands in [2^14, 2^15)
            assert 2.0 ** 14 <= float(np.max(np.abs(scaled))) < 2.0 ** 15
        back = scaled.astype(np.float16).astype(np.float64) * 2.0 ** -sg
        err = np.abs(back - v.astype(np.float64))
        keep = np.abs(v) >= m * 2.0 ** -31
        assert np.all(err[keep] == 0.0)
        assert np.all(err <= m * 2.0 ** -39)


def test_an_element_below_the_bound_can_lose_bits():
    v = np.zeros(256, dtype=np.float32)
    v[0] = 1.0                                            # sigma = 14
    v[1] = np.float32(255 * 2.0 ** -40)                   # 8 significant bits at 2^-33 .. 2^-40
    sg = sigma_of(1.0)
    back = float(np.float16(v[1] * 2.0 ** sg)) * 2.0 ** -sg
    assert back != float(v[1])
