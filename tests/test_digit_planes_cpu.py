"""The exact E2M1 digit-plane split of a bf16 activation block, on the CPU.

The decode path feeds bf16 activations (x, and h before the second GEMM) to
the block-scaled FP4 tensor core by writing each 32-element block as 8 planes
of E2M1 digits, plane p at the UE8M0 scale 2^(E0 - 2p) with
2^E0 < max|v| <= 2^(E0 + 1), each digit the nearest half of the remainder.
The pages fix only the weight format (FP4 E2M1 + UE8M0, 10100.com article
151357339, section "moe专家的容量瓶颈") and bf16 activations, so this split is
a design reading; these tests pin the numerical claims it rests on, written
out here from that definition (not from the kernel):

- every digit is one of 0, +-0.5, +-1, +-1.5, +-2 and its 4-bit code decodes
  back to it through the OCP E2M1 table (tests/golden/e2m1_table.txt);
- after 8 planes each element is off by at most 2^(E0 - 16) < max|v| * 2^-16;
- every element with |v| >= max|v| * 2^-8 is represented exactly, and that
  bound is tight: an element within 2^9 of the maximum may not be;
- the float32 remainder updates are exact (the same digits as in exact
  rational arithmetic);
- scaling a block by a power of two leaves the digits unchanged and shifts the
  plane scales, which is what makes the power-of-two invariants of the layer
  hold bit for bit on the GPU.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest

from fp4_routed_expert_router_b200 import synth
from tests.helpers import e2m1_table

PLANES = 8


def block_exponent(mb: float) -> int:
    """E0 with 2^E0 < mb <= 2^(E0 + 1), for mb > 0."""
    m, e = np.frexp(np.float64(mb))   # mb = m * 2^e, 0.5 <= m < 1
    return int(e) - 1 if m > 0.5 else int(e) - 2


def split_f32(v: np.ndarray):
    """Digit planes of one block in float32 arithmetic: (E0, [(s, digits)])."""
    v = np.asarray(v, dtype=np.float32)
    mb = float(np.max(np.abs(v)))
    if mb == 0.0:
        return None, []
    e0 = block_exponent(mb)
    r = v.copy()
    planes = []
    for p in range(PLANES):
        s = e0 - 2 * p
        if s < -127:
            break
        d = (np.rint(np.float32(2.0) * (r * np.float32(2.0 ** -s))) * np.float32(0.5)).astype(np.float32)
        planes.append((s, d))
        r = (r - d * np.float32(2.0 ** s)).astype(np.float32)
    return e0, planes


def split_exact(v: np.ndarray):
    """The same split in exact rational arithmetic (round half to even)."""
    vals = [Fraction(float(t)) for t in np.asarray(v, dtype=np.float32)]
    mb = max(abs(t) for t in vals)
    e0 = block_exponent(float(mb))
    r = vals
    planes = []
    for p in range(PLANES):
        s = e0 - 2 * p
        if s < -127:
            break
        d = [Fraction(round(2 * t / Fraction(2) ** s), 2) for t in r]   # round() is half to even
        planes.append((s, d))
        r = [t - q * Fraction(2) ** s for t, q in zip(r, d)]
    return e0, planes


def reconstruct(planes) -> np.ndarray:
    out = np.zeros(32, dtype=np.float64)
    for s, d in planes:
        out += np.asarray(d, dtype=np.float64) * 2.0 ** s
    return out


def bf16_blocks(n: int, seed: int) -> np.ndarray:
    """n blocks of 32 bf16 values (as float32) with varied dynamic range,
    signed zeros, exact powers of two and subnormal magnitudes."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((n, 32)).astype(np.float32)
    spread = rng.integers(0, 24, size=(n, 1))                  # per-block dynamic range in binades
    z *= np.exp2(-rng.uniform(0, 1, size=(n, 32)) * spread).astype(np.float32)
    z *= np.exp2(rng.integers(-120, 120, size=(n, 1))).astype(np.float32)   # block magnitude
    z[rng.random((n, 32)) < 0.05] = 0.0
    z[rng.random((n, 32)) < 0.02] = -0.0
    pw = rng.random((n, 32)) < 0.03
    z[pw] = np.exp2(rng.integers(-20, 20, size=pw.sum())).astype(np.float32) * np.sign(z[pw] + 0.5)
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(z)).reshape(n, 32)


BLOCKS = bf16_blocks(400, 20260917)


def test_digits_are_e2m1_values_and_codes_decode_through_the_table():
    table = e2m1_table()
    for v in BLOCKS[:100]:
        _, planes = split_f32(v)
        for _, d in planes:
            assert np.all(np.isin(np.abs(d), [0.0, 0.5, 1.0, 1.5, 2.0]))
            code = (2.0 * np.abs(d)).astype(np.int64) | np.where(d < 0, 8, 0)
            assert np.array_equal(table[code], d.astype(np.float64))


def test_error_bound_and_exact_elements():
    for v in BLOCKS:
        e0, planes = split_f32(v)
        if e0 is None:
            continue
        mb = float(np.max(np.abs(v)))
        err = np.abs(reconstruct(planes) - v.astype(np.float64))
        if e0 - 2 * (PLANES - 1) >= -127:   # all 8 planes present
            assert np.all(err <= 2.0 ** (e0 - 16))
            assert np.all(err < mb * 2.0 ** -16)
            big = np.abs(v) >= mb * 2.0 ** -8
            assert np.all(err[big] == 0.0), "an element within 2^8 of the block maximum is not exact"


def test_within_2_to_the_9_is_not_always_exact():
    # max 1.5 (E0 = 0): 255 * 2^-16 is within 2^9 of it but has a bit below 2^-15
    v = np.zeros(32, dtype=np.float32)
    v[0] = 1.5
    v[1] = np.float32(255 * 2.0 ** -16)
    assert v[1] >= 1.5 * 2.0 ** -9
    _, planes = split_f32(v)
    assert reconstruct(planes)[1] != v[1]
    v[1] = np.float32(255 * 2.0 ** -15)                       # within 2^8: exact
    _, planes = split_f32(v)
    assert reconstruct(planes)[1] == v[1]


def test_float32_remainders_are_exact():
    for v in BLOCKS[:60]:
        e0, planes = split_f32(v)
        if e0 is None:
            continue
        e0x, exact = split_exact(v)
        assert e0 == e0x
        assert len(planes) == len(exact)
        for (s, d), (sx, dx) in zip(planes, exact):
            assert s == sx
            assert [Fraction(float(t)) for t in d] == dx


@pytest.mark.parametrize("k", [-9, -1, 1, 7])
def test_power_of_two_scaling_shifts_the_scales_only(k):
    for v in BLOCKS[:100]:
        mb = float(np.max(np.abs(v)))
        if mb == 0.0 or not 2.0 ** -100 < mb * 2.0 ** k < 2.0 ** 100:
            continue
        if float(np.min(np.abs(v[v != 0]))) * 2.0 ** k < 2.0 ** -100:   # keep every element normal
            continue
        e0, planes = split_f32(v)
        e1, scaled = split_f32((v * np.float32(2.0 ** k)).astype(np.float32))
        assert e1 == e0 + k
        for (s, d), (s2, d2) in zip(planes, scaled):
            assert s2 == s + k
            assert np.array_equal(d, d2)


def test_plane_scales_are_ue8m0_bytes():
    for v in BLOCKS:
        e0, planes = split_f32(v)
        for s, _ in planes:
            assert 0 <= s + 127 <= 254
