"""Pins of the CPU oracle against facts fixed outside it: the numbers the pages
print, the OCP MX format definitions, IEEE/bfloat16 rounding, brute force on
tiny shapes, closed forms and exact invariants.  CPU only."""
import math
import struct

import numpy as np
import pytest

import oracle
from fp4_routed_expert_router_b200 import synth
from tests import helpers


# ---------------------------------------------------------------- shapes / bytes
def test_expert_bytes_match_printed_numbers():
    g = helpers.golden_kv("expert_bytes.txt")
    per = oracle.expert_bytes(g["hidden"], g["inter"])
    assert per == g["expert_bytes"] == 18_800_640
    assert g["total_experts"] == g["layers"] * g["experts_per_layer"]
    total = per * g["total_experts"]
    assert round(total / 1e8) == g["total_gb_x10"]            # ~288.8 GB
    weights = 3 * g["inter"] * g["hidden"] * g["experts_per_layer"] * g["layers"]
    assert round(weights / 1e8) == g["total_weights_e8"]      # ~5436e8
    lay = synth.expert_layout(g["hidden"], g["inter"])
    codes = lay["s1"][0]                                      # codes come first
    assert round(codes / 1e5) == g["weight_mb_x10"]           # ~17.7 MB
    assert round((per - codes) / 1e5) == g["scale_mb_x10"]    # ~1.1 MB
    assert round(3 * g["hidden"] * g["inter"] / 1e5) == g["expert_params_e5"]
    assert lay["total"] == per


def test_expert_bytes_tiny_shape():
    # hidden 256, inter 128: 2*(128*128 + 128*8) + (256*64 + 256*4)
    assert oracle.expert_bytes(256, 128) == 2 * (128 * 128 + 128 * 8) + (256 * 64 + 256 * 4)


# ---------------------------------------------------------------- formats
def test_e2m1_matches_ocp_table():
    tab = helpers.e2m1_table()
    for c in range(16):
        v = oracle.e2m1(c)
        assert v == tab[c]
        assert math.copysign(1.0, v) == math.copysign(1.0, tab[c])   # -0.0 for 0x8


def test_ue8m0_matches_ieee_exponent_field():
    # 2^(e-127) is the fp32 number whose exponent field is e and mantissa 0
    for e in range(1, 255):
        f = struct.unpack("<f", struct.pack("<I", e << 23))[0]
        assert oracle.ue8m0(e) == f
    assert oracle.ue8m0(0) == 2.0 ** -127
    assert math.isnan(oracle.ue8m0(255))


def test_bf16_rounding_against_fp32_integer_rounding():
    rng = np.random.default_rng(1)
    f = (rng.standard_normal(20000) * np.exp2(rng.integers(-30, 30, 20000))).astype(np.float32)
    ref = synth.f32_to_bf16_bits(f)
    got = np.array([oracle.bf16_rne(float(v)) for v in f], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rounding_ties_and_single_rounding():
    assert oracle.bf16_rne(1.0 + 2.0 ** -8) == 0x3F80          # tie -> even (down)
    assert oracle.bf16_rne(1.0 + 3 * 2.0 ** -8) == 0x3F82      # tie -> even (up)
    # just above a tie: one rounding from fp64 goes up; via fp32 it would tie down
    assert oracle.bf16_rne(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    assert oracle.bf16_rne(-2.5) == 0xC020
    assert oracle.bf16_rne(1e39) == 0x7F80
    assert oracle.bf16_rne(2.0 ** -133) == 0x0001               # smallest subnormal
    rng = np.random.default_rng(2)
    for v in rng.standard_normal(300) * 10.0 ** rng.integers(-5, 5, 300):
        b = oracle.bf16_rne(float(v))
        assert oracle.bf16_to_double(b) == helpers.bf16_exact_round(float(v))


def test_dequantised_weights_are_exact_in_bf16():
    # E2M1 * 2^(e-127) has <= 2 significant bits: exact in bf16 for e in [0, 252]
    for e in list(range(0, 12)) + list(range(110, 140)) + list(range(240, 253)):
        for c in range(16):
            v = oracle.e2m1(c) * oracle.ue8m0(e)
            assert oracle.bf16_to_double(oracle.bf16_rne(v)) == v


# ---------------------------------------------------------------- router
def test_route_brute_force_with_ties():
    rng = np.random.default_rng(3)
    T, E, k = 64, 40, 6
    logits = rng.integers(-3, 4, size=(T, E)).astype(np.float32)   # many ties
    logits[0, 5] = -0.0
    logits[0, 2] = 0.0
    ids, w = oracle.route(logits, k)
    bids, bw = helpers.brute_route(logits, k)
    assert np.array_equal(ids, bids)
    np.testing.assert_allclose(w, bw, rtol=1e-14, atol=0)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)


def test_route_special_cases():
    E = 16
    logits = np.random.default_rng(4).standard_normal((5, E)).astype(np.float32)
    ids, w = oracle.route(logits, 1)
    assert np.all(w == 1.0)
    assert np.array_equal(ids[:, 0], np.argmax(logits, axis=1))
    eq = np.zeros((3, E), dtype=np.float32)
    ids, w = oracle.route(eq, E)
    assert np.array_equal(ids, np.tile(np.arange(E), (3, 1)))
    assert np.all(w == 1.0 / E)


def test_route_mask_and_errors():
    rng = np.random.default_rng(5)
    E, k = 32, 4
    logits = rng.standard_normal((10, E)).astype(np.float32)
    keep = np.zeros(E, np.uint8)
    keep[::3] = 1
    ids, _ = oracle.route(logits, k, keep)
    bids, _ = helpers.brute_route(logits, k, keep)
    assert np.array_equal(ids, bids)
    assert np.all(keep[ids] == 1)
    with pytest.raises(ValueError):
        oracle.route(logits, 12, keep)          # only 11 routable
    bad = logits.copy()
    bad[3, 7] = np.nan
    with pytest.raises(ValueError):
        oracle.route(bad, k)


def test_permute_brute_force():
    rng = np.random.default_rng(6)
    T, k, E = 50, 3, 12
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    counts, offsets, perm = oracle.permute(ids, E)
    flat = ids.reshape(-1)
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    ref = np.array(sorted(range(T * k), key=lambda i: (flat[i], i)), dtype=np.int32)
    assert np.array_equal(perm, ref)


# ---------------------------------------------------------------- expert FFN
def _tiny_expert(seed, H=64, I=96, lo=120, hi=126):
    return synth.gen_expert(seed, 0, 0, H, I, lo, hi)


def _silu(z):
    return z / (1.0 + np.exp(-z))


def test_dequant_matches_table_decode():
    t = _tiny_expert(7)
    for m in ("w1", "w3", "w2"):
        s = "s" + m[1]
        np.testing.assert_array_equal(oracle.dequant(t[m], t[s]),
                                      helpers.dense_from_table(t[m], t[s]))


def test_single_weight_orientation_and_nibble_order():
    H, I = 64, 96
    t = {k: np.zeros_like(v) for k, v in _tiny_expert(8, H, I).items()}
    for s in ("s1", "s3", "s2"):
        t[s][:] = 127
    t["w1"][3, 5] = 0x0A        # low nibble -1.0 at k = 10, high nibble 0 at k = 11
    t["w3"][3, 5] = 0x40        # high nibble 2.0 at k = 11
    t["w2"][7, 1] = 0x70        # high nibble 6.0 at (n = 7, i = 3), low nibble 0 at i = 2
    x = synth.gen_x(9, 1, H)[0]
    xd = helpers.bf16_bits_to_f64(x)
    h, o = oracle.expert_ffn(x, t)
    a1, a3 = -xd[10], 2.0 * xd[11]
    hv = helpers.bf16_exact_round(float(_silu(a1) * a3))
    hd = helpers.bf16_bits_to_f64(h)
    assert hv != 0.0
    assert hd[3] == hv and np.count_nonzero(hd) == 1
    assert o[7] == 6.0 * hv and np.count_nonzero(o) == 1


def test_expert_ffn_brute_force_dense():
    H, I = 64, 96
    for seed in range(3):
        t = _tiny_expert(10 + seed, H, I)
        W1 = helpers.dense_from_table(t["w1"], t["s1"])
        W3 = helpers.dense_from_table(t["w3"], t["s3"])
        W2 = helpers.dense_from_table(t["w2"], t["s2"])
        x = synth.gen_x(20 + seed, 2, H)
        for r in range(2):
            xd = helpers.bf16_bits_to_f64(x[r])
            a1, a3 = W1 @ xd, W3 @ xd
            href = np.array([helpers.bf16_exact_round(float(v)) for v in _silu(a1) * a3])
            oref = W2 @ href
            h, o = oracle.expert_ffn(x[r], t)
            np.testing.assert_array_equal(helpers.bf16_bits_to_f64(h), href)
            np.testing.assert_allclose(o, oref, rtol=1e-12, atol=1e-12 * np.abs(oref).max())


def test_moe_forward_closed_form_all_ones():
    # every code 1.0 (0x22), scale 127: a1 = a3 = sum(x), h = bf16(silu(s)*s), o = I*h
    H, I, E, k, T = 64, 96, 4, 2, 3
    lay = synth.expert_layout(H, I)
    obj = np.empty(lay["total"], np.uint8)
    obj[:lay["s1"][0]] = 0x22
    obj[lay["s1"][0]:] = 127
    x = synth.gen_x(30, T, H)
    logits = np.random.default_rng(31).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(logits, k)
    y = oracle.moe_forward(x, ids, w, {e: obj for e in range(E)}, E, H, I)
    for t in range(T):
        s = float(helpers.bf16_bits_to_f64(x[t]).sum())
        h = helpers.bf16_exact_round(s / (1.0 + math.exp(-s)) * s)
        np.testing.assert_allclose(y[t], I * h * w[t].sum(), rtol=1e-13)


def _tiny_layer(seed, H=64, I=96, E=8):
    objs = {e: synth.expert_object(synth.gen_expert(seed, 0, e, H, I, 120, 126), H, I)
            for e in range(E)}
    return objs


def test_moe_forward_brute_force_and_combine():
    H, I, E, k, T = 64, 96, 8, 3, 5
    objs = _tiny_layer(40, H, I, E)
    lay = synth.expert_layout(H, I)
    x = synth.gen_x(41, T, H)
    logits = np.random.default_rng(42).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(logits, k)
    y = oracle.moe_forward(x, ids, w, objs, E, H, I)

    def part(obj, name):
        off, (r, c) = lay[name]
        return obj[off:off + r * c].reshape(r, c)

    for t in range(T):
        xd = helpers.bf16_bits_to_f64(x[t])
        acc = np.zeros(H)
        for j in range(k):
            ob = objs[int(ids[t, j])]
            W1 = helpers.dense_from_table(part(ob, "w1"), part(ob, "s1"))
            W3 = helpers.dense_from_table(part(ob, "w3"), part(ob, "s3"))
            W2 = helpers.dense_from_table(part(ob, "w2"), part(ob, "s2"))
            h = np.array([helpers.bf16_exact_round(float(v)) for v in _silu(W1 @ xd) * (W3 @ xd)])
            acc += w[t, j] * (W2 @ h)
        np.testing.assert_allclose(y[t], acc, rtol=1e-11, atol=1e-12 * np.abs(acc).max())


def test_moe_forward_power_of_two_invariants():
    # w2 scales + 1 => y doubles exactly; w3 scales + 1 => h doubles => y doubles
    H, I, E, k, T = 64, 96, 6, 2, 4
    objs = _tiny_layer(50, H, I, E)
    lay = synth.expert_layout(H, I)
    x = synth.gen_x(51, T, H)
    logits = np.random.default_rng(52).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(logits, k)
    y = oracle.moe_forward(x, ids, w, objs, E, H, I)
    for name in ("s2", "s3"):
        off, (r, c) = lay[name]
        bumped = {}
        for e, ob in objs.items():
            b = ob.copy()
            b[off:off + r * c] += 1
            bumped[e] = b
        y2 = oracle.moe_forward(x, ids, w, bumped, E, H, I)
        np.testing.assert_array_equal(y2, 2.0 * y)


def test_moe_forward_relabel_invariance():
    # renaming experts (weights and logits together) leaves y unchanged
    H, I, E, k, T = 64, 96, 6, 2, 4
    objs = _tiny_layer(60, H, I, E)
    x = synth.gen_x(61, T, H)
    logits = np.random.default_rng(62).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(logits, k)
    y = oracle.moe_forward(x, ids, w, objs, E, H, I)
    p = np.array([3, 0, 5, 1, 4, 2])          # new id of old expert e is p[e]
    logits2 = np.empty_like(logits)
    logits2[:, p] = logits
    objs2 = {int(p[e]): objs[e] for e in range(E)}
    ids2, w2 = oracle.route(logits2, k)
    np.testing.assert_array_equal(ids2, p[ids])
    y2 = oracle.moe_forward(x, ids2, w2, objs2, E, H, I)
    np.testing.assert_array_equal(y2, y)


def test_residual_rounds_once():
    x = synth.gen_x(70, 2, 64)
    y = np.random.default_rng(71).standard_normal((2, 64)) * 1e-3
    out = oracle.residual(x, y)
    ref = [helpers.bf16_exact_round(float(a + b))
           for a, b in zip(helpers.bf16_bits_to_f64(x).ravel(), y.ravel())]
    np.testing.assert_array_equal(helpers.bf16_bits_to_f64(out).ravel(), ref)


def test_saliency_brute_force_dense():
    # saliency = sum over entries routed to e of w * ||o||_2, with o from dense
    # table-decoded matrices (independent of the oracle's decoder)
    H, I, E, k, T = 64, 96, 8, 3, 7
    objs = _tiny_layer(60, H, I, E)
    lay = synth.expert_layout(H, I)
    x = synth.gen_x(61, T, H)
    logits = np.random.default_rng(62).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(logits, k)
    sal = oracle.saliency(x, ids, w, objs, E, H, I)

    def part(obj, name):
        off, (r, c) = lay[name]
        return obj[off:off + r * c].reshape(r, c)

    ref = np.zeros(E)
    for t in range(T):
        xd = helpers.bf16_bits_to_f64(x[t])
        for j in range(k):
            e = int(ids[t, j])
            ob = objs[e]
            W1 = helpers.dense_from_table(part(ob, "w1"), part(ob, "s1"))
            W3 = helpers.dense_from_table(part(ob, "w3"), part(ob, "s3"))
            W2 = helpers.dense_from_table(part(ob, "w2"), part(ob, "s2"))
            h = np.array([helpers.bf16_exact_round(float(v)) for v in _silu(W1 @ xd) * (W3 @ xd)])
            ref[e] += w[t, j] * math.sqrt(float(np.sum((W2 @ h) ** 2)))
    np.testing.assert_allclose(sal, ref, rtol=1e-11, atol=0)
    unused = np.setdiff1d(np.arange(E), np.unique(ids))
    assert np.all(sal[unused] == 0.0)


def test_saliency_power_of_two_invariants():
    # w2 scales + 1 => every output doubles => saliency doubles exactly;
    # doubling the router weights doubles it too
    H, I, E, k, T = 64, 96, 6, 2, 5
    objs = _tiny_layer(70, H, I, E)
    lay = synth.expert_layout(H, I)
    x = synth.gen_x(71, T, H)
    logits = np.random.default_rng(72).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(logits, k)
    sal = oracle.saliency(x, ids, w, objs, E, H, I)
    off, (r, c) = lay["s2"]
    bumped = {}
    for e, ob in objs.items():
        b = ob.copy()
        b[off:off + r * c] += 1
        bumped[e] = b
    np.testing.assert_array_equal(oracle.saliency(x, ids, w, bumped, E, H, I), 2.0 * sal)
    np.testing.assert_array_equal(oracle.saliency(x, ids, 2.0 * w, objs, E, H, I), 2.0 * sal)
