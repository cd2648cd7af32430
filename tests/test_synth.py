"""The seeded input generators: known-answer values, determinism, layout, and
the routing statistics they are calibrated to reproduce.  CPU only."""
import os

import numpy as np

import oracle
from fp4_routed_expert_router_b200 import synth
from tests import helpers


def test_splitmix64_known_answer():
    with open(os.path.join(helpers.GOLDEN_DIR, "splitmix64.txt")) as f:
        vals = [int(l, 16) for l in f if l.strip() and not l.startswith("#")]
    got = [int(v) for v in synth.splitmix64_stream(0, 3)]
    assert got == vals
    assert synth.mix64(synth.GOLDEN) == vals[0]
    # counter mode: any window of the stream equals the same slice of the whole
    whole = synth.splitmix64_stream(12345, 100)
    assert np.array_equal(synth.splitmix64_stream(12345, 10, start=37), whole[37:47])


def test_expert_tensors_deterministic_and_distinct():
    a = synth.gen_expert(1, 0, 3, 256, 128, 120, 126)
    b = synth.gen_expert(1, 0, 3, 256, 128, 120, 126)
    c = synth.gen_expert(1, 0, 4, 256, 128, 120, 126)
    for k in a:
        assert np.array_equal(a[k], b[k])
        assert not np.array_equal(a[k], c[k])
    assert a["w1"].shape == (128, 128) and a["s1"].shape == (128, 8)
    assert a["w2"].shape == (256, 64) and a["s2"].shape == (256, 4)
    for s in ("s1", "s3", "s2"):
        assert a[s].min() >= 120 and a[s].max() <= 126
        assert len(np.unique(a[s])) == 7
    nib = np.concatenate([a["w1"].ravel() & 15, a["w1"].ravel() >> 4])
    counts = np.bincount(nib, minlength=16)
    assert counts.min() > 0.8 * nib.size / 16


def test_expert_object_layout():
    t = synth.gen_expert(2, 1, 5, 256, 128, 120, 126)
    obj = synth.expert_object(t, 256, 128)
    lay = synth.expert_layout(256, 128)
    assert obj.size == lay["total"] == oracle.expert_bytes(256, 128)
    for name in ("w1", "w3", "w2", "s1", "s3", "s2"):
        off, (r, c) = lay[name]
        assert np.array_equal(obj[off:off + r * c].reshape(r, c), t[name])


def test_bf16_activations():
    x = synth.gen_x(3, 4, 512)
    f = synth.bf16_bits_to_f32(x)
    assert x.dtype == np.uint16 and x.shape == (4, 512)
    assert abs(float(f.mean())) < 0.1 and 0.9 < float(f.std()) < 1.1
    assert np.array_equal(synth.f32_to_bf16_bits(f), x)


def test_zipf_bias_reproduces_hit_curve():
    """10100.com article, section "热专家与Prefill隔离": keeping the 3000 / 4000 /
    5000 most frequent of 15,360 experts predicts about 80.5 / 85.5 / 89.1 %
    LRU hits.  With alpha = 0.5 the synthetic router concentrates its choices
    similarly: the top 19.5 / 26 / 32.6 % of one layer's experts take most hits."""
    wl = synth.WORKLOADS["decode_b1"]
    logits = synth.gen_logits(wl.seed, 0, 4096, wl.n_experts, wl.zipf_alpha)
    ids, _ = oracle.route(logits, wl.top_k)
    freq = np.sort(np.bincount(ids.ravel(), minlength=wl.n_experts))[::-1]
    cum = np.cumsum(freq) / freq.sum()
    for frac, page in ((3000 / 15360, 0.805), (4000 / 15360, 0.855), (5000 / 15360, 0.891)):
        got = cum[int(round(frac * wl.n_experts)) - 1]
        assert abs(got - page) < 0.05, (frac, got, page)


def test_prefill_chunk_touches_most_experts():
    """Same article: one prefill layer of a 2048-token chunk touches 370-381 of
    384 experts.  The weak bias (alpha = 0.47) lands in that neighbourhood."""
    wl = synth.WORKLOADS["prefill_2048"]
    logits = synth.gen_logits(wl.seed, 0, wl.tokens, wl.n_experts, wl.zipf_alpha)
    ids, _ = oracle.route(logits, wl.top_k)
    active = len(np.unique(ids))
    assert 360 <= active <= 384, active


def test_keep_mask_has_the_stated_size():
    wl = synth.WORKLOADS["stack40_b1"]
    for layer in (0, 17, 39):
        m = synth.keep_mask(wl.seed, layer, wl.n_experts, wl.n_keep)
        assert m.sum() == 154
    assert wl.n_slots == 6160
    assert wl.n_slots * wl.expert_bytes == 115_811_942_400
