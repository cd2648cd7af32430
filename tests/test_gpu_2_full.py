"""GPU parity at the full V4.1-Flash layer size (hidden 5120, inter 2304, 384
experts, top-6): decode batch 1 and 64, a 2048-token prefill chunk, and the
40-layer stack with residual.  Routing is compared for every token; outputs
for tokens the oracle can afford (fp64, one (token, expert) pair at a time)."""
import numpy as np
import pytest
import torch

import oracle
from fp4_routed_expert_router_b200 import moe, synth
from tests.gpu_helpers import Filled, check_routing, check_y, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer():
    f = Filled(synth.WORKLOADS["decode_b1"], max_tokens=2048)
    yield f
    f.close()


def _step(f, wl, T, step, path=moe.PATH_AUTO):
    logits, mask = synth.layer_inputs(wl, 0, step, tokens=T)
    x = synth.gen_x(wl.seed, T, wl.hidden, step)
    f.ctx.set_path(path)
    r = f.ctx.route(0, to_dev(logits))
    y = f.ctx.forward(0, to_dev(x), r).cpu().numpy()
    rc, msg = f.ctx.last_error()
    assert rc == moe.OK, msg
    ids, w = check_routing(r, logits, wl.top_k, wl.n_experts)
    return x, ids, w, y


@pytest.mark.parametrize("step", [0, 1, 2])
def test_decode_b1(layer, step):
    wl = synth.WORKLOADS["decode_b1"]
    x, ids, w, y = _step(layer, wl, 1, step)
    check_y(y, layer.oracle_y(0, x, ids, w, [0]))


def _sample_tokens(ids, n, rng):
    """Tokens routed to the most loaded experts plus random ones."""
    flat = ids.reshape(-1)
    hot = np.argsort(np.bincount(flat, minlength=384))[::-1][:3]
    pick = set()
    for e in hot:
        pick.add(int(np.nonzero((ids == e).any(1))[0][-1]))
    pick.update(int(t) for t in rng.choice(ids.shape[0], n, replace=False))
    return sorted(pick)[: n + 3]


@pytest.mark.parametrize("path", [moe.PATH_AUTO, moe.PATH_GEMV])
def test_decode_b64(layer, path):
    wl = synth.WORKLOADS["decode_b64"]
    x, ids, w, y = _step(layer, wl, 64, 5, path)
    toks = _sample_tokens(ids, 6, np.random.default_rng(0))
    check_y(y[toks], layer.oracle_y(0, x, ids, w, toks))


def test_prefill_2048(layer):
    wl = synth.WORKLOADS["prefill_2048"]
    x, ids, w, y = _step(layer, wl, 2048, 7)
    assert len(np.unique(ids)) >= 360
    toks = _sample_tokens(ids, 8, np.random.default_rng(1))
    toks.append(2047)
    check_y(y[toks], layer.oracle_y(0, x, ids, w, toks))


def test_unmapped_expert_reports_eslot(layer):
    wl = synth.WORKLOADS["decode_b1"]
    logits, _ = synth.layer_inputs(wl, 0, 11, tokens=1)
    x = synth.gen_x(wl.seed, 1, wl.hidden, 11)
    ids, w = oracle.route(logits, wl.top_k)
    victim = int(ids[0, 2])
    layer.ctx.load_expert_slot(0, victim, -1, None)
    try:
        r = layer.ctx.route(0, to_dev(logits))
        y = layer.ctx.forward(0, to_dev(x), r).cpu().numpy()
        rc, msg = layer.ctx.last_error()
        assert rc == moe.ESLOT, msg
        # the other five experts still contribute exactly as without the victim
        keep = [j for j in range(wl.top_k) if j != 2]
        y_ref = oracle.moe_forward(x, ids[:, keep], w[:, keep],
                                   {int(e): layer.host_object(0, int(e)) for e in ids[0, keep]},
                                   wl.n_experts, wl.hidden, wl.inter)
        check_y(y, y_ref)
    finally:
        slot = layer.slot_of[(0, victim)]
        staging = torch.empty(wl.expert_bytes, dtype=torch.uint8, device="cuda")
        moe.synth_fill_expert(staging, wl.seed, 0, victim, wl.hidden, wl.inter, wl.scale_lo, wl.scale_hi)
        layer.ctx.load_expert_object(0, victim, slot, staging)
        torch.cuda.synchronize()


def test_stack40_b1_residual_chain():
    """40 layers x 154 kept experts (6,160 slots, 115.8 GB arena), router masked
    to each layer's kept set, x <- bf16(x + y) between layers."""
    wl = synth.WORKLOADS["stack40_b1"]
    f = Filled(wl, max_tokens=8)
    try:
        x = synth.gen_x(wl.seed, 1, wl.hidden, 0)
        xd = to_dev(x)
        x_ref = x.copy()
        for l in range(wl.n_layers):
            logits, mask = synth.layer_inputs(wl, l, 0, tokens=1)
            r = f.ctx.route(l, to_dev(logits), to_dev(mask))
            y = f.ctx.forward(l, xd, r, x_out=xd).cpu().numpy()
            ids, w = check_routing(r, logits, wl.top_k, wl.n_experts, mask)
            y_ref = f.oracle_y(l, x_ref, ids, w, [0])
            check_y(y, y_ref)
            x_ref = oracle.residual(x_ref, y_ref)
        rc, msg = f.ctx.last_error()
        assert rc == moe.OK, msg
        got = xd.cpu().numpy().view(np.uint16)
        xr, xg = synth.bf16_bits_to_f32(x_ref), synth.bf16_bits_to_f32(got)
        rms = np.sqrt(np.mean(xr.astype(np.float64) ** 2))
        assert np.max(np.abs(xg - xr)) <= 1e-2 * rms
    finally:
        f.close()
