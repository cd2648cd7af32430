"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Routing (ids, counts, offsets, perm) must match bit for bit; fp32 outputs
must satisfy max|y - y_ref| <= 1e-2 * rms(y_ref) per token."""
import numpy as np
import pytest
import torch

import oracle
from fp4_routed_expert_router_b200 import moe, synth
from tests.gpu_helpers import Filled, check_routing, check_y, routing_to_host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    f = Filled(synth.WORKLOADS["tiny"], max_tokens=256, from_host=True)
    yield f
    f.close()


def _run(f: Filled, T: int, step: int, layer: int = 0, path: int = moe.PATH_AUTO):
    wl = f.wl
    logits, mask = synth.layer_inputs(wl, layer, step, tokens=T)
    x = synth.gen_x(wl.seed, T, wl.hidden, step)
    f.ctx.set_path(path)
    r = f.ctx.route(layer, to_dev(logits), to_dev(mask) if mask is not None else None)
    y = f.ctx.forward(layer, to_dev(x), r)
    torch.cuda.synchronize()
    rc, msg = f.ctx.last_error()
    assert rc == moe.OK, msg
    return logits, mask, x, r, y.cpu().numpy()


@pytest.mark.parametrize("T", [1, 2, 3, 4, 7, 17, 64, 200])
def test_tiny_layer_parity(tiny, T):
    wl = tiny.wl
    logits, mask, x, r, y = _run(tiny, T, step=T)
    ids, w = check_routing(r, logits, wl.top_k, wl.n_experts, mask)
    y_ref = tiny.oracle_y(0, x, ids, w, range(T))
    check_y(y, y_ref)


@pytest.mark.parametrize("path", [moe.PATH_GEMV, moe.PATH_TC])
@pytest.mark.parametrize("T", [1, 5, 33, 130])
def test_tiny_forced_paths(tiny, path, T):
    """Both expert-FFN engines on the same inputs: the decode kernel (block-scaled
    FP4 tensor cores) and the tcgen05 f16 grouped GEMM (token chunks of 1..128,
    ragged tails)."""
    wl = tiny.wl
    logits, mask, x, r, y = _run(tiny, T, step=1000 + T, path=path)
    ids, w = check_routing(r, logits, wl.top_k, wl.n_experts, mask)
    y_ref = tiny.oracle_y(0, x, ids, w, range(T))
    check_y(y, y_ref)


@pytest.mark.parametrize("T", [1, 4, 7])
def test_tiny_route_forward_one_launch(tiny, T):
    """moe_fp4_route_forward routes inside the layer kernel (every CTA routes,
    the first writes the routing): routing bit-exact against the oracle, y
    within the bar, and identical, bit for bit, to route + forward."""
    wl = tiny.wl
    logits, _ = synth.layer_inputs(wl, 0, 3000 + T, tokens=T)
    x = to_dev(synth.gen_x(wl.seed, T, wl.hidden, 3000 + T))
    tiny.ctx.set_path(moe.PATH_AUTO)
    r, y = tiny.ctx.route_forward(0, to_dev(logits), x)
    torch.cuda.synchronize()
    rc, msg = tiny.ctx.last_error()
    assert rc == moe.OK, msg
    ids, w = check_routing(r, logits, wl.top_k, wl.n_experts)
    check_y(y.cpu().numpy(), tiny.oracle_y(0, synth.gen_x(wl.seed, T, wl.hidden, 3000 + T), ids, w, range(T)))
    r2 = tiny.ctx.route(0, to_dev(logits))
    y2 = tiny.ctx.forward(0, x, r2)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    assert torch.equal(r.weights, r2.weights)


def test_tiny_zero_tokens(tiny):
    r = tiny.ctx.alloc_routing(0)
    logits = torch.empty((0, tiny.wl.n_experts), dtype=torch.float32, device="cuda")
    tiny.ctx.route(0, logits, out=r)
    y = tiny.ctx.forward(0, torch.empty((0, tiny.wl.hidden), dtype=torch.int16, device="cuda"), r)
    torch.cuda.synchronize()
    assert y.shape == (0, tiny.wl.hidden)
    assert int(r.counts.sum()) == 0 and int(r.offsets[-1]) == 0


@pytest.mark.parametrize("T", [5, 16, 40])   # one-warp path (T*k <= 32) and the grid path
def test_tiny_routing_ties_and_mask(tiny, T):
    wl = tiny.wl
    rng = np.random.default_rng(5 + T)
    logits = rng.integers(-2, 3, size=(T, wl.n_experts)).astype(np.float32)
    logits[0, 3] = -0.0
    logits[0, 1] = 0.0
    keep = np.ones(wl.n_experts, np.uint8)
    keep[[2, 5, 11]] = 0
    for m in (None, keep):
        r = tiny.ctx.route(0, to_dev(logits), to_dev(m) if m is not None else None)
        torch.cuda.synchronize()
        check_routing(r, logits, wl.top_k, wl.n_experts, m)


def test_device_generator_matches_host():
    for name in ("tiny", "decode_b1"):
        wl = synth.WORKLOADS[name]
        buf = torch.empty(wl.expert_bytes, dtype=torch.uint8, device="cuda")
        for layer, e in ((0, 0), (3, 17 % wl.n_experts)):
            moe.synth_fill_expert(buf, wl.seed, layer, e, wl.hidden, wl.inter, wl.scale_lo, wl.scale_hi)
            host = synth.expert_object(synth.gen_expert(wl.seed, layer, e, wl.hidden, wl.inter, wl.scale_lo,
                                                        wl.scale_hi), wl.hidden, wl.inter)
            assert np.array_equal(buf.cpu().numpy(), host)


def test_power_of_two_invariants_bit_exact(tiny):
    """Raising every w2 (or w3) scale by one doubles y exactly on the GPU too."""
    wl = tiny.wl
    T = 9
    logits, _ = synth.layer_inputs(wl, 0, 77, tokens=T)
    x = synth.gen_x(wl.seed, T, wl.hidden, 77)
    ctx = moe.Context(wl.hidden, wl.inter, wl.n_experts, wl.top_k, 1, wl.n_experts, 16)
    ys = []
    for bump in (None, "s2", "s3"):
        for e in range(wl.n_experts):
            t = synth.gen_expert(wl.seed, 0, e, wl.hidden, wl.inter, wl.scale_lo, wl.scale_hi)
            if bump:
                t[bump] = t[bump] + 1
            ctx.load_expert_slot(0, e, e, t)
        r = ctx.route(0, to_dev(logits))
        ys.append(ctx.forward(0, to_dev(x), r).cpu().numpy())
    torch.cuda.synchronize()
    assert ctx.last_error()[0] == moe.OK
    np.testing.assert_array_equal(ys[1], 2 * ys[0])
    np.testing.assert_array_equal(ys[2], 2 * ys[0])
    ctx.close()


def test_residual_output(tiny):
    """x_out = bf16(x + y): against the oracle's residual of its own y; the two
    may differ by one bf16 unit where y differs within tolerance."""
    wl = tiny.wl
    T = 5
    logits, _ = synth.layer_inputs(wl, 0, 9, tokens=T)
    x = synth.gen_x(wl.seed, T, wl.hidden, 9)
    xd = to_dev(x)
    r = tiny.ctx.route(0, to_dev(logits))
    xo = torch.empty_like(xd)
    tiny.ctx.forward(0, xd, r, x_out=xo)
    torch.cuda.synchronize()
    ids, w = oracle.route(logits, wl.top_k)
    x_ref = oracle.residual(x, tiny.oracle_y(0, x, ids, w, range(T)))
    got = xo.cpu().numpy().view(np.uint16).astype(np.int32)
    diff = np.abs(got - x_ref.astype(np.int32))      # same sign: bit distance = ulps
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.97


@pytest.mark.parametrize("path,T", [(moe.PATH_GEMV, 17), (moe.PATH_TC, 130), (moe.PATH_AUTO, 200)])
def test_tiny_saliency(tiny, path, T):
    """Per-expert saliency (router weight x ||expert output||_2, summed) of a
    forward against the oracle; experts nobody chose stay untouched; a second
    call on the same forward adds the same amount again (exactly, in fp64)."""
    wl = tiny.wl
    logits, mask, x, r, y = _run(tiny, T, step=2000 + T, path=path)
    ids, w = check_routing(r, logits, wl.top_k, wl.n_experts, mask)
    sal = torch.zeros(wl.n_experts, dtype=torch.float64, device="cuda")
    tiny.ctx.saliency(r, sal)
    s1 = sal.cpu().numpy().copy()
    tiny.ctx.saliency(r, sal)
    s2 = sal.cpu().numpy()
    rc, msg = tiny.ctx.last_error()
    assert rc == moe.OK, msg
    objs = {int(e): tiny.host_object(0, int(e)) for e in np.unique(ids)}
    ref = oracle.saliency(x, ids, w, objs, wl.n_experts, wl.hidden, wl.inter)
    used = np.unique(ids)
    np.testing.assert_allclose(s1[used], ref[used], rtol=2e-3)
    assert np.all(s1[np.setdiff1d(np.arange(wl.n_experts), used)] == 0.0)
    np.testing.assert_array_equal(s2, 2.0 * s1)
