"""GPU parity for a drafter-shaped MoE: 128 routed experts, top-3 (the
drafter model's expert count and fan-out as ai-shiz.ru "DeepSeek-V4.1-Flash
дома" describes it, section "Что за модель"), at the layer's hidden 5120 /
inter 2304.  The same kernels serve it: the 128-expert router instantiation,
the decode kernel for small batches and the tcgen05 path for large ones."""
import numpy as np
import pytest

from fp4_routed_expert_router_b200 import moe, synth
from tests.gpu_helpers import Filled, check_routing, check_y, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def drafter():
    f = Filled(synth.WORKLOADS["drafter_b1"], max_tokens=256)
    yield f
    f.close()


def _run(f, wl, T, step, path):
    logits, _ = synth.layer_inputs(wl, 0, step, tokens=T)
    x = synth.gen_x(wl.seed, T, wl.hidden, step)
    f.ctx.set_path(path)
    r = f.ctx.route(0, to_dev(logits))
    y = f.ctx.forward(0, to_dev(x), r).cpu().numpy()
    rc, msg = f.ctx.last_error()
    assert rc == moe.OK, msg
    ids, w = check_routing(r, logits, wl.top_k, wl.n_experts)
    return x, ids, w, y


@pytest.mark.parametrize("step", [0, 1])
def test_drafter_decode_b1(drafter, step):
    wl = synth.WORKLOADS["drafter_b1"]
    x, ids, w, y = _run(drafter, wl, 1, step, moe.PATH_AUTO)
    check_y(y, drafter.oracle_y(0, x, ids, w, [0]))


@pytest.mark.parametrize("path", [moe.PATH_AUTO, moe.PATH_GEMV, moe.PATH_TC])
def test_drafter_batch256(drafter, path):
    wl = synth.WORKLOADS["drafter_b256"]
    x, ids, w, y = _run(drafter, wl, 256, 3, path)
    counts = np.bincount(ids.reshape(-1), minlength=wl.n_experts)
    hot = int(np.argmax(counts))
    rng = np.random.default_rng(5)
    toks = sorted({int(np.nonzero((ids == hot).any(1))[0][-1]), 255, *map(int, rng.choice(256, 5, replace=False))})
    check_y(y[toks], drafter.oracle_y(0, x, ids, w, toks))


def test_drafter_batch256_paths_agree_on_every_token(drafter):
    """The decode kernel (groups of two entries, 768 entries) and the tcgen05 path
    on the same 256-token batch: every token within twice the bar of each other
    (both are within the bar of the oracle on the sampled tokens above)."""
    wl = synth.WORKLOADS["drafter_b256"]
    ys = {path: _run(drafter, wl, 256, 3, path)[3] for path in (moe.PATH_GEMV, moe.PATH_TC)}
    drafter.ctx.set_path(moe.PATH_AUTO)
    check_y(ys[moe.PATH_GEMV], ys[moe.PATH_TC].astype(np.float64), tol=2e-2)
