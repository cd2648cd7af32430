"""The bounded-wait abort path, made to run out on purpose without faulting
anything: the context's wait limit is set to 1 us, so that waits for weights
in flight and for accumulators (and, on the decode kernel, the grid
barriers) give up.  The tcgen05 case runs the V4.1 layer at 64 tokens, whose
items take tens of microseconds.  The call
must report MOE_FP4_ETIMEOUT through moe_fp4_last_error, the kernels must
still let every copy in flight land and free what they hold, and with the
default limit restored the same context must produce oracle-exact routing and
outputs within the parity bar again."""
import pytest
import torch

from fp4_routed_expert_router_b200 import moe, synth
from tests.gpu_helpers import Filled, check_routing, check_y, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    f = Filled(synth.WORKLOADS["tiny"], max_tokens=256, from_host=True)
    yield f
    f.close()


@pytest.fixture(scope="module")
def v41():
    f = Filled(synth.WORKLOADS["decode_b64"], max_tokens=64)
    yield f
    f.close()


def _layer(f, T, step):
    wl = f.wl
    logits, _ = synth.layer_inputs(wl, 0, step, tokens=T)
    x = synth.gen_x(wl.seed, T, wl.hidden, step)
    r = f.ctx.route(0, to_dev(logits))
    y = f.ctx.forward(0, to_dev(x), r)
    torch.cuda.synchronize()
    return logits, x, r, y


@pytest.mark.parametrize("which,path,T", [("tiny", moe.PATH_GEMV, 4), ("v41", moe.PATH_TC, 64)])
def test_wait_limit_runs_out_then_context_recovers(request, which, path, T):
    tiny = request.getfixturevalue(which)
    wl = tiny.wl
    tiny.ctx.set_path(path)
    assert tiny.ctx.last_error()[0] == moe.OK
    tiny.ctx.set_wait_limit_us(1)
    try:
        _layer(tiny, T, 6000 + T)
        rc, msg = tiny.ctx.last_error()
        assert rc == moe.ETIMEOUT, (rc, msg)
        assert "timed out" in msg
    finally:
        tiny.ctx.set_wait_limit_us(0)
    for step in (6100 + T, 6200 + T):          # the same context, twice, with the default limit
        logits, x, r, y = _layer(tiny, T, step)
        rc, msg = tiny.ctx.last_error()
        assert rc == moe.OK, msg
        ids, w = check_routing(r, logits, wl.top_k, wl.n_experts)
        check_y(y.cpu().numpy(), tiny.oracle_y(0, x, ids, w, range(T)))
    tiny.ctx.set_path(moe.PATH_AUTO)
