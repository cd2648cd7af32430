"""The expert-parallel building blocks on the GPU: moe_fp4_expert_outputs on
a forward's (token, slot) entries followed by moe_fp4_combine must reproduce
moe_fp4_forward bit for bit (same per-expert grouping, same kernels), and the
expert-parallel driver over a one-rank NCCL group, with either dispatch plan,
must give the same y and meet the oracle bar on every token."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from fp4_routed_expert_router_b200 import ep, moe, synth
from tests.gpu_helpers import Filled, check_y, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    f = Filled(synth.WORKLOADS["tiny"], max_tokens=256)
    yield f
    f.close()


@pytest.fixture(scope="module")
def v41():
    f = Filled(synth.WORKLOADS["decode_b64"], max_tokens=64)
    yield f
    f.close()


def _pieces_vs_forward(f, T, step, path):
    wl = f.wl
    logits, _ = synth.layer_inputs(wl, 0, step, tokens=T)
    xd = to_dev(synth.gen_x(wl.seed, T, wl.hidden, step))
    f.ctx.set_path(path)
    r = f.ctx.route(0, to_dev(logits))
    y = f.ctx.forward(0, xd, r).clone()
    rows = xd.repeat_interleave(wl.top_k, dim=0).contiguous()           # entry t*k+j -> row of token t
    o = f.ctx.expert_outputs(0, rows, r.ids.reshape(-1).contiguous())
    y2 = f.ctx.combine(o, r.weights)
    torch.cuda.synchronize()
    rc, msg = f.ctx.last_error()
    assert rc == moe.OK, msg
    assert torch.equal(y, y2)
    return r, xd, y


@pytest.mark.parametrize("path,T", [(moe.PATH_GEMV, 17), (moe.PATH_TC, 130), (moe.PATH_AUTO, 200)])
def test_tiny_expert_outputs_and_combine_equal_forward(tiny, path, T):
    _pieces_vs_forward(tiny, T, 4000 + T, path)


@pytest.mark.parametrize("path", [moe.PATH_GEMV, moe.PATH_TC])
def test_v41_expert_outputs_and_combine_equal_forward(v41, path):
    _pieces_vs_forward(v41, 64, 4100, path)


@pytest.mark.parametrize("device_plan", [True, False])
def test_expert_parallel_driver_one_rank_nccl(tiny, device_plan):
    """The driver over a one-rank NCCL group, with the device plan (fixed-capacity
    slots padded with expert id -1, no host read) or the host plan: y equals
    moe_fp4_forward bit for bit and meets the oracle bar on every token."""
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        T, step = 33, 4200
        r, xd, y = _pieces_vs_forward(tiny, T, step, moe.PATH_AUTO)
        wl = tiny.wl
        layer = ep.ExpertParallel(wl.n_experts, wl.top_k, wl.hidden, max_tokens=48)
        y_ep = layer.forward(xd, r.ids, r.weights, ep.gpu_expert_fn(tiny.ctx, 0), ep.gpu_combine_fn(tiny.ctx),
                             device_plan=device_plan)
        torch.cuda.synchronize()
        rc, msg = tiny.ctx.last_error()
        assert rc == moe.OK, msg
        assert torch.equal(y_ep, y)
        x = synth.gen_x(wl.seed, T, wl.hidden, step)
        check_y(y_ep.cpu().numpy(), tiny.oracle_y(0, x, r.ids.cpu().numpy(), r.weights.cpu().numpy(), range(T)))
    finally:
        dist.destroy_process_group()
