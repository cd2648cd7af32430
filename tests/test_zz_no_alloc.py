"""moe_fp4_forward_noalloc: the forward for callers that may not allocate
device memory (for example a plugin whose host framework owns all device
memory and forbids allocation on its execution path).  Its scratch is a
library-owned static device array, so the call takes only caller-provided
inputs and outputs.  Checked through the C ABI against moe_fp4_forward on the
same arena and routing, on two calls in a row (the second reuses scratch the
first left behind), and for its size limit."""
import numpy as np
import pytest
import torch

from fp4_routed_expert_router_b200 import moe, synth
from tests.gpu_helpers import Filled, check_y, to_dev

pytestmark = pytest.mark.gpu


def _slot_table(f: Filled) -> torch.Tensor:
    wl = f.wl
    t = np.full((f.L, wl.n_experts), -1, dtype=np.int32)
    for (layer, e), s in f.slot_of.items():
        t[layer, e] = s
    return torch.from_numpy(t).cuda()


@pytest.mark.parametrize("name,T", [("tiny", 4), ("tiny", 37), ("decode_b1", 1), ("decode_b1", 8)])
def test_noalloc_matches_forward_twice(name, T):
    wl = synth.WORKLOADS[name]
    f = Filled(wl, max_tokens=max(T, 8), from_host=(name == "tiny"))
    try:
        table = _slot_table(f)
        err = torch.zeros(4, dtype=torch.int32, device="cuda")
        for step in (0, 1):                      # two calls in a row, different tokens
            logits, _ = synth.layer_inputs(wl, 0, 500 + step, tokens=T)
            x = to_dev(synth.gen_x(wl.seed, T, wl.hidden, 500 + step))
            r = f.ctx.route(0, to_dev(logits))
            y_ref = f.ctx.forward(0, x, r)
            y = torch.full_like(y_ref, float("nan"))
            xo = torch.empty_like(x)
            rc = moe.forward_noalloc(f.ctx.cfg, f.ctx.arena_ptr(), table, 0, x, r, y, x_out=xo, err=err)
            assert rc == moe.OK
            torch.cuda.synchronize()
            assert int(err[0]) == 0
            assert f.ctx.last_error()[0] == moe.OK
            check_y(y.cpu().numpy(), y_ref.cpu().numpy().astype(np.float64))
            xr = synth.bf16_bits_to_f32(x.cpu().numpy().view(np.uint16)) + y.cpu().numpy()
            assert np.array_equal(xo.cpu().numpy().view(np.uint16), synth.f32_to_bf16_bits(xr))
    finally:
        f.close()


def _need(T: int, wl, sms: int) -> int:
    """Scratch bytes of a call, as the header states them (the middle parts rounded up to 256)."""
    H, I, k = wl.hidden, wl.inter, wl.top_k
    KU, KD = H // 128, I // 128
    parts = [T * KU * 512, T * KU * 128, T * k * KD * 512, T * k * KD * 128, sms * 6144]
    return 656640 + sum((p + 255) // 256 * 256 for p in parts) + T * k * H * 4


def test_noalloc_rejects_sizes_beyond_the_limits():
    wl = synth.WORKLOADS["decode_b1"]
    cfg = moe.Config(wl.hidden, wl.inter, wl.n_experts, wl.top_k, 1, 1, 4096)
    # the largest T whose scratch fits the 16 MiB array
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    T_ok = max(T for T in range(1, 512) if _need(T, wl, sms) <= (16 << 20))
    if sms == 148:
        assert T_ok == 69
    T = T_ok + 1
    x = torch.zeros((T, wl.hidden), dtype=torch.int16, device="cuda")
    y = torch.empty((T, wl.hidden), dtype=torch.float32, device="cuda")
    r = moe.Routing(torch.zeros((T, 6), dtype=torch.int32, device="cuda"),
                    torch.zeros((T, 6), dtype=torch.float32, device="cuda"),
                    torch.zeros(384, dtype=torch.int32, device="cuda"),
                    torch.zeros(385, dtype=torch.int32, device="cuda"),
                    torch.zeros(T * 6, dtype=torch.int32, device="cuda"))
    arena = torch.empty(256, dtype=torch.uint8, device="cuda")
    table = torch.full((1, 384), -1, dtype=torch.int32, device="cuda")
    assert moe.forward_noalloc(cfg, arena.data_ptr(), table, 0, x, r, y) == moe.EINVAL
    assert moe.forward_noalloc(cfg, arena.data_ptr(), table, 0, x[:T_ok], r, y) == moe.OK
    # router weights that are not 4-byte aligned are an argument error, before any launch
    wbad = r.weights.reshape(-1).view(torch.uint8)[1:]
    assert moe.forward_noalloc(cfg, arena.data_ptr(), table, 0, x[:1],
                               moe.Routing(r.ids, wbad, r.counts, r.offsets, r.perm), y) == moe.EINVAL
    torch.cuda.synchronize()
