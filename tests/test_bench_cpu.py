"""Host logic of bench.py and of the expert-parallel dispatch plan, on CPU:
the roofline bound follows the arithmetic intensity, stored ncu traffic is
used only while the kernel sources match its digest, and the dispatch plan
orders entries by (owner rank, token, slot)."""
import importlib.util
import json
import os
import socket

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PEAKS = {"hbm_gbs": 6547.5, "bf16_tflops": 1674.6, "bf16_tflops_sustained": 1363.4}


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def test_decode_roofline_is_hbm_with_algorithmic_bytes(bench):
    """The one-kernel decode step: its algorithmic bytes are the six experts'
    full objects (w1, w3, w2 codes and scales), 6 x 18,800,640 bytes."""
    from fp4_routed_expert_router_b200 import synth
    wl = synth.WORKLOADS["decode_b1"]
    r = bench.roofline(wl, {"kernel_ms": {"decode_layer": 0.030}, "active": 6.0}, PEAKS, "test")
    layer_bytes = 6 * (3 * 2304 * 5120 // 2 + 3 * 2304 * 5120 // 32)
    assert r["bound"] == "hbm" and r["kernel"] == "decode_layer"
    assert r["algorithmic_bytes_per_launch"] == layer_bytes == 112_803_840
    assert r["achieved"] == pytest.approx(layer_bytes / 30e-6 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["hbm_gbs"])


def test_prefill_roofline_picks_the_bound_by_intensity(bench):
    from fp4_routed_expert_router_b200 import synth
    wl = synth.WORKLOADS["prefill_2048"]
    # 378.8 active experts: 122 FLOP/B, below the ridge (256 FLOP/B) -> HBM-bound, tensor as "other"
    r = bench.roofline(wl, {"kernel_ms": {"tc_up": 3.0}, "active": 378.8}, PEAKS, "test")
    assert r["bound"] == "hbm" and r["other"]["bound"] == "tensor"
    assert r["other"]["algorithmic_flops_per_launch"] == 2.0 * 2.0 * 5120 * 2304 * 2048 * 6
    # few active experts for the same tokens: intensity above the ridge -> tensor-bound
    r = bench.roofline(wl, {"kernel_ms": {"tc_up": 3.0}, "active": 100.0}, PEAKS, "test")
    assert r["bound"] == "tensor" and r["other"]["bound"] == "hbm"


def test_stored_traffic_requires_matching_sources(bench, tmp_path):
    files = ["fp4_cvt.cuh", "slot_layout.cuh"]
    rec = {"k@w": {"bytes_per_launch": 1234, "files": files, "source_digest": bench.source_digest(files)}}
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(rec))
    assert bench.stored_traffic("k", "w", str(p)) == 1234
    assert bench.stored_traffic("k", "other", str(p)) is None
    rec["k@w"]["source_digest"] = "0" * 16              # sources changed since the capture
    p.write_text(json.dumps(rec))
    assert bench.stored_traffic("k", "w", str(p)) is None
    rec["k@w"]["files"] = ["no_such_file.cuh"]
    p.write_text(json.dumps(rec))
    assert bench.stored_traffic("k", "w", str(p)) is None


def test_dispatch_plan_orders_by_owner_then_entry():
    import torch.distributed as dist
    from fp4_routed_expert_router_b200 import ep
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        layer = ep.ExpertParallel(16, 2, 8)
        ids = torch.tensor([[3, 9], [15, 0], [9, 2]])
        p = layer.plan(ids, "cpu")
        assert p.order.tolist() == [0, 1, 2, 3, 4, 5]          # one rank owns everything: entry order kept
        assert p.send_counts == [6] and p.recv_counts == [6]
        # owner of each entry under 4 ranks of 4 experts, ordered stably
        dest = ids.reshape(-1) // 4
        want = sorted(range(6), key=lambda i: (int(dest[i]), i))
        assert np.array_equal(np.argsort(dest.numpy(), kind="stable"), np.array(want))
    finally:
        dist.destroy_process_group()
