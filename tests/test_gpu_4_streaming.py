"""Expert streaming into an arena smaller than the expert set
(moe_fp4_stream_experts): each step routes on the GPU, streams the chosen
experts' checkpoint objects from pinned host memory into LRU slots, and runs
the forward; outputs must match the oracle, and slots / hit counts must match
a least-recently-used model of the same requests."""
import numpy as np
import pytest
import torch

import oracle
from fp4_routed_expert_router_b200 import moe, synth
from tests.gpu_helpers import check_routing, check_y, to_dev

pytestmark = pytest.mark.gpu


def _lru(n_slots):
    owner, last, clock = [None] * n_slots, [0] * n_slots, [0]

    def request(keys):
        clock[0] += 1
        where = {k: s for s, k in enumerate(owner) if k is not None}
        for k in keys:
            if k in where:
                last[where[k]] = clock[0]
        slots, hits = [], 0
        for k in keys:
            if k in where:
                slots.append(where[k])
                hits += 1
                continue
            free = [s for s in range(n_slots) if owner[s] is None]
            v = free[0] if free else min((s for s in range(n_slots) if last[s] < clock[0]),
                                         key=lambda s: (last[s], s))
            if owner[v] is not None:
                del where[owner[v]]
            owner[v] = k
            where[k] = v
            last[v] = clock[0]
            slots.append(v)
        return slots, hits
    return request


def _objects(wl, experts):
    out = {}
    for e in experts:
        t = synth.gen_expert(wl.seed, 0, int(e), wl.hidden, wl.inter, wl.scale_lo, wl.scale_hi)
        out[int(e)] = torch.from_numpy(synth.expert_object(t, wl.hidden, wl.inter)).pin_memory()
    return out


@pytest.mark.parametrize("name,n_slots,T,steps", [("tiny", 5, 2, 14), ("decode_b1", 12, 1, 5)])
def test_streamed_forward_matches_oracle_and_lru(name, n_slots, T, steps):
    wl = synth.WORKLOADS[name]
    ctx = moe.Context(wl.hidden, wl.inter, wl.n_experts, wl.top_k, 1, n_slots, 8)
    model = _lru(n_slots)
    objs = {}
    hits = misses = 0
    try:
        for step in range(steps):
            logits, _ = synth.layer_inputs(wl, 0, 300 + step, tokens=T)
            x = synth.gen_x(wl.seed, T, wl.hidden, 300 + step)
            r = ctx.route(0, to_dev(logits))
            ids, w = check_routing(r, logits, wl.top_k, wl.n_experts)
            need = sorted({int(e) for e in ids.reshape(-1)})
            objs.update(_objects(wl, [e for e in need if e not in objs]))
            slots = ctx.stream_experts(0, need, [objs[e] for e in need])
            want_slots, h = model(need)
            assert slots == want_slots
            hits += h
            misses += len(need) - h
            y = ctx.forward(0, to_dev(x), r).cpu().numpy()
            rc, msg = ctx.last_error()
            assert rc == moe.OK, msg
            ref = oracle.moe_forward(x, ids, w, {e: objs[e].numpy() for e in need}, wl.n_experts, wl.hidden,
                                     wl.inter)
            check_y(y, ref)
        st = ctx.residency_stats()
        assert st == (hits, misses, misses * wl.expert_bytes)
        assert misses > n_slots            # the arena really was recycled
    finally:
        ctx.close()


def test_stream_experts_rejects_bad_requests():
    wl = synth.WORKLOADS["tiny"]
    ctx = moe.Context(wl.hidden, wl.inter, wl.n_experts, wl.top_k, 1, 3, 8)
    objs = _objects(wl, range(4))
    try:
        for experts, objects in [([1, 1], [objs[1], objs[1]]),          # repeated
                                 ([0, 1, 2, 3], [objs[e] for e in range(4)]),   # more than the slots
                                 ([2], [None]),                         # not resident, no object
                                 ([16], [objs[0]])]:                    # out of range
            with pytest.raises(moe.MoeError) as ex:
                ctx.stream_experts(0, experts, objects)
            assert ex.value.status == moe.EINVAL
        assert ctx.residency_stats() == (0, 0, 0)
        assert ctx.stream_experts(0, [2], [objs[2]]) == [0]
        assert ctx.stream_experts(0, [2], [None]) == [0]            # resident: no object needed
        assert ctx.residency_stats() == (1, 1, wl.expert_bytes)
    finally:
        ctx.close()
