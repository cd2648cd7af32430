"""Expert-parallel dispatch / combine (fp4_routed_expert_router_b200.ep) on
CPU gloo ranks, with the oracle as each rank's expert computation: the
sharded result must equal the single-process oracle layer bit for bit (the
same fp64 expert outputs, combined in the same slot order)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
H, I, E, K = 64, 96, 8, 3


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(seed):
    from fp4_routed_expert_router_b200 import synth
    objs = {}
    for e in range(E):
        t = synth.gen_expert(seed, 0, e, H, I, 118, 124)
        objs[e] = synth.expert_object(t, H, I)
    return objs


def _tokens(rank, T):
    import oracle
    from fp4_routed_expert_router_b200 import synth
    x = synth.gen_x(900 + rank, T, H)
    logits = np.random.default_rng(910 + rank).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(logits, K) if T else (np.zeros((0, K), np.int32), np.zeros((0, K)))
    return x, ids, w


def _rank_main(rank, world, port, tokens_per_rank, out):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    from fp4_routed_expert_router_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        layer = ep.ExpertParallel(E, K, H)
        all_objs = _layer(77)
        mine = {e: all_objs[e] for e in layer.owned()}        # this rank holds only its shard

        def expert_fn(x_rows, experts):
            xe = x_rows.numpy().view(np.uint16)
            e = experts.numpy().astype(np.int32).reshape(-1, 1)
            o = oracle.moe_forward(xe, e, np.ones(e.shape), mine, E, H, I)
            return torch.from_numpy(o)

        def combine_fn(o, weights):
            o = o.numpy().reshape(-1, K, H)
            w = weights.numpy()
            y = np.zeros((o.shape[0], H))
            for j in range(K):
                y += w[:, j:j + 1] * o[:, j]
            return torch.from_numpy(y)

        x, ids, w = _tokens(rank, tokens_per_rank[rank])
        y = layer.forward(torch.from_numpy(x.view(np.int16)), torch.from_numpy(ids.astype(np.int64)),
                          torch.from_numpy(w), expert_fn, combine_fn)
        out[rank] = y.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,tokens", [(2, [5, 3]), (4, [4, 0, 7, 2])])
def test_expert_parallel_matches_single_process(world, tokens):
    import oracle
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, tokens, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    objs = _layer(77)
    for r in range(world):
        x, ids, w = _tokens(r, tokens[r])
        want = oracle.moe_forward(x, ids, w, objs, E, H, I) if tokens[r] else np.zeros((0, H))
        assert np.array_equal(out[r], want), f"rank {r}"
