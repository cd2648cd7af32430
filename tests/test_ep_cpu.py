"""Expert-parallel dispatch / combine (fp4_routed_expert_router_b200.ep) on
CPU gloo ranks, with the oracle as each rank's expert computation: the
sharded result must equal the single-process oracle layer bit for bit (the
same fp64 expert outputs, combined in the same slot order), under both
dispatch plans; and the device plan must not read anything back to the host
(counted by wrapping the tensor methods that do)."""
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


def _oracle_fns(mine):
    import oracle

    def expert_fn(x_rows, experts):
        """o rows of the owned experts; rows with expert id -1 are empty slots (zero)."""
        e_all = experts.numpy().astype(np.int32)
        o = np.zeros((e_all.shape[0], H))
        live = np.nonzero(e_all >= 0)[0]
        if live.size:
            xe = x_rows.numpy().view(np.uint16)[live]
            o[live] = oracle.moe_forward(xe, e_all[live].reshape(-1, 1), np.ones((live.size, 1)), mine, E, H, I)
        return torch.from_numpy(o)

    def combine_fn(o, weights):
        o = o.numpy().reshape(-1, K, H)
        w = weights.numpy()
        y = np.zeros((o.shape[0], H))
        for j in range(K):
            y += w[:, j:j + 1] * o[:, j]
        return torch.from_numpy(y)

    return expert_fn, combine_fn


def _rank_main(rank, world, port, tokens_per_rank, device_plan, out):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    from fp4_routed_expert_router_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        layer = ep.ExpertParallel(E, K, H, max_tokens=max(tokens_per_rank))
        all_objs = _layer(77)
        mine = {e: all_objs[e] for e in layer.owned()}        # this rank holds only its shard
        expert_fn, combine_fn = _oracle_fns(mine)
        x, ids, w = _tokens(rank, tokens_per_rank[rank])
        y = layer.forward(torch.from_numpy(x.view(np.int16)), torch.from_numpy(ids.astype(np.int64)),
                          torch.from_numpy(w), expert_fn, combine_fn, device_plan=device_plan)
        out[rank] = y.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("device_plan", [False, True])
@pytest.mark.parametrize("world,tokens", [(2, [5, 3]), (4, [4, 0, 7, 2]),
                                          (3, [5, 2, 4]),         # 8 experts as 3 + 3 + 2
                                          (5, [3, 1, 0, 4, 2])])  # 2 + 2 + 2 + 2 + 0: a rank owns none
def test_expert_parallel_matches_single_process(world, tokens, device_plan):
    import oracle
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, tokens, device_plan, out))
             for r in range(world)]
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


def _count_rank(rank, world, port, device_plan, out):
    """One layer on a gloo rank with every host read of a tensor counted, except
    inside the expert and combine callables (their host work is the oracle's)."""
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from fp4_routed_expert_router_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    counting = {"on": False, "n": 0, "what": []}
    patched = {}

    def wrap(name):
        orig = getattr(torch.Tensor, name)

        def f(self, *a, **kw):
            # a .to() is a host read when it names the host explicitly (moves to the
            # data's own device are not, and on CPU ranks that device is the host)
            host = name != "to" or any(isinstance(v, str) and v.startswith("cpu") for v in list(a) + list(kw.values()))
            if counting["on"] and host:
                counting["n"] += 1
                counting["what"].append(name)
            return orig(self, *a, **kw)
        patched[name] = orig
        setattr(torch.Tensor, name, f)

    try:
        for name in ("item", "tolist", "cpu", "numpy", "__bool__", "to"):
            wrap(name)
        layer = ep.ExpertParallel(E, K, H, max_tokens=6)
        all_objs = _layer(77)
        mine = {e: all_objs[e] for e in layer.owned()}
        efn, cfn = _oracle_fns(mine)

        def expert_fn(x_rows, experts):
            counting["on"] = False
            try:
                return efn(x_rows, experts)
            finally:
                counting["on"] = True

        def combine_fn(o, weights):
            counting["on"] = False
            try:
                return cfn(o, weights)
            finally:
                counting["on"] = True

        x, ids, w = _tokens(rank, 6)
        xt, it, wt = torch.from_numpy(x.view(np.int16)), torch.from_numpy(ids.astype(np.int64)), torch.from_numpy(w)
        counting["on"] = True
        y = layer.forward(xt, it, wt, expert_fn, combine_fn, device_plan=device_plan)
        counting["on"] = False
        out[rank] = (counting["n"], counting["what"], y.numpy())
    finally:
        for name, orig in patched.items():
            setattr(torch.Tensor, name, orig)
        dist.destroy_process_group()


def test_device_plan_reads_nothing_back_to_the_host():
    """The device plan's dispatch makes no host read (no .item/.tolist/.cpu/
    .numpy/bool/.to('cpu') on any tensor outside the expert and combine calls);
    the host plan needs its split sizes on the host; both give the oracle layer."""
    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    res = {}
    for device_plan in (True, False):
        mgr = ctx.Manager()
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_count_rank, args=(r, world, port, device_plan, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
            assert p.exitcode == 0
        res[device_plan] = dict(out)
    objs = _layer(77)
    for r in range(world):
        n_dev, what_dev, y_dev = res[True][r]
        n_host, _, y_host = res[False][r]
        assert n_dev == 0, f"rank {r}: device plan read back {what_dev}"
        assert n_host > 0
        x, ids, w = _tokens(r, 6)
        want = oracle.moe_forward(x, ids, w, objs, E, H, I)
        assert np.array_equal(y_dev, want) and np.array_equal(y_host, want), f"rank {r}"
