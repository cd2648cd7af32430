"""Benchmark of the routed-expert FP4 FFN layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_b1|decode_b64|prefill_2048]

One step = one pass of the whole path (route + w1/w3 GEMM + SwiGLU + w2 GEMM
+ combine) over one batch of fresh synthetic tokens of one DeepSeek-V4.1-Flash
layer (hidden 5120, inter 2304, 384 experts resident in the arena, top-6).
The JSON line's value is the --workload (default decode batch 1); the other
workloads of the same layer (decode batch 64, prefill 2048 tokens) are timed
on the same arena right after it, then decode batch 1 with only 25 % of the
experts resident and the rest streamed from pinned host memory, then the
40-layer stack (batch 1 and 8, its own 115.8 GB arena), all reported under
"workloads".
Inputs are resident in HBM when a timed step starts; L2 is flushed between
timed steps (a 2x L2-sized write whose lines are then discarded), so expert
bytes really come from HBM, and the step's small inputs (x, logits) are
written after the flush, as the preceding layer of a model leaves them.
Rank 0 prints one JSON line.  Under torchrun each rank runs an independent
replica (data parallel, no collective on the data path): weak scaling.

``--impl reference`` times the CPU oracle (oracle/) on the host cores, on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp4_routed_expert_router_b200 import synth  # noqa: E402

METRIC = "MoE FP4 expert-FFN: decode HBM GB/s & tok/s (b=1); prefill TFLOP/s @2048 tok"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="decode_b1", choices=["decode_b1", "decode_b64", "prefill_2048"])
    p.add_argument("--experts", type=int, default=0,
                   help="resident experts override (a smaller arena for ncu captures; 0 = the workload's)")
    p.add_argument("--no-graph", action="store_true", help="launch eagerly instead of a CUDA graph")
    p.add_argument("--only", action="store_true",
                   help="time only --workload (skip the other workloads of the same layer)")
    return p.parse_args()


def workload_config(wl: synth.Workload) -> dict:
    """The workload a line measures; identical for both arms (how it is launched is reported apart)."""
    return {
        "workload": f"{wl.name}: one DeepSeek-V4.1-Flash routed-expert layer, {wl.notes}",
        "hidden": wl.hidden, "inter": wl.inter, "n_experts": wl.n_experts, "top_k": wl.top_k,
        "tokens_per_step": wl.tokens, "experts_resident": wl.n_experts,
        "expert_bytes": wl.expert_bytes, "weights": "fp4 e2m1 + ue8m0 per 32 along K",
        "logits": f"N(0,1) + Zipf(1.1) bias, alpha {wl.zipf_alpha}",
        "scale_exponents": f"uniform {wl.scale_lo}..{wl.scale_hi}",
        "l2": "flushed between timed steps (2x L2 write, then its lines discarded); the step's small inputs "
              "(x, logits) are written after the flush, as the preceding layer leaves them, the expert "
              "weights come from HBM",
        "parallelism": "replicas (one independent layer per GPU)",
    }


def launch_desc(wl: synth.Workload, graph: bool) -> str:
    return (("cuda graph of moe_fp4_route_forward" if graph else "eager moe_fp4_route_forward") +
            (" (one persistent kernel per step)" if wl.tokens * wl.top_k <= 64 else
             " (route kernel, then the expert kernels)"))


# ============================================================================ oracle arm
def _oracle_step(wl, step, cache, n_threads):
    """One step of the oracle: route + forward of wl.tokens fresh tokens.
    Returns (tokens, seconds) with expert generation excluded from the time."""
    import oracle
    logits, _ = synth.layer_inputs(wl, 0, step)
    x = synth.gen_x(wl.seed, wl.tokens, wl.hidden, step)
    t0 = time.perf_counter()
    ids, w = oracle.route(logits, wl.top_k)
    t_route = time.perf_counter() - t0
    objs = {}
    for e in np.unique(ids):
        e = int(e)
        if e not in cache:
            cache[e] = synth.expert_object(synth.gen_expert(wl.seed, 0, e, wl.hidden, wl.inter, wl.scale_lo,
                                                            wl.scale_hi), wl.hidden, wl.inter)
        objs[e] = cache[e]
    t1 = time.perf_counter()
    oracle.moe_forward(x, ids, w, objs, wl.n_experts, wl.hidden, wl.inter, n_threads=n_threads)
    return wl.tokens, t_route + time.perf_counter() - t1


def cpu_baseline(wl: synth.Workload, budget_s: float = 15.0, max_steps: int = 64) -> dict:
    """The oracle timed on this host's cores on a bounded sample of the workload."""
    import oracle
    n_threads = oracle.max_threads()
    if wl.tokens > 8:   # sample 8-token batches of the big workloads
        wl = synth.Workload(**{**wl.__dict__, "tokens": 8})
    cache, toks, secs, steps = {}, 0, 0.0, 0
    while steps < max_steps and secs < budget_s:
        n, s = _oracle_step(wl, 10_000 + steps, cache, n_threads)
        toks += n
        secs += s
        steps += 1
    return {"value": toks / secs, "unit": "tok/s", "cores": n_threads, "kind": "oracle",
            "sample": f"{steps} steps x {wl.tokens} token(s) of {wl.name} (fp64 oracle, OpenMP over "
                      f"(token, expert) pairs, expert generation excluded), {secs:.1f} s"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    n_threads = oracle.max_threads()
    swl = wl if wl.tokens <= 8 else synth.Workload(**{**wl.__dict__, "tokens": 8})
    cache = {}
    for i in range(args.warmup):
        _oracle_step(swl, 20_000 + i, cache, n_threads)
    toks, secs = 0, 0.0
    for i in range(args.steps):
        n, s = _oracle_step(swl, 30_000 + i, cache, n_threads)
        toks += n
        secs += s
    value = toks / secs
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "launch": "fp64 oracle on the host cores (OpenMP over token-expert pairs)",
            "cpu_baseline": {"value": value, "unit": "tok/s", "cores": n_threads, "kind": "oracle",
                             "sample": f"{args.steps} steps x {swl.tokens} token(s) of {wl.name}"},
            "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ============================================================================ GPU arm
class ClockSampler:
    """SM clock and throttle-reason sampling DURING the timed region: an NVML
    reader thread polling every ~0.5 ms (read-only queries), with nvidia-smi
    as a fallback when NVML is unavailable."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_index: int):
        self.idx = device_index
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = False

    def _poll(self, nv, h):
        masks = [(n, getattr(nv, c, 0)) for n, c in self.REASONS]
        while not self._stop:
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for n, m in masks:
                    if m and (r & m):
                        self.reasons.add(n)
            except Exception:
                break
            time.sleep(0.0005)

    def __enter__(self):
        import threading
        self._thread = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self._physical_index())
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def _physical_index(self) -> int:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                return int(vis.split(",")[self.idx])
            except (ValueError, IndexError):
                pass
        return self.idx

    def __exit__(self, *exc):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def measured_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def source_digest(files) -> str:
    """Digest of the listed CUDA sources (sha256 over name, NUL, bytes, in list
    order): a stored ncu traffic figure is used only while the sources of the
    kernel it was taken from are unchanged."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fp4_routed_expert_router_b200", "csrc")
    for name in files:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str, path: str | None = None):
    """DRAM bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)
    recorded in profiles/traffic.json (or ``path``) for this kernel and
    workload, or None when there is none or its sources changed since the
    capture."""
    p = path or os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(f"{kernel}@{workload}")
    if not rec:
        return None
    try:
        if source_digest(rec["files"]) != rec["source_digest"]:
            return None
    except OSError:
        return None
    return rec.get("bytes_per_launch")


class Bench:
    """One resident layer (all experts in the arena) and the timing loops."""

    def __init__(self, wl, local, rank, max_tokens):
        import torch
        from fp4_routed_expert_router_b200 import moe
        self.torch, self.moe = torch, moe
        self.dev = torch.device("cuda", local)
        self.rank = rank
        self.wl = wl
        self.ctx = moe.Context(wl.hidden, wl.inter, wl.n_experts, wl.top_k, 1, wl.n_experts, max_tokens,
                               device=local)
        staging = torch.empty(wl.expert_bytes, dtype=torch.uint8, device=self.dev)
        for e in range(wl.n_experts):
            moe.synth_fill_expert(staging, wl.seed, 0, e, wl.hidden, wl.inter, wl.scale_lo, wl.scale_hi)
            self.ctx.load_expert_object(0, e, e, staging)
        torch.cuda.synchronize()
        rc, msg = self.ctx.last_error()
        assert rc == moe.OK, msg
        l2 = torch.cuda.get_device_properties(self.dev).L2_cache_size
        self.flush = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=self.dev)
        self.stream = torch.cuda.Stream(device=self.dev)

    def run(self, wl, steps, warmup, graph_ok, npool, clocks=False, e2e=False):
        torch, moe, ctx = self.torch, self.moe, self.ctx
        T, dev, stream = wl.tokens, self.dev, self.stream
        pool_x = torch.empty((npool, T, wl.hidden), dtype=torch.int16, device=dev)
        pool_l = torch.empty((npool, T, wl.n_experts), dtype=torch.float32, device=dev)
        for i in range(npool):
            st = self.rank * 100_000 + i
            pool_x[i] = torch.from_numpy(synth.gen_x(wl.seed, T, wl.hidden, st).view(np.int16))
            pool_l[i] = torch.from_numpy(synth.layer_inputs(wl, 0, st)[0])
        x_buf = torch.empty((T, wl.hidden), dtype=torch.int16, device=dev)
        l_buf = torch.empty((T, wl.n_experts), dtype=torch.float32, device=dev)
        y_buf = torch.empty((T, wl.hidden), dtype=torch.float32, device=dev)
        routing = ctx.alloc_routing(T)
        flush = self.flush

        def step_launch():
            ctx.route_forward(0, l_buf, x_buf, out=routing, y=y_buf, stream=stream)

        def stage(i):   # L2 flushed, then the step's inputs written (as the preceding layer leaves them)
            moe.l2_flush(flush, float(i), stream)
            x_buf.copy_(pool_x[i % npool], non_blocking=True)
            l_buf.copy_(pool_l[i % npool], non_blocking=True)

        out = {}
        graph = None
        with torch.cuda.stream(stream):
            stage(0)
            step_launch()
            stream.synchronize()
            if graph_ok:
                try:
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        step_launch()
                    graph = g
                except Exception as ex:  # graph capture unavailable: launch eagerly
                    print(f"# cuda graph capture failed ({ex}); launching eagerly", file=sys.stderr)
                    graph = None
            run = graph.replay if graph is not None else step_launch
            for i in range(warmup):
                stage(i)
                run()
            stream.synchronize()
            rc, msg = ctx.last_error()
            assert rc == moe.OK, msg

            # ---- timed region: K steps, events on the launching stream, L2 flushed between steps
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(steps)]
            if self.world > 1:
                self.dist.barrier()
            torch.cuda.synchronize()
            clk = ClockSampler(dev.index) if clocks else None
            if clk:
                clk.__enter__()
            for i in range(steps):
                stage(1000 + i)
                ev[i][0].record(stream)
                run()
                ev[i][1].record(stream)
            torch.cuda.synchronize()
            if clk:
                clk.__exit__(None, None, None)
                out["clocks"] = clk.summary()
            if self.world > 1:
                self.dist.barrier()
            out["total_ms"] = sum(a.elapsed_time(b) for a, b in ev)

            # ---- per-kernel pass: same steps, events around every kernel
            ctx.set_profile(True)
            ctx.profile_read()
            n_active = []
            for i in range(steps):
                stage(1000 + i)
                step_launch()
                n_active.append(int((routing.counts > 0).sum()))
            recs = ctx.profile_read()
            ctx.set_profile(False)
            out["launches_per_step"] = len(recs) / steps
            per_kernel = {}
            for name, ms in recs:
                per_kernel.setdefault(name, []).append(ms)
            out["kernel_ms"] = {k: sum(v) / len(v) for k, v in per_kernel.items()}
            out["active"] = float(np.mean(n_active))

            if e2e:   # ---- end to end through the public API with host buffers
                hx = torch.empty((npool, T, wl.hidden), dtype=torch.int16, pin_memory=True)
                hl = torch.empty((npool, T, wl.n_experts), dtype=torch.float32, pin_memory=True)
                hx.copy_(pool_x.cpu())
                hl.copy_(pool_l.cpu())
                hy = torch.empty((T, wl.hidden), dtype=torch.float32, pin_memory=True)
                e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                          for _ in range(steps)]
                for i in range(steps):
                    moe.l2_flush(flush, float(i), stream)
                    e2e_ev[i][0].record(stream)
                    x_buf.copy_(hx[i % npool], non_blocking=True)
                    l_buf.copy_(hl[i % npool], non_blocking=True)
                    run()
                    hy.copy_(y_buf, non_blocking=True)
                    e2e_ev[i][1].record(stream)
                torch.cuda.synchronize()
                out["e2e_ms"] = sum(a.elapsed_time(b) for a, b in e2e_ev)
        rc, msg = ctx.last_error()
        assert rc == moe.OK, msg
        del graph
        return out


def run_stack(wls, local, rank, steps, warmup, graph_ok, peaks, world, dist):
    """The 40-layer expert-FFN stack: each layer keeps its n_keep most popular
    experts in one arena (40 x 154 = 6,160 slots, 115.8 GB), the router is
    masked to the kept set, and x <- bf16(x + y) between layers, in place.
    One step = 40 x (route + forward) for one batch of fresh tokens, captured
    in one CUDA graph.  Returns {workload name: summary} for each of ``wls``
    (same layers and experts, different batch sizes), sharing one arena."""
    import torch
    from fp4_routed_expert_router_b200 import moe
    wl0 = wls[0]
    dev = torch.device("cuda", local)
    L, E, H, I, k = wl0.n_layers, wl0.n_experts, wl0.hidden, wl0.inter, wl0.top_k
    kept = wl0.n_keep
    tmax = max(w.tokens for w in wls)
    ctx = moe.Context(H, I, E, k, L, kept * L, max(tmax, 8), device=local)
    staging = torch.empty(wl0.expert_bytes, dtype=torch.uint8, device=dev)
    slot = 0
    for layer in range(L):
        for e in synth.resident_experts(wl0, layer):
            moe.synth_fill_expert(staging, wl0.seed, layer, int(e), H, I, wl0.scale_lo, wl0.scale_hi)
            ctx.load_expert_object(layer, int(e), slot, staging)
            slot += 1
    del staging
    masks = [torch.from_numpy(synth.keep_mask(wl0.seed, l, E, kept)).to(dev) for l in range(L)]
    torch.cuda.synchronize()
    rc, msg = ctx.last_error()
    assert rc == moe.OK, msg
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    out = {}
    for wl in wls:
        T = wl.tokens
        npool = 8
        pool_x = torch.empty((npool, T, H), dtype=torch.int16, device=dev)
        pool_l = torch.empty((npool, L, T, E), dtype=torch.float32, device=dev)
        for i in range(npool):
            st = rank * 100_000 + i
            pool_x[i] = torch.from_numpy(synth.gen_x(wl.seed, T, H, st).view(np.int16))
            for l in range(L):
                pool_l[i, l] = torch.from_numpy(synth.layer_inputs(wl, l, st)[0])
        x_buf = torch.empty((T, H), dtype=torch.int16, device=dev)
        l_buf = torch.empty((L, T, E), dtype=torch.float32, device=dev)
        y_buf = torch.empty((T, H), dtype=torch.float32, device=dev)
        routes = [ctx.alloc_routing(T) for _ in range(L)]

        def step_launch():
            for l in range(L):
                ctx.route_forward(l, l_buf[l], x_buf, keep=masks[l], out=routes[l], y=y_buf, x_out=x_buf,
                                  stream=stream)

        def stage(i):   # L2 flushed, then the step's inputs written (as the preceding layer leaves them)
            moe.l2_flush(flush, float(i), stream)
            x_buf.copy_(pool_x[i % npool], non_blocking=True)
            l_buf.copy_(pool_l[i % npool], non_blocking=True)

        graph = None
        with torch.cuda.stream(stream):
            stage(0)
            step_launch()
            stream.synchronize()
            if graph_ok:
                try:
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        step_launch()
                    graph = g
                except Exception as ex:
                    print(f"# cuda graph capture failed ({ex}); launching eagerly", file=sys.stderr)
            run = graph.replay if graph is not None else step_launch
            for i in range(warmup):
                stage(i)
                run()
            stream.synchronize()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(steps)]
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            clk = ClockSampler(dev.index)
            clk.__enter__()
            active = []
            for i in range(steps):
                stage(1000 + i)
                ev[i][0].record(stream)
                run()
                ev[i][1].record(stream)
            torch.cuda.synchronize()
            clk.__exit__(None, None, None)
            if world > 1:
                dist.barrier()
            for r in routes:     # active experts of the last step, per layer
                active.append(int((r.counts > 0).sum()))
        rc, msg = ctx.last_error()
        assert rc == moe.OK, msg
        total_ms = sum(a.elapsed_time(b) for a, b in ev)
        if world > 1:
            total_ms = max_over_ranks([total_ms], dist, dev)[0]
        ms = total_ms / steps
        nbytes = sum(active) * wl.expert_bytes
        out[wl.name] = {"steps": steps, "tok_s": T * world / (ms * 1e-3), "ms_per_step": ms,
                        "layers": L, "slots": kept * L, "arena_bytes": kept * L * wl.expert_bytes,
                        "expert_bytes_per_step": nbytes, "active_experts_per_step": sum(active),
                        "hbm_gbs_step": nbytes / (ms * 1e-3) / 1e9,
                        "hbm_frac_step": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                        "launch": "one cuda graph of 40 x moe_fp4_route_forward" if graph is not None else "eager",
                        "clocks": clk.summary()}
        del graph
    ctx.close()
    return out


def run_streaming(wl, local, resident_frac, steps, warmup):
    """Decode with an arena smaller than the layer: only resident_frac of the
    experts have slots, the rest stream in on demand from pinned host memory
    (moe_fp4_stream_experts, least recently used slots).  One step = route ->
    chosen ids to the host -> stream the misses -> forward, for one token; the
    host takes part in every step, so the time is wall-clock around the step
    with the device synchronised at both ends."""
    import torch
    from fp4_routed_expert_router_b200 import moe
    dev = torch.device("cuda", local)
    E = wl.n_experts
    n_slots = max(wl.top_k, int(round(resident_frac * E)))
    ctx = moe.Context(wl.hidden, wl.inter, E, wl.top_k, 1, n_slots, 8, device=local)
    staging = torch.empty(wl.expert_bytes, dtype=torch.uint8, device=dev)
    host = []
    for e in range(E):   # the expert store: every expert's checkpoint object in pinned host memory
        moe.synth_fill_expert(staging, wl.seed, 0, e, wl.hidden, wl.inter, wl.scale_lo, wl.scale_hi)
        h = torch.empty(wl.expert_bytes, dtype=torch.uint8, pin_memory=True)
        h.copy_(staging)
        host.append(h)
    del staging
    T = wl.tokens
    npool = 64
    pool_x = [torch.from_numpy(synth.gen_x(wl.seed, T, wl.hidden, 50_000 + i).view(np.int16)).to(dev)
              for i in range(npool)]
    pool_l = [torch.from_numpy(synth.layer_inputs(wl, 0, 50_000 + i)[0]).to(dev) for i in range(npool)]
    r = ctx.alloc_routing(T)
    y = torch.empty((T, wl.hidden), dtype=torch.float32, device=dev)

    def step(i):
        ctx.route(0, pool_l[i % npool], out=r)
        need = sorted({int(e) for e in r.ids.reshape(-1).tolist()})
        ctx.stream_experts(0, need, [host[e] for e in need])
        ctx.forward(0, pool_x[i % npool], r, y=y)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    h0 = ctx.residency_stats()
    t0 = time.perf_counter()
    for i in range(steps):
        step(warmup + i)
    torch.cuda.synchronize()
    sec = time.perf_counter() - t0
    h1 = ctx.residency_stats()
    rc, msg = ctx.last_error()
    assert rc == moe.OK, msg
    hits, misses, nbytes = (h1[j] - h0[j] for j in range(3))
    ctx.close()
    return {"steps": steps, "warmup_steps": warmup, "tok_s": T * steps / sec, "ms_per_step": 1e3 * sec / steps,
            "resident_slots": n_slots, "resident_fraction": n_slots / E,
            "hit_rate": hits / max(1, hits + misses), "misses_per_step": misses / steps,
            "h2d_gbs": nbytes / sec / 1e9, "timing": "wall clock, host in the loop (ids read back every step)",
            "expert_store": "pinned host memory, checkpoint layout"}


def roofline(wl, res, peaks, peak_src):
    """Roofline of the step's dominant kernel.  Decode batches run the whole
    layer in one kernel (decode_layer): its algorithmic bytes are every active
    expert's weights, codes + scales (18,800,640 B each).  Larger batches run
    the tcgen05 GEMMs; the w1/w3 one (tc_up) dominates: active experts x w1/w3
    codes + scales.  Algorithmic FLOPs = 2 H I per matrix per token-expert
    pair.  The bound is the one the arithmetic intensity selects against the
    measured ridge point; a tensor-core kernel also reports its fraction of
    the bf16 peak."""
    E, H, I, k, T = wl.n_experts, wl.hidden, wl.inter, wl.top_k, wl.tokens
    avg, act = res["kernel_ms"], res["active"]
    if "decode_layer" in avg:
        kern = "decode_layer"
        nbytes = act * wl.expert_bytes
        flops = 6.0 * H * I * T * k
    else:
        kern = "tc_up" if "tc_up" in avg else max(avg, key=avg.get)
        nbytes = act * 2 * (I * H // 2 + I * H // 32)
        flops = 2.0 * 2.0 * H * I * T * k
    sec = avg[kern] * 1e-3
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    gbs, tfs = nbytes / sec / 1e9, flops / sec / 1e12
    out_hbm = {"bound": "hbm", "kernel": kern, "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
               "frac": gbs / peaks["hbm_gbs"], "traffic": stored_traffic(kern, wl.name),
               "peak_source": f"{peak_src} hbm_gbs", "algorithmic_bytes_per_launch": nbytes,
               "intensity_flop_per_byte": flops / nbytes, "ridge_flop_per_byte": ridge}
    out_tc = {"bound": "tensor", "kernel": kern, "achieved": tfs, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
              "frac": tfs / peaks["bf16_tflops"], "traffic": stored_traffic(kern, wl.name),
              "peak_source": f"{peak_src} bf16_tflops (burst; kernel timed per launch)",
              "algorithmic_flops_per_launch": flops}
    hbm_bound = flops / nbytes < ridge
    main = dict(out_hbm if hbm_bound else out_tc)
    if kern == "tc_up":
        main["other"] = out_tc if hbm_bound else out_hbm
    return main


def summary(wl, res, steps, world, peaks, peak_src):
    E, H, I, k, T = wl.n_experts, wl.hidden, wl.inter, wl.top_k, wl.tokens
    ms = res["total_ms"] / steps
    act = res["active"]
    layer_bytes = act * (2 * (I * H // 2 + I * H // 32) + H * I // 2 + H * I // 32)
    flops = 6.0 * H * I * T * k
    return {"tok_s": T * world / (ms * 1e-3), "ms_per_step": ms,
            "expert_bytes_per_step": layer_bytes,
            "hbm_gbs_step": layer_bytes / (ms * 1e-3) / 1e9,
            "hbm_frac_step": layer_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "tflops_step": flops / (ms * 1e-3) / 1e12,
            "tensor_frac_step": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"],
            "active_experts_per_step": act, "kernel_ms": res["kernel_ms"],
            "roofline": roofline(wl, res, peaks, peak_src)}


def max_over_ranks(values, dist, device):
    """Element-wise maximum of per-rank timings over the process group (every
    rank takes this same collective step).  The multi-GPU number is the
    slowest rank's device time."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    # the other workloads of the same layer (same experts and seed), measured on the same arena
    others = [] if args.only else [n for n in ("decode_b1", "decode_b64", "prefill_2048")
                                   if n != wl.name and synth.WORKLOADS[n].n_experts == wl.n_experts]
    max_tokens = max([wl.tokens] + [synth.WORKLOADS[n].tokens for n in others] + [8])
    bench = Bench(wl, local, rank, max_tokens)
    bench.world, bench.dist = world, dist
    peaks, peak_src = measured_peaks()

    res = bench.run(wl, args.steps, args.warmup, not args.no_graph, 64, clocks=True, e2e=True)
    sec = {}
    for n in others:
        w2 = synth.WORKLOADS[n]
        steps2 = min(args.steps, 20)
        r2 = bench.run(w2, steps2, max(3, min(args.warmup, 5)), not args.no_graph, 8, clocks=True)
        sec[n] = {"steps": steps2, **summary(w2, r2, steps2, world, peaks, peak_src), "clocks": r2["clocks"]}

    if not args.only and wl.name == "decode_b1" and world == 1:   # host memory and PCIe are shared by ranks
        # steady state of the LRU: 200 warm-up steps, then 200 timed ones, whatever --steps / --warmup
        sec["stream_decode_b1_25pct"] = run_streaming(wl, local, 0.25, 200, 200)
    if not args.only and wl.n_experts == synth.WORKLOADS["stack40_b1"].n_experts:
        bench.ctx.close()
        bench.ctx = None
        torch.cuda.empty_cache()
        stack = [synth.WORKLOADS[n] for n in ("stack40_b1", "stack40_b8")]
        sec.update(run_stack(stack, local, rank, min(args.steps, 20), max(3, min(args.warmup, 5)),
                             not args.no_graph, peaks, world, dist))

    total_ms, e2e_ms = res["total_ms"], res["e2e_ms"]
    if world > 1:
        total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dist, dev)
        res["total_ms"] = total_ms

    s = summary(wl, res, args.steps, world, peaks, peak_src)
    T = wl.tokens
    toks = T * args.steps * world
    line = {
        "metric": METRIC, "value": toks / (total_ms * 1e-3), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(wl), "launch": launch_desc(wl, not args.no_graph),
        "hbm_gbs_step": s["hbm_gbs_step"], "hbm_frac_step": s["hbm_frac_step"],
        "kernel_ms": s["kernel_ms"],
        "roofline": s["roofline"],
        "active_experts_per_step": s["active_experts_per_step"],
        "e2e": {"value": toks / (e2e_ms * 1e-3), "unit": "tok/s",
                "h2d_bytes_per_step": T * (wl.hidden * 2 + wl.n_experts * 4),
                "d2h_bytes_per_step": T * wl.hidden * 4},
        "gpu_launches": int(round(res["launches_per_step"] * args.steps)),
        "clocks": res["clocks"],
        "workloads": sec,
    }
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if bench.ctx is not None:
        bench.ctx.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    wl = synth.WORKLOADS[args.workload]
    if args.experts:
        import dataclasses
        wl = dataclasses.replace(wl, name=f"{wl.name}_e{args.experts}", n_experts=args.experts,
                                 notes=f"{wl.notes} (profiling case: {args.experts} experts)")
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
