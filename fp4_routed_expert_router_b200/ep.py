"""Expert-parallel execution of one routed-expert layer over a process group.

Rank r of G holds experts [r*S, min((r+1)*S, E)) in its arena, S = ceil(E/G)
(so the last ranks may hold fewer, or none, when G does not divide E).  Each rank routes
its own tokens; the (token, selected expert) entries then take one exchange
step to the ranks owning their experts and the expert outputs take one
exchange step back, after which each rank combines its tokens' outputs:

  1. dispatch plan: the rank's T*k entries ordered by (owner rank, token,
     slot); per-destination counts exchanged with all_to_all_single;
  2. x rows and expert ids of the entries sent with all_to_all_single;
  3. the owner computes o = expert(x) for everything it received
     (moe_fp4_expert_outputs on the GPU);
  4. o rows sent back with all_to_all_single, into the same order;
  5. o rows put back in (token, slot) order and combined
     (y[t] = sum_j w[t,j] o[t,j], moe_fp4_combine on the GPU).

The exchanges use torch.distributed (NCCL on GPUs, gloo on CPU); this module
only plans and moves rows.  The expert work and the combine are callables so
that the same plan runs over the CUDA library or, in CPU tests, over the
oracle.  Every rank takes the same collective steps in the same order.

Two plans.  The device plan (decode-sized batches) never reads anything back
to the host: every destination gets a fixed capacity of C = max_tokens * k
slots (max_tokens: the most tokens a rank brings to a layer), an
entry's slot (destination * C + its rank among the entries for that
destination, in (token, slot) order) comes from a stable sort and counts on
the device, unused slots carry expert id -1 (skipped by the expert call),
and the exchanges have equal split sizes.  It moves world * C rows each way
instead of the T*k routed ones.  The host plan (large batches) sends exactly the routed
rows; all_to_all_single needs its split sizes on the host, so it reads the
per-destination counts back once per layer.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


# Largest exchange buffer (bytes of x rows, world * T*k * H * 2) the device plan uses.
DEVICE_PLAN_MAX_BYTES = 64 << 20


@dataclass
class DispatchPlan:
    order: torch.Tensor         # int64 [T*k]: entries (t*k + j) in send order
    send_counts: list[int]      # entries sent to each rank
    recv_counts: list[int]      # entries received from each rank


class ExpertParallel:
    """Contiguous expert shards: rank r owns experts [r*S, min((r+1)*S, E)), S = ceil(E/G)."""

    def __init__(self, n_experts: int, top_k: int, hidden: int, group=None, max_tokens: int | None = None):
        """max_tokens: the most tokens any rank brings to one layer; it sets the
        device plan's capacity (max_tokens * top_k slots per destination) and
        enables that plan."""
        self.group = group
        self.max_tokens = max_tokens
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if n_experts < 1:
            raise ValueError("no experts to shard")
        self.E, self.k, self.H = n_experts, top_k, hidden
        self.per_rank = -(-n_experts // self.world)        # ceil: expert e lives on rank e // per_rank

    def owned(self) -> range:
        lo = min(self.rank * self.per_rank, self.E)
        return range(lo, min(lo + self.per_rank, self.E))

    def plan(self, ids: torch.Tensor, device) -> DispatchPlan:
        """Send order and counts for this rank's routed ids [T, k]; the counts
        are exchanged on `device` (the data's device: CUDA for NCCL, CPU for
        gloo)."""
        flat = ids.reshape(-1).to("cpu", torch.int64)
        dest = flat // self.per_rank
        order = torch.argsort(dest, stable=True)           # (owner, t, j): stable keeps (t, j) order
        send = torch.bincount(dest, minlength=self.world).to(torch.int64)
        send_d = send.to(device)
        recv_d = torch.empty_like(send_d)
        dist.all_to_all_single(recv_d, send_d, group=self.group)
        return DispatchPlan(order, send.tolist(), recv_d.cpu().tolist())

    def plan_device(self, ids: torch.Tensor, cap: int) -> torch.Tensor:
        """Send slot of every entry t*k+j, on the ids' device without a host read:
        destination * cap + rank among the entries for that destination, in
        (token, slot) order (a stable sort of the destinations).  cap >= T*k, so
        no destination overflows."""
        flat = ids.reshape(-1).to(torch.int64)
        n = flat.numel()
        dest = torch.div(flat, self.per_rank, rounding_mode="floor").clamp_(0, self.world - 1)
        order = torch.sort(dest, stable=True).indices
        counts = torch.zeros(self.world, dtype=torch.int64, device=flat.device)
        counts.scatter_add_(0, dest, torch.ones_like(dest))
        starts = torch.cumsum(counts, 0) - counts
        d_sorted = dest.index_select(0, order)
        pos = torch.arange(n, device=flat.device) - starts.index_select(0, d_sorted)
        slot = torch.empty(n, dtype=torch.int64, device=flat.device)
        slot[order] = d_sorted * cap + pos
        return slot

    def _exchange_equal(self, rows: torch.Tensor) -> torch.Tensor:
        """all_to_all with equal splits (rows.shape[0] / world to and from each
        rank), as raw bytes."""
        shape = tuple(rows.shape[1:])
        width = rows.element_size()
        for d in shape:
            width *= d
        flat = rows.contiguous().reshape(rows.shape[0], width // rows.element_size()).view(torch.uint8)
        out = torch.empty_like(flat)
        dist.all_to_all_single(out, flat, group=self.group)
        return out.view(rows.dtype).reshape((rows.shape[0],) + shape)

    def _exchange(self, rows: torch.Tensor, send: list[int], recv: list[int]) -> torch.Tensor:
        """Rows to the other ranks (send[i] rows to rank i, recv[i] from rank i),
        moved as raw bytes so that any row type crosses any backend."""
        shape = tuple(rows.shape[1:])
        width = rows.element_size()
        for d in shape:
            width *= d
        if rows.shape[0] == 0:   # nothing to send (an empty tensor's strides need not allow the byte view)
            flat = torch.empty((0, width), dtype=torch.uint8, device=rows.device)
        else:
            flat = rows.contiguous().reshape(rows.shape[0], width // rows.element_size()).view(torch.uint8)
        out = torch.empty((sum(recv), width), dtype=torch.uint8, device=rows.device)
        dist.all_to_all_single(out, flat, recv, send, group=self.group)
        return out.view(rows.dtype).reshape((sum(recv),) + shape)

    def forward(self, x: torch.Tensor, ids: torch.Tensor, weights: torch.Tensor, expert_fn, combine_fn,
                device_plan: bool | None = None):
        """x [T, H] (bf16 bits), ids/weights [T, k] of this rank's tokens.
        expert_fn(x_rows [n, H], experts [n] int32) -> o [n, H] fp32 for
        experts this rank owns, rows with expert id -1 being empty slots (their
        o rows are never read), and n may be 0 (a rank that received nothing);
        combine_fn(o [T*k, H], weights) -> y [T, H].
        device_plan: True / False forces a plan; None takes the device plan
        when its exchange buffer is at most DEVICE_PLAN_MAX_BYTES.  Every rank
        must take the same plan; the default depends only on the constructor's
        max_tokens, so all ranks agree.  An expert id this
        rank does not own arrives only through a routing error; the expert
        call then latches EINVAL (CUDA library) or raises (oracle)."""
        T = x.shape[0]
        fits = self.max_tokens is not None and T <= self.max_tokens
        if device_plan is None:
            device_plan = fits and self.world * self.max_tokens * self.k * self.H * 2 <= DEVICE_PLAN_MAX_BYTES
        if device_plan:
            if not fits:
                raise ValueError(f"the device plan needs max_tokens >= T ({self.max_tokens} < {T})")
            return self._forward_device(x, ids, weights, expert_fn, combine_fn)
        p = self.plan(ids, x.device)
        order_dev = p.order.to(x.device)
        x_send = x.index_select(0, order_dev // self.k)
        e_send = ids.reshape(-1).to(torch.int32).index_select(0, order_dev.to(ids.device)).to(x.device)
        x_recv = self._exchange(x_send, p.send_counts, p.recv_counts)
        e_recv = self._exchange(e_send, p.send_counts, p.recv_counts)
        o_recv = expert_fn(x_recv, e_recv)      # zero rows too: every rank's o rows get expert_fn's dtype
        o_back = self._exchange(o_recv, p.recv_counts, p.send_counts)
        o = torch.empty((T * self.k, self.H), dtype=o_back.dtype, device=o_back.device)
        o[order_dev.to(o.device)] = o_back
        return combine_fn(o, weights)

    def _forward_device(self, x, ids, weights, expert_fn, combine_fn):
        """The device plan: fixed capacity C = max_tokens * k slots per
        destination (the same on every rank), no host read."""
        T, H, k = x.shape[0], self.H, self.k
        cap = max(1, self.max_tokens * k)
        slot = self.plan_device(ids, cap).to(x.device)
        entry_tok = torch.arange(T * k, device=x.device) // k
        x_send = torch.zeros((self.world * cap, H), dtype=x.dtype, device=x.device)
        x_send[slot] = x.index_select(0, entry_tok)
        e_send = torch.full((self.world * cap,), -1, dtype=torch.int32, device=x.device)
        e_send[slot] = ids.reshape(-1).to(device=x.device, dtype=torch.int32)
        x_recv = self._exchange_equal(x_send)
        e_recv = self._exchange_equal(e_send)
        o_recv = expert_fn(x_recv, e_recv)
        o_back = self._exchange_equal(o_recv)
        return combine_fn(o_back.index_select(0, slot), weights)


def gpu_expert_fn(ctx, layer: int):
    """expert_fn over the CUDA library: moe_fp4_expert_outputs on this rank's arena."""
    def fn(x_rows, experts):
        return ctx.expert_outputs(layer, x_rows, experts.to(torch.int32).contiguous())
    return fn


def gpu_combine_fn(ctx):
    def fn(o, weights):
        return ctx.combine(o, weights.contiguous())
    return fn
