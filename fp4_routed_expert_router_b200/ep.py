"""Expert-parallel execution of one routed-expert layer over a process group.

Rank r of G holds experts [r*E/G, (r+1)*E/G) in its arena.  Each rank routes
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
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class DispatchPlan:
    order: torch.Tensor         # int64 [T*k]: entries (t*k + j) in send order
    send_counts: list[int]      # entries sent to each rank
    recv_counts: list[int]      # entries received from each rank


class ExpertParallel:
    """Contiguous expert shards: rank r owns experts [r*E/G, (r+1)*E/G)."""

    def __init__(self, n_experts: int, top_k: int, hidden: int, group=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if n_experts % self.world:
            raise ValueError(f"{n_experts} experts do not split evenly over {self.world} ranks")
        self.E, self.k, self.H = n_experts, top_k, hidden
        self.per_rank = n_experts // self.world

    def owned(self) -> range:
        return range(self.rank * self.per_rank, (self.rank + 1) * self.per_rank)

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

    def _exchange(self, rows: torch.Tensor, send: list[int], recv: list[int]) -> torch.Tensor:
        """Rows to the other ranks (send[i] rows to rank i, recv[i] from rank i),
        moved as raw bytes so that any row type crosses any backend."""
        shape = tuple(rows.shape[1:])
        width = rows.element_size()
        for d in shape:
            width *= d
        flat = rows.contiguous().reshape(rows.shape[0], width // rows.element_size()).view(torch.uint8)
        out = torch.empty((sum(recv), width), dtype=torch.uint8, device=rows.device)
        dist.all_to_all_single(out, flat, recv, send, group=self.group)
        return out.view(rows.dtype).reshape((sum(recv),) + shape)

    def forward(self, x: torch.Tensor, ids: torch.Tensor, weights: torch.Tensor, expert_fn, combine_fn):
        """x [T, H] (bf16 bits), ids/weights [T, k] of this rank's tokens.
        expert_fn(x_rows [n, H], experts [n] int32) -> o [n, H] fp32 for
        experts this rank owns; combine_fn(o [T*k, H], weights) -> y [T, H]."""
        T = x.shape[0]
        p = self.plan(ids, x.device)
        order_dev = p.order.to(x.device)
        x_send = x.index_select(0, order_dev // self.k)
        e_send = ids.reshape(-1).to(torch.int32).index_select(0, order_dev.to(ids.device)).to(x.device)
        x_recv = self._exchange(x_send, p.send_counts, p.recv_counts)
        e_recv = self._exchange(e_send, p.send_counts, p.recv_counts)
        if x_recv.shape[0]:
            lo = self.rank * self.per_rank
            bad = (e_recv < lo) | (e_recv >= lo + self.per_rank)
            if bool(bad.any()):
                raise RuntimeError("received an entry for an expert this rank does not own")
            o_recv = expert_fn(x_recv, e_recv)
        else:
            o_recv = torch.empty((0, self.H), dtype=torch.float32, device=x.device)
        o_back = self._exchange(o_recv, p.recv_counts, p.send_counts)
        o = torch.empty((T * self.k, self.H), dtype=o_back.dtype, device=o_back.device)
        o[order_dev.to(o.device)] = o_back
        return combine_fn(o, weights)


def gpu_expert_fn(ctx, layer: int):
    """expert_fn over the CUDA library: moe_fp4_expert_outputs on this rank's arena."""
    def fn(x_rows, experts):
        return ctx.expert_outputs(layer, x_rows, experts.to(torch.int32).contiguous())
    return fn


def gpu_combine_fn(ctx):
    def fn(o, weights):
        return ctx.combine(o, weights.contiguous())
    return fn
