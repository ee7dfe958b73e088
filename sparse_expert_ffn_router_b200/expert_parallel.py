"""Expert-parallel MoE layer over several GPUs (one process per GPU, torch.distributed).

The pages place experts on GPUs by device order and move tokens to them peer to peer
(www.mhpq.cn/news/563172 §2.2: expert-parallel communication of 512 tokens over 8 GPUs;
www.0539edu.com/news/4774449 §2.2: experts spread over the GPUs of a node).  Here rank g owns the
contiguous experts [g E / G, (g + 1) E / G) and one forward is

    Gate + Scatter on the rank's own tokens      colibri_route_noalloc (rows grouped by expert, so
                                                 the rows bound for each rank are contiguous)
    count exchange                               all-to-all of the per-(rank, local expert) counts
    dispatch                                     all-to-all-v of the grouped rows
    expert compute                               colibri_moe_forward_routed on the received rows:
                                                 one slot per row, its local expert, weight 1
    return                                       all-to-all-v of the output rows, back in the
                                                 order they were sent
    Gather                                       colibri_combine with the rank's own routing

Every step of the layer's arithmetic runs in the library's CUDA kernels; this module only moves
rows between ranks (NCCL through torch.distributed) and builds the split sizes, which the
all-to-all-v needs on the host (one device-to-host copy of the exchanged counts per forward).
The exchange functions below take tensors on any device, so the same bookkeeping runs on CPU
ranks over gloo.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch
import torch.distributed as dist

from . import (COLIBRI_BF16, COLIBRI_F32, MoELayer, colibri_combine, colibri_moe_forward_routed,
               colibri_route_noalloc)


def owned_experts(num_experts: int, world: int, rank: int) -> range:
    """The experts rank `rank` holds: a contiguous range, E / G of them."""
    if num_experts % world:
        raise ValueError(f"num_experts={num_experts} must be a multiple of the world size {world}")
    n = num_experts // world
    return range(rank * n, (rank + 1) * n)


@dataclass
class ExchangePlan:
    """Split sizes of one forward's all-to-all-v (rows), and the received rows' local experts."""
    send_rows: List[int]        # rows this rank sends to each rank (its grouped rows, in order)
    recv_rows: List[int]        # rows this rank receives from each rank
    recv_counts: torch.Tensor   # [world, E / G] rows received per (source rank, local expert)


def exchange_counts(counts: torch.Tensor, world: int, group=None) -> ExchangePlan:
    """Count exchange.  `counts` [E] int32: the rows of each expert among this rank's grouped rows.
    Sends each rank the counts of the experts it owns; returns the split sizes of both
    all-to-alls and the counts received per (source rank, local expert)."""
    E = counts.numel()
    per = counts.to(torch.int32).reshape(world, E // world).contiguous()  # [dest rank, local expert]
    recv = torch.empty_like(per)
    if world > 1:
        dist.all_to_all_single(recv, per, group=group)
    else:
        recv.copy_(per)
    host_send = per.sum(dim=1).cpu().tolist()
    host_recv = recv.sum(dim=1).cpu().tolist()
    return ExchangePlan([int(v) for v in host_send], [int(v) for v in host_recv], recv)


def dispatch_rows(rows: torch.Tensor, plan: ExchangePlan, group=None) -> torch.Tensor:
    """All-to-all-v of the grouped rows: rank g receives, from every rank in rank order, the rows of
    the experts it owns (each source's rows in that source's expert order)."""
    world = len(plan.send_rows)
    out = torch.empty((sum(plan.recv_rows),) + tuple(rows.shape[1:]), dtype=rows.dtype, device=rows.device)
    if world > 1:
        dist.all_to_all_single(out, rows[: sum(plan.send_rows)].contiguous(), output_split_sizes=plan.recv_rows,
                               input_split_sizes=plan.send_rows, group=group)
    else:
        out.copy_(rows[: out.shape[0]])
    return out


def return_rows(rows: torch.Tensor, plan: ExchangePlan, group=None) -> torch.Tensor:
    """The reverse all-to-all-v: each output row goes back to the rank that sent its input row, in
    the order it was sent (so the result lines up with the sender's grouped rows)."""
    world = len(plan.send_rows)
    out = torch.empty((sum(plan.send_rows),) + tuple(rows.shape[1:]), dtype=rows.dtype, device=rows.device)
    if world > 1:
        dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=plan.send_rows,
                               input_split_sizes=plan.recv_rows, group=group)
    else:
        out.copy_(rows)
    return out


def received_experts(plan: ExchangePlan) -> torch.Tensor:
    """The local expert of every received row, [rows, 1] int32, in received order (source rank
    major, then the source's expert order)."""
    n_local = plan.recv_counts.shape[1]
    ids = torch.arange(n_local, dtype=torch.int32, device=plan.recv_counts.device).repeat(plan.recv_counts.shape[0])
    return torch.repeat_interleave(ids, plan.recv_counts.reshape(-1).to(torch.int64)).reshape(-1, 1).contiguous()


class ExpertParallelMoE:
    """One MoE layer whose experts are spread over the ranks of a process group.

    Each rank passes its own tokens x [T, d] (T <= max_tokens), the full router weights, and the
    weights of the experts it owns (`owned_experts`) in the library's expert-buffer layout with
    E / G experts.  The layer description is that of colibri_init with num_experts = E; weights
    int8 / int4 carry their scales for the owned experts.  No shared expert.
    """

    def __init__(self, d_model: int, d_ff: int, num_experts: int, top_k: int, act_dtype: int = COLIBRI_BF16,
                 weight_dtype: int = COLIBRI_BF16, max_tokens: int = 1, device_id: int = 0, group=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.d, self.f, self.E, self.k = d_model, d_ff, num_experts, top_k
        self.act = act_dtype
        self.owned = owned_experts(num_experts, self.world, self.rank)
        # the received rows: at most every slot of every rank's tokens
        self.max_recv = max_tokens * top_k * self.world
        self.local = MoELayer(d_model, d_ff, len(self.owned), 1, 0, act_dtype, weight_dtype,
                              max_tokens=self.max_recv, device_id=device_id)
        self.max_tokens = max_tokens
        self.device = torch.device("cuda", device_id)

    @property
    def expert_stride(self) -> int:
        return self.local.expert_stride

    def forward(self, x: torch.Tensor, router_w: torch.Tensor, router_b: Optional[torch.Tensor],
                expert_w_local: torch.Tensor, y: torch.Tensor, expert_scales_local: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        T, d, k, E = x.shape[0], self.d, self.k, self.E
        if T > self.max_tokens:
            raise ValueError(f"T={T} exceeds max_tokens={self.max_tokens}")
        dev, adt = self.device, x.dtype
        stream = stream or torch.cuda.current_stream(dev)
        with torch.cuda.stream(stream):
            i32 = dict(dtype=torch.int32, device=dev)
            idx = torch.empty(T, k, **i32)
            w = torch.empty(T, k, dtype=torch.float32, device=dev)
            counts = torch.empty(E, **i32)
            offsets = torch.empty(E + 1, **i32)
            src_row = torch.empty(T * k, **i32)
            dst_row = torch.empty(T, k, **i32)
            Xp = torch.empty(T * k, d, dtype=adt, device=dev)
            if T > 0:
                colibri_route_noalloc(x, self.act, T, d, router_w, router_b, E, k, idx, w, counts, offsets, src_row,
                                      dst_row, Xp, stream)
            else:
                counts.zero_()
            plan = exchange_counts(counts, self.world, self.group)
            recv = dispatch_rows(Xp, plan, self.group)
            R = recv.shape[0]
            y_recv = torch.empty(R, d, dtype=adt, device=dev)
            if R > 0:
                local_idx = received_experts(plan)
                ones = torch.ones(R, 1, dtype=torch.float32, device=dev)
                colibri_moe_forward_routed(self.local.ctx, recv, R, local_idx, ones, expert_w_local,
                                           expert_scales_local, None, y_recv, stream)
            back = return_rows(y_recv, plan, self.group)
            if T > 0:
                colibri_combine(back, self.act, dst_row, w, T, k, d, y, stream)
        return y

    def close(self):
        self.local.close()


__all__ = ["owned_experts", "ExchangePlan", "exchange_counts", "dispatch_rows", "return_rows", "received_experts",
           "ExpertParallelMoE", "COLIBRI_F32", "COLIBRI_BF16"]
