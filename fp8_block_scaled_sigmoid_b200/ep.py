"""Expert parallelism: the exchange of routed rows between ranks.

"DeepSeek_V3_Report：Annotation", "Low-Precision Communication" (activations
are quantised to FP8 before the dispatch; the combine's rows travel back)
and "No Token-Dropping"; [INFRA] describes the same dispatch/combine pair as
an all-to-all over the expert-parallel group.  On B200 the group is the
GPUs of one NVLink 5 / NVSwitch domain, one process per GPU, and the
exchanges are NCCL all-to-alls (``torch.distributed``).

Each rank owns a contiguous block of E / world routed experts.  After the
local permutation (``moe_permute``) a rank's routed rows are sorted by
expert, so the rows for rank r's experts are one contiguous run: the
dispatch is a single all-to-all with one split per destination, and a
receiver gets, from every source in rank order, that source's rows of its
experts sorted by expert.  The return exchange sends the expert outputs
back with the splits swapped, so each sender gets its rows in exactly the
order it sent them and the combine runs unchanged.

This module is plumbing (split sizes and the collectives); the rows it moves
are produced and consumed by the library's kernels.  Planning reads the
per-destination split sizes to the host once per step, which NCCL's
variable-size all-to-all needs.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class ExpertShard:
    """Routed experts [e0, e1) of ``rank`` in a group of ``world`` ranks."""
    E: int
    world: int
    rank: int

    def __post_init__(self):
        if self.world <= 0 or not 0 <= self.rank < self.world or self.E % self.world != 0:
            raise ValueError(f"{self.E} experts do not split evenly over {self.world} ranks")

    @property
    def per_rank(self) -> int:
        return self.E // self.world

    @property
    def e0(self) -> int:
        return self.rank * self.per_rank

    @property
    def e1(self) -> int:
        return self.e0 + self.per_rank


@dataclass
class DispatchPlan:
    """Split sizes of one step's exchange.

    send_splits[r]  rows this rank sends to rank r (its rows of r's experts)
    recv_splits[s]  rows this rank receives from rank s
    recv_counts     int32 [world][E/world]: rows from source s for local expert e
                    (on the counts' device; the receiver's per-source segments)
    """
    send_splits: list[int]
    recv_splits: list[int]
    recv_counts: torch.Tensor

    @property
    def n_recv(self) -> int:
        return sum(self.recv_splits)


def plan_dispatch(counts: torch.Tensor, shard: ExpertShard, process_group=None) -> DispatchPlan:
    """counts: int32 [E] routed rows of this rank per expert (moe_permute's
    counts).  Exchanges the per-expert counts (a small all-to-all), then
    reads the split sizes to the host."""
    import torch.distributed as dist
    if counts.dim() != 1 or counts.numel() != shard.E:
        raise ValueError("counts must be [E]")
    send = counts.to(torch.int32).reshape(shard.world, shard.per_rank).contiguous()
    recv = torch.empty_like(send)
    if shard.world == 1:
        recv.copy_(send)
    else:
        dist.all_to_all_single(recv, send, group=process_group)
    both = torch.stack([send.sum(1), recv.sum(1)]).cpu()
    return DispatchPlan(send_splits=[int(v) for v in both[0]],
                        recv_splits=[int(v) for v in both[1]], recv_counts=recv)


def exchange_rows(rows: torch.Tensor, send_splits: list[int], recv_splits: list[int],
                  process_group=None, out: torch.Tensor | None = None) -> torch.Tensor:
    """All-to-all of row blocks: rows [sum(send_splits)][...] -> [sum(recv_splits)][...],
    block r of the input to rank r, block s of the output from rank s."""
    import torch.distributed as dist
    if rows.shape[0] != sum(send_splits):
        raise ValueError("rows do not match the send splits")
    shape = (sum(recv_splits),) + tuple(rows.shape[1:])
    if out is None:
        out = torch.empty(shape, dtype=rows.dtype, device=rows.device)
    elif tuple(out.shape) != shape:
        raise ValueError("output does not match the receive splits")
    if len(send_splits) == 1:
        out.copy_(rows)
        return out
    dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=recv_splits,
                           input_split_sizes=send_splits, group=process_group)
    return out


def dispatch(xq_routed: torch.Tensor, xs_routed: torch.Tensor, plan: DispatchPlan,
             process_group=None):
    """Send each rank the FP8 rows (and their 1x128 scales) of its experts."""
    return (exchange_rows(xq_routed, plan.send_splits, plan.recv_splits, process_group),
            exchange_rows(xs_routed, plan.send_splits, plan.recv_splits, process_group))


def combine_return(y_recv: torch.Tensor, plan: DispatchPlan, process_group=None,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """Send the expert outputs of the received rows back to their senders;
    each sender gets them in its own send order."""
    return exchange_rows(y_recv, plan.recv_splits, plan.send_splits, process_group, out)
