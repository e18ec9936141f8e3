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


class MoELayerEP:
    """Forward of one layer with the routed experts sharded over the ranks of
    ``process_group`` (one process per GPU).  Every step runs in the library's
    kernels; this class only sequences them around the two exchanges:

        moe_route -> fp8_quant_1x128 -> moe_permute (all E experts, with shared)
        -> plan_dispatch -> dispatch (FP8 rows + scales)
        -> moe_segment_ids -> moe_permute (received rows by local expert, K = 1)
        -> grouped GEMM 1 (SwiGLU + requantisation) -> grouped GEMM 2
        -> back to receive order (moe_combine with K = 1, gate 1, zero residual)
        -> combine_return -> shared expert on the local tokens (grouped GEMMs)
        -> moe_combine -> moe_bias_update (counts summed over the ranks)

    The weight stacks hold this rank's E/world routed experts followed by a
    replica of the shared expert ([E/world + 1][...]).  centroids and bias
    cover all E experts (routing is replicated).  With one rank the result is
    bit-identical to MoELayer.forward: every row's GEMMs and the combine see
    the same operands in the same order."""

    def __init__(self, cfg, centroids, bias, w1q, w1s, w2q, w2s, shard: ExpertShard,
                 process_group=None, T: int | None = None):
        from . import _abi
        if shard.E != cfg.E:
            raise ValueError("the shard must cover the config's experts")
        if w1q.shape[0] != shard.per_rank + cfg.n_shared:
            raise ValueError("weights must hold the local experts and the shared expert")
        self._abi = _abi
        self.cfg = cfg
        self.shard = shard
        self.pg = process_group
        self.T = cfg.T if T is None else T
        self.centroids, self.bias = centroids, bias
        self.w1q, self.w1s, self.w2q, self.w2s = w1q, w1s, w2q, w2s
        dev = centroids.device
        self.dev = dev
        T, d, K, E, I = self.T, cfg.d, cfg.K, cfg.E, cfg.I
        P = T * K
        self.pairs = P
        i32, f32, u8 = torch.int32, torch.float32, torch.uint8
        self.idx = torch.empty(T, K, dtype=i32, device=dev)
        self.gate = torch.empty(T, K, dtype=f32, device=dev)
        self.route_ws = torch.empty(max(_abi.moe_route_workspace_size(T, d, E), 16), dtype=u8,
                                    device=dev)
        self.Xq = torch.empty(P + T, d, dtype=u8, device=dev)
        self.Xs = torch.empty(P + T, d // 128, dtype=f32, device=dev)
        self.perm = {"xq_perm": self.Xq[:P], "xs_perm": self.Xs[:P]}
        self.dev_err = torch.zeros(1, dtype=i32, device=dev)
        # the shared expert's rows are the local tokens: one segment of T rows
        self.shared_offsets = torch.tensor([0, T], dtype=i32, device=dev)
        self.shared_tiles = (T + 127) // 128
        self.shared_table = _abi.moe_tile_table(self.shared_offsets, self.shared_tiles)
        self.H_sh = torch.empty(T, I, dtype=u8, device=dev)
        self.Hs_sh = torch.empty(T, I // 128, dtype=f32, device=dev)
        self.Y_sh = torch.empty(T, d, dtype=f32, device=dev)
        self.out = torch.empty(T, d, dtype=f32, device=dev)

    def forward(self, u: torch.Tensor, update_bias: bool = True) -> torch.Tensor:
        a, c, sh = self._abi, self.cfg, self.shard
        T, d, K, E, I, P = self.T, c.d, c.K, c.E, c.I, self.pairs
        El = sh.per_rank
        assert u.shape == (T, d) and u.dtype == torch.bfloat16
        a.moe_route(u, self.centroids, self.bias, c.G, c.M, K, self.idx, self.gate,
                    ws=self.route_ws, dev_err=self.dev_err)
        a.fp8_quant_1x128(u, self.Xq[P:], self.Xs[P:])
        p = a.moe_permute(self.idx, E, self.Xq[P:], self.Xs[P:], True, out=self.perm,
                          dev_err=self.dev_err)
        plan = plan_dispatch(p["counts"], sh, self.pg)
        rq, rs = dispatch(self.Xq[:P], self.Xs[:P], plan, self.pg)
        R = plan.n_recv
        y_recv = torch.empty(R, d, dtype=torch.float32, device=self.dev)
        if R > 0:
            ids = a.moe_segment_ids(plan.recv_counts, El, R, dev_err=self.dev_err)
            p2 = a.moe_permute(ids.view(R, 1), El, rq, rs, False, dev_err=self.dev_err)
            h2, hs2 = a.grouped_gemm_fp8_blockscaled(
                p2["xq_perm"], p2["xs_perm"], self.w1q[:El], self.w1s[:El], p2["offsets"],
                p2["tile_group"], p2["tile_start"], p2["n_tiles"], p2["max_tiles"],
                a.EP_SWIGLU_QUANT, dev_err=self.dev_err)
            y2 = a.grouped_gemm_fp8_blockscaled(
                h2, hs2, self.w2q[:El], self.w2s[:El], p2["offsets"], p2["tile_group"],
                p2["tile_start"], p2["n_tiles"], p2["max_tiles"], a.EP_F32,
                dev_err=self.dev_err)
            # back to receive order: y_recv[r] = 0 + 1 * y2[dst_of[r]] (exact)
            ones = torch.ones(R, 1, dtype=torch.float32, device=self.dev)
            zeros = torch.zeros(R, d, dtype=torch.bfloat16, device=self.dev)
            a.moe_combine(y2, p2["dst_of"], ones, None, zeros, out=y_recv)
        y_back = combine_return(y_recv, plan, self.pg)
        # the shared expert on this rank's own tokens
        tg, ts, nt = self.shared_table
        a.grouped_gemm_fp8_blockscaled(self.Xq[P:], self.Xs[P:], self.w1q[El:], self.w1s[El:],
                                       self.shared_offsets, tg, ts, nt, self.shared_tiles,
                                       a.EP_SWIGLU_QUANT, self.H_sh, self.Hs_sh,
                                       dev_err=self.dev_err)
        a.grouped_gemm_fp8_blockscaled(self.H_sh, self.Hs_sh, self.w2q[El:], self.w2s[El:],
                                       self.shared_offsets, tg, ts, nt, self.shared_tiles,
                                       a.EP_F32, self.Y_sh, dev_err=self.dev_err)
        a.moe_combine(y_back, p["dst_of"], self.gate, self.Y_sh, u, self.out)
        if update_bias:
            from .layer import reduce_load_counts
            counts, T_all = reduce_load_counts(p["counts"], T, self.pg)
            a.moe_bias_update(counts, T_all, K, c.gamma, self.bias)
        return self.out

    def check(self) -> None:
        self._abi.raise_dev_err(self.dev_err)
