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


def plan_dispatch(counts: torch.Tensor, shard: ExpertShard, process_group=None,
                  dev_err: torch.Tensor | None = None, recv_counts: torch.Tensor | None = None
                  ) -> DispatchPlan:
    """counts: int32 [E] routed rows of this rank per expert (moe_permute's
    counts).  Exchanges the per-expert counts (a small all-to-all), then
    reads the split sizes to the host.  ``dev_err`` (the layer's device error
    word) travels to the host in the same copy: a non-zero code (for instance
    an expert index out of range, which leaves the counts short of the rows)
    raises before any row is exchanged.  The received counts are written
    into ``recv_counts`` when given."""
    import torch.distributed as dist
    if counts.dim() != 1 or counts.numel() != shard.E:
        raise ValueError("counts must be [E]")
    send = counts.to(torch.int32).reshape(shard.world, shard.per_rank).contiguous()
    recv = torch.empty_like(send) if recv_counts is None else recv_counts.view_as(send)
    if shard.world == 1:
        recv.copy_(send)
    else:
        dist.all_to_all_single(recv, send, group=process_group)
    parts = [send.sum(1), recv.sum(1)]
    if dev_err is not None:
        parts.append(dev_err.reshape(1).to(torch.int64).expand(shard.world))
    both = torch.stack([p.to(torch.int64) for p in parts]).cpu()
    if dev_err is not None and int(both[2, 0]) != 0:
        from . import _abi
        raise _abi.MoEError(f"device-side error {int(both[2, 0])} before the dispatch: "
                            f"{_abi.DEVERR.get(int(both[2, 0]), 'unknown')}")
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
    kernels; this class owns the buffers (all allocated once, here) and
    sequences the calls around the two exchanges:

        stage_dispatch:  moe_route -> moe_permute_index over all E experts
                         -> fp8_quant_1x128_scatter (the tokens into the
                         receive buffer's head, their routed rows into the
                         send buffer, expert-sorted)
        plan + dispatch: per-expert counts all-to-all, split sizes to the host,
                         FP8 rows + scales all-to-all into the receive buffer
        stage_experts:   moe_segment_ids (the rank's T own tokens = group 0,
                         the shared expert; received rows = 1 + local expert)
                         -> moe_permute (K = 1) regroups them
                         -> grouped GEMM 1 (SwiGLU + requantisation)
                         -> grouped GEMM 2, its fp32 rows written straight back
                            in receive order through the permutation's row map
        return:          the received rows' outputs all-to-all back to their
                         senders, in each sender's own send order
        stage_combine:   moe_combine (+ shared expert rows, + residual)
                         -> moe_bias_update (counts summed over the ranks)

    The shared expert is the first segment of the local grouped GEMMs, so a
    step runs the same two GEMM launches as the single-GPU layer.  The weight
    stacks hold the shared expert followed by this rank's E/world routed
    experts ([1 + E/world][...]; make_fp8_weights(experts=[E, e0, .., e1-1])).
    centroids and bias cover all E experts (routing is replicated).

    recv_capacity bounds the rows a rank can receive (default T*K*world, the
    most it can be sent); a step that would receive more raises before the
    exchange.  Each received row meets the same FP8 operands as in the
    single-GPU layer, and per-row results do not depend on a row's tile, so
    the output equals MoELayer.forward on the same tokens bit for bit."""

    def __init__(self, cfg, centroids, bias, w1q, w1s, w2q, w2s, shard: ExpertShard,
                 process_group=None, T: int | None = None, recv_capacity: int | None = None):
        from . import _abi
        if shard.E != cfg.E:
            raise ValueError("the shard must cover the config's experts")
        if cfg.n_shared != 1:
            raise ValueError("the expert-parallel layer runs one shared expert")
        if w1q.shape[0] != shard.per_rank + 1:
            raise ValueError("weights must hold the shared expert and the local experts")
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
        El = shard.per_rank
        Rcap = P * shard.world if recv_capacity is None else int(recv_capacity)
        self.recv_capacity = Rcap
        i32, f32, u8 = torch.int32, torch.float32, torch.uint8
        self.idx = torch.empty(T, K, dtype=i32, device=dev)
        self.gate = torch.empty(T, K, dtype=f32, device=dev)
        self.route_ws = torch.empty(max(_abi.moe_route_workspace_size(T, d, E), 16), dtype=u8,
                                    device=dev)
        self.dev_err = torch.zeros(1, dtype=i32, device=dev)
        self.sched = torch.zeros(1, dtype=i32, device=dev)   # the GEMMs' work counter
        # receive side: [own T tokens | received rows], then regrouped copies
        rows = T + Rcap
        self.RX = torch.empty(rows, d, dtype=u8, device=dev)
        self.RXs = torch.empty(rows, d // 128, dtype=f32, device=dev)
        # send side: routed rows sorted by expert over all E experts.  With one
        # rank every row goes to this rank in send order, so the send buffer
        # is the receive area itself and the dispatch moves nothing.
        self.local = shard.world == 1
        if self.local:
            self.Xsend, self.Xs_send = self.RX[T:T + P], self.RXs[T:T + P]
        else:
            self.Xsend = torch.empty(P, d, dtype=u8, device=dev)
            self.Xs_send = torch.empty(P, d // 128, dtype=f32, device=dev)
        self.perm = {"xq_perm": self.Xsend, "xs_perm": self.Xs_send}
        self.perm_ws = torch.empty(max(_abi.moe_permute_workspace_size(T, K, E), 16), dtype=u8,
                                   device=dev)
        self.ids = torch.empty(rows, dtype=i32, device=dev)
        self.X2 = torch.empty(rows, d, dtype=u8, device=dev)
        self.X2s = torch.empty(rows, d // 128, dtype=f32, device=dev)
        mt2 = _abi.moe_max_m_tiles(rows, 1, El + 1, False)
        self.perm2 = {"xq_perm": self.X2, "xs_perm": self.X2s,
                      "counts": torch.empty(El + 1, dtype=i32, device=dev),
                      "offsets": torch.empty(El + 2, dtype=i32, device=dev),
                      "src_row": torch.empty(rows, dtype=i32, device=dev),
                      "dst_of": torch.empty(rows, 1, dtype=i32, device=dev),
                      "tile_group": torch.empty(max(mt2, 1), dtype=i32, device=dev),
                      "tile_start": torch.empty(El + 2, dtype=i32, device=dev),
                      "n_tiles": torch.empty(1, dtype=i32, device=dev)}
        self.perm2_ws = torch.empty(max(_abi.moe_permute_workspace_size(rows, 1, El + 1), 16),
                                    dtype=u8, device=dev)
        self.H2 = torch.empty(rows, I, dtype=u8, device=dev)
        self.H2s = torch.empty(rows, I // 128, dtype=f32, device=dev)
        self.Yr = torch.empty(rows, d, dtype=f32, device=dev)     # receive order
        # send order (with one rank the same rows: receive order is send order)
        self.Yback = self.Yr[T:T + P] if self.local else torch.empty(P, d, dtype=f32, device=dev)
        self.recv_counts = torch.empty(shard.world, El, dtype=i32, device=dev)
        self.out = torch.empty(T, d, dtype=f32, device=dev)
        self.plan: DispatchPlan | None = None
        self.R = 0

    # -- stages (the emulation of several ranks on one GPU calls them) -----
    def stage_dispatch(self, u: torch.Tensor) -> torch.Tensor:
        """Route, then quantise the rank's tokens once: into the receive
        buffer's head, and their routed rows, sorted by expert, into the send
        buffer.  Returns the per-expert counts (device int32 [E])."""
        a, c = self._abi, self.cfg
        T = self.T
        assert u.shape == (T, c.d) and u.dtype == torch.bfloat16
        a.moe_route(u, self.centroids, self.bias, c.G, c.M, c.K, self.idx, self.gate,
                    ws=self.route_ws, dev_err=self.dev_err)
        a.moe_permute_index(self.idx, c.E, False, out=self.perm, ws=self.perm_ws,
                            dev_err=self.dev_err)
        a.fp8_quant_1x128_scatter(u, self.perm["dst_of"], self.Xsend, self.Xs_send,
                                  self.RX[:T], self.RXs[:T])
        return self.perm["counts"]

    def send_rows(self):
        """The rows (and scales) to dispatch, one contiguous run per destination."""
        return self.Xsend, self.Xs_send

    def recv_rows(self, plan: DispatchPlan):
        """Adopt the step's plan and return the receive buffers (rows and
        scales) the dispatch writes into, in source-rank order."""
        R = plan.n_recv
        if R > self.recv_capacity:
            raise ValueError(f"{R} rows to receive exceed the capacity {self.recv_capacity}")
        self.plan, self.R = plan, R
        if plan.recv_counts.data_ptr() != self.recv_counts.data_ptr():
            self.recv_counts.copy_(plan.recv_counts.reshape(self.recv_counts.shape))
        T = self.T
        return self.RX[T:T + R], self.RXs[T:T + R]

    def stage_experts(self) -> None:
        """Regroup [own tokens | received rows] by group (shared expert first,
        then the local experts) and run both grouped GEMMs; GEMM 2 writes
        every row's output back to its receive-buffer position."""
        a, c = self._abi, self.cfg
        T, R, El = self.T, self.R, self.shard.per_rank
        n = T + R
        a.moe_segment_ids(self.recv_counts, El, n, ids=self.ids[:n], dev_err=self.dev_err,
                          lead_rows=T)
        p2 = a.moe_permute(self.ids[:n].view(n, 1), El + 1, self.RX[:n], self.RXs[:n], False,
                           out=self.perm2, ws=self.perm2_ws, dev_err=self.dev_err)
        mt = a.moe_max_m_tiles(n, 1, El + 1, False)
        a.grouped_gemm_fp8_blockscaled(self.X2[:n], self.X2s[:n], self.w1q, self.w1s,
                                       p2["offsets"], p2["tile_group"], p2["tile_start"],
                                       p2["n_tiles"], mt, a.EP_SWIGLU_QUANT, self.H2[:n],
                                       self.H2s[:n], dev_err=self.dev_err, sched=self.sched)
        a.grouped_gemm_fp8_blockscaled(self.H2[:n], self.H2s[:n], self.w2q, self.w2s,
                                       p2["offsets"], p2["tile_group"], p2["tile_start"],
                                       p2["n_tiles"], mt, a.EP_F32, self.Yr[:n],
                                       dev_err=self.dev_err, d_rows=p2["src_row"][:n],
                                       sched=self.sched)

    def return_rows(self):
        """The received rows' outputs to send back (receive order)."""
        T = self.T
        return self.Yr[T:T + self.R]

    def stage_combine(self, u: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        """out = u + shared expert + gate-weighted routed outputs (Yback holds
        the returned rows in this rank's send order)."""
        out = self.out if out is None else out
        self._abi.moe_combine(self.Yback, self.perm["dst_of"], self.gate, self.Yr[:self.T], u,
                              out=out)
        return out

    def stage_bias_update(self, counts: torch.Tensor, total_tokens: int) -> None:
        self._abi.moe_bias_update(counts, total_tokens, self.cfg.K, self.cfg.gamma, self.bias)

    # -- one step with the process group's exchanges ------------------------
    def forward(self, u: torch.Tensor, update_bias: bool = True) -> torch.Tensor:
        counts = self.stage_dispatch(u)
        if self.local:
            # one rank: every split is known on the host (all T*K rows stay),
            # the counts "exchange" is a device copy and the rows are already
            # in place, so the step needs no host synchronisation
            self.recv_counts.copy_(counts.view(1, -1))
            self.recv_rows(DispatchPlan([self.pairs], [self.pairs], self.recv_counts))
            self.stage_experts()
        else:
            plan = plan_dispatch(counts, self.shard, self.pg, dev_err=self.dev_err,
                                 recv_counts=self.recv_counts)
            rq, rs = self.recv_rows(plan)
            xq, xs = self.send_rows()
            exchange_rows(xq, plan.send_splits, plan.recv_splits, self.pg, out=rq)
            exchange_rows(xs, plan.send_splits, plan.recv_splits, self.pg, out=rs)
            self.stage_experts()
            exchange_rows(self.return_rows(), plan.recv_splits, plan.send_splits, self.pg,
                          out=self.Yback)
        out = self.stage_combine(u)
        if update_bias:
            from .layer import reduce_load_counts
            total, T_all = reduce_load_counts(counts, self.T, self.pg)
            self.stage_bias_update(total, T_all)
        return out

    def check(self) -> None:
        self._abi.raise_dev_err(self.dev_err)
