"""Multi-rank host logic on CPU (gloo ranks).

Each data-parallel rank routes its own batch; the bias update needs the load
of the whole batch ("DeepSeek_V3_Report：Annotation", "Auxiliary-Loss-Free
Load Balancing"), so the per-expert counts are summed over ranks first.  The
test checks that every rank then computes the same new bias, equal to the
oracle's update on the concatenated batch, and that timings reduce to the
slowest rank.  The weight gradients of data-parallel training are summed the
same way.  Under expert parallelism the routed rows are exchanged with two
all-to-alls (dispatch and return), checked row by row on 2 and 3 ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as O

E, K, T = 32, 4, 50


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_idx(rank):
    rng = np.random.default_rng(100 + rank)
    return np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from fp8_block_scaled_sigmoid_b200.layer import max_over_ranks, reduce_load_counts
    counts, _, _, _ = O.permute(_rank_idx(rank), E)
    total, t_all = reduce_load_counts(torch.from_numpy(counts), T, dist.group.WORLD)
    b0 = np.linspace(-0.01, 0.01, E).astype(np.float32)
    nb = O.bias_update(total.numpy(), t_all, K, 0.001, b0)
    slowest = max_over_ranks(1.0 + rank, "cpu", dist.group.WORLD)
    q.put((rank, total.numpy(), t_all, nb, slowest))
    dist.barrier()
    dist.destroy_process_group()


def test_bias_update_over_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in procs], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    both = np.concatenate([_rank_idx(0), _rank_idx(1)])
    counts_all, _, _, _ = O.permute(both, E)
    b0 = np.linspace(-0.01, 0.01, E).astype(np.float32)
    want = O.bias_update(counts_all, 2 * T, K, 0.001, b0)
    for rank, total, t_all, nb, slowest in res:
        assert np.array_equal(total, counts_all) and t_all == 2 * T
        assert np.array_equal(nb, want)
        assert slowest == 2.0


def _grad_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from fp8_block_scaled_sigmoid_b200.layer import reduce_weight_grads
    rng = np.random.default_rng(200 + rank)
    g = {"dW1": torch.from_numpy(rng.normal(0, 1, (3, 8, 4)).astype(np.float32)),
         "dW2": torch.from_numpy(rng.normal(0, 1, (3, 4, 8)).astype(np.float32))}
    local = {k: v.clone() for k, v in g.items()}
    reduce_weight_grads(g, dist.group.WORLD)
    q.put((rank, {k: v.numpy() for k, v in local.items()}, {k: v.numpy() for k, v in g.items()}))
    dist.barrier()
    dist.destroy_process_group()


def test_weight_grads_sum_over_two_ranks():
    """Data-parallel training: each rank's expert weight gradients (fp32,
    "Mixed Precision Framework") are summed over the ranks, so both hold the
    gradient of the whole batch."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_grad_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in procs], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for k in ("dW1", "dW2"):
        want = res[0][1][k] + res[1][1][k]
        for _, _, reduced in res:
            assert np.array_equal(reduced[k], want)


# ---------------------------------------------------------------------------
# Expert parallelism: the dispatch / return exchange (ep.py) on CPU ranks.
EP_E, EP_K, EP_T, EP_D = 12, 3, 40, 256


def _ep_rank_data(rank):
    """A rank's routed rows after its local permutation: expert-sorted FP8
    rows and scales (the oracle's quantiser and permutation)."""
    rng = np.random.default_rng(300 + rank)
    idx = np.stack([rng.permutation(EP_E)[:EP_K] for _ in range(EP_T)]).astype(np.int32)
    u = rng.normal(0, 1, (EP_T, EP_D)).astype(np.float32)
    xq, xs = O.quant_1x128(u)
    counts, offsets, src_row, dst_of = O.permute(idx, EP_E)
    expert_of_row = np.repeat(np.arange(EP_E), counts)
    return counts, xq[src_row], xs[src_row], expert_of_row


def _ep_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from fp8_block_scaled_sigmoid_b200 import ep
    shard = ep.ExpertShard(EP_E, world, rank)
    counts, xq, xs, expert_of_row = _ep_rank_data(rank)
    plan = ep.plan_dispatch(torch.from_numpy(counts), shard, dist.group.WORLD)
    rq, rs = ep.dispatch(torch.from_numpy(xq), torch.from_numpy(xs), plan, dist.group.WORLD)
    # a stand-in expert on the receiver: row -> dequantised row * (expert + 1),
    # the expert read from the plan's per-source segments
    rc = plan.recv_counts.numpy()
    local_expert = np.concatenate([np.repeat(np.arange(shard.e0, shard.e1), rc[s])
                                   for s in range(world)]).astype(np.int64)
    y = (O.dequant_1x128(rq.numpy(), rs.numpy()) * (local_expert[:, None] + 1)).astype(np.float32)
    back = ep.combine_return(torch.from_numpy(y), plan, dist.group.WORLD)
    q.put((rank, plan.send_splits, plan.recv_splits, rc, rq.numpy(), rs.numpy(), back.numpy()))
    dist.barrier()
    dist.destroy_process_group()


def _run_ep(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in procs], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res



@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_dispatch_and_return(world):
    """Each rank receives, from every source in rank order, exactly that
    source's rows of its own experts (expert-sorted, token order kept inside an
    expert), and the return exchange hands every sender its rows back in its
    own send order."""
    res = _run_ep(world)
    per = EP_E // world
    data = [_ep_rank_data(r) for r in range(world)]
    for rank, send_splits, recv_splits, rc, rq, rs, back in res:
        counts, xq, xs, expert_of_row = data[rank]
        e0, e1 = rank * per, (rank + 1) * per
        assert send_splits == [int(counts[r * per:(r + 1) * per].sum()) for r in range(world)]
        want_q, want_s = [], []
        for s in range(world):
            cs, xqs, xss, eor = data[s]
            sel = (eor >= e0) & (eor < e1)
            want_q.append(xqs[sel])
            want_s.append(xss[sel])
            assert np.array_equal(rc[s], cs[e0:e1])
        assert recv_splits == [len(w) for w in want_q]
        assert np.array_equal(rq, np.concatenate(want_q)) and np.array_equal(rs, np.concatenate(want_s))
        ref = O.dequant_1x128(xq, xs) * (expert_of_row[:, None] + 1)
        assert np.array_equal(back, ref.astype(np.float32))


def test_expert_shard_bounds():
    from fp8_block_scaled_sigmoid_b200 import ep
    s = ep.ExpertShard(256, 8, 3)
    assert (s.e0, s.e1, s.per_rank) == (96, 128, 32)
    with pytest.raises(ValueError):
        ep.ExpertShard(250, 8, 0)
    with pytest.raises(ValueError):
        ep.ExpertShard(256, 8, 8)


def test_expert_parallel_single_rank_is_identity():
    """world = 1: the plan keeps every row and both exchanges are copies."""
    from fp8_block_scaled_sigmoid_b200 import ep
    counts, xq, xs, _ = _ep_rank_data(0)
    shard = ep.ExpertShard(EP_E, 1, 0)
    plan = ep.plan_dispatch(torch.from_numpy(counts), shard)
    assert plan.send_splits == plan.recv_splits == [int(counts.sum())]
    assert np.array_equal(plan.recv_counts.numpy()[0], counts)
    rq, rs = ep.dispatch(torch.from_numpy(xq), torch.from_numpy(xs), plan)
    assert np.array_equal(rq.numpy(), xq) and np.array_equal(rs.numpy(), xs)
    y = torch.from_numpy(O.dequant_1x128(xq, xs).astype(np.float32))
    assert torch.equal(ep.combine_return(y, plan), y)
    with pytest.raises(ValueError):
        ep.exchange_rows(torch.zeros(3, 4), [2], [2])
