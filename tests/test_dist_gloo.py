"""Multi-rank host logic on CPU (gloo, world size 2).

Each data-parallel rank routes its own batch; the bias update needs the load
of the whole batch ("DeepSeek_V3_Report：Annotation", "Auxiliary-Loss-Free
Load Balancing"), so the per-expert counts are summed over ranks first.  The
test checks that every rank then computes the same new bias, equal to the
oracle's update on the concatenated batch, and that timings reduce to the
slowest rank.
"""
import os
import socket

import numpy as np
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
