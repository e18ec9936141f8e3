"""Expert parallelism on one GPU: the receive-side labelling kernel, the
expert-parallel forward with one rank, and several ranks emulated in one
process.

"DeepSeek_V3_Report：Annotation", "Low-Precision Communication" (FP8 rows
dispatched to the experts' ranks, outputs returned for the combine) and
"Auxiliary-Loss-Free Load Balancing" (the bias update sees the load of the
whole batch).  Ranks that wait on one another are not run as processes on one
GPU: the emulation runs every rank's stages from one process, in order, and
does each exchange as the device-side copies an all-to-all would make (rank
s's block for rank r lands in r's receive buffer after the blocks of the
sources before s).  No kernel waits on another rank.
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import MoELayer, _abi, configs, ep, inputs, make_fp8_weights
from oracle import moe_oracle as O
from tests._util import assert_within_rms, e4m3_step_distance, np32, npraw

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S,E", [(1, 16), (4, 8), (8, 32)])
def test_segment_ids(cuda_dev, S, E):
    rng = np.random.default_rng(S * 100 + E)
    counts = rng.integers(0, 300, (S, E)).astype(np.int32)
    counts[0, 1] = 0
    n = int(counts.sum())
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    ids = _abi.moe_segment_ids(torch.from_numpy(counts).to(cuda_dev), E, n, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = np.repeat(np.tile(np.arange(E, dtype=np.int32), S), counts.reshape(-1))
    assert np.array_equal(npraw(ids), want)
    # with a lead group: the first 77 rows are group 0, the rest shift by one
    ids2 = _abi.moe_segment_ids(torch.from_numpy(counts).to(cuda_dev), E, n + 77, dev_err=err,
                                lead_rows=77)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(npraw(ids2), np.concatenate([np.zeros(77, np.int32), want + 1]))


def test_segment_ids_inconsistent_counts(cuda_dev):
    counts = torch.tensor([[3, 4]], dtype=torch.int32, device=cuda_dev)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    ids = _abi.moe_segment_ids(counts, 2, 9, dev_err=err)   # the counts sum to 7, not 9
    torch.cuda.synchronize()
    assert int(err.item()) == 2                               # MOE_DEVERR_BAD_TABLE
    assert npraw(ids)[:7].tolist() == [0, 0, 0, 1, 1, 1, 1]


def test_gemm_row_map(cuda_dev):
    """grouped_gemm_fp8_blockscaled with d_rows writes row j's output to row
    d_rows[j] and nothing else; a bad entry is reported and skipped."""
    rng = np.random.default_rng(3)
    rows, K, N = 300, 256, 256
    a = torch.from_numpy(rng.normal(0, 1, (rows, K)).astype(np.float32)).to(cuda_dev)
    w = torch.from_numpy(rng.normal(0, 0.05, (2, N, K)).astype(np.float32)).to(cuda_dev)
    aq, sa = _abi.fp8_quant_1x128(a.bfloat16())
    bq, sb = _abi.fp8_quant_128x128(w.bfloat16())
    offs = torch.tensor([0, 170, rows], dtype=torch.int32, device=cuda_dev)
    mt = 3
    tg, ts, nt = _abi.moe_tile_table(offs, mt)
    plain = _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, mt)
    perm = torch.from_numpy(rng.permutation(rows).astype(np.int32)).to(cuda_dev)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    D = torch.full((rows, N), -7.0, dtype=torch.float32, device=cuda_dev)
    _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, mt, D=D, d_rows=perm,
                                      dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = torch.empty_like(plain)
    want[perm.long()] = plain
    assert torch.equal(D, want)
    bad = perm.clone()
    bad[5] = rows + 3
    D2 = torch.full((rows, N), -7.0, dtype=torch.float32, device=cuda_dev)
    _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, mt, D=D2, d_rows=bad,
                                      dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 2
    keep = torch.ones(rows, dtype=torch.bool, device=cuda_dev)
    keep[perm[5].long()] = False
    assert torch.equal(D2[keep], want[keep])
    assert torch.all(D2[perm[5].long()] == -7.0)


def _oracle_same_operands(layer, cfg, u, w, gate):
    """The single-GPU layer against the oracle on its own FP8 operands:
    SwiGLU + requantisation within one E4M3 step of the oracle's on the same
    GEMM-1 inputs; GEMM 2, the combine and the output within 2e-3 RMS of the
    oracle's fp64 evaluation on the same h."""
    w1q, w1s, w2q, w2s = w
    P = cfg.T * cfg.K
    offs = npraw(layer.perm["offsets"])
    gu = O.grouped_gemm(npraw(layer.Xq), npraw(layer.Xs), w1q, w1s, offs)
    hq, _ = O.swiglu_quant(gu, cfg.I)
    dist = e4m3_step_distance(npraw(layer.H), hq)
    assert dist.max() <= 1 and (dist > 0).mean() < 2e-2
    Y = O.grouped_gemm(npraw(layer.H), npraw(layer.Hs), w2q, w2s, offs)
    assert_within_rms(npraw(layer.Y), Y, what="GEMM-2 rows")
    out = O.combine(Y[:P], npraw(layer.perm["dst_of"]), gate, Y[P:], np32(u))
    assert_within_rms(npraw(layer.out), out, what="layer output")


def _stack_for(w, E, e0, e1):
    """A rank's weight stack: the shared expert (index E) first, then its
    routed experts e0..e1-1."""
    ids = torch.tensor([E] + list(range(e0, e1)), device=w[0].device)
    return [t.index_select(0, ids).contiguous() for t in w]


def _emulate_step(layers, us):
    """One expert-parallel step of every rank, run from one process.  Each
    exchange is done as the copies an all-to-all makes: the counts (rank s's
    block r -> rank r's row s), the FP8 rows and scales (rank s's run for
    rank r's experts, sources in order), the outputs back (the reverse)."""
    world = len(layers)
    El = layers[0].shard.per_rank
    counts = [L.stage_dispatch(u) for L, u in zip(layers, us)]
    cmat = [c.view(world, El) for c in counts]
    for r, L in enumerate(layers):
        for s in range(world):
            L.recv_counts[s].copy_(cmat[s][r])
    send = [c.sum(1).tolist() for c in cmat]             # send[s][r]
    plans = []
    for r, L in enumerate(layers):
        plan = ep.DispatchPlan(send_splits=send[r], recv_splits=[send[s][r] for s in range(world)],
                               recv_counts=L.recv_counts)
        plans.append(plan)
        rq, rs = L.recv_rows(plan)
        o = 0
        for s in range(world):
            xs_q, xs_s = layers[s].send_rows()
            a = sum(send[s][:r])
            n = send[s][r]
            rq[o:o + n].copy_(xs_q[a:a + n])
            rs[o:o + n].copy_(xs_s[a:a + n])
            o += n
    for L in layers:
        L.stage_experts()
    for s, L in enumerate(layers):
        o = 0
        for r in range(world):
            back = layers[r].return_rows()
            a = sum(send[q][r] for q in range(s))            # rank s's rows inside r's buffer
            n = send[s][r]
            L.Yback[o:o + n].copy_(back[a:a + n])
            o += n
    for L, u in zip(layers, us):
        L.stage_combine(u)
    total = torch.stack(counts).sum(0, dtype=torch.int32)
    T_all = sum(L.T for L in layers)
    for L in layers:
        L.stage_bias_update(total, T_all)
    return counts, plans


@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("cfg", [
    configs.TINY,
    configs.TINY.with_(name="small", T=333, d=512, E=32, G=4, M=2, K=6, I=256),
], ids=lambda c: c.name)
def test_ep_emulated_ranks(cuda_dev, cfg, world):
    E, T, K = cfg.E, cfg.T, cfg.K
    El = E // world
    w = make_fp8_weights(cfg, cuda_dev)
    cent = inputs.draw_centroids(cfg, cuda_dev)
    bias0 = inputs.draw_bias(cfg, cuda_dev)
    us = [inputs.draw_u(cfg.with_(seed=cfg.seed + r), cuda_dev) for r in range(world)]
    layers = [ep.MoELayerEP(cfg, cent, bias0.clone(), *_stack_for(w, E, r * El, (r + 1) * El),
                            ep.ExpertShard(E, world, r)) for r in range(world)]
    counts, plans = _emulate_step(layers, us)
    torch.cuda.synchronize()
    for L in layers:
        L.check()
    # several sources really interleave on the receive side
    assert all(sum(1 for v in p.recv_splits if v > 0) > 1 for p in plans)
    w1q, w1s, w2q, w2s = (npraw(t) for t in w)
    all_counts = np.zeros(E, np.int64)
    for r, (L, u) in enumerate(zip(layers, us)):
        ref = MoELayer(cfg, cent, bias0.clone(), *w)
        out_ref = ref.forward(u, update_bias=False)
        torch.cuda.synchronize()
        ref.check()
        # routing, counts and the dispatched FP8 rows: bit-exact with the
        # single-GPU layer on the same tokens
        assert torch.equal(L.idx, ref.idx) and torch.equal(L.gate, ref.gate)
        assert torch.equal(counts[r], ref.perm["counts"])
        assert torch.equal(L.Xsend, ref.Xq[:T * K]) and torch.equal(L.Xs_send, ref.Xs[:T * K])
        # the received rows: from every source in rank order, its rows of
        # this rank's experts
        want = []
        for s, Ls in enumerate(layers):
            off = npraw(Ls.perm["offsets"])
            want.append(npraw(Ls.Xsend)[off[r * El]:off[(r + 1) * El]])
        assert np.array_equal(npraw(L.RX[T:T + L.R]), np.concatenate(want))
        # the output: bit for bit the single-GPU layer's, which the oracle
        # checks on the same FP8 operands (the contract's comparison)
        assert torch.equal(L.out, out_ref)
        _oracle_same_operands(ref, cfg, u, (w1q, w1s, w2q, w2s), gate=npraw(ref.gate))
        all_counts += npraw(counts[r])
    # the bias update sees the load of every rank's tokens
    want_b = O.bias_update(all_counts, T * world, K, cfg.gamma, npraw(bias0))
    for L in layers:
        assert np.array_equal(npraw(L.bias), want_b)


@pytest.mark.parametrize("cfg", [
    configs.TINY,
    configs.TINY.with_(name="small", T=333, d=512, E=32, G=4, M=2, K=6, I=256),
], ids=lambda c: c.name)
def test_ep_single_rank_matches_layer(cuda_dev, cfg):
    w = make_fp8_weights(cfg, cuda_dev)
    cent = inputs.draw_centroids(cfg, cuda_dev)
    bias = inputs.draw_bias(cfg, cuda_dev)
    u = inputs.draw_u(cfg, cuda_dev)
    ref = MoELayer(cfg, cent, bias.clone(), *w)
    out_ref = ref.forward(u).clone()
    layer = ep.MoELayerEP(cfg, cent, bias.clone(), *_stack_for(w, cfg.E, 0, cfg.E),
                          ep.ExpertShard(cfg.E, 1, 0))
    for _ in range(2):     # the preallocated buffers serve every step
        out = layer.forward(u, update_bias=False)
    layer.forward(u)
    torch.cuda.synchronize()
    ref.check()
    layer.check()
    assert torch.equal(out, out_ref)
    assert torch.equal(layer.bias, ref.bias)


def test_ep_bad_index_raises_before_the_exchange(cuda_dev):
    """A device error recorded before the dispatch (here planted in the
    error word, as an out-of-range expert index would) stops the step at the
    plan's host read, before any row is exchanged."""
    cfg = configs.TINY
    w = make_fp8_weights(cfg, cuda_dev)
    layer = ep.MoELayerEP(cfg, inputs.draw_centroids(cfg, cuda_dev), inputs.draw_bias(cfg, cuda_dev),
                          *_stack_for(w, cfg.E, 0, cfg.E), ep.ExpertShard(cfg.E, 1, 0))
    counts = layer.stage_dispatch(inputs.draw_u(cfg, cuda_dev))
    layer.dev_err.fill_(3)
    with pytest.raises(_abi.MoEError):
        ep.plan_dispatch(counts, layer.shard, dev_err=layer.dev_err)
