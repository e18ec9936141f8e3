"""GPU parity of the sequence-wise balance loss against the oracle: the
three-pass form from logits (moe_seq_balance_loss) and the form fused into
moe_route's selection pass (moe_balance_loss).

"DeepSeek_V3_Report：Annotation", "Complementary Sequence-Wise Auxiliary
Loss", eqs. (17)-(20).  The oracle runs on the GPU's own fp32 logits:
* membership counts (f * K * S / E) are integers and must match exactly,
  except that a token whose K-th and (K+1)-th affinities differ by less than
  1e-6 (fp32 vs fp64 sigmoid) may move one expert in or out;
* P and the loss are fp32 sums of S terms: within 1e-4 relative.
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import _abi
from oracle import moe_oracle as O
from tests._util import npraw

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,E,K,S,std", [
    (64, 16, 4, 32, 1.0),
    (300, 40, 6, 100, 2.0),
    (384, 384, 6, 128, 1.0),
    (4096, 256, 8, 4096, 0.5),     # V3 prefill shape, one sequence
    (4096, 256, 8, 1024, 0.5),     # four sequences
])
def test_seq_balance_loss_parity(cuda_dev, T, E, K, S, std):
    g = torch.Generator(device=cuda_dev).manual_seed(T + E + K)
    z = torch.randn(T, E, generator=g, device=cuda_dev) * std
    loss, f, P = _abi.moe_seq_balance_loss(z, K, S, alpha=1e-4, with_fp=True)
    loss2 = _abi.moe_seq_balance_loss(z, K, S, alpha=1e-4)
    torch.cuda.synchronize()
    assert torch.equal(loss, loss2), "not deterministic"
    lo, fo, Po, margin = O.seq_balance_loss(npraw(z).astype(np.float64), K, S, 1e-4)
    n_seq = T // S
    cnt_g = np.rint(npraw(f) * K * S / E).astype(np.int64)
    cnt_o = np.rint(fo * K * S / E).astype(np.int64)
    near = (margin < 1e-6).reshape(n_seq, S).sum(axis=1)
    for q in range(n_seq):
        assert cnt_g[q].sum() == K * S
        assert np.abs(cnt_g[q] - cnt_o[q]).sum() <= 2 * near[q], (q, near[q])
    assert np.allclose(npraw(P), Po, rtol=1e-4, atol=1e-7)
    clean = near == 0
    assert np.allclose(npraw(loss)[clean], lo[clean], rtol=1e-4, atol=0)
    print(f"T={T} E={K}/{E} S={S}: loss {npraw(loss)} oracle {lo}, near-tie tokens {near.sum()}")


def test_seq_balance_loss_uniform_is_alpha(cuda_dev):
    """Equal logits: the ties go to experts 0..K-1 and L = alpha (eq. 17 with
    f = E/K on K experts and P = 1/E)."""
    T, E, K, S = 256, 64, 8, 128
    z = torch.full((T, E), 0.25, device=cuda_dev)
    loss, f, P = _abi.moe_seq_balance_loss(z, K, S, alpha=1e-4, with_fp=True)
    torch.cuda.synchronize()
    assert np.allclose(npraw(loss), 1e-4, rtol=1e-5, atol=0)
    want = np.zeros(E, np.float32)
    want[:K] = E / K
    assert np.array_equal(npraw(f), np.stack([want, want]))


def test_layer_seq_balance_loss(cuda_dev):
    """Through the layer: the loss of the step's own router logits matches
    the oracle's on the same logits."""
    from fp8_block_scaled_sigmoid_b200 import MoELayer, configs, inputs, make_fp8_weights
    cfg = configs.TINY
    w1q, w1s, w2q, w2s = make_fp8_weights(cfg, cuda_dev)
    layer = MoELayer(cfg, inputs.draw_centroids(cfg, cuda_dev), inputs.draw_bias(cfg, cuda_dev),
                     w1q, w1s, w2q, w2s, keep_logits=True, balance_loss=True,
                     seq_len=cfg.T // 2)
    layer.forward(inputs.draw_u(cfg, cuda_dev))
    loss = layer.seq_balance_loss().clone()
    loss3 = _abi.moe_seq_balance_loss(layer.logits, cfg.K, cfg.T // 2)
    torch.cuda.synchronize()
    lo, _, _, margin = O.seq_balance_loss(npraw(layer.logits).astype(np.float64), cfg.K,
                                          cfg.T // 2, 1e-4)
    clean = (margin < 1e-6).reshape(2, -1).sum(axis=1) == 0
    assert np.allclose(npraw(loss)[clean], lo[clean], rtol=1e-4, atol=0)
    assert torch.allclose(loss, loss3, rtol=1e-5, atol=0)


@pytest.mark.parametrize("cfg_name,S", [("tiny", 64), ("tiny", 8), ("v3_prefill", 4096),
                                        ("v3_prefill", 1024), ("v4_pro", 2048)])
def test_route_fused_loss_matches_three_pass(cuda_dev, cfg_name, S):
    """The loss fused into the router's selection (integer sums, the last
    block of each sequence finishes it) gives the three-pass loss on the same
    logits: the membership counts (hence f) exactly, P and the loss up to the
    rounding of the sums; the routing itself is unchanged; two calls give
    the same bits and leave the state zeroed."""
    from fp8_block_scaled_sigmoid_b200 import configs, inputs
    cfg = configs.PRESETS[cfg_name]
    if cfg.T > 4096:
        cfg = cfg.with_(T=4096)
    u = inputs.draw_u(cfg, cuda_dev)
    cent = inputs.draw_centroids(cfg, cuda_dev)
    bias = inputs.draw_bias(cfg, cuda_dev)
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=cuda_dev)
    st = _abi.BalanceLossState(cfg.T, cfg.E, S, 1e-4, with_fp=True, device=cuda_dev)
    idx, gate = _abi.moe_route(u, cent, bias, cfg.G, cfg.M, cfg.K, logits_out=logits, aux=st)
    la, fa, Pa = st.loss.clone(), st.f.clone(), st.P.clone()
    idx2, gate2 = _abi.moe_route(u, cent, bias, cfg.G, cfg.M, cfg.K, aux=st)
    idx3, gate3 = _abi.moe_route(u, cent, bias, cfg.G, cfg.M, cfg.K)
    lb, fb, Pb = _abi.moe_seq_balance_loss(logits, cfg.K, S, with_fp=True)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx3) and torch.equal(gate, gate3)   # routing unchanged
    assert torch.equal(idx2, idx3) and torch.equal(gate2, gate3)
    assert torch.equal(la, st.loss) and torch.equal(fa, st.f) and torch.equal(Pa, st.P), \
        "not deterministic"
    assert not st.acc.any() and not st.cnt.any() and not st.done.any(), "state not zeroed"
    assert torch.equal(fa, fb)
    # every token counts K members
    assert torch.all(torch.round(fa * cfg.K * S / cfg.E).sum(1) == cfg.K * S)
    # the three-pass P is an fp32 sum over 32-token chunks and then over the
    # chunks: up to (32 + S/32) roundings of 2^-24 relative
    tol = (32 + S / 32) * 2.0 ** -24
    assert torch.allclose(Pa, Pb, rtol=tol, atol=1e-9)
    assert torch.allclose(la, lb, rtol=tol, atol=0)
    # and against the oracle on the same logits
    lo, fo, Po, margin = O.seq_balance_loss(npraw(logits).astype(np.float64), cfg.K, S, 1e-4)
    near = (margin < 1e-6).reshape(-1, S).sum(axis=1)
    assert np.allclose(npraw(Pa), Po, rtol=1e-4, atol=1e-7)
    clean = near == 0
    assert np.allclose(npraw(la)[clean], lo[clean], rtol=1e-4, atol=0)


def test_fused_loss_in_a_cuda_graph(cuda_dev):
    """The fused loss's state zeroes itself, so a step captured in a CUDA
    graph gives the eager step's loss on every replay (same bits), and the
    state is zero after each."""
    from fp8_block_scaled_sigmoid_b200 import MoELayer, configs, inputs, make_fp8_weights
    cfg = configs.TINY
    w1q, w1s, w2q, w2s = make_fp8_weights(cfg, cuda_dev)
    layer = MoELayer(cfg, inputs.draw_centroids(cfg, cuda_dev), inputs.draw_bias(cfg, cuda_dev),
                     w1q, w1s, w2q, w2s, balance_loss=True, seq_len=cfg.T // 4)
    u = inputs.draw_u(cfg, cuda_dev)
    layer.forward(u, update_bias=False)
    eager = layer.seq_balance_loss().clone()
    graph, _ = layer.capture(u, update_bias=False)
    b = layer.balance
    for _ in range(2):
        b.loss.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(b.loss[:b.n_seq], eager)
        assert not b.acc.any() and not b.cnt.any() and not b.done.any()
    del graph
