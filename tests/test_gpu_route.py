"""GPU parity of moe_route and moe_bias_update against the oracle.

"DeepSeek_V3_Report：Annotation", eqs. (13)-(16), "Node-Limited Routing",
"Auxiliary-Loss-Free Load Balancing".

* logits: tensor-core fp32 accumulation vs the oracle's fp64 product of the
  same bf16 values, within a bound derived from the K-length sum;
* selection: the oracle runs on the GPU's own fp32 logits; expert indices must
  match exactly except for tokens whose K-th vs (K+1)-th biased score (or M-th
  vs (M+1)-th group score) differ by less than 1e-6 -- those are counted and
  only checked for validity; tokens whose chosen experts are tied inside the
  top-K (ordering only) are compared as sets;
* gates: within 4 fp32 ulps of the fp64 value (an ulp of the gate's own
  binade), as the parity contract states.
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import _abi, configs, inputs
from oracle import moe_oracle as O
from tests._util import np32, npraw

pytestmark = pytest.mark.gpu

MARGIN = 1e-6


def _check_selection(z32, bias, G, M, K, idx_g, gate_g):
    idx_o, gate_o, info = O.route_select(z32.astype(np.float64), bias.astype(np.float64), G, M, K)
    T, E = z32.shape
    near = (info["k_margin"] < MARGIN) | (info["g_margin"] < MARGIN)
    order_amb = info["o_margin"] < MARGIN
    exact = ~near & ~order_amb
    assert np.array_equal(idx_g[exact], idx_o[exact]), \
        f"{int((idx_g[exact] != idx_o[exact]).any(1).sum())} tokens differ"
    sets = ~near & order_amb
    for t in np.flatnonzero(sets):
        assert sorted(idx_g[t]) == sorted(idx_o[t])
    # every token's choice is valid: K distinct experts, at most M groups
    for t in range(T):
        assert len(set(idx_g[t])) == K and idx_g[t].min() >= 0 and idx_g[t].max() < E
        if M < G:
            assert len(set(idx_g[t] // (E // G))) <= M
    ok = exact | sets
    go = gate_o[ok]
    ulp = np.ldexp(1.0, np.frexp(go)[1] - 24)          # fp32 ulp at |gate|
    ulps = np.abs(gate_g[ok] - go) / ulp
    print(f"gate error: max {ulps.max():.2f} fp32 ulps, mean {ulps.mean():.3f}")
    assert ulps.max() <= 4.0, f"gate error {ulps.max():.2f} fp32 ulps"
    # gates of every token renormalise its own chosen raw scores
    s = 1.0 / (1.0 + np.exp(-z32.astype(np.float64)))
    for t in range(0, T, max(1, T // 64)):
        sel = s[t, idx_g[t]]
        assert np.allclose(gate_g[t], sel / sel.sum(), rtol=2.0 ** -20, atol=0)
    return int(near.sum()), int(order_amb.sum())


@pytest.mark.parametrize("cfg", [
    configs.TINY,
    configs.TINY.with_(T=333, E=64, G=8, M=2, K=6, d=512),
    configs.V3_PREFILL,
    configs.V3_DECODE,
    configs.V4_PRO.with_(T=2048),
])
def test_route_parity(cuda_dev, cfg):
    u = inputs.draw_u(cfg, cuda_dev)
    cent = inputs.draw_centroids(cfg, cuda_dev)
    bias = inputs.draw_bias(cfg, cuda_dev)
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=cuda_dev)
    idx, gate = _abi.moe_route(u, cent, bias, cfg.G, cfg.M, cfg.K, logits_out=logits)
    torch.cuda.synchronize()
    # logits vs fp64 product of the same bf16 values
    un, cn = np32(u), np32(cent)
    rows = np.arange(0, cfg.T, max(1, cfg.T // 256))
    z64 = O.router_logits(un[rows], cn)
    zg = npraw(logits)[rows]
    bound = 4 * 2.0 ** -24 * np.sqrt(cfg.d) * (np.abs(un[rows]) @ np.abs(cn).T) + 1e-6
    assert np.all(np.abs(zg - z64) <= bound), float(np.max(np.abs(zg - z64) - bound))
    near, amb = _check_selection(npraw(logits), npraw(bias), cfg.G, cfg.M, cfg.K,
                                 npraw(idx), npraw(gate))
    print(f"{cfg.name}: near-ties excluded {near}, order-only ties {amb} of {cfg.T}")


def test_route_end_to_end_against_fp64_logits(cuda_dev):
    """Selection from the oracle's own fp64 logits: identical except near-ties."""
    cfg = configs.TINY.with_(T=512)
    u = inputs.draw_u(cfg, cuda_dev)
    cent = inputs.draw_centroids(cfg, cuda_dev)
    bias = inputs.draw_bias(cfg, cuda_dev)
    idx, _ = _abi.moe_route(u, cent, bias, cfg.G, cfg.M, cfg.K)
    torch.cuda.synchronize()
    idx_o, _, info = O.route(np32(u), np32(cent), npraw(bias), cfg.G, cfg.M, cfg.K)
    # fp32 tensor-core logits differ from fp64 by ~1e-6; widen the margin to it
    near = (info["k_margin"] < 1e-4) | (info["g_margin"] < 1e-4) | (info["o_margin"] < 1e-4)
    assert np.array_equal(npraw(idx)[~near], idx_o[~near])


def test_bias_update_bit_exact(cuda_dev):
    rng = np.random.default_rng(0)
    for E, T, K in [(16, 128, 4), (256, 4096, 8), (384, 16384, 6)]:
        counts = rng.integers(0, 3 * T * K // E, E).astype(np.int32)
        counts[: E // 4] = T * K // E                    # exactly at the mean
        b = rng.uniform(-0.05, 0.05, E).astype(np.float32)
        bd = torch.from_numpy(b).to(cuda_dev)
        _abi.moe_bias_update(torch.from_numpy(counts).to(cuda_dev), T, K, 0.001, bd)
        torch.cuda.synchronize()
        assert np.array_equal(npraw(bd), O.bias_update(counts, T, K, 0.001, b))
