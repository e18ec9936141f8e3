"""Seeded synthetic inputs shared by the CUDA path and the oracle.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no routing, no quantisation, no GEMM).  Every tensor is
drawn from its own ``torch.Generator`` keyed by (config seed, tensor id,
expert), so one expert's weights can be re-drawn alone, on the host or on the
device, without drawing the others.

Value distributions (per tensor):
  u            ~ N(0, 1), rounded to bf16                       [T][d]
  centroids e  ~ N(0, 1/d) drawn in fp32, rounded to bf16        [E][d]
  bias b       ~ U(lo, hi) in fp32, or a load-shaping profile    [E]
  W1 (per expert, gate/up block-interleaved rows) ~ N(0, 1/d)    [2I][d]
  W2 (per expert)                                 ~ N(0, 1/I)    [d][I]
Expert index E is the shared expert.

W1 row layout: rows [256j, 256j+128) hold the gate projection's output
channels 128j..128j+127 and rows [256j+128, 256j+256) the matching up
projection channels.  Both are drawn from the same distribution, so the
interleave changes no statistics; it lets one 256-row weight tile carry one
128-wide slice of both halves of SwiGLU.
"""
from __future__ import annotations

import math

import torch

from .configs import GemmConfig, MoEConfig

# tensor ids (part of every generator key)
_ID_U, _ID_CENT, _ID_BIAS, _ID_W1, _ID_W2, _ID_PERM, _ID_HOT = 1, 2, 3, 4, 5, 6, 7
_ID_GA, _ID_GB, _ID_GMASK = 11, 12, 13


def _gen(device, seed: int, tid: int, sub: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tid * 10_007 + sub) & 0x7FFF_FFFF_FFFF)
    return g


def draw_u(cfg: MoEConfig, device="cpu", T: int | None = None) -> torch.Tensor:
    T = cfg.T if T is None else T
    g = _gen(device, cfg.seed, _ID_U)
    return torch.randn(T, cfg.d, generator=g, device=device).to(torch.bfloat16)


def draw_centroids(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    g = _gen(device, cfg.seed, _ID_CENT)
    e = torch.randn(cfg.E, cfg.d, generator=g, device=device) * (1.0 / math.sqrt(cfg.d))
    return e.to(torch.bfloat16)


def draw_bias(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    """fp32 [E].  'uniform': U(lo, hi).  'zipf': b_i = c*ln(p_i/p_1) with
    p_i ∝ rank_i^-s over a seeded ordering of the experts, which tilts the
    selection toward a few hot experts.  'hot': U(lo, hi) plus a boost of
    ``hot_delta`` on a seeded ``hot_frac`` share of the experts."""
    g = _gen(device, cfg.seed, _ID_BIAS)
    base = torch.rand(cfg.E, generator=g, device=device, dtype=torch.float64)
    b = cfg.bias_lo + (cfg.bias_hi - cfg.bias_lo) * base
    if cfg.load_shape == "zipf":
        gp = _gen(device, cfg.seed, _ID_PERM)
        order = torch.randperm(cfg.E, generator=gp, device=device)
        rank = torch.empty(cfg.E, dtype=torch.float64, device=device)
        rank[order] = torch.arange(1, cfg.E + 1, dtype=torch.float64, device=device)
        b = -cfg.zipf_c * cfg.zipf_s * torch.log(rank)
    elif cfg.load_shape == "hot":
        gh = _gen(device, cfg.seed, _ID_HOT)
        n_hot = int(round(cfg.hot_frac * cfg.E))
        hot = torch.randperm(cfg.E, generator=gh, device=device)[:n_hot]
        b = b.clone()
        b[hot] += cfg.hot_delta
    return b.to(torch.float32)


def hot_experts(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    gh = _gen(device, cfg.seed, _ID_HOT)
    n_hot = int(round(cfg.hot_frac * cfg.E))
    return torch.randperm(cfg.E, generator=gh, device=device)[:n_hot]


def draw_w1(cfg: MoEConfig, expert: int, device="cpu") -> torch.Tensor:
    """bf16 [2I][d] for one expert (index E is the shared expert)."""
    g = _gen(device, cfg.seed, _ID_W1, expert)
    w = torch.randn(2 * cfg.I, cfg.d, generator=g, device=device) * (1.0 / math.sqrt(cfg.d))
    return w.to(torch.bfloat16)


def draw_w2(cfg: MoEConfig, expert: int, device="cpu") -> torch.Tensor:
    """bf16 [d][I] for one expert (index E is the shared expert)."""
    g = _gen(device, cfg.seed, _ID_W2, expert)
    w = torch.randn(cfg.d, cfg.I, generator=g, device=device) * (1.0 / math.sqrt(cfg.I))
    return w.to(torch.bfloat16)


def draw_layer(cfg: MoEConfig, device="cpu", with_weights: bool = True) -> dict:
    """All inputs of one layer.  Weights are [E+1][...] stacks (shared last)."""
    out = {
        "u": draw_u(cfg, device),
        "centroids": draw_centroids(cfg, device),
        "bias": draw_bias(cfg, device),
    }
    if with_weights:
        out["w1"] = torch.stack([draw_w1(cfg, e, device) for e in range(cfg.E + cfg.n_shared)])
        out["w2"] = torch.stack([draw_w2(cfg, e, device) for e in range(cfg.E + cfg.n_shared)])
    return out


def draw_gemm(cfg: GemmConfig, device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """A bf16 [M][K] ~ N(0,1) with a seeded 1% of elements multiplied by 50;
    B^T bf16 [N][K] ~ N(0, b_std^2)."""
    ga = _gen(device, cfg.seed, _ID_GA)
    a = torch.randn(cfg.M, cfg.K, generator=ga, device=device)
    gm = _gen(device, cfg.seed, _ID_GMASK)
    mask = torch.rand(cfg.M, cfg.K, generator=gm, device=device) < cfg.a_outlier_frac
    a = torch.where(mask, a * cfg.a_outlier_mult, a)
    gb = _gen(device, cfg.seed, _ID_GB)
    bt = torch.randn(cfg.N, cfg.K, generator=gb, device=device) * cfg.b_std
    return a.to(torch.bfloat16), bt.to(torch.bfloat16)


def draw_matrix(rows: int, cols: int, seed: int, tid: int, std: float = 1.0,
                device="cpu", outlier_frac: float = 0.0, outlier_mult: float = 1.0) -> torch.Tensor:
    """Generic bf16 N(0, std^2) matrix with optional multiplicative outliers."""
    g = _gen(device, seed, 100 + tid)
    x = torch.randn(rows, cols, generator=g, device=device) * std
    if outlier_frac > 0:
        gm = _gen(device, seed, 200 + tid)
        m = torch.rand(rows, cols, generator=gm, device=device) < outlier_frac
        x = torch.where(m, x * outlier_mult, x)
    return x.to(torch.bfloat16)
