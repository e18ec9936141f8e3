"""Named MoE-layer shapes and the value distributions of their synthetic inputs.

Plain data only: no arithmetic of the method lives here.

Dimensions follow DeepSeek-V3 as summarised on "DeepSeek_V3_Report：Annotation"
(model hyper-parameters: hidden 7168, 1 shared + 256 routed experts of
intermediate width 2048, 8 activated experts per token, at most 4 of 8 nodes)
and the V4-Pro figures on "DeepSeek V3 / V4 Infra" (overlap-budget section:
intermediate 3072, 384 routed experts, 6 activated).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int            # tokens in the batch
    d: int            # hidden width
    E: int            # routed experts
    G: int            # expert groups (the pages' nodes); G=1 means no group limit
    M: int            # groups a token may use (the pages' M)
    K: int            # routed experts per token (the pages' K_r)
    I: int            # expert intermediate width (shared and routed)
    n_shared: int = 1
    gamma: float = 0.001          # bias update speed
    bias_lo: float = -0.01        # b_i ~ U(bias_lo, bias_hi) unless a load shape is given
    bias_hi: float = 0.01
    load_shape: str = "uniform"   # "uniform" | "zipf" | "hot"
    zipf_s: float = 1.1
    zipf_c: float = 0.12          # b_i = zipf_c * ln(p_i / p_1), p_i ~ i^-s over a seeded order
    hot_frac: float = 0.1         # share of experts given a bias boost
    hot_delta: float = 0.045      # bias boost of the hot experts
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def pairs(self) -> int:
        return self.T * self.K

    @property
    def gemm_flops(self) -> float:
        """Algorithmic FLOPs of the expert FFNs: 6*d*I per token-expert pair
        (gate, up and down projections), routed pairs plus one shared pass per
        token."""
        return 6.0 * self.d * self.I * (self.pairs + self.n_shared * self.T)

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


TINY = MoEConfig("tiny", T=128, d=256, E=16, G=4, M=2, K=4, I=128,
                 bias_lo=-0.01, bias_hi=0.01)
V3_PREFILL = MoEConfig("v3_prefill", T=4096, d=7168, E=256, G=8, M=4, K=8, I=2048,
                       bias_lo=-0.05, bias_hi=0.05)
V3_DECODE = MoEConfig("v3_decode", T=256, d=7168, E=256, G=8, M=4, K=8, I=2048,
                      load_shape="zipf")
V4_PRO = MoEConfig("v4_pro", T=16384, d=7168, E=384, G=1, M=1, K=6, I=3072,
                   load_shape="hot", bias_lo=-0.01, bias_hi=0.01)

# Profiling case: V3 prefill's per-expert shapes (~128 rows per expert,
# d=7168, I=2048) with 32 experts, so an ncu capture holds ~1.5 GB.
V3_PREFILL_E32 = MoEConfig("v3_prefill_e32", T=512, d=7168, E=32, G=8, M=4, K=8, I=2048,
                           bias_lo=-0.05, bias_hi=0.05)

# Profiling case for the token-sized kernels (route, quantisation,
# permutation, combine): V3 prefill's T, d and top-8, but 32 experts, so the
# weights take ~1.5 GB and multi-pass captures stay small.
V3_TOKENS_E32 = MoEConfig("v3_tokens_e32", T=4096, d=7168, E=32, G=8, M=4, K=8, I=2048,
                          bias_lo=-0.05, bias_hi=0.05)

# Profiling case for the backward: V3's d and I with ~128 tokens per expert
# (16 routed experts, top-8 within 4 of 8 groups), so its fp32 weight
# gradients (17 experts) take ~3 GB and a multi-pass capture stays small.
V3_BWD_E16 = MoEConfig("v3_bwd_e16", T=256, d=7168, E=16, G=8, M=4, K=8, I=2048,
                       bias_lo=-0.05, bias_hi=0.05)

PRESETS = {c.name: c for c in (TINY, V3_PREFILL, V3_DECODE, V4_PRO, V3_PREFILL_E32, V3_TOKENS_E32,
                               V3_BWD_E16)}


@dataclass(frozen=True)
class GemmConfig:
    """Standalone block-scaled GEMM: A [M][K] (1x128 tiles) times B^T, B stored
    as [N][K] (128x128 blocks), fp32 out."""
    name: str = "gemm_4096x7168x2048"
    M: int = 4096
    K: int = 7168
    N: int = 2048
    a_outlier_frac: float = 0.01
    a_outlier_mult: float = 50.0
    b_std: float = 0.02
    seed: int = 0

    @property
    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K


STANDALONE_GEMM = GemmConfig()
