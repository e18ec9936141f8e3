"""CPU oracle for the DeepSeekMoE layer forward with FP8 block-scaled expert GEMMs.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only the tests, the smoke check and the benchmark's CPU-baseline leg do.  It
shares no code with the CUDA library and reads no value the library produced
unless a test hands it one explicitly (e.g. the GPU's FP8 operands, so that a
GEMM is checked on identical inputs).

Plain numpy, fp64 unless a passage fixes another precision.  Every function
names the passage it follows.  Pages:
  [ANN]  "DeepSeek_V3_Report：Annotation" (annotated translation of the V3 report)
  [NOTES] "DeepSeek-V3：671B/37B MoE、FP8 训练与 DualPipe 的算法—基础设施协同设计"
  [INFRA] "DeepSeek V3 / V4 Infra：把 all-to-all 藏进计算"
  [BLOG]  "从MLA到MTP，从FP8到DualPipe：DeepSeek-V3——一场关于效率、智能与工程哲学的“全栈式”架构革命"

Readings taken where the pages leave a step open (each also listed in the
design notes):
  * quantisation scale stored as the fp32 dequantisation multiplier
    fl32(max(amax, eps)/448), eps = 1e-4; the quantised value is
    E4M3(fl32(x / scale)), round-to-nearest-even, saturating at +-448;
  * group score = sum of the top K/M *biased* scores of the group;
  * ties in every top-k go to the lower index; the selected experts are
    ordered by biased score descending, then index ascending;
  * bias update uses sign(c_i - T*K/E) with sign(0) = 0;
  * Swish beta = 1 (SiLU); shared expert has the routed experts' width and
    gate 1; expert outputs and the layer output are fp32/fp64, not bf16;
  * the balance loss's TopK (eq. 18) is over the raw affinities of all
    routed experts, ties to the lower index;
  * a power-of-two scale is the fp32 scale above rounded up to the next
    power of two (nothing saturates; x / scale is exact).

Parity pins: every function here is pinned by tests that do not re-type its
formula (brute-force enumeration, exhaustive code tables, closed forms,
invariants).  No function is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0          # largest finite E4M3 value (1.75 * 2^8)
QUANT_EPS = np.float32(1e-4)
TILE = 128                # 1x128 activation tiles, 128x128 weight blocks


# ---------------------------------------------------------------------------
# E4M3 format.  [ANN] "Mantissa over Exponents": E4M3 (4 exponent bits,
# 3 mantissa bits) for every tensor; [ANN] "Online Quantization": Q_max = 448.
# Exponent bias 7; exponent field 0 holds subnormals m * 2^-9; field 15 with
# mantissa 7 is NaN; no infinities.
# ---------------------------------------------------------------------------
def e4m3_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    sign = np.where(codes & 0x80, -1.0, 1.0)
    ef = ((codes >> 3) & 0xF).astype(np.int64)
    mf = (codes & 0x7).astype(np.float64)
    normal = (1.0 + mf / 8.0) * np.ldexp(1.0, ef - 7)
    sub = mf * 2.0 ** -9
    val = np.where(ef == 0, sub, normal)
    val = np.where((ef == 15) & (mf == 7), np.nan, val)
    return sign * val


def e4m3_encode(v) -> np.ndarray:
    """Round each finite value to the nearest E4M3 value (ties to even mantissa),
    saturating magnitudes above 448 to 448, and return its code byte."""
    v = np.asarray(v, dtype=np.float64)
    if np.isnan(v).any():
        raise ValueError("e4m3_encode: NaN input")
    neg = np.signbit(v)
    a = np.abs(v)
    # binade of a: a = f * 2^ex with f in [0.5, 1)  =>  floor(log2 a) = ex - 1
    _, ex = np.frexp(a)
    e = np.maximum(ex - 1, -6)                 # below 2^-6 the spacing stays 2^-9
    quantum = np.ldexp(1.0, e - 3)              # 3 mantissa bits
    n = np.rint(a / quantum)                    # rint: half to even
    r = np.minimum(n * quantum, E4M3_MAX)       # saturate (satfinite)
    r = np.where(a >= E4M3_MAX, E4M3_MAX, r)
    # encode the representable magnitude r
    _, rex = np.frexp(r)
    re = rex - 1
    is_sub = r < 2.0 ** -6
    ef = np.where(is_sub, 0, re + 7)
    mf = np.where(is_sub, np.rint(r / 2.0 ** -9), np.rint((r / np.ldexp(1.0, re) - 1.0) * 8.0))
    mf = np.where(r == 0, 0, mf)
    ef = np.where(r == 0, 0, ef)
    code = (ef.astype(np.int64) << 3) | mf.astype(np.int64)
    code = np.where(neg, code | 0x80, code)
    return code.astype(np.uint8)


# ---------------------------------------------------------------------------
# Online fine-grained quantisation.  [ANN] "Fine-Grained Quantization" (1x128
# activation tiles per token, 128x128 weight blocks) and "Online
# Quantization" (scale from the current tile's max |x|, s = Q_max/max(A_max,
# eps), x_fp8 = round(x * s), dequantisation x_fp8 * s^-1).  The stored scale
# is the dequantisation multiplier s^-1 = max(A_max, eps)/448 in fp32; the
# quantised value divides by it in fp32.
# ---------------------------------------------------------------------------
def _scale_of(amax32: np.ndarray) -> np.ndarray:
    a = np.maximum(amax32.astype(np.float32), QUANT_EPS)
    return (a / np.float32(E4M3_MAX)).astype(np.float32)


def quant_1x128(x) -> tuple[np.ndarray, np.ndarray]:
    """x [rows][cols] (values exactly representable in fp32), cols % 128 == 0.
    Returns q uint8 [rows][cols], scale fp32 [rows][cols/128]."""
    x = np.asarray(x, dtype=np.float32)
    rows, cols = x.shape
    assert cols % TILE == 0
    tiles = x.reshape(rows, cols // TILE, TILE)
    amax = np.abs(tiles).max(axis=2)
    scale = _scale_of(amax)
    y = (tiles / scale[:, :, None]).astype(np.float32)
    q = e4m3_encode(y).reshape(rows, cols)
    return q, scale


def quant_128x128(w) -> tuple[np.ndarray, np.ndarray]:
    """w [rows][cols] (nn.Linear layout: output channels x input channels),
    cols % 128 == 0; a ragged last row-block is allowed.  Returns q uint8
    [rows][cols], scale fp32 [ceil(rows/128)][cols/128]."""
    w = np.asarray(w, dtype=np.float32)
    rows, cols = w.shape
    assert cols % TILE == 0
    rb = -(-rows // TILE)
    q = np.empty((rows, cols), dtype=np.uint8)
    scale = np.empty((rb, cols // TILE), dtype=np.float32)
    for i in range(rb):
        blk = w[i * TILE:(i + 1) * TILE]
        for j in range(cols // TILE):
            b = blk[:, j * TILE:(j + 1) * TILE]
            s = _scale_of(np.abs(b).max())
            scale[i, j] = s
            q[i * TILE:(i + 1) * TILE, j * TILE:(j + 1) * TILE] = e4m3_encode((b / s).astype(np.float32))
    return q, scale


# ---------------------------------------------------------------------------
# Power-of-two scales.  [ANN] "Low-Precision Storage and Communication": the
# activations quantised before the dispatch to the MoE up-projection (like the
# input of the Linear after attention) carry scaling factors that are integral
# powers of 2.  Reading: the power of two is the fp32 scale above rounded UP
# (the smallest 2^e >= fl32(max(amax, eps)/448)), so no element saturates and
# x / 2^e is exact in fp32.  The block-scaled variant applies the same rounding
# to the 128x128 weight blocks and to the SwiGLU output, so that every operand
# scale of both expert GEMMs is a pure exponent (UE8M0).
# ---------------------------------------------------------------------------
def pow2_ceil(s) -> np.ndarray:
    """Smallest power of two >= s, for positive finite s (returned in fp32)."""
    s = np.asarray(s, np.float64)
    if (s <= 0).any() or not np.isfinite(s).all():
        raise ValueError("pow2_ceil: positive finite scales only")
    m, ex = np.frexp(s)                  # s = m * 2^ex, m in [0.5, 1)
    return np.where(m == 0.5, s, np.ldexp(1.0, ex)).astype(np.float32)


def quant_1x128_pow2(x) -> tuple[np.ndarray, np.ndarray]:
    """quant_1x128 with each tile's scale rounded up to a power of two."""
    x = np.asarray(x, dtype=np.float32)
    rows, cols = x.shape
    assert cols % TILE == 0
    tiles = x.reshape(rows, cols // TILE, TILE)
    scale = pow2_ceil(_scale_of(np.abs(tiles).max(axis=2)))
    y = (tiles / scale[:, :, None]).astype(np.float32)
    return e4m3_encode(y).reshape(rows, cols), scale


def quant_128x128_pow2(w) -> tuple[np.ndarray, np.ndarray]:
    """quant_128x128 with each block's scale rounded up to a power of two."""
    w = np.asarray(w, dtype=np.float32)
    rows, cols = w.shape
    assert cols % TILE == 0
    rb = -(-rows // TILE)
    q = np.empty((rows, cols), dtype=np.uint8)
    scale = np.empty((rb, cols // TILE), dtype=np.float32)
    for i in range(rb):
        for j in range(cols // TILE):
            b = w[i * TILE:(i + 1) * TILE, j * TILE:(j + 1) * TILE]
            s = pow2_ceil(_scale_of(np.abs(b).max()))
            scale[i, j] = s
            q[i * TILE:(i + 1) * TILE, j * TILE:(j + 1) * TILE] = e4m3_encode((b / s).astype(np.float32))
    return q, scale


def dequant_1x128(q, scale) -> np.ndarray:
    """x_dequant = x_fp8 * (stored scale), per 1x128 tile."""
    return e4m3_decode(q) * np.repeat(np.asarray(scale, np.float64), TILE, axis=1)


def dequant_128x128(q, scale) -> np.ndarray:
    q = np.asarray(q)
    rows, cols = q.shape
    s = np.repeat(np.repeat(np.asarray(scale, np.float64), TILE, axis=0), TILE, axis=1)
    return e4m3_decode(q) * s[:rows, :cols]


# ---------------------------------------------------------------------------
# Router.  [ANN] "Basic Architecture of DeepSeekMoE", eqs. (12)-(15):
# s_{i,t} = Sigmoid(u_t^T e_i); g'_{i,t} = s_{i,t} for the top-K_r experts,
# g_{i,t} = g'_{i,t} / sum_j g'_{j,t}.  "Auxiliary-Loss-Free Load Balancing",
# eq. (16): the top-K_r is taken over s_{i,t} + b_i, the gate still comes from
# the raw s_{i,t}.  "Node-Limited Routing": a token uses at most M nodes,
# chosen by the sum of the highest K_r/M affinities of the experts on each
# node (here: G contiguous expert groups).
# ---------------------------------------------------------------------------
def router_logits(u, centroids) -> np.ndarray:
    """z[t, i] = u_t . e_i in fp64 (the gating stays in high precision,
    [ANN] "Mixed Precision Framework")."""
    return np.asarray(u, np.float64) @ np.asarray(centroids, np.float64).T


def sigmoid(z) -> np.ndarray:
    z = np.asarray(z, np.float64)
    return 1.0 / (1.0 + np.exp(-z))


def _order_desc(vals: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Positions of vals sorted by value descending, then id ascending."""
    return np.lexsort((ids, -vals))


def route_select(z, bias, G: int, M: int, K: int, group_score: str = "biased"):
    """Selection and gating for every token, from logits z [T][E].

    Returns (idx int32 [T][K], gate fp64 [T][K], info) where info holds, per
    token, the margins used to set aside near-ties in parity comparisons:
      k_margin  = beta_(K) - beta_(K+1) among the allowed experts
      g_margin  = score_(M) - score_(M+1) among the groups (inf without limit)
      o_margin  = smallest gap between consecutive selected beta (ordering)
    """
    z = np.asarray(z, np.float64)
    T, E = z.shape
    b = np.asarray(bias, np.float64)
    assert E % G == 0
    gs = E // G
    s = sigmoid(z)
    beta = s + b[None, :]
    idx = np.zeros((T, K), np.int32)
    gate = np.zeros((T, K), np.float64)
    k_margin = np.full(T, np.inf)
    g_margin = np.full(T, np.inf)
    o_margin = np.full(T, np.inf)
    experts = np.arange(E)
    groups = np.arange(G)
    limited = M < G
    if limited:
        assert K % M == 0, "group score uses the top K/M experts of a group"
        n_top = K // M
    for t in range(T):
        allowed = np.ones(E, bool)
        if limited:
            src = beta[t] if group_score == "biased" else s[t]
            gscore = np.array([np.sort(src[g * gs:(g + 1) * gs])[::-1][:n_top].sum()
                               for g in groups])
            gord = _order_desc(gscore, groups)
            keep = gord[:M]
            g_margin[t] = gscore[gord[M - 1]] - gscore[gord[M]]
            allowed[:] = False
            for g in keep:
                allowed[g * gs:(g + 1) * gs] = True
        cand = experts[allowed]
        cb = beta[t, cand]
        ordr = _order_desc(cb, cand)
        sel = cand[ordr[:K]]
        if len(cand) > K:
            k_margin[t] = cb[ordr[K - 1]] - cb[ordr[K]]
        if K > 1:
            o_margin[t] = np.min(-np.diff(cb[ordr[:K]]))
        idx[t] = sel
        gate[t] = s[t, sel] / s[t, sel].sum()
    return idx, gate, {"k_margin": k_margin, "g_margin": g_margin, "o_margin": o_margin,
                       "s": s, "beta": beta}


def route(u, centroids, bias, G, M, K, group_score="biased"):
    z = router_logits(u, centroids)
    idx, gate, info = route_select(z, bias, G, M, K, group_score)
    info["z"] = z
    return idx, gate, info


# ---------------------------------------------------------------------------
# Local permutation by expert.  Stands in for the dispatch step: activations
# are quantised to FP8 before dispatch ([ANN] "Low-Precision Communication")
# and no token is dropped ([ANN] "No Token-Dropping").  Pairs (t, k) are
# grouped by expert; inside an expert, by ascending token.  The shared
# expert's segment (all T tokens in order) follows the routed pairs.
# ---------------------------------------------------------------------------
def permute(idx, E: int):
    idx = np.asarray(idx, np.int64)
    T, K = idx.shape
    flat = idx.reshape(-1)                       # pair p = t*K + k
    order = np.argsort(flat, kind="stable")      # expert-major, token order kept
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    src_row = (order // K).astype(np.int32)
    dst_of = np.empty(T * K, np.int32)
    dst_of[order] = np.arange(T * K, dtype=np.int32)
    return counts, offsets, src_row, dst_of.reshape(T, K)


def segment_offsets_with_shared(offsets, T: int) -> np.ndarray:
    """Append the shared expert's segment (rows pairs .. pairs+T)."""
    offsets = np.asarray(offsets, np.int64)
    return np.concatenate([offsets, [offsets[-1] + T]]).astype(np.int32)


def mtile_table(offsets, tile_m: int = TILE):
    """128-row tiles of every segment, in segment order.
    Returns (tile_group int32 [n_tiles], tile_start int32 [groups+1])."""
    offsets = np.asarray(offsets, np.int64)
    cnt = np.diff(offsets)
    mt = -(-cnt // tile_m)
    start = np.concatenate([[0], np.cumsum(mt)]).astype(np.int32)
    grp = np.repeat(np.arange(len(cnt)), mt).astype(np.int32)
    return grp, start


# ---------------------------------------------------------------------------
# Block-scaled grouped GEMM.  [ANN] "Fine-Grained Quantization" /
# "Increasing Accumulation Precision": per-group scales along the inner
# dimension K, accumulation in high precision.  Written as the definition:
# D = deq(A) . deq(B)^T per segment, in fp64.
# ---------------------------------------------------------------------------
def grouped_gemm(aq, sa, bq, sb, offsets) -> np.ndarray:
    """aq uint8 [rows][K], sa fp32 [rows][K/128]; bq uint8 [groups][N][K],
    sb fp32 [groups][N/128][K/128]; offsets [groups+1].  fp64 [rows][N]."""
    aq = np.asarray(aq)
    bq = np.asarray(bq)
    rows = aq.shape[0]
    groups, N, _ = bq.shape
    out = np.zeros((rows, N), np.float64)
    a = dequant_1x128(aq, sa)
    for g in range(groups):
        r0, r1 = int(offsets[g]), int(offsets[g + 1])
        if r1 > r0:
            out[r0:r1] = a[r0:r1] @ dequant_128x128(bq[g], sb[g]).T
    return out


# ---------------------------------------------------------------------------
# SwiGLU expert.  [ANN] "SwiGLU 运算符的特殊处理": SwiGLU(x) = Swish(x W1) ⊗ (x W2),
# Swish(x) = x * sigma(beta x), beta = 1.  The first GEMM's weight rows are
# block-interleaved: columns [256j, 256j+128) of its output are gate channels
# 128j.., the next 128 are the matching up channels.
# ---------------------------------------------------------------------------
def silu(x) -> np.ndarray:
    x = np.asarray(x, np.float64)
    return x / (1.0 + np.exp(-x))


def swiglu(gu, I: int) -> np.ndarray:
    gu = np.asarray(gu, np.float64)
    rows = gu.shape[0]
    assert gu.shape[1] == 2 * I and I % TILE == 0
    blk = gu.reshape(rows, I // TILE, 2, TILE)
    h = silu(blk[:, :, 0, :]) * blk[:, :, 1, :]
    return h.reshape(rows, I)


def swiglu_quant(gu, I: int, pow2: bool = False):
    """SwiGLU, then 1x128 online quantisation of its fp32 value (the input of
    the down projection is FP8 like every other GEMM input); ``pow2`` rounds
    the scales up to powers of two."""
    h = swiglu(gu, I).astype(np.float32)
    return quant_1x128_pow2(h) if pow2 else quant_1x128(h)


# ---------------------------------------------------------------------------
# Combine.  [ANN] eq. (12): h'_t = u_t + sum_s FFN_s(u_t) + sum_i g_{i,t} FFN_i(u_t).
# ---------------------------------------------------------------------------
def combine(Y, dst_of, gate, Y_shared, u) -> np.ndarray:
    Y = np.asarray(Y, np.float64)
    out = np.asarray(u, np.float64).copy()
    if Y_shared is not None:
        out += np.asarray(Y_shared, np.float64)
    dst_of = np.asarray(dst_of)
    gate = np.asarray(gate, np.float64)
    for k in range(dst_of.shape[1]):
        out += gate[:, k:k + 1] * Y[dst_of[:, k]]
    return out


# ---------------------------------------------------------------------------
# Auxiliary-loss-free bias update.  [ANN] "Auxiliary-Loss-Free Load
# Balancing": at the end of each step, over the whole batch, an overloaded
# expert's b_i drops by gamma and an underloaded one's rises by gamma;
# [BLOG] 1.2.2 reads "overloaded" as receiving more than the average number
# of tokens.  Loads count routed pairs; the shared expert is excluded.
# ---------------------------------------------------------------------------
def bias_update(counts, T: int, K: int, gamma: float, bias) -> np.ndarray:
    counts = np.asarray(counts, np.int64)
    E = counts.shape[0]
    mean = T * K / E                              # exact in fp64 for these sizes
    sgn = np.sign(counts.astype(np.float64) - mean)
    b = np.asarray(bias, np.float32).astype(np.float64)
    g = np.float64(np.float32(gamma))
    return (b - g * sgn).astype(np.float32)


# ---------------------------------------------------------------------------
# Complementary sequence-wise balance loss.  [ANN] "Complementary
# Sequence-Wise Auxiliary Loss", eqs. (17)-(20), for each sequence of T
# tokens:
#   L_Bal = alpha * sum_i f_i P_i,
#   f_i   = N_r / (K_r T) * #{t : s_{i,t} in TopK({s_{j,t}}_j, K_r)},
#   s'_{i,t} = s_{i,t} / sum_j s_{j,t},   P_i = (1/T) sum_t s'_{i,t};
# alpha = 0.0001 for DeepSeek-V3 ([ANN] training hyper-parameters; [BLOG]
# 1.2.3).  Reading: the TopK of eq. (18) is taken over the raw affinities of
# all N_r routed experts, as written (no bias, no group limit), ties to the
# lower index.
# ---------------------------------------------------------------------------
def seq_balance_loss(z, K: int, seq_len: int, alpha: float = 1e-4):
    """Per sequence of seq_len consecutive tokens of the logits z [T][E]:
    (loss [n_seq], f [n_seq][E], P [n_seq][E], k_margin [T]) with k_margin the
    per-token gap between the K-th and (K+1)-th raw affinity (for setting
    aside near-ties when the membership counts are compared)."""
    z = np.asarray(z, np.float64)
    T, E = z.shape
    assert T % seq_len == 0 and 0 < K <= E
    s = sigmoid(z)
    member = np.zeros((T, E), bool)
    k_margin = np.full(T, np.inf)
    experts = np.arange(E)
    for t in range(T):
        ordr = _order_desc(s[t], experts)
        member[t, ordr[:K]] = True
        if K < E:
            k_margin[t] = s[t, ordr[K - 1]] - s[t, ordr[K]]
    s_norm = s / s.sum(axis=1, keepdims=True)
    n_seq = T // seq_len
    f = np.zeros((n_seq, E))
    P = np.zeros((n_seq, E))
    for q in range(n_seq):
        rows = slice(q * seq_len, (q + 1) * seq_len)
        f[q] = E / (K * seq_len) * member[rows].sum(axis=0)
        P[q] = s_norm[rows].sum(axis=0) / seq_len
    loss = alpha * (f * P).sum(axis=1)
    return loss, f, P, k_margin


# ---------------------------------------------------------------------------
# Whole layer, composed from the steps above.
# ---------------------------------------------------------------------------
def quantise_weights(w1, w2, pow2: bool = False):
    """Per expert 128x128 block quantisation of the stacked bf16 weights
    (``pow2``: scales rounded up to powers of two)."""
    w1 = np.asarray(w1, np.float32)
    w2 = np.asarray(w2, np.float32)
    qf = quant_128x128_pow2 if pow2 else quant_128x128
    q1, s1 = zip(*[qf(w) for w in w1])
    q2, s2 = zip(*[qf(w) for w in w2])
    return np.stack(q1), np.stack(s1), np.stack(q2), np.stack(s2)


def moe_layer(u, centroids, bias, w1q, w1s, w2q, w2s, G, M, K, gamma,
              h_override=None, pow2: bool = False):
    """Forward of one layer plus the bias update.  Weights are given already
    quantised ([E+1] stacks, shared expert last).  ``h_override`` =
    (hq, hs) makes the second GEMM consume given FP8 activations (used to
    check the second GEMM and the combine on the CUDA path's own operands).
    ``pow2`` quantises the activations and the SwiGLU output with power-of-two
    scales (the weights must then be quantised with ``pow2`` too)."""
    u = np.asarray(u, np.float32)
    T, d = u.shape
    E = np.asarray(centroids).shape[0]
    I = np.asarray(w1q).shape[1] // 2
    idx, gate, rinfo = route(u, centroids, bias, G, M, K)
    xq_tok, xs_tok = quant_1x128_pow2(u) if pow2 else quant_1x128(u)
    counts, offsets, src_row, dst_of = permute(idx, E)
    pairs = T * K
    xq = np.concatenate([xq_tok[src_row], xq_tok])
    xs = np.concatenate([xs_tok[src_row], xs_tok])
    offs = segment_offsets_with_shared(offsets, T)
    gu = grouped_gemm(xq, xs, w1q, w1s, offs)
    # the SwiGLU input, cached in FP8 for the backward pass ([ANN] "Low-Precision Activation")
    guq, gus = quant_1x128_pow2(gu.astype(np.float32)) if pow2 else quant_1x128(gu.astype(np.float32))
    if h_override is None:
        hq, hs = swiglu_quant(gu, I, pow2)
    else:
        hq, hs = h_override
    Y = grouped_gemm(hq, hs, w2q, w2s, offs)
    out = combine(Y[:pairs], dst_of, gate, Y[pairs:], u)
    new_bias = bias_update(counts, T, K, gamma, bias)
    return {"idx": idx, "gate": gate, "route": rinfo, "xq_tok": xq_tok, "xs_tok": xs_tok,
            "counts": counts, "offsets": offs, "src_row": src_row, "dst_of": dst_of,
            "xq": xq, "xs": xs, "gu": gu, "guq": guq, "gus": gus, "hq": hq, "hs": hs, "Y": Y,
            "out": out, "bias": new_bias}


# ---------------------------------------------------------------------------
# Backward of the expert FFNs.  [ANN] "Mixed Precision Framework": the three
# GEMMs of a linear operator -- Fprop, Dgrad (activation gradient) and Wgrad
# (weight gradient) -- take FP8 inputs and give high-precision outputs; the
# weight gradients stay in high precision.  "Low-Precision Activation": the
# SwiGLU input is cached in FP8 and the SwiGLU output is recomputed in the
# backward pass.  "Low-Precision Communication": the activation gradient
# before the MoE down-projection is quantised to FP8 with power-of-two
# scales.  "Support for Transposed GEMM Operations": an operand whose
# reduction runs over tokens is re-quantised in 128x1 tiles (128 tokens of one
# channel).
# Readings (also in the design notes): every gradient quantisation is 1x128
# along the channels with power-of-two scales (activation gradients are never
# block-quantised: [INFRA] "V3 FP8" reports divergence for 128x128 Dgrad
# gradients); a
# 128x1 operand is quantised from the fp32 value where the backward pass
# computes it (dy, dgu, the recomputed h) and from the dequantised FP8 cache
# for x; each expert's token segment is zero-padded to a multiple of 128
# tokens for its Wgrad; the router's gradient (not an FP8 GEMM) is not part
# of this path.
# ---------------------------------------------------------------------------
def transpose_weights(q, s):
    """FP8 weight stack [G][N][K] with 128x128 block scales [G][N/128][K/128]
    -> the transposed stack [G][K][N] and scales [G][K/128][N/128].  Exact:
    every 128x128 block keeps its own scale."""
    return (np.ascontiguousarray(np.swapaxes(np.asarray(q), 1, 2)),
            np.ascontiguousarray(np.swapaxes(np.asarray(s), 1, 2)))


def wgrad_segments(offsets):
    """Column offsets koff [groups+1] of the token-major (transposed) Wgrad
    operands: segment g's rows, zero-padded to a multiple of 128."""
    offsets = np.asarray(offsets, np.int64)
    kpad = [-(-(int(offsets[g + 1]) - int(offsets[g])) // TILE) * TILE
            for g in range(len(offsets) - 1)]
    return np.concatenate([[0], np.cumsum(kpad)]).astype(np.int64)


def quant_128x1_pow2(m, offsets):
    """m [rows][C] (fp32 values) in token segments [offsets[g], offsets[g+1]).
    Each column of each segment is quantised in blocks of 128 tokens (the
    segment zero-padded to a multiple of 128) with a power-of-two scale.
    Returns the transposed codes qt uint8 [C][Ktot], scales st fp32
    [C][Ktot/128] and koff [groups+1] (segment g = columns koff[g]..koff[g+1])."""
    m = np.asarray(m, np.float32)
    C = m.shape[1]
    offsets = np.asarray(offsets, np.int64)
    koff = wgrad_segments(offsets)
    qt = np.zeros((C, int(koff[-1])), np.uint8)
    st = np.zeros((C, int(koff[-1]) // TILE), np.float32)
    for g in range(len(offsets) - 1):
        r0, r1 = int(offsets[g]), int(offsets[g + 1])
        for b in range(0, r1 - r0, TILE):
            blk = m[r0 + b:min(r1, r0 + b + TILE)]          # up to 128 tokens x C
            scale = pow2_ceil(_scale_of(np.abs(blk).max(axis=0)))
            col = int(koff[g]) + b
            st[:, col // TILE] = scale
            qt[:, col:col + blk.shape[0]] = e4m3_encode((blk / scale[None, :]).astype(np.float32)).T
    return qt, st, koff


def dequant_rows(qt, st) -> np.ndarray:
    """Codes [C][Ktot] with one scale per row per 128 columns."""
    return e4m3_decode(qt) * np.repeat(np.asarray(st, np.float64), TILE, axis=1)


def wgrad(at, bt, koff) -> np.ndarray:
    """Per segment g: dW[g] = At[:, seg g] . Bt[:, seg g]^T (fp64), from two
    dequantised token-major operands At [Ca][Ktot], Bt [Cb][Ktot]."""
    G = len(koff) - 1
    out = np.zeros((G, at.shape[0], bt.shape[0]), np.float64)
    for g in range(G):
        k0, k1 = int(koff[g]), int(koff[g + 1])
        if k1 > k0:
            out[g] = at[:, k0:k1] @ bt[:, k0:k1].T
    return out


def swiglu_backward(dh, gu, I: int):
    """SwiGLU backward ([ANN] SwiGLU operator notes, Swish beta = 1): for the
    block-interleaved input gu [rows][2I] (gate blocks, then the matching up
    blocks) and dh = dL/dh [rows][I]: sigma = 1/(1+e^-g), dg = dh u sigma
    (1 + g (1 - sigma)), du = dh g sigma.  Returns dgu [rows][2I] (same
    interleaving) and the recomputed h = g sigma u [rows][I], fp64."""
    gu = np.asarray(gu, np.float64)
    rows = gu.shape[0]
    blk = gu.reshape(rows, I // TILE, 2, TILE)
    g, u = blk[:, :, 0, :], blk[:, :, 1, :]
    with np.errstate(over="ignore"):
        sg = 1.0 / (1.0 + np.exp(-g))
    silu_g = g * sg
    dsilu = sg * (1.0 + g * (1.0 - sg))
    dh4 = np.asarray(dh, np.float64).reshape(rows, I // TILE, TILE)
    dgu = np.stack([dh4 * u * dsilu, dh4 * silu_g], axis=2).reshape(rows, 2 * I)
    return dgu, (silu_g * u).reshape(rows, I)


def unpermute_add(dx, dst_of, dout) -> np.ndarray:
    """du_t = dout_t + dx[T*K + t] + sum_k dx[dst_of[t][k]] (fp64)."""
    dst_of = np.asarray(dst_of)
    T, K = dst_of.shape
    dx = np.asarray(dx, np.float64)
    du = np.asarray(dout, np.float64) + dx[T * K:T * K + T]
    for k in range(K):
        du = du + dx[dst_of[:, k]]
    return du


def expert_backward(dout, fwd, w1q, w1s, w2q, w2s, quantize: bool = True):
    """Gradients of the expert FFNs for the upstream gradient dout [T][d] of
    the layer output, with the routing of the forward pass ``fwd`` (a
    moe_layer result).  ``quantize=False`` replaces every FP8 quantisation
    of the backward pass by the exact value (and uses the exact SwiGLU input
    and x) -- the plain chain rule, for checking against finite differences.
    Returns dy, dh, dgu, h, dx (per permuted row), du [T][d] (gradient of the
    layer input through the experts and the residual), dW1 [G][2I][d],
    dW2 [G][d][I] (fp64) and the FP8 operands of each GEMM."""
    dout = np.asarray(dout, np.float32)
    T, d = dout.shape
    dst_of, gate, offs = fwd["dst_of"], np.asarray(fwd["gate"], np.float32), fwd["offsets"]
    K = dst_of.shape[1]
    P = T * K
    rows = P + T
    I = np.asarray(w2q).shape[2]
    w1 = np.stack([dequant_128x128(q, s) for q, s in zip(w1q, w1s)])
    w2 = np.stack([dequant_128x128(q, s) for q, s in zip(w2q, w2s)])
    r = {}

    def seg_gemm(a, w):   # rows of segment g times w[g]^T
        o = np.zeros((a.shape[0], w.shape[1]), np.float64)
        for g in range(len(offs) - 1):
            r0, r1 = int(offs[g]), int(offs[g + 1])
            if r1 > r0:
                o[r0:r1] = a[r0:r1] @ w[g].T
        return o

    # 1. the gradient at every expert output row: gate * dout for a routed
    #    pair (one fp32 product), dout itself for the shared expert's row
    dy = np.empty((rows, d), np.float32)
    for k in range(K):
        dy[dst_of[:, k]] = gate[:, k:k + 1] * dout
    dy[P:] = dout
    r["dy"] = dy
    if quantize:
        r["dyq"], r["dys"] = quant_1x128_pow2(dy)
        dy_in = dequant_1x128(r["dyq"], r["dys"])
    else:
        dy_in = dy.astype(np.float64)
    # 2. Dgrad of the down projection: dh = dy . W2 (the GEMM's B is W2^T)
    dh = seg_gemm(dy_in, np.swapaxes(w2, 1, 2))
    r["dh"] = dh
    # 3. SwiGLU backward on its cached input (gate/up blocks interleaved)
    gu = dequant_1x128(fwd["guq"], fwd["gus"]) if quantize else np.asarray(fwd["gu"], np.float64)
    dgu, h = swiglu_backward(dh, gu, I)
    r["dgu"], r["h"] = dgu, h
    dgu32 = dgu.astype(np.float32)
    if quantize:
        r["dguq"], r["dgus"] = quant_1x128_pow2(dgu32)
        dgu_in = dequant_1x128(r["dguq"], r["dgus"])
    else:
        dgu_in = dgu
    # 4. Dgrad of the up projection: dx = dgu . W1
    dx = seg_gemm(dgu_in, np.swapaxes(w1, 1, 2))
    r["dx"] = dx
    # 5. back to the tokens: the residual plus every expert row of the token
    r["du"] = unpermute_add(dx, dst_of, dout)
    # 6. Wgrad: token-major operands, 128x1 tiles
    x = dequant_1x128(fwd["xq"], fwd["xs"])
    koff = wgrad_segments(offs)
    r["koff"] = koff
    if quantize:
        r["dyt"] = quant_128x1_pow2(dy, offs)[:2]
        r["ht"] = quant_128x1_pow2(h.astype(np.float32), offs)[:2]
        r["dgut"] = quant_128x1_pow2(dgu32, offs)[:2]
        r["xt"] = quant_128x1_pow2(x.astype(np.float32), offs)[:2]
        ops = {k: dequant_rows(*r[k]) for k in ("dyt", "ht", "dgut", "xt")}
    else:
        def tm(m):   # token-major, zero-padded segments, exact
            out = np.zeros((m.shape[1], int(koff[-1])), np.float64)
            for gi in range(len(offs) - 1):
                r0, r1 = int(offs[gi]), int(offs[gi + 1])
                out[:, int(koff[gi]):int(koff[gi]) + r1 - r0] = m[r0:r1].T
            return out
        ops = {"dyt": tm(dy.astype(np.float64)), "ht": tm(h), "dgut": tm(dgu), "xt": tm(x)}
    r["dW2"] = wgrad(ops["dyt"], ops["ht"], koff)
    r["dW1"] = wgrad(ops["dgut"], ops["xt"], koff)
    return r
