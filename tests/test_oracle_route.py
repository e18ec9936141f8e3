"""Pins of the oracle's router, permutation, GEMM, SwiGLU, combine and bias
update (CPU only).

Each pin computes the same quantity another way: brute-force enumeration of
expert and group subsets, exact rational arithmetic, per-element Python loops,
or a closed form / invariant from "DeepSeek_V3_Report：Annotation"
(eqs. (12)-(16), "Auxiliary-Loss-Free Load Balancing", "Node-Limited
Routing", "No Token-Dropping").
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import moe_oracle as ONP


# ---------------------------------------------------------------- routing --
def _bruteforce_select(beta_row, G, M, K):
    """Best group subset by enumeration, then best expert subset by enumeration.
    Scores are exact (fp64 sums of dyadic grid values).  Ties: the subset whose
    sorted index tuple is lexicographically smallest wins."""
    E = len(beta_row)
    gs = E // G
    if M < G:
        n = K // M
        gscore = []
        for g in range(G):
            vals = beta_row[g * gs:(g + 1) * gs]
            gscore.append(max(sum(c) for c in itertools.combinations(vals, n)))
        best = None
        for sub in itertools.combinations(range(G), M):
            sc = sum(gscore[g] for g in sub)
            if best is None or sc > best[0]:
                best = (sc, sub)
        allowed = [e for g in best[1] for e in range(g * gs, (g + 1) * gs)]
    else:
        allowed = list(range(E))
    best = None
    for sub in itertools.combinations(sorted(allowed), K):
        sc = sum(beta_row[e] for e in sub)
        if best is None or sc > best[0]:
            best = (sc, sub)
    chosen = list(best[1])
    chosen.sort(key=lambda e: (-beta_row[e], e))
    return chosen


def _grid_logits(rng, T, E, ties=False):
    """Logits whose sigmoid+bias lands on a dyadic grid (exact sums): pick the
    biased score beta on a 1/64 grid and solve for (z, b) with b = 0."""
    beta = rng.integers(4, 60, (T, E)) / 64.0
    if ties:
        beta[:, 1::3] = beta[:, 0::3][:, : beta[:, 1::3].shape[1]]
    z = np.log(beta / (1.0 - beta))
    return z, beta


@pytest.mark.parametrize("G,M,K", [(4, 2, 4), (4, 4, 4), (8, 4, 8), (2, 1, 2), (1, 1, 3)])
def test_route_select_matches_bruteforce(O, G, M, K):
    rng = np.random.default_rng(10 + G * 7 + M + K)
    E = 16
    for ties in (False, True):
        z, _ = _grid_logits(rng, 60, E, ties)
        bias = np.zeros(E)
        idx, gate, info = O.route_select(z, bias, G, M, K)
        beta = info["beta"]
        for t in range(z.shape[0]):
            want = _bruteforce_select(list(beta[t]), G, M, K)
            assert list(idx[t]) == want, (t, list(idx[t]), want)


def _bruteforce_select_int(s_int, b_int, G, M, K):
    """Exhaustive selection on exact integers: beta = s + b, both given as
    integer multiples of a common power of two (so every sum is exact).
    Groups: every C(G, M) subset, scored by the sum over its groups of the
    best K/M-subset sum of beta; experts: every K-subset of the allowed
    experts.  Ties: the lexicographically smallest sorted index tuple."""
    E = len(s_int)
    beta = [s_int[e] + b_int[e] for e in range(E)]
    gs = E // G
    if M < G:
        n = K // M
        gscore = [max(sum(beta[e] for e in c) for c in itertools.combinations(range(g * gs, (g + 1) * gs), n))
                  for g in range(G)]
        best = max(itertools.combinations(range(G), M),
                   key=lambda sub: (sum(gscore[g] for g in sub), [-g for g in sub]))
        allowed = [e for g in sorted(best) for e in range(g * gs, (g + 1) * gs)]
    else:
        allowed = list(range(E))
    best = max(itertools.combinations(allowed, K),
               key=lambda sub: (sum(beta[e] for e in sub), [-e for e in sub]))
    return sorted(best, key=lambda e: (-beta[e], e))


SCALE = 2 ** 70   # s in (2^-16, 1) has its last bit at or above 2^-69


def _as_int(x):
    """Exact integer multiple of 2^-70 of an fp64 value (asserted exact)."""
    v = float(x) * SCALE
    assert v == int(v)
    return int(v)


@pytest.mark.parametrize("G,M,K,seed", [(4, 2, 4, 0), (8, 4, 8, 1), (4, 1, 2, 2), (2, 1, 4, 3)])
def test_route_select_with_bias_matches_bruteforce(O, G, M, K, seed):
    """Selection with a non-zero bias b_i ([ANN] eq. (16): the top-K is taken
    over s_{i,t} + b_i) and the group limit of "Node-Limited Routing", each
    group ranked by its biased scores.  Exhaustive enumeration over 2500
    tokens per case (10^4 over the four), on exact integers: s comes from the
    oracle's sigmoid (pinned against math.exp), b is a multiple of 1/64, and
    beta = s + b is summed without rounding.  A third of the tokens copy
    logits and biases between experts and between whole groups, forcing
    exact ties in beta and in the group scores."""
    rng = np.random.default_rng(100 + seed)
    T, E = 2500, 16
    gs = E // G
    z = rng.uniform(-6, 6, (T, E))
    bias = rng.integers(-4, 5, E) / 64.0
    # forced ties: the same logit (and so the same s) on expert pairs that
    # share a bias value, and whole groups copied onto another group
    tied = rng.random(T) < 1 / 3
    bias[gs:2 * gs] = bias[:gs]
    for t in np.flatnonzero(tied):
        z[t, gs:2 * gs] = z[t, :gs]                  # group 1 == group 0, exactly
        same_b = [(i, j) for i in range(E) for j in range(i + 1, E) if bias[i] == bias[j]]
        i, j = same_b[rng.integers(len(same_b))]
        z[t, j] = z[t, i]
    idx, gate, info = O.route_select(z, bias, G, M, K)
    s = O.sigmoid(z)
    b_int = [_as_int(v) for v in bias]
    n_raw_differs = 0
    for t in range(T):
        s_int = [_as_int(v) for v in s[t]]
        want = _bruteforce_select_int(s_int, b_int, G, M, K)
        assert list(idx[t]) == want, (t, list(idx[t]), want)
        # the gates come from the raw affinities of the chosen experts
        assert np.allclose(gate[t], s[t, want] / s[t, want].sum(), rtol=1e-14, atol=0)
        if M < G:
            raw = _bruteforce_select_int(s_int, [0] * E, G, M, K)
            if set(raw) != set(want):
                n_raw_differs += 1
    if M < G:
        # the bias decides the selection of many tokens, so ranking the groups
        # or the experts by raw affinity would fail this pin
        assert n_raw_differs > T // 20, n_raw_differs


def test_group_score_uses_the_biased_scores(O):
    """Hand-built token (E = 8 experts in G = 4 groups of 2, M = 2, K = 2,
    so each group is scored by its best biased score).  Raw affinities
    s = (.9, .1 | .8, .1 | .5, .1 | .45, .1) rank the groups 0, 1, 2, 3;
    a bias of +0.5 on expert 6 makes group 3 score .95 and beat groups 1 and
    0.  The biased reading selects groups {3, 0} and experts (6, 0): beta
    .95 > .9.  Ranking groups by raw s would pick groups {0, 1} and experts
    (0, 2).  The gates are the raw s of the chosen experts normalised:
    (.45, .9) / 1.35 = (1/3, 2/3)."""
    s = np.array([0.9, 0.1, 0.8, 0.1, 0.5, 0.1, 0.45, 0.1])
    z = np.log(s / (1.0 - s))[None, :]
    b = np.array([0, 0, 0, 0, 0, 0, 0.5, 0.0])
    idx, gate, _ = O.route_select(z, b, 4, 2, 2)
    assert list(idx[0]) == [6, 0]
    assert np.allclose(gate[0], [1 / 3, 2 / 3], rtol=1e-12, atol=0)
    raw_idx, _, _ = O.route_select(z, b, 4, 2, 2, group_score="raw")
    assert list(raw_idx[0]) == [0, 2]


def test_raw_group_score_fails_the_pin(O):
    """Negative control: the raw-affinity group ranking (a plausible mistake)
    disagrees with the exhaustive biased selection on many tokens."""
    rng = np.random.default_rng(7)
    T, E, G, M, K = 400, 16, 4, 2, 4
    z = rng.uniform(-6, 6, (T, E))
    bias = rng.integers(-4, 5, E) / 64.0
    idx, _, _ = O.route_select(z, bias, G, M, K, group_score="raw")
    s = O.sigmoid(z)
    b_int = [_as_int(v) for v in bias]
    wrong = sum(list(idx[t]) != _bruteforce_select_int([_as_int(v) for v in s[t]], b_int, G, M, K)
                for t in range(T))
    assert wrong > T // 20, wrong


def test_no_group_limit_is_plain_topk(O):
    rng = np.random.default_rng(5)
    T, E, K = 200, 64, 6
    z = rng.normal(0, 1, (T, E))
    b = rng.uniform(-0.05, 0.05, E)
    idx, _, _ = O.route_select(z, b, 1, 1, K)
    s = 1.0 / (1.0 + np.exp(-z))
    for t in range(T):
        beta = [s[t, e] + b[e] for e in range(E)]
        want = sorted(range(E), key=lambda e: (-beta[e], e))[:K]
        assert list(idx[t]) == want
    # M == G behaves like no limit
    idx2, _, _ = O.route_select(z, b, 8, 8, K)
    assert np.array_equal(idx, idx2)


def test_sigmoid_against_math_exp(O):
    z = np.array([-30.0, -2.5, -1e-3, 0.0, 0.7, 12.0])
    want = np.array([1.0 / (1.0 + math.exp(-v)) for v in z])
    assert np.allclose(O.sigmoid(z), want, rtol=1e-15, atol=0)


def test_gates_normalised_and_bias_only_selects(O):
    rng = np.random.default_rng(6)
    T, E, G, M, K = 300, 32, 4, 2, 4
    z = rng.normal(0, 1, (T, E))
    b0 = np.zeros(E)
    b1 = rng.uniform(-0.1, 0.1, E)
    i0, g0, _ = O.route_select(z, b0, G, M, K)
    i1, g1, info = O.route_select(z, b1, G, M, K)
    assert np.allclose(g1.sum(axis=1), 1.0, atol=1e-12, rtol=0)
    s = info["s"]
    # eq. (13): gates are the raw affinities of the chosen experts, normalised
    for t in range(T):
        raw = [s[t, e] for e in i1[t]]
        assert np.allclose(g1[t], np.array(raw) / sum(raw), rtol=1e-14, atol=0)
    # eq. (16): the bias changes which experts are chosen, never the gate of a
    # given chosen set
    same = [t for t in range(T) if set(i0[t]) == set(i1[t])]
    assert 0 < len(same) < T
    for t in same:
        m0 = dict(zip(i0[t], g0[t]))
        m1 = dict(zip(i1[t], g1[t]))
        for e in m0:   # same set, possibly summed in another order
            assert math.isclose(m0[e], m1[e], rel_tol=2e-15, abs_tol=0)


def test_route_with_group_limit_uses_at_most_m_groups(O):
    rng = np.random.default_rng(7)
    T, E, G, M, K = 500, 64, 8, 3, 6
    z = rng.normal(0, 1, (T, E))
    idx, _, _ = O.route_select(z, rng.uniform(-0.05, 0.05, E), G, M, K)
    for t in range(T):
        assert len(set(idx[t] // (E // G))) <= M
        assert len(set(idx[t])) == K


# ----------------------------------------------------------- permutation --
def test_permute_bruteforce(O):
    rng = np.random.default_rng(8)
    T, E, K = 97, 12, 3
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    counts, offsets, src_row, dst_of = O.permute(idx, E)
    assert counts.sum() == T * K                               # no token dropped
    slot = 0
    for e in range(E):
        toks = [t for t in range(T) if e in idx[t]]            # ascending tokens
        assert counts[e] == len(toks) and offsets[e] == slot
        for t in toks:
            assert src_row[slot] == t
            k = list(idx[t]).index(e)
            assert dst_of[t, k] == slot
            slot += 1
    assert offsets[E] == T * K


def test_mtile_table_bruteforce(O):
    offs = np.array([0, 0, 5, 133, 261, 262, 600], np.int64)
    grp, start = O.mtile_table(offs)
    want = []
    for g in range(len(offs) - 1):
        n = offs[g + 1] - offs[g]
        want += [g] * math.ceil(n / 128)
    assert list(grp) == want
    assert list(start) == [0, 0, 1, 2, 3, 4, 7]


# -------------------------------------------------------------------- GEMM --
def _exact_block_gemm(aq, sa, bq, sb):
    """D[m][n] = sum_kb sa[m,kb] sb[n/128,kb] sum_k deq(a) deq(b), exactly."""
    dec = {c: Fraction(float(ONP.e4m3_decode(np.uint8(c)))) for c in range(256) if c not in (0x7F, 0xFF)}
    M, K = aq.shape
    N = bq.shape[0]
    out = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            tot = Fraction(0)
            for kb in range(K // 128):
                part = sum(dec[int(aq[m, k])] * dec[int(bq[n, k])] for k in range(kb * 128, kb * 128 + 128))
                tot += Fraction(float(sa[m, kb])) * Fraction(float(sb[n // 128, kb])) * part
            out[m, n] = float(tot)
    return out


def test_grouped_gemm_exact_small(O):
    rng = np.random.default_rng(9)
    K, N = 256, 128
    aq = rng.integers(0, 0x7E, (5, K)).astype(np.uint8) | (rng.integers(0, 2, (5, K)) << 7).astype(np.uint8)
    bq = rng.integers(0, 0x7E, (2, N, K)).astype(np.uint8)
    sa = rng.uniform(0.01, 2, (5, 2)).astype(np.float32)
    sb = rng.uniform(0.01, 2, (2, 1, 2)).astype(np.float32)
    offs = np.array([0, 2, 5])
    got = O.grouped_gemm(aq, sa, bq, sb, offs)
    cols = [0, 1, 77, 127]
    want0 = _exact_block_gemm(aq[:2], sa[:2], bq[0][cols], sb[0])
    want1 = _exact_block_gemm(aq[2:], sa[2:], bq[1][cols], sb[1])
    assert np.allclose(got[:2][:, cols], want0, rtol=1e-13, atol=1e-13)
    assert np.allclose(got[2:][:, cols], want1, rtol=1e-13, atol=1e-13)


def test_grouped_gemm_integer_operands_exact(O):
    # codes whose E4M3 values are small integers, unit scales: exact integers
    rng = np.random.default_rng(11)
    ints = {int(v): c for c, v in zip(range(0x7F), O.e4m3_decode(np.arange(0x7F, dtype=np.uint8)))
            if float(v).is_integer() and 0 < v <= 8}
    keys = sorted(ints)
    av = rng.choice(keys, (3, 128))
    bv = rng.choice(keys, (1, 128, 128))
    aq = np.vectorize(ints.get)(av).astype(np.uint8)
    bq = np.vectorize(ints.get)(bv).astype(np.uint8)
    got = O.grouped_gemm(aq, np.ones((3, 1), np.float32), bq, np.ones((1, 1, 1), np.float32), [0, 3])
    want = av.astype(np.int64) @ bv[0].T.astype(np.int64)
    assert np.array_equal(got, want.astype(np.float64))


def test_empty_segments_leave_rows_zero(O):
    aq = np.full((4, 128), 0x38, np.uint8)       # all 1.0
    bq = np.full((3, 128, 128), 0x38, np.uint8)
    sa = np.ones((4, 1), np.float32)
    sb = np.stack([np.full((1, 1), 2.0 ** i, np.float32) for i in range(3)])
    got = O.grouped_gemm(aq, sa, bq, sb, [0, 0, 4, 4])
    assert np.all(got == 128.0 * 2.0)             # every row in segment 1 (scale 2)


# ----------------------------------------------------------------- SwiGLU --
def test_swiglu_layout_and_values(O):
    rng = np.random.default_rng(12)
    I = 256
    gu = rng.normal(0, 2, (3, 2 * I))
    h = O.swiglu(gu, I)
    for r in range(3):
        for c in (0, 5, 127, 128, 200, 255):
            j, o = divmod(c, 128)
            g = gu[r, 256 * j + o]
            u = gu[r, 256 * j + 128 + o]
            assert math.isclose(h[r, c], g / (1 + math.exp(-g)) * u, rel_tol=1e-14)
    assert O.silu(0.0) == 0.0
    assert math.isclose(float(O.silu(40.0)), 40.0, rel_tol=1e-15)
    assert abs(float(O.silu(-40.0))) < 1e-15


def test_swiglu_quant_roundtrip(O):
    rng = np.random.default_rng(13)
    gu = rng.normal(0, 1, (4, 512)).astype(np.float32)
    q, s = O.swiglu_quant(gu, 256)
    assert q.shape == (4, 256) and s.shape == (4, 2)
    h = O.swiglu(gu, 256)
    deq = O.dequant_1x128(q, s)
    assert np.all(np.abs(deq - h) <= np.abs(h) * 2.0 ** -4 + np.repeat(s, 128, 1) * 2.0 ** -9)


# ---------------------------------------------------------------- combine --
def test_combine_bruteforce(O):
    rng = np.random.default_rng(14)
    T, K, d = 5, 3, 8
    Y = rng.normal(0, 1, (T * K, d))
    Ys = rng.normal(0, 1, (T, d))
    u = rng.normal(0, 1, (T, d))
    dst = np.stack([rng.permutation(T * K)[:K] for _ in range(T)])
    gate = rng.uniform(0, 1, (T, K))
    out = O.combine(Y, dst, gate, Ys, u)
    for t in range(T):
        for j in range(d):
            want = u[t, j] + Ys[t, j] + sum(gate[t, k] * Y[dst[t, k], j] for k in range(K))
            assert math.isclose(out[t, j], want, rel_tol=1e-13, abs_tol=1e-13)
    # gates summing to 1 over identical rows reproduce that row
    Yc = np.tile(rng.normal(0, 1, (1, d)), (T * K, 1))
    g1 = gate / gate.sum(1, keepdims=True)
    assert np.allclose(O.combine(Yc, dst, g1, None, np.zeros((T, d))), np.tile(Yc[:1], (T, 1)))


# ------------------------------------------------------------ bias update --
def test_bias_update_hand_example(O):
    counts = np.array([3, 1, 2, 2])               # T=2, K=4, E=4: mean load 2
    b = np.array([0.01, -0.02, 0.03, 0.0], np.float32)
    nb = O.bias_update(counts, 2, 4, 0.001, b)
    g = np.float32(0.001)
    assert nb.dtype == np.float32
    assert nb[0] == np.float32(b[0] - g)          # overloaded: minus gamma
    assert nb[1] == np.float32(b[1] + g)          # underloaded: plus gamma
    assert nb[2] == b[2] and nb[3] == b[3]        # at the mean: unchanged


def test_bias_update_fp32_exact(O):
    rng = np.random.default_rng(15)
    E = 256
    counts = rng.integers(0, 300, E)
    b = rng.uniform(-0.05, 0.05, E).astype(np.float32)
    nb = O.bias_update(counts, 4096, 8, 0.001, b)
    mean = 4096 * 8 / E
    for i in range(E):
        if counts[i] > mean:
            assert nb[i] == np.float32(b[i]) - np.float32(0.001)
        elif counts[i] < mean:
            assert nb[i] == np.float32(b[i]) + np.float32(0.001)
        else:
            assert nb[i] == b[i]


# ----------------------------------------------------------- whole layer --
def test_tiny_layer_invariants(O):
    from fp8_block_scaled_sigmoid_b200 import configs, inputs
    cfg = configs.TINY
    inp = inputs.draw_layer(cfg)
    u = inp["u"].float().numpy()
    w1q, w1s, w2q, w2s = O.quantise_weights(inp["w1"].float().numpy(), inp["w2"].float().numpy())
    r = O.moe_layer(u, inp["centroids"].float().numpy(), inp["bias"].numpy(),
                    w1q, w1s, w2q, w2s, cfg.G, cfg.M, cfg.K, cfg.gamma)
    T, K = cfg.T, cfg.K
    assert r["counts"].sum() == T * K
    assert np.allclose(r["gate"].sum(1), 1.0)
    # eq. (12) rebuilt from the per-row expert outputs
    Y = r["Y"]
    out = u.astype(np.float64) + Y[T * K:]
    for t in range(T):
        for k in range(K):
            out[t] += r["gate"][t, k] * Y[r["dst_of"][t, k]]
    assert np.allclose(out, r["out"], rtol=1e-12, atol=1e-12)
    # the expert outputs of token t under expert e equal the dense FFN of t
    t, k = 3, 1
    e = r["idx"][t, k]
    x = O.dequant_1x128(r["xq_tok"][t:t + 1], r["xs_tok"][t:t + 1])
    gu = x @ O.dequant_128x128(w1q[e], w1s[e]).T
    hq, hs = O.swiglu_quant(gu, cfg.I)
    y = O.dequant_1x128(hq, hs) @ O.dequant_128x128(w2q[e], w2s[e]).T
    assert np.allclose(y[0], Y[r["dst_of"][t, k]], rtol=1e-12, atol=1e-12)


# ----------------------------------------------- sequence-wise balance loss --
# [ANN] "Complementary Sequence-Wise Auxiliary Loss", eqs. (17)-(20).
def test_seq_balance_loss_hand_example(O):
    """Two tokens, three experts, K=1, one sequence, alpha=1.  The logits are
    chosen so the affinities are exact: sigmoid(ln 3) = 3/4, sigmoid(0) = 1/2,
    sigmoid(-ln 3) = 1/4.
      token 0: s = (3/4, 1/2, 1/4), sum 3/2 -> s' = (1/2, 1/3, 1/6), top-1 = 0
      token 1: s = (1/4, 3/4, 1/2), sum 3/2 -> s' = (1/6, 1/2, 1/3), top-1 = 1
      f = 3/(1*2) * (1, 1, 0) = (3/2, 3/2, 0)
      P = ((1/2+1/6)/2, (1/3+1/2)/2, (1/6+1/3)/2) = (1/3, 5/12, 1/4)
      L = 3/2*1/3 + 3/2*5/12 = 9/8"""
    l3 = math.log(3.0)
    z = np.array([[l3, 0.0, -l3], [-l3, l3, 0.0]])
    loss, f, P, _ = O.seq_balance_loss(z, K=1, seq_len=2, alpha=1.0)
    assert np.allclose(f[0], [1.5, 1.5, 0.0], rtol=0, atol=1e-15)
    assert np.allclose(P[0], [1 / 3, 5 / 12, 1 / 4], rtol=0, atol=1e-15)
    assert abs(loss[0] - 9 / 8) < 1e-14


@pytest.mark.parametrize("E,K,S", [(4, 2, 4), (16, 4, 8), (64, 8, 16)])
def test_seq_balance_loss_uniform_affinities(O, E, K, S):
    """Equal logits: every s' = 1/E, the ties go to experts 0..K-1, so
    f = E/K on them and 0 elsewhere, and L = alpha * K * (E/K) * (1/E) = alpha."""
    z = np.full((2 * S, E), 0.3)
    loss, f, P, _ = O.seq_balance_loss(z, K=K, seq_len=S, alpha=1e-4)
    assert np.allclose(loss, 1e-4, rtol=1e-14, atol=0)
    want_f = np.zeros(E)
    want_f[:K] = E / K
    assert np.array_equal(f, np.stack([want_f, want_f]))
    assert np.allclose(P, 1.0 / E, rtol=1e-14, atol=0)


def test_seq_balance_loss_invariants_and_sequences(O):
    """Random logits: sum_i f_i = N_r (each token counts K experts, scaled by
    N_r/(K T)); sum_i P_i = 1 (each s' row sums to 1); 0 < L <= alpha*N_r/K
    (P sums to 1, f_i <= N_r/K); sequences are independent (the loss of each
    sequence equals the loss computed on it alone)."""
    rng = np.random.default_rng(17)
    E, K, S = 32, 6, 24
    z = rng.normal(0, 1.5, (3 * S, E))
    loss, f, P, _ = O.seq_balance_loss(z, K=K, seq_len=S, alpha=2e-4)
    assert np.allclose(f.sum(axis=1), E, rtol=1e-13, atol=0)
    assert np.allclose(P.sum(axis=1), 1.0, rtol=1e-13, atol=0)
    assert (loss > 0).all() and (loss <= 2e-4 * E / K + 1e-18).all()
    for q in range(3):
        lq, fq, Pq, _ = O.seq_balance_loss(z[q * S:(q + 1) * S], K=K, seq_len=S, alpha=2e-4)
        assert lq[0] == loss[q] and np.array_equal(fq[0], f[q]) and np.array_equal(Pq[0], P[q])
    # a token whose affinity mass sits on its own top-K raises the loss it
    # would have with flat affinities: concentrating every token on the same
    # K experts gives f = N_r/K there and P close to 1/K, so L -> alpha*N_r/K
    zc = np.full((S, E), -30.0)
    zc[:, :K] = 30.0
    lc, _, _, _ = O.seq_balance_loss(zc, K=K, seq_len=S, alpha=1.0)
    assert abs(lc[0] - E / K) < 1e-9
