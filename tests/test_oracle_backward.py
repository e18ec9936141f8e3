"""Pins of the oracle's expert-FFN backward (CPU only).

"DeepSeek_V3_Report：Annotation", "Mixed Precision Framework" (Fprop, Dgrad
and Wgrad GEMMs in FP8), "Low-Precision Activation" (SwiGLU input cached in
FP8, output recomputed) and "Support for Transposed GEMM Operations" (128x1
re-quantisation).  The chain rule is pinned by central finite differences of
a forward written here from eq. (12) with the routing held fixed; the FP8
pieces by exact identities (transposed weights dequantise to the transpose,
a 128x1 tile is the 1x128 tile of the transpose, zero padding) and by
brute-force sums over tokens.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O

T, d, E, G, M, K, I = 7, 256, 4, 2, 1, 2, 128


def _problem(seed=0, pow2=True):
    rng = np.random.default_rng(seed)
    u = rng.normal(0, 1, (T, d)).astype(np.float32)
    cent = rng.normal(0, 0.05, (E, d)).astype(np.float32)
    bias = np.zeros(E, np.float32)
    w1 = rng.normal(0, 1 / np.sqrt(d), (E + 1, 2 * I, d)).astype(np.float32)
    w2 = rng.normal(0, 1 / np.sqrt(I), (E + 1, d, I)).astype(np.float32)
    w1q, w1s, w2q, w2s = O.quantise_weights(w1, w2, pow2=pow2)
    fwd = O.moe_layer(u, cent, bias, w1q, w1s, w2q, w2s, G, M, K, 0.001, pow2=pow2)
    dout = rng.normal(0, 1, (T, d)).astype(np.float32)
    return u, fwd, (w1q, w1s, w2q, w2s), dout


def _loss(x_rows, w1, w2, fwd, dout):
    """L = sum_t <dout_t, out_t> with out_t = u_t + sum_s FFN_s + sum_i g_i FFN_i
    (eq. (12)), the experts' input rows x held as the variable, routing and
    gates fixed, no quantisation."""
    offs, dst, gate = fwd["offsets"], fwd["dst_of"], fwd["gate"].astype(np.float64)
    rows = x_rows.shape[0]
    P = T * K
    y = np.zeros((rows, d))
    for g in range(len(offs) - 1):
        r0, r1 = int(offs[g]), int(offs[g + 1])
        if r1 == r0:
            continue
        gu = x_rows[r0:r1] @ w1[g].T
        blk = gu.reshape(r1 - r0, I // 128, 2, 128)
        gg, uu = blk[:, :, 0, :], blk[:, :, 1, :]
        h = (gg / (1 + np.exp(-gg)) * uu).reshape(r1 - r0, I)
        y[r0:r1] = h @ w2[g].T
    out = y[P:].copy()
    for k in range(K):
        out += gate[:, k:k + 1] * y[dst[:, k]]
    return float(np.sum(out * dout))


def test_chain_rule_against_finite_differences():
    _, fwd, (w1q, w1s, w2q, w2s), dout = _problem(1)
    w1 = np.stack([O.dequant_128x128(q, s) for q, s in zip(w1q, w1s)])
    w2 = np.stack([O.dequant_128x128(q, s) for q, s in zip(w2q, w2s)])
    x = O.dequant_1x128(fwd["xq"], fwd["xs"])
    # the exact (unquantised) backward must use the exact SwiGLU input of x
    fwd = dict(fwd)
    gu = np.zeros((x.shape[0], 2 * I))
    offs = fwd["offsets"]
    for g in range(len(offs) - 1):
        gu[offs[g]:offs[g + 1]] = x[offs[g]:offs[g + 1]] @ w1[g].T
    fwd["gu"] = gu
    r = O.expert_backward(dout, fwd, w1q, w1s, w2q, w2s, quantize=False)
    rng = np.random.default_rng(7)
    eps = 1e-5

    def fd(fn, arr, idx):
        a0 = arr[idx]
        arr[idx] = a0 + eps
        lp = fn()
        arr[idx] = a0 - eps
        lm = fn()
        arr[idx] = a0
        return (lp - lm) / (2 * eps)

    L = lambda: _loss(x, w1, w2, fwd, dout)
    for _ in range(6):
        i = (int(rng.integers(x.shape[0])), int(rng.integers(d)))
        assert abs(fd(L, x, i) - r["dx"][i]) <= 1e-6 * (1 + abs(r["dx"][i])), ("dx", i)
    used = [g for g in range(E + 1) if offs[g + 1] > offs[g]]
    for _ in range(6):
        g = int(rng.choice(used))
        i = (g, int(rng.integers(2 * I)), int(rng.integers(d)))
        assert abs(fd(L, w1, i) - r["dW1"][i]) <= 1e-6 * (1 + abs(r["dW1"][i])), ("dW1", i)
        j = (g, int(rng.integers(d)), int(rng.integers(I)))
        assert abs(fd(L, w2, j) - r["dW2"][j]) <= 1e-6 * (1 + abs(r["dW2"][j])), ("dW2", j)
    # du: the residual plus every row of the token (the input reaches each
    # expert through x = u's rows)
    P = T * K
    du = dout.astype(np.float64) + r["dx"][P:]
    for k in range(K):
        du += r["dx"][fwd["dst_of"][:, k]]
    assert np.allclose(r["du"], du, rtol=0, atol=1e-12)


def test_quantised_backward_close_to_exact():
    _, fwd, (w1q, w1s, w2q, w2s), dout = _problem(2)
    rq = O.expert_backward(dout, fwd, w1q, w1s, w2q, w2s, quantize=True)
    re = O.expert_backward(dout, fwd, w1q, w1s, w2q, w2s, quantize=False)
    for k in ("dh", "dx", "du", "dW1", "dW2"):
        err = np.linalg.norm(rq[k] - re[k]) / np.linalg.norm(re[k])
        assert err < 0.1, (k, err)       # a few E4M3 half-steps (2^-4) of relative noise
    # the FP8 operands are what the quantisers give
    qy, sy = O.quant_1x128_pow2(rq["dy"])
    assert np.array_equal(qy, rq["dyq"]) and np.array_equal(sy, rq["dys"])


def test_transpose_weights_exact():
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, (2, 256, 384)).astype(np.float32)
    q, s = zip(*[O.quant_128x128_pow2(x) for x in w])
    q, s = np.stack(q), np.stack(s)
    qt, st = O.transpose_weights(q, s)
    assert qt.shape == (2, 384, 256) and st.shape == (2, 3, 2)
    for g in range(2):
        assert np.array_equal(O.dequant_128x128(qt[g], st[g]), O.dequant_128x128(q[g], s[g]).T)


def test_quant_128x1_is_1x128_of_the_transpose():
    rng = np.random.default_rng(4)
    m = (rng.normal(0, 1, (300, 256)) * np.exp2(rng.integers(-4, 4, (300, 1)))).astype(np.float32)
    offsets = [0, 0, 130, 131, 300]            # an empty, a ragged and a one-token segment
    qt, st, koff = O.quant_128x1_pow2(m, offsets)
    assert list(koff) == [0, 0, 256, 384, 640]
    assert qt.shape == (256, 640) and st.shape == (256, 5)
    for g in range(4):
        r0, r1 = offsets[g], offsets[g + 1]
        if r1 == r0:
            continue
        kp = koff[g + 1] - koff[g]
        pad = np.zeros((kp, 256), np.float32)
        pad[:r1 - r0] = m[r0:r1]
        q1, s1 = O.quant_1x128_pow2(pad.T)
        assert np.array_equal(qt[:, koff[g]:koff[g + 1]], q1)
        # a block with real tokens takes its scale from them; padding codes are zero
        assert np.array_equal(st[:, koff[g] // 128:koff[g + 1] // 128], s1)
        assert np.all(qt[:, koff[g] + (r1 - r0):koff[g + 1]] == 0)
    # brute force: a column block's maximum maps into [224, 448]
    deq = O.dequant_rows(qt, st)
    c, blk = 17, 1                             # segment 1 (rows 0..129), its second block: 2 tokens
    vals = np.abs(deq[c, 128:130]) / st[c, 1]
    assert 224 <= vals.max() <= 448


def test_wgrad_is_a_sum_over_tokens():
    rng = np.random.default_rng(5)
    rows = 150
    a = rng.integers(-4, 5, (rows, 128)).astype(np.float32)     # exact in E4M3 with scale 1
    b = rng.integers(-4, 5, (rows, 256)).astype(np.float32)
    offsets = [0, 40, 150]
    at = O.quant_128x1_pow2(a, offsets)
    bt = O.quant_128x1_pow2(b, offsets)
    dw = O.wgrad(O.dequant_rows(*at[:2]), O.dequant_rows(*bt[:2]), at[2])
    for g in range(2):
        ref = np.zeros((128, 256))
        for r in range(offsets[g], offsets[g + 1]):         # brute force over tokens
            ref += np.outer(a[r], b[r])
        assert np.allclose(dw[g], ref, rtol=0, atol=1e-9)
