"""Cross-check of the two oracles: the numpy one (oracle/moe_oracle.py) and the
single-threaded C++ one (oracle/moe_oracle_ref.cpp), written separately from
the same passages of "DeepSeek_V3_Report：Annotation" (eqs. (12)-(16),
"Fine-Grained Quantization", "Online Quantization", "Auxiliary-Loss-Free Load
Balancing").  Integer and byte results must agree exactly; fp64 results up to
the rounding of different summation orders.
"""
import numpy as np
import pytest

from oracle import cpp_oracle as C
from oracle import moe_oracle as N
from tests._util import e4m3_step_distance


def test_e4m3_codec_agrees_everywhere():
    codes = np.arange(256, dtype=np.uint8)
    a, b = N.e4m3_decode(codes), C.e4m3_decode(codes)
    assert np.array_equal(np.isnan(a), np.isnan(b))
    fin = ~np.isnan(a)
    assert np.array_equal(a[fin], b[fin])
    # every representable value, every midpoint, and values around them
    v = np.sort(a[fin])
    mids = (v[:-1] + v[1:]) / 2
    probe = np.concatenate([v, mids, np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf),
                            [-0.0, 0.0, 448.0, 464.0, 480.0, 1e30, -1e30]])
    assert np.array_equal(N.e4m3_encode(probe), C.e4m3_encode(probe))


@pytest.mark.parametrize("pow2", [False, True])
def test_quantisers_agree(pow2):
    rng = np.random.default_rng(1)
    x = rng.normal(0, 1, (96, 512)) * np.where(rng.random((96, 512)) < 0.01, 50.0, 1.0)
    x = x.astype(np.float32)
    x[5, 128:256] = 0.0                           # an all-zero tile (eps floor)
    x[7, :128] = 1e-6                              # a tile below eps
    f1 = (N.quant_1x128_pow2, C.quant_1x128_pow2) if pow2 else (N.quant_1x128, C.quant_1x128)
    f2 = (N.quant_128x128_pow2, C.quant_128x128_pow2) if pow2 else (N.quant_128x128, C.quant_128x128)
    for fn, fc in (f1, f2):
        qn, sn = fn(x)
        qc, sc = fc(x)
        assert np.array_equal(qn, qc) and np.array_equal(sn, sc)


@pytest.mark.parametrize("G,M,K,E", [(8, 4, 8, 64), (1, 1, 6, 48), (8, 2, 4, 32)])
def test_routing_and_permutation_agree(G, M, K, E):
    rng = np.random.default_rng(G * 10 + K)
    z = rng.normal(0, 1.5, (700, E))
    b = rng.uniform(-0.05, 0.05, E)
    i1, g1, r1 = N.route_select(z, b, G, M, K)
    i2, g2, r2 = C.route_select(z, b, G, M, K)
    assert np.array_equal(i1, i2)
    assert np.allclose(g1, g2, rtol=1e-14, atol=0)
    # margins: differences of sigmoids, equal up to the last bits of exp()
    assert np.allclose(r1["k_margin"], r2["k_margin"], rtol=0, atol=1e-15)
    assert np.allclose(r1["g_margin"], r2["g_margin"], rtol=0, atol=1e-15)
    for a, c in zip(N.permute(i1, E), C.permute(i2, E)):
        assert np.array_equal(a, c)


def test_tiny_layer_agrees():
    from fp8_block_scaled_sigmoid_b200 import configs, inputs
    cfg = configs.TINY
    inp = inputs.draw_layer(cfg)
    u = inp["u"].float().numpy()
    cent = inp["centroids"].float().numpy()
    bias = inp["bias"].numpy()
    wn = N.quantise_weights(inp["w1"].float().numpy(), inp["w2"].float().numpy())
    wc = C.quantise_weights(inp["w1"].float().numpy(), inp["w2"].float().numpy())
    for a, c in zip(wn, wc):
        assert np.array_equal(a, c)
    rn = N.moe_layer(u, cent, bias, *wn, cfg.G, cfg.M, cfg.K, cfg.gamma)
    rc = C.moe_layer(u, cent, bias, *wn, cfg.G, cfg.M, cfg.K, cfg.gamma)
    for k in ("idx", "counts", "offsets", "src_row", "dst_of", "xq_tok", "xs_tok", "xq", "xs",
              "bias"):
        assert np.array_equal(rn[k], rc[k]), k
    assert np.allclose(rn["route"]["z"], rc["route"]["z"], rtol=1e-13, atol=1e-13)
    assert np.allclose(rn["gate"], rc["gate"], rtol=1e-14, atol=0)
    assert np.allclose(rn["gu"], rc["gu"], rtol=1e-12, atol=1e-12)
    # h is rounded to fp32 and then quantised: a summation-order difference in
    # gu can move an element across a rounding boundary, by one code at most
    dist = e4m3_step_distance(rn["hq"], rc["hq"])
    assert dist.max() <= 1 and (dist > 0).mean() < 1e-3
    # the second GEMM and the combine on identical FP8 inputs
    rc2 = C.moe_layer(u, cent, bias, *wn, cfg.G, cfg.M, cfg.K, cfg.gamma,
                      h_override=(rn["hq"], rn["hs"]))
    assert np.allclose(rn["Y"], rc2["Y"], rtol=1e-12, atol=1e-12)
    assert np.allclose(rn["out"], rc2["out"], rtol=1e-12, atol=1e-12)


def test_balance_loss_agrees():
    rng = np.random.default_rng(4)
    z = rng.normal(0, 1.2, (96, 40))
    ln, fn, Pn, kn = N.seq_balance_loss(z, 6, 32, 1e-4)
    lc, fc, Pc, kc = C.seq_balance_loss(z, 6, 32, 1e-4)
    assert np.array_equal(fn, fc) and np.array_equal(kn, kc)
    assert np.allclose(Pn, Pc, rtol=1e-13, atol=0) and np.allclose(ln, lc, rtol=1e-13, atol=0)
