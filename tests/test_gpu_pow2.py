"""GPU parity of the power-of-two scale variant.

"DeepSeek_V3_Report：Annotation", "Low-Precision Storage and Communication"
(scaling factors that are integral powers of 2) and "Suggestions on Hardware
Design" (tensor cores that apply the group scales).  The quantisers must
match the oracle byte for byte; the block-scaled GEMM (the tensor core applies
the UE8M0 exponents) must meet max|err| <= 2e-3 * RMS(ref) against the fp64
oracle on the very FP8 operands it consumed; the layer is compared like the
fp32-scale layer.
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import MoELayer, _abi, configs, inputs, make_fp8_weights
from oracle import moe_oracle as O
from tests._util import assert_within_rms, e4m3_step_distance, np32, npraw

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols,outl", [(1, 128, 0.0), (37, 384, 0.01), (1000, 7168, 0.001)])
def test_quant_1x128_pow2_bitexact(cuda_dev, rows, cols, outl):
    x = inputs.draw_matrix(rows, cols, seed=rows + cols, tid=30, outlier_frac=outl,
                           outlier_mult=80.0)
    x[0, :128] = 0                                  # an all-zero tile
    q, s = _abi.fp8_quant_1x128(x.to(cuda_dev), pow2=True)
    torch.cuda.synchronize()
    qo, so = O.quant_1x128_pow2(np32(x))
    assert np.array_equal(npraw(s), so)
    assert np.array_equal(npraw(q), qo)


@pytest.mark.parametrize("rows,cols", [(128, 128), (200, 384), (2 * 2048, 1024)])
def test_quant_128x128_pow2_bitexact(cuda_dev, rows, cols):
    w = inputs.draw_matrix(rows, cols, seed=rows * 3 + cols, tid=31, std=0.02,
                           outlier_frac=0.001, outlier_mult=30.0)
    q, s = _abi.fp8_quant_128x128(w.to(cuda_dev), pow2=True)
    torch.cuda.synchronize()
    qo, so = O.quant_128x128_pow2(np32(w))
    assert np.array_equal(npraw(s), so)
    assert np.array_equal(npraw(q), qo)


def _operands(dev, rows, K, groups, N, seed):
    a = inputs.draw_matrix(rows, K, seed=seed, tid=32, outlier_frac=0.002, outlier_mult=50.0)
    b = torch.stack([inputs.draw_matrix(N, K, seed=seed + g, tid=33, std=1.0 / np.sqrt(K))
                     for g in range(groups)])
    aq, sa = _abi.fp8_quant_1x128(a.to(dev), pow2=True)
    bq, sb = _abi.fp8_quant_128x128(b.to(dev), pow2=True)
    return aq, sa, bq, sb


def _tables(dev, offsets, max_tiles):
    offs = torch.tensor(offsets, dtype=torch.int32, device=dev)
    tg, ts, nt = _abi.moe_tile_table(offs, max_tiles)
    return offs, tg, ts, nt


# K blocks 1, 3, 5 (a partial group of four), 8 and 56; empty segments, a
# leading offset and ragged tails
@pytest.mark.parametrize("K,N,counts,start", [
    (128, 256, [1], 0),
    (384, 512, [0, 1, 130, 300, 17], 0),
    (640, 256, [129, 0, 255], 3),
    (512, 256, [31, 32, 33, 64, 65, 96, 97, 160, 225], 0),   # every A box size
    (1024, 768, [5, 0, 0, 256, 129], 10),
    (7168, 512, [200, 60], 0),
])
def test_gemm_pow2_ragged(cuda_dev, K, N, counts, start):
    rows = start + sum(counts) + 7
    G = len(counts)
    aq, sa, bq, sb = _operands(cuda_dev, rows, K, G, N, seed=K + N + 1)
    offsets = list(np.cumsum([start] + counts))
    max_tiles = sum((c + 127) // 128 for c in counts) + 2
    offs, tg, ts, nt = _tables(cuda_dev, offsets, max_tiles)
    D = torch.full((rows, N), float("nan"), dtype=torch.float32, device=cuda_dev)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, max_tiles, D=D,
                                      dev_err=err, pow2=True)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    Dn = npraw(D)
    lo, hi = offsets[0], offsets[-1]
    assert np.isnan(Dn[:lo]).all() and np.isnan(Dn[hi:]).all(), "rows outside segments written"
    ref = O.grouped_gemm(npraw(aq), npraw(sa), npraw(bq), npraw(sb), offsets)
    rel = assert_within_rms(Dn[lo:hi], ref[lo:hi], what=f"pow2 K={K} N={N}")
    # the promoting GEMM on the same operands agrees too
    D2 = _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, max_tiles)
    torch.cuda.synchronize()
    assert_within_rms(npraw(D2)[lo:hi], Dn[lo:hi], what="pow2 vs promoting GEMM")
    print(f"pow2 GEMM K={K} N={N}: max|err|/RMS = {rel:.2e}")


def test_gemm_pow2_standalone_4096x7168x2048(cuda_dev):
    cfg = configs.STANDALONE_GEMM
    a, bt = inputs.draw_gemm(cfg, cuda_dev)
    aq, sa = _abi.fp8_quant_1x128(a, pow2=True)
    bq, sb = _abi.fp8_quant_128x128(bt.unsqueeze(0), pow2=True)
    offs, tg, ts, nt = _tables(cuda_dev, [0, cfg.M], cfg.M // 128)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    D = _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, cfg.M // 128,
                                          dev_err=err, pow2=True)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = O.grouped_gemm(npraw(aq), npraw(sa), npraw(bq), npraw(sb), [0, cfg.M])
    rel = assert_within_rms(npraw(D), ref, what="pow2 standalone gemm")
    print(f"pow2 standalone GEMM max|err|/RMS = {rel:.2e}")


def test_gemm_pow2_rejects_other_scales(cuda_dev):
    """fp32 amax/448 scales are not powers of two: the kernel records it."""
    K, N, rows = 256, 256, 128
    a = inputs.draw_matrix(rows, K, seed=1, tid=34)
    b = inputs.draw_matrix(N, K, seed=2, tid=35, std=0.05).unsqueeze(0)
    aq, sa = _abi.fp8_quant_1x128(a.to(cuda_dev))
    bq, sb = _abi.fp8_quant_128x128(b.to(cuda_dev))
    offs, tg, ts, nt = _tables(cuda_dev, [0, rows], 1)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, 1, dev_err=err, pow2=True)
    torch.cuda.synchronize()
    assert int(err.item()) == 4        # MOE_DEVERR_BAD_SCALE


def _compare_h(hq_g, hs_g, hq_o, hs_o, max_flip=1e-3, max_off=2e-2, what=""):
    """h bytes per 1x128 tile: where the power-of-two scales agree, codes
    within one E4M3 step; a tile whose amax sits on a power-of-two boundary
    may take the neighbouring scale (fp32 vs fp64 accumulation), then its
    dequantised values agree within one step of the coarser scale."""
    rows, I = hq_g.shape
    sg, so = hs_g.reshape(rows, I // 128), hs_o.reshape(rows, I // 128)
    same = sg == so
    assert np.all(same | (sg == 2 * so) | (2 * sg == so)), what
    assert (~same).mean() <= max_flip, (what, (~same).mean())
    tile_same = np.repeat(same, 128, axis=1)
    dist = e4m3_step_distance(hq_g, hq_o)
    assert dist[tile_same].max(initial=0) <= 1, what
    assert (dist[tile_same] > 0).mean() < max_off, (what, (dist[tile_same] > 0).mean())
    if (~same).any():
        dg = O.dequant_1x128(hq_g, hs_g)
        do = O.dequant_1x128(hq_o, hs_o)
        coarse = np.repeat(np.maximum(sg, so), 128, axis=1)
        bad = ~tile_same
        # one E4M3 step at the tile maximum's binade (<= 32 for [256, 448]) times the scale
        assert np.all(np.abs(dg - do)[bad] <= 32.0 * coarse[bad]), what
    return (dist[tile_same] > 0).mean(), (~same).mean()


@pytest.mark.parametrize("K,I,counts", [(256, 128, [3, 129, 0, 64]), (7168, 2048, [140, 9])])
def test_swiglu_pow2_epilogue(cuda_dev, K, I, counts):
    N = 2 * I
    rows = sum(counts)
    G = len(counts)
    aq, sa, bq, sb = _operands(cuda_dev, rows, K, G, N, seed=5 * K + I)
    offsets = list(np.cumsum([0] + counts))
    max_tiles = sum((c + 127) // 128 for c in counts)
    offs, tg, ts, nt = _tables(cuda_dev, offsets, max_tiles)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    gu = _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, max_tiles,
                                           dev_err=err, pow2=True)
    h, hs = _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, max_tiles,
                                              ep=_abi.EP_SWIGLU_QUANT, dev_err=err, pow2=True)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    hsn = npraw(hs)
    m, _ = np.frexp(hsn.astype(np.float64))
    assert np.all(m == 0.5)
    # on the kernel's own fp32 accumulators (the F32 run computes the same sums)
    hq_o, hs_o = O.swiglu_quant(npraw(gu), I, pow2=True)
    off1, flip1 = _compare_h(npraw(h), hsn, hq_o, hs_o, what="same accumulators")
    # against the fp64 GEMM
    gu_o = O.grouped_gemm(npraw(aq), npraw(sa), npraw(bq), npraw(sb), offsets)
    hq_o2, hs_o2 = O.swiglu_quant(gu_o, I, pow2=True)
    off2, flip2 = _compare_h(npraw(h), hsn, hq_o2, hs_o2, max_flip=5e-3, what="fp64 GEMM")
    print(f"pow2 swiglu: off-by-one bytes {off1:.2e} / {off2:.2e}, scale flips {flip1:.2e} / {flip2:.2e}")


@pytest.mark.parametrize("cfg", [
    configs.TINY,
    configs.TINY.with_(name="small", T=333, d=512, E=32, G=4, M=2, K=6, I=256),
])
def test_layer_pow2_parity(cuda_dev, cfg):
    w1q, w1s, w2q, w2s = make_fp8_weights(cfg, cuda_dev, pow2=True)
    cent = inputs.draw_centroids(cfg, cuda_dev)
    bias0 = inputs.draw_bias(cfg, cuda_dev)
    layer = MoELayer(cfg, cent, bias0.clone(), w1q, w1s, w2q, w2s, pow2=True)
    u = inputs.draw_u(cfg, cuda_dev)
    out = layer.forward(u)
    torch.cuda.synchronize()
    layer.check()
    w1q, w1s, w2q, w2s = (npraw(t) for t in (w1q, w1s, w2q, w2s))
    m, _ = np.frexp(np.concatenate([w1s.ravel(), w2s.ravel()]).astype(np.float64))
    assert np.all(m == 0.5)
    un = np32(u)
    T, K, P = cfg.T, cfg.K, cfg.T * cfg.K
    r = O.moe_layer(un, np32(cent), npraw(bias0), w1q, w1s, w2q, w2s, cfg.G, cfg.M, cfg.K,
                    cfg.gamma, pow2=True)
    assert np.array_equal(npraw(layer.Xq[P:]), r["xq_tok"])
    assert np.array_equal(npraw(layer.Xs[P:]), r["xs_tok"])
    idx_g, dst_g = npraw(layer.idx), npraw(layer.perm["dst_of"])
    near = (r["route"]["k_margin"] < 1e-5) | (r["route"]["g_margin"] < 1e-5)
    keep = np.flatnonzero(~near)
    rows_g = {(int(t), int(idx_g[t, k])): int(dst_g[t, k]) for t in keep for k in range(K)}
    rows_o = {(int(t), int(r["idx"][t, k])): int(r["dst_of"][t, k]) for t in keep for k in range(K)}
    assert set(rows_g) == set(rows_o)
    pg = np.array([rows_g[k] for k in rows_o])
    po = np.array([rows_o[k] for k in rows_o])
    Hg, Hsg = npraw(layer.H), npraw(layer.Hs)
    _compare_h(Hg[pg], Hsg[pg], r["hq"][po], r["hs"][po], max_flip=5e-3, what="routed h")
    _compare_h(Hg[P:], Hsg[P:], r["hq"][P:], r["hs"][P:], max_flip=5e-3, what="shared h")
    # second GEMM and the output on the CUDA path's own h
    h_in, hs_in = r["hq"].copy(), r["hs"].copy()
    h_in[po], hs_in[po] = Hg[pg], Hsg[pg]
    h_in[P:], hs_in[P:] = Hg[P:], Hsg[P:]
    r2 = O.moe_layer(un, np32(cent), npraw(bias0), w1q, w1s, w2q, w2s, cfg.G, cfg.M, cfg.K,
                     cfg.gamma, h_override=(h_in, hs_in), pow2=True)
    Yg = npraw(layer.Y)
    assert_within_rms(Yg[pg], r2["Y"][po], what="pow2 GEMM-2 rows")
    assert_within_rms(Yg[P:], r2["Y"][P:], what="pow2 GEMM-2 shared rows")
    og = npraw(out)
    assert_within_rms(og[keep], r2["out"][keep], what="pow2 layer output (same h)")
    e = assert_within_rms(og[keep], r["out"][keep], what="pow2 layer output (independent)")
    print(f"{cfg.name} pow2: independent max|err|/RMS {e:.2e}")
