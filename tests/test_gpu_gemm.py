"""GPU parity of grouped_gemm_fp8_blockscaled, swiglu_quant and moe_combine.

"DeepSeek_V3_Report：Annotation", "Fine-Grained Quantization" and "Increasing
Accumulation Precision" (per-128-K scales, fp32 accumulation), SwiGLU
operator notes, eq. (12).  The oracle consumes the very FP8 bytes and scales
the GPU consumed; the float bar is max|err| <= 2e-3 * RMS(ref).
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import _abi, configs, inputs
from oracle import moe_oracle as O
from tests._util import assert_within_rms, e4m3_step_distance, np32, npraw

pytestmark = pytest.mark.gpu


def _quantised_operands(dev, rows, K, groups, N, seed, a_outl=0.0, b_std=None):
    a = inputs.draw_matrix(rows, K, seed=seed, tid=10, outlier_frac=a_outl, outlier_mult=50.0)
    b = torch.stack([inputs.draw_matrix(N, K, seed=seed + g, tid=11,
                                        std=b_std or 1.0 / np.sqrt(K)) for g in range(groups)])
    aq, sa = _abi.fp8_quant_1x128(a.to(dev))
    bq, sb = _abi.fp8_quant_128x128(b.to(dev))
    return aq, sa, bq, sb


def _tables(dev, offsets, max_tiles):
    offs = torch.tensor(offsets, dtype=torch.int32, device=dev)
    tg, ts, nt = _abi.moe_tile_table(offs, max_tiles)
    return offs, tg, ts, nt


def test_standalone_gemm_4096x7168x2048(cuda_dev):
    cfg = configs.STANDALONE_GEMM
    a, bt = inputs.draw_gemm(cfg, cuda_dev)
    aq, sa = _abi.fp8_quant_1x128(a)
    bq, sb = _abi.fp8_quant_128x128(bt.unsqueeze(0))
    offs, tg, ts, nt = _tables(cuda_dev, [0, cfg.M], cfg.M // 128)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    D = _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, cfg.M // 128,
                                          dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = O.grouped_gemm(npraw(aq), npraw(sa), npraw(bq), npraw(sb), [0, cfg.M])
    rel = assert_within_rms(npraw(D), ref, what="standalone gemm")
    print(f"standalone GEMM max|err|/RMS = {rel:.2e}")


@pytest.mark.parametrize("K,N,counts,start", [
    (128, 256, [1], 0),
    (512, 512, [0, 1, 130, 300, 17], 0),
    (1024, 768, [5, 0, 0, 256, 129], 10),
    (7168, 512, [200, 60], 0),
])
def test_grouped_gemm_ragged(cuda_dev, K, N, counts, start):
    rows = start + sum(counts) + 7
    G = len(counts)
    aq, sa, bq, sb = _quantised_operands(cuda_dev, rows, K, G, N, seed=K + N)
    offsets = list(np.cumsum([start] + counts))
    max_tiles = sum((c + 127) // 128 for c in counts) + 2
    offs, tg, ts, nt = _tables(cuda_dev, offsets, max_tiles)
    D = torch.full((rows, N), float("nan"), dtype=torch.float32, device=cuda_dev)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, max_tiles, D=D,
                                      dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    Dn = npraw(D)
    lo, hi = offsets[0], offsets[-1]
    assert np.isnan(Dn[:lo]).all() and np.isnan(Dn[hi:]).all(), "rows outside segments written"
    ref = O.grouped_gemm(npraw(aq), npraw(sa), npraw(bq), npraw(sb), offsets)
    assert_within_rms(Dn[lo:hi], ref[lo:hi], what=f"ragged K={K} N={N}")


@pytest.mark.parametrize("K,I,counts", [(256, 128, [3, 129, 0, 64]), (7168, 2048, [140, 9])])
def test_swiglu_epilogue(cuda_dev, K, I, counts):
    N = 2 * I
    rows = sum(counts)
    G = len(counts)
    aq, sa, bq, sb = _quantised_operands(cuda_dev, rows, K, G, N, seed=3 * K + I)
    offsets = list(np.cumsum([0] + counts))
    max_tiles = sum((c + 127) // 128 for c in counts)
    offs, tg, ts, nt = _tables(cuda_dev, offsets, max_tiles)
    gu = _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, max_tiles)
    h, hs = _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, max_tiles,
                                              ep=_abi.EP_SWIGLU_QUANT)
    h2, hs2 = _abi.swiglu_quant(gu, I)
    torch.cuda.synchronize()
    # fused epilogue == standalone kernel on the same fp32 accumulators
    assert np.array_equal(npraw(hs), npraw(hs2))
    assert np.array_equal(npraw(h), npraw(h2))
    # standalone kernel on identical fp32 input vs the oracle: SiLU goes
    # through expf on the GPU, so a byte may move by one E4M3 step where the
    # value sits on a rounding boundary; scales agree to fp32 rounding
    hq_o, hs_o = O.swiglu_quant(npraw(gu), I)
    assert np.allclose(npraw(hs2), hs_o, rtol=2.0 ** -21, atol=0)
    dist = e4m3_step_distance(npraw(h2), hq_o)
    assert dist.max() <= 1 and (dist > 0).mean() < 1e-3, (dist.max(), (dist > 0).mean())
    # against the fp64 GEMM: scales within accumulation error, bytes within a step
    gu_o = O.grouped_gemm(npraw(aq), npraw(sa), npraw(bq), npraw(sb), offsets)
    hq_o2, hs_o2 = O.swiglu_quant(gu_o, I)
    assert np.allclose(npraw(hs), hs_o2, rtol=1e-4, atol=0)
    dist2 = e4m3_step_distance(npraw(h), hq_o2)
    assert dist2.max() <= 1 and (dist2 > 0).mean() < 2e-2, (dist2.max(), (dist2 > 0).mean())
    print(f"swiglu: bytes off by one step {(dist > 0).mean():.2e} (same input), "
          f"{(dist2 > 0).mean():.2e} (vs fp64 GEMM)")


def test_combine(cuda_dev):
    rng = np.random.default_rng(5)
    T, K, d = 300, 6, 1024
    P = T * K
    Y = torch.from_numpy(rng.normal(0, 1, (P + T, d)).astype(np.float32)).to(cuda_dev)
    dst = np.stack([rng.permutation(P)[:K] for _ in range(T)]).astype(np.int32)
    gate = rng.uniform(0, 1, (T, K)).astype(np.float32)
    gate /= gate.sum(1, keepdims=True)
    u = inputs.draw_matrix(T, d, seed=1, tid=20)
    out = _abi.moe_combine(Y, torch.from_numpy(dst).to(cuda_dev), torch.from_numpy(gate).to(cuda_dev),
                           Y[P:], u.to(cuda_dev))
    torch.cuda.synchronize()
    Yn = npraw(Y)
    ref = O.combine(Yn[:P], dst, gate, Yn[P:], np32(u))
    assert np.allclose(npraw(out), ref, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("ep", ["f32", "swiglu"])
def test_tail_tiles_and_dynamic_schedule(cuda_dev, ep):
    """m-tiles of at most 32 rows (an expert's rows past a whole 128-row
    tile, or an expert with few rows) take the transposed tail path; every
    tail size from 1 to 33 rows, partial tiles of every A box size and a few
    whole tiles are checked against the oracle on the same FP8 operands.  The dynamic schedule (a work counter)
    gives the same bytes as the static one."""
    K, N = 1024, 512
    # also every A box size (a partial m-tile loads 32, 64, 96 or 128 rows):
    # 63/64/65, 96/97 and their repeats past a whole tile
    counts = [1, 2, 7, 16, 17, 31, 32, 33, 0, 128 + 1, 128 + 31, 128 + 32, 128 + 33, 256 + 5, 64,
              100, 127, 128, 63, 65, 96, 97, 128 + 64, 128 + 65, 128 + 96, 128 + 97]
    G = len(counts)
    rows = sum(counts)
    aq, sa, bq, sb = _quantised_operands(cuda_dev, rows, K, G, N, seed=77)
    offsets = [int(x) for x in np.cumsum([0] + counts)]
    max_tiles = sum(-(-c // 128) for c in counts)
    offs, tg, ts, nt = _tables(cuda_dev, offsets, max_tiles)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    sched = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    mode = _abi.EP_F32 if ep == "f32" else _abi.EP_SWIGLU_QUANT
    out_s = _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, max_tiles, mode,
                                              dev_err=err)
    out_d = _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, max_tiles, mode,
                                              dev_err=err, sched=sched)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    gu = O.grouped_gemm(npraw(aq), npraw(sa), npraw(bq), npraw(sb), offsets)
    if ep == "f32":
        assert torch.equal(out_s, out_d)
        assert_within_rms(npraw(out_s), gu, what="tail/whole tiles")
        # every row is within the bound on its own: the tails are not hidden
        # behind the whole tiles' magnitude
        g = npraw(out_s)
        for r in range(rows):
            assert_within_rms(g[r], gu[r], what=f"row {r}")
    else:
        (h_s, hs_s), (h_d, hs_d) = out_s, out_d
        assert torch.equal(h_s, h_d) and torch.equal(hs_s, hs_d)
        hq, hs = O.swiglu_quant(gu, N // 2)
        d = e4m3_step_distance(npraw(h_s), hq)
        assert d.max() <= 1 and (d > 0).mean() < 2e-2
        assert np.allclose(npraw(hs_s), hs, rtol=1e-4, atol=0)
