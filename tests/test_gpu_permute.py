"""GPU parity of moe_permute / moe_tile_table: bit-exact against the oracle.

"DeepSeek_V3_Report：Annotation", "Low-Precision Communication" (FP8 rows are
what gets dispatched) and "No Token-Dropping".  Cases: ragged T, empty
experts, a single hot expert, T=1, the V3 and V4-Pro batch shapes.
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import _abi
from oracle import moe_oracle as O
from tests._util import npraw

pytestmark = pytest.mark.gpu


def _idx(T, E, K, rng, hot=None):
    rows = []
    for _ in range(T):
        if hot is not None and rng.random() < 0.7:
            rest = rng.permutation([e for e in range(E) if e != hot])[: K - 1]
            rows.append(np.concatenate([[hot], rest]))
        else:
            rows.append(rng.permutation(E)[:K])
    return np.array(rows, np.int32)


@pytest.mark.parametrize("T,E,K,d,hot", [
    (1, 16, 4, 256, None), (333, 64, 6, 512, None), (300, 40, 3, 256, 7),
    (4096, 256, 8, 7168, None), (16384, 384, 6, 1024, None)])
def test_permute_bit_exact(cuda_dev, T, E, K, d, hot):
    rng = np.random.default_rng(T + E)
    if E == 64:
        idx = _idx(T, E // 2, K, rng) * 2        # odd experts stay empty
    else:
        idx = _idx(T, E, K, rng, hot)
    xq = torch.from_numpy(rng.integers(0, 256, (T, d), dtype=np.uint8)).to(cuda_dev)
    xs = torch.from_numpy(rng.uniform(0.1, 1, (T, d // 128)).astype(np.float32)).to(cuda_dev)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    out = _abi.moe_permute(torch.from_numpy(idx).to(cuda_dev), E, xq, xs, True, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    counts, offsets, src_row, dst_of = O.permute(idx, E)
    assert np.array_equal(npraw(out["counts"]), counts)
    offs = O.segment_offsets_with_shared(offsets, T)
    assert np.array_equal(npraw(out["offsets"]), offs)
    assert np.array_equal(npraw(out["src_row"]), src_row)
    assert np.array_equal(npraw(out["dst_of"]), dst_of)
    grp, start = O.mtile_table(offs)
    n = int(out["n_tiles"].item())
    assert n == len(grp) and n <= out["max_tiles"]
    assert np.array_equal(npraw(out["tile_group"])[:n], grp)
    assert np.array_equal(npraw(out["tile_start"]), start)
    xqn, xsn = npraw(xq), npraw(xs)
    assert np.array_equal(npraw(out["xq_perm"]), xqn[src_row])
    assert np.array_equal(npraw(out["xs_perm"]), xsn[src_row])


def test_permute_flags_bad_index(cuda_dev):
    idx = torch.tensor([[0, 1], [2, 99]], dtype=torch.int32, device=cuda_dev)
    xq = torch.zeros(2, 128, dtype=torch.uint8, device=cuda_dev)
    xs = torch.ones(2, 1, dtype=torch.float32, device=cuda_dev)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    _abi.moe_permute(idx, 4, xq, xs, True, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 3


def test_tile_table_bit_exact(cuda_dev):
    offs = np.array([0, 0, 5, 133, 261, 262, 600, 600, 1000], np.int32)
    grp, start = O.mtile_table(offs)
    tg, ts, nt = _abi.moe_tile_table(torch.from_numpy(offs).to(cuda_dev), 64)
    torch.cuda.synchronize()
    n = int(nt.item())
    assert n == len(grp)
    assert np.array_equal(npraw(tg)[:n], grp) and np.array_equal(npraw(ts), start)


def test_tile_table_flags_decreasing_offsets(cuda_dev):
    offs = torch.tensor([0, 10, 5, 20], dtype=torch.int32, device=cuda_dev)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    _abi.moe_tile_table(offs, 8, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 2


@pytest.mark.parametrize("T,E,K,d,hot,pow2", [
    (1, 16, 4, 256, None, False), (333, 64, 6, 512, None, False), (300, 40, 3, 256, 7, True),
    (4096, 256, 8, 7168, None, False), (16384, 384, 6, 1024, None, True)])
def test_permute_index_and_quant_scatter(cuda_dev, T, E, K, d, hot, pow2):
    """moe_permute_index + fp8_quant_1x128_scatter (the layer's path) give the
    index tables of the oracle's permutation and, row for row, the bytes and
    scales of fp8_quant_1x128 followed by moe_permute's gather."""
    rng = np.random.default_rng(T + E + 1)
    idx = _idx(T, E // 2, K, rng) * 2 if E == 64 else _idx(T, E, K, rng, hot)
    idx_d = torch.from_numpy(idx).to(cuda_dev)
    g = torch.Generator(device=cuda_dev).manual_seed(T)
    u = (torch.randn(T, d, generator=g, device=cuda_dev) *
         torch.where(torch.rand(T, d, generator=g, device=cuda_dev) < 0.01, 50.0, 1.0)).bfloat16()
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    p = _abi.moe_permute_index(idx_d, E, True, dev_err=err)
    P = T * K
    q_all = torch.empty(P + T, d, dtype=torch.uint8, device=cuda_dev)
    s_all = torch.empty(P + T, d // 128, dtype=torch.float32, device=cuda_dev)
    _abi.fp8_quant_1x128_scatter(u, p["dst_of"], q_all[:P], s_all[:P], q_all[P:], s_all[P:],
                                 pow2=pow2)
    q_ref, s_ref = _abi.fp8_quant_1x128(u, pow2=pow2)
    ref = _abi.moe_permute(idx_d, E, q_ref, s_ref, True)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    counts, offsets, src_row, dst_of = O.permute(idx, E)
    assert np.array_equal(npraw(p["counts"]), counts)
    assert np.array_equal(npraw(p["offsets"]), O.segment_offsets_with_shared(offsets, T))
    assert np.array_equal(npraw(p["src_row"]), src_row)
    assert np.array_equal(npraw(p["dst_of"]), dst_of)
    n = int(p["n_tiles"].item())
    assert n == int(ref["n_tiles"].item())
    assert torch.equal(p["tile_group"][:n], ref["tile_group"][:n])
    assert torch.equal(p["tile_start"], ref["tile_start"])
    assert torch.equal(q_all[P:], q_ref) and torch.equal(s_all[P:], s_ref)
    assert torch.equal(q_all[:P], ref["xq_perm"]) and torch.equal(s_all[:P], ref["xs_perm"])
    # the bytes themselves against the oracle's quantiser on a few rows
    rows = sorted({0, T // 2, T - 1})
    qo, so = (O.quant_1x128_pow2 if pow2 else O.quant_1x128)(u[rows].float().cpu().numpy())
    assert np.array_equal(npraw(q_all[P:])[rows], qo) and np.array_equal(npraw(s_all[P:])[rows], so)


def test_quant_scatter_skips_flagged_rows(cuda_dev):
    """A -1 destination (left by a flagged bad expert index) writes nothing."""
    u = torch.randn(2, 128, device=cuda_dev).bfloat16()
    dst = torch.tensor([[1, -1], [0, 2]], dtype=torch.int32, device=cuda_dev)
    q = torch.full((4, 128), 0xAB, dtype=torch.uint8, device=cuda_dev)
    s = torch.full((4, 1), -1.0, dtype=torch.float32, device=cuda_dev)
    _abi.fp8_quant_1x128_scatter(u, dst, q, s)
    q_ref, s_ref = _abi.fp8_quant_1x128(u)
    torch.cuda.synchronize()
    assert torch.equal(q[1], q_ref[0]) and torch.equal(q[0], q_ref[1]) and torch.equal(q[2], q_ref[1])
    assert torch.all(q[3] == 0xAB) and float(s[3, 0]) == -1.0
