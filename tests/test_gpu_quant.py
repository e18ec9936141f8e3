"""GPU parity of the FP8 quantisers against the oracle: bit-exact bytes and scales.

"DeepSeek_V3_Report：Annotation", "Fine-Grained Quantization" / "Online
Quantization".  The shapes span several tiles and blocks, a ragged last
row-block, an ld larger than cols, outliers (the standalone-GEMM recipe: 1%
of elements x50), all-zero tiles, a single row, and the full 4096 x 7168
activation and one V3 expert's 4096 x 7168 weight.
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import _abi, inputs
from oracle import moe_oracle as O
from tests._util import np32, npraw

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols,ld,outl", [
    (1, 128, 128, 0.0), (3, 384, 512, 0.0), (300, 1024, 1024, 0.01), (4096, 7168, 7168, 0.01)])
def test_quant_1x128_bit_exact(cuda_dev, rows, cols, ld, outl):
    x = inputs.draw_matrix(rows, ld, seed=rows, tid=1, outlier_frac=outl, outlier_mult=50.0)
    if rows >= 3:
        x[2, :128] = 0                         # an all-zero tile
    xd = x.to(cuda_dev)
    q, s = _abi.fp8_quant_1x128(xd[:, :cols])
    torch.cuda.synchronize()
    qo, so = O.quant_1x128(np32(x[:, :cols]))
    assert np.array_equal(npraw(s), so), "scales differ"
    qg = npraw(q)
    bad = np.argwhere(qg != qo)
    assert bad.size == 0, f"{len(bad)} FP8 bytes differ, first {bad[:5]}"


@pytest.mark.parametrize("rows,cols", [(128, 128), (200, 384), (4096, 7168)])
def test_quant_128x128_bit_exact(cuda_dev, rows, cols):
    w = inputs.draw_matrix(rows, cols, seed=7, tid=2, std=1.0 / np.sqrt(cols))
    w[5, min(130, cols - 1)] = 0.75            # a block outlier
    q, s = _abi.fp8_quant_128x128(w.to(cuda_dev))
    torch.cuda.synchronize()
    qo, so = O.quant_128x128(np32(w))
    assert np.array_equal(npraw(s), so)
    assert np.array_equal(npraw(q), qo)


def test_quant_128x128_stack_layout(cuda_dev):
    w = torch.stack([inputs.draw_matrix(256, 256, seed=e, tid=3) for e in range(3)])
    q, s = _abi.fp8_quant_128x128(w.to(cuda_dev))
    torch.cuda.synchronize()
    assert q.shape == (3, 256, 256) and s.shape == (3, 2, 2)
    for e in range(3):
        qo, so = O.quant_128x128(np32(w[e]))
        assert np.array_equal(npraw(q[e]), qo) and np.array_equal(npraw(s[e]), so)


def test_quant_rejects_bad_shapes(cuda_dev):
    x = torch.zeros(4, 200, dtype=torch.bfloat16, device=cuda_dev)
    with pytest.raises(_abi.MoEError):
        _abi.fp8_quant_1x128(x)
