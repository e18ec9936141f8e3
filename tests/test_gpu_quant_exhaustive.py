"""Exhaustive check of the bf16 quantisers' division.

fp8_quant_1x128 / fp8_quant_128x128 divide each bf16 value x by the tile
scale s = fl32(max(amax, 1e-4) / 448) ("DeepSeek_V3_Report：Annotation",
"Online Quantization") with one correctly rounded reciprocal per tile and a
per-element FMA correction.  Both x and amax are bf16, so every (x, s) pair
the kernels can meet is enumerable: for each of the 32639 positive finite
bf16 values of amax, every bf16 x with |x| <= amax, both signs (about 1.07e9
pairs).  Each row of the test input is one 1x128 tile holding amax and 127 of
those x.  The scales must equal the fp32 formula bit for bit and the bytes
must equal IEEE fp32 division followed by round-to-nearest-even E4M3
(PyTorch's float8_e4m3fn cast, with the +-448 saturation applied first).
"""
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import _abi

pytestmark = pytest.mark.gpu

N_AMAX = 0x7F80  # bf16 patterns 1 .. 0x7F7F are the positive finite values


def _batch_rows(dev, a0, a1):
    """Rows for amax patterns a0 .. a1-1: column 0 = amax, columns 1..127 =
    the x patterns +-0 .. +-amax (zero-padded at the end of each amax)."""
    A = torch.arange(a0, a1, dtype=torch.int64, device=dev)
    n = 2 * (A + 1)                                    # x patterns per amax
    rows = (n + 126) // 127
    row_a = torch.repeat_interleave(A, rows)
    row_n = torch.repeat_interleave(n, rows)
    first = torch.cumsum(rows, 0) - rows
    row_j = torch.arange(int(rows.sum()), device=dev) - torch.repeat_interleave(first, rows)
    k = row_j[:, None] * 127 + torch.arange(127, device=dev)[None, :]
    pat = torch.where(k % 2 == 0, k // 2, 0x8000 | (k // 2))
    pat = torch.where(k < row_n[:, None], pat, torch.zeros_like(pat))
    allp = torch.cat([row_a[:, None], pat], dim=1)
    signed = torch.where(allp >= 0x8000, allp - 0x10000, allp).to(torch.int16)
    return signed.view(torch.bfloat16)


def test_quant_division_exhaustive(cuda_dev):
    dev = cuda_dev
    eps = torch.tensor(1e-4, dtype=torch.float32, device=dev)
    a0, checked = 1, 0
    while a0 < N_AMAX:
        # about 64M pairs per batch
        a1 = a0
        tot = 0
        while a1 < N_AMAX and tot < (1 << 26):
            tot += 2 * (a1 + 1)
            a1 += 1
        x = _batch_rows(dev, a0, a1)
        q, s = _abi.fp8_quant_1x128(x)
        xf = x.float()
        amax = xf.abs().amax(dim=1)
        # tensor / tensor: elementwise IEEE division (PyTorch divides by a
        # Python scalar through a host-side reciprocal, which is not)
        s_ref = torch.maximum(amax, eps) / torch.full_like(amax, 448.0)
        assert torch.equal(s[:, 0], s_ref), f"scales differ for amax patterns {a0}..{a1}"
        y = (xf / s_ref[:, None]).clamp(-448.0, 448.0)
        q_ref = y.to(torch.float8_e4m3fn).view(torch.uint8)
        bad = (q != q_ref)
        assert not bool(bad.any()), (
            f"{int(bad.sum())} bytes differ for amax patterns {a0}..{a1}; first at "
            f"{bad.nonzero()[0].tolist()}")
        checked += int(x.numel())
        a0 = a1
        del x, q, s, xf, y, q_ref
    assert checked > 1_000_000_000
