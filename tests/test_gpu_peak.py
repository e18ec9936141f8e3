"""The FP8 MMA loop that measures the tensor-core peak (moe_fp8_mma_peak).

It is the denominator of the expert GEMMs' roofline, so it must really run
its MMAs: the accumulator it leaves behind grows linearly with the number of
K blocks ("DeepSeek_V3_Report：Annotation", "Fine-Grained Quantization":
E4M3 operands, fp32 accumulation), and the block-scaled instruction with unit
scales gives the same products as the plain one.
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import _abi

pytestmark = pytest.mark.gpu


def _run(dev, block_scaled, iters, ctas=4):
    sink = torch.full((ctas,), float("nan"), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flops = _abi.moe_fp8_mma_peak(block_scaled, iters, ctas, sink, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert flops == ctas * iters * 4 * 2 * 128 * 256 * 32
    return sink.cpu().numpy().astype(np.float64)


def test_peak_loop_accumulates(cuda_dev):
    # block-scaled: one accumulator, D = iters * P
    s1 = _run(cuda_dev, True, 1)
    s4 = _run(cuda_dev, True, 4)
    assert np.all(np.isfinite(s1)) and np.any(s1 != 0)
    assert np.allclose(s4, 4 * s1, rtol=1e-5, atol=1e-6)
    # plain kind::f8f6f4: two alternating accumulators, D0 = ceil(iters/2) * P
    p2 = _run(cuda_dev, False, 2)
    p8 = _run(cuda_dev, False, 8)
    assert np.allclose(p2, s1, rtol=1e-5, atol=1e-6)
    assert np.allclose(p8, 4 * s1, rtol=1e-5, atol=1e-6)


def test_peak_rate_is_measurable(cuda_dev):
    sms = torch.cuda.get_device_properties(cuda_dev).multi_processor_count
    sink = torch.empty(sms, dtype=torch.float32, device=cuda_dev)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    for bs in (False, True):
        _abi.moe_fp8_mma_peak(bs, 256, sms, sink, err)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        flops = _abi.moe_fp8_mma_peak(bs, 2048, sms, sink, err)
        b.record()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        tflops = flops / (a.elapsed_time(b) / 1e3) / 1e12
        # a loose sanity window around the part's nominal 4.5 PFLOP/s dense
        assert 500 < tflops < 10000, tflops
