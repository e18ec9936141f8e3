"""CPU checks of the C ABI: the library loads, exports every entry point that
include/moefp8.h declares, and rejects bad arguments on the host before any
launch (these calls never reach a GPU)."""
import ctypes
import os
import re

import pytest

from fp8_block_scaled_sigmoid_b200 import _abi

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "moefp8.h")


_BL = []


def _bl(seq_len):
    """Address of a moe_balance_loss with the given seq_len and NULL buffers
    (kept alive for the test session)."""
    b = _abi._BalanceLoss(seq_len, 1e-4, None, None, None, None, None, None)
    _BL.append(b)
    return ctypes.addressof(b)


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:moe_status|int|const char\*)\s+(\w+)\(", src, re.M)))


def test_library_exports_every_declared_symbol():
    L = _abi.lib()
    names = _declared()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_abi.exported_symbols())
    assert L.moe_abi_version() == 4


def test_status_strings():
    L = _abi.lib()
    for s in range(7):
        assert L.moe_status_string(s)
    assert L.moe_status_string(0) == b"ok"


def test_max_m_tiles_bound():
    L = _abi.lib()
    # sum over experts of ceil(c_e/128) <= (T*K + 127*E)/128, plus the shared tiles
    assert L.moe_max_m_tiles(4096, 8, 256, 0) == (4096 * 8 + 127 * 256) // 128
    assert L.moe_max_m_tiles(4096, 8, 256, 1) == (4096 * 8 + 127 * 256) // 128 + 32
    assert L.moe_max_m_tiles(1, 1, 1, 1) == 2


@pytest.mark.parametrize("call,code", [
    (lambda L: L.fp8_quant_1x128(None, 200, 4, 200, None, None, None), 2),   # cols % 128
    (lambda L: L.fp8_quant_1x128(None, 128, -1, 128, None, None, None), 1),  # negative rows
    (lambda L: L.fp8_quant_1x128(None, 128, 4, 128, None, None, None), 1),   # NULL buffers
    (lambda L: L.fp8_quant_1x128(16, 128, 4, 128, 8, 4, None), 3),          # misaligned
    (lambda L: L.fp8_quant_128x128(None, 64, 4, 128, None, None, None), 2),  # ld < cols
    (lambda L: L.moe_route(None, 256, None, None, 8, 256, 20, 4, 2, 4, None, None, None,
                           None, None, 0, None, None), 2),                    # E % 16
    (lambda L: L.moe_route(None, 256, None, None, 8, 256, 64, 8, 3, 8, None, None, None,
                           None, None, 0, None, None), 2),                    # K % M
    (lambda L: L.moe_route(None, 256, None, None, 8, 256, 2048, 8, 4, 8, None, None, None,
                           None, None, 0, None, None), 4),                    # E > 1024
    (lambda L: L.moe_route(None, 256, None, None, 96, 256, 16, 4, 2, 4, None, None, None,
                           _bl(30), None, 0, None, None), 2),                # T % seq_len
    (lambda L: L.moe_route(None, 256, None, None, 100, 256, 16, 4, 2, 4, None, None, None,
                           _bl(50), None, 0, None, None), 2),                # seq_len % 8
    (lambda L: L.moe_route(None, 256, None, None, 96, 256, 16, 4, 2, 4, None, None, None,
                           _bl(0), None, 0, None, None), 1),                 # seq_len 0
    (lambda L: L.grouped_gemm_fp8_blockscaled(None, None, 10, None, None, None, None, None,
                                              None, 4, 1, 384, 128, 0, None, None, None,
                                              None, None, None), 2),          # N % 256
    (lambda L: L.grouped_gemm_fp8_blockscaled(None, None, 10, None, None, None, None, None,
                                              None, 4, 1, 256, 128, 7, None, None, None,
                                              None, None, None), 1),          # bad epilogue
    (lambda L: L.grouped_gemm_fp8_blockscaled(None, None, 10, None, None, None, None, None,
                                              None, 4, 1, 256, 128, 1, None, None, 16, None,
                                              None, None), 1),                # row map with SwiGLU
    (lambda L: L.swiglu_quant(None, 4, 100, None, None, None), 2),
    (lambda L: L.moe_seq_balance_loss(None, 100, 16, 4, 30, ctypes.c_float(1e-4), None, None,
                                      None, None, 0, None), 2),              # T % seq_len
    (lambda L: L.moe_seq_balance_loss(None, 100, 16, 40, 50, ctypes.c_float(1e-4), None, None,
                                      None, None, 0, None), 2),              # K > 32
    (lambda L: L.moe_seq_balance_loss(None, 100, 2048, 4, 50, ctypes.c_float(1e-4), None, None,
                                      None, None, 0, None), 4),              # E > 1024
    (lambda L: L.moe_seq_balance_loss(None, 100, 16, 4, 50, ctypes.c_float(1e-4), None, None,
                                      None, None, 0, None), 1),              # NULL logits
    (lambda L: L.moe_combine(None, None, None, None, None, 4, 40, 128, None, None), 4),
    (lambda L: L.moe_bias_update(None, 4, 8, 2, ctypes.c_float(0.001), None, None), 1),
    # power-of-two variant
    (lambda L: L.fp8_quant_1x128_pow2(None, 200, 4, 200, None, None, None), 2),
    (lambda L: L.fp8_quant_128x128_pow2(None, 64, 4, 128, None, None, None), 2),
    (lambda L: L.grouped_gemm_fp8_pow2(None, None, 10, None, None, None, None, None, None, 4, 1,
                                       384, 128, 0, None, None, None, None, None, None), 2),
    (lambda L: L.swiglu_quant_pow2(None, 4, 100, None, None, None), 2),
    # backward
    (lambda L: L.fp8_quant_1x128_f32(None, 200, 4, 200, 0, None, None, None), 2),
    (lambda L: L.fp8_quant_1x128_f32(None, 128, 4, 128, 1, None, None, None), 1),
    (lambda L: L.moe_combine_backward(None, None, None, 4, 4, 200, None, None, None, None), 2),
    (lambda L: L.moe_combine_backward(None, None, None, 4, 40, 128, None, None, None, None), 4),
    (lambda L: L.swiglu_backward(None, None, None, 4, 100, None, None, None, None, None), 2),
    (lambda L: L.fp8_quant_128x1_pow2(None, 128, None, None, None, None, 4, 128, None, 512, None,
                                      None, None), 1),                        # NULL source
    (lambda L: L.fp8_quant_128x1_pow2(16, 128, None, None, None, None, 4, 100, None, 512, None,
                                      None, None), 2),                        # C % 128
    (lambda L: L.fp8_quant_128x1_pow2(16, 256, None, None, None, None, 4, 256, None, 256, None,
                                      None, None), 2),                        # ldt < 128 * tiles
    (lambda L: L.fp8_quant_128x1_pow2(16, 256, None, None, None, None, 2, 256, None, 384, None,
                                      32, None), 2),                          # atoms need ldt % 512
    (lambda L: L.fp8_requant_128x1_pow2(None, None, 128, None, None, None, None, 4, 128, None, 512,
                                        None, None, None), 1),
    (lambda L: L.fp8_transpose_128x128(None, None, 2, 100, 128, None, None, None), 2),
    (lambda L: L.moe_unpermute_add(None, None, None, 4, 40, 128, None, None), 4),
    (lambda L: L.grouped_gemm_fp8_wgrad(None, None, None, None, 512, 100, 256, None, 2, None,
                                        None, None), 2),                      # Ma % 128
    (lambda L: L.grouped_gemm_fp8_wgrad(None, None, None, None, 500, 128, 256, None, 2, None,
                                        None, None), 2),                      # ldt % 512
    (lambda L: L.grouped_gemm_fp8_wgrad(None, None, None, None, 512, 128, 256, None, 2, None,
                                        None, None), 1),                      # NULL buffers
    # expert parallelism
    (lambda L: L.moe_segment_ids(None, 12, 8, 0, 100, None, None, None), 2),    # segments % E
    (lambda L: L.moe_segment_ids(None, 2048, 8, 0, 100, None, None, None), 4),  # > 1024 segments
    (lambda L: L.moe_segment_ids(None, 16, 8, 0, 100, None, None, None), 1),    # NULL buffers
    (lambda L: L.moe_segment_ids(None, 16, 0, 0, 100, None, None, None), 1),    # E = 0
    (lambda L: L.moe_segment_ids(None, 16, 8, 101, 100, None, None, None), 1),  # lead > rows
    # FP8 peak measurement loop
    (lambda L: L.moe_fp8_mma_peak(0, 0, 4, 16, None, None), 1),              # iters < 1
    (lambda L: L.moe_fp8_mma_peak(1, 100, 4, None, None, None), 1),          # NULL sink
    (lambda L: L.moe_fp8_mma_peak(0, (1 << 21) + 1, 4, 16, None, None), 4),  # beyond the wait
])
def test_host_validation(call, code):
    assert call(_abi.lib()) == code


def test_empty_batches_are_no_ops():
    L = _abi.lib()
    assert L.fp8_quant_1x128(None, 128, 0, 128, None, None, None) == 0
    assert L.moe_combine(None, None, None, None, None, 0, 8, 128, None, None) == 0
    assert L.swiglu_quant(None, 0, 128, None, None, None) == 0
    assert L.moe_combine_backward(None, None, None, 0, 4, 128, None, None, None, None) == 0
    assert L.swiglu_backward(None, None, None, 0, 128, None, None, None, None, None) == 0
    assert L.fp8_quant_128x1_pow2(16, 128, None, None, None, None, 0, 128, None, 0, None, None,
                                  None) == 0
    assert L.grouped_gemm_fp8_wgrad(None, None, None, None, 512, 128, 256, None, 0, None, None,
                                    None) == 0
    assert L.moe_segment_ids(None, 16, 8, 0, 0, None, None, None) == 0
