"""B200-native (sm_100a) forward pass of one DeepSeekMoE layer with FP8
block-scaled expert GEMMs.

The compute lives in libmoefp8.so (C ABI, include/moefp8.h); this package is
its ctypes binding (`_abi`), the layer's call sequence (`layer`), named
shapes (`configs`) and the seeded synthetic inputs (`inputs`).  The library
is loaded on first use and its absence is an error: there is no CPU path.
"""
from . import configs, inputs  # noqa: F401
from ._abi import (EP_F32, EP_SWIGLU_QUANT, MoEError, fp8_quant_128x128,  # noqa: F401
                   fp8_quant_1x128, grouped_gemm_fp8_blockscaled, moe_bias_update,
                   moe_combine, moe_max_m_tiles, moe_permute, moe_route, moe_tile_table,
                   swiglu_quant)
from .layer import MoELayer, make_fp8_weights  # noqa: F401
