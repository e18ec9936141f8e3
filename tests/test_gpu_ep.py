"""Expert parallelism on one GPU: the receive-side labelling kernel and the
whole expert-parallel forward with a single rank.

"DeepSeek_V3_Report：Annotation", "Low-Precision Communication" (FP8 rows
dispatched to the experts' ranks, outputs returned for the combine).  With one
rank both exchanges are copies, and the forward must equal the single-GPU
layer bit for bit: every row meets the same operands in the same order.
Ranks that wait on one another are not run as processes on one GPU; the
exchange between ranks is tested on CPU ranks (tests/test_dist_gloo.py).
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import MoELayer, _abi, configs, ep, inputs, make_fp8_weights
from tests._util import npraw

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S,E", [(1, 16), (4, 8), (8, 32)])
def test_segment_ids(cuda_dev, S, E):
    rng = np.random.default_rng(S * 100 + E)
    counts = rng.integers(0, 300, (S, E)).astype(np.int32)
    counts[0, 1] = 0
    n = int(counts.sum())
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    ids = _abi.moe_segment_ids(torch.from_numpy(counts).to(cuda_dev), E, n, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = np.repeat(np.tile(np.arange(E, dtype=np.int32), S), counts.reshape(-1))
    assert np.array_equal(npraw(ids), want)


def test_segment_ids_inconsistent_counts(cuda_dev):
    counts = torch.tensor([[3, 4]], dtype=torch.int32, device=cuda_dev)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    ids = _abi.moe_segment_ids(counts, 2, 9, dev_err=err)   # the counts sum to 7, not 9
    torch.cuda.synchronize()
    assert int(err.item()) == 2                               # MOE_DEVERR_BAD_TABLE
    assert npraw(ids)[:7].tolist() == [0, 0, 0, 1, 1, 1, 1]


@pytest.mark.parametrize("cfg", [
    configs.TINY,
    configs.TINY.with_(name="small", T=333, d=512, E=32, G=4, M=2, K=6, I=256),
])
def test_ep_single_rank_matches_layer(cuda_dev, cfg):
    w = make_fp8_weights(cfg, cuda_dev)
    cent = inputs.draw_centroids(cfg, cuda_dev)
    bias = inputs.draw_bias(cfg, cuda_dev)
    u = inputs.draw_u(cfg, cuda_dev)
    ref = MoELayer(cfg, cent, bias.clone(), *w)
    out_ref = ref.forward(u).clone()
    layer = ep.MoELayerEP(cfg, cent, bias.clone(), *w, ep.ExpertShard(cfg.E, 1, 0))
    out = layer.forward(u)
    torch.cuda.synchronize()
    ref.check()
    layer.check()
    assert torch.equal(out, out_ref)
    assert torch.equal(layer.bias, ref.bias)
