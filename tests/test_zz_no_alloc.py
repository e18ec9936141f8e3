"""moe_permute_noalloc: the permutation for callers that cannot allocate.

Some callers cannot allocate device memory when they call the library (a
plugin inside an inference runtime that owns all device memory and offers no
workspace; a latency-critical path that must avoid cudaMalloc's implicit
synchronisation).  For them moe_permute_noalloc uses a fixed 1 MiB device
array inside the library instead of a caller workspace.  This test calls it
through the C ABI twice in a row (a large batch, then a smaller one that
leaves the first call's contents behind in the shared array) and checks every
output against the regular moe_permute on the same inputs: the work is
integer, so the match must be exact.  It also checks that a batch needing more
than 1 MiB of scratch is refused on the host.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from fp8_block_scaled_sigmoid_b200 import _abi

pytestmark = pytest.mark.gpu

NAMES = ["counts", "offsets", "src_row", "dst_of", "xq_perm", "xs_perm", "tile_start", "n_tiles"]


def _inputs(dev, T, E, K, d, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    xq = torch.from_numpy(rng.integers(0, 256, (T, d), dtype=np.uint8)).to(dev)
    xs = torch.from_numpy(rng.uniform(0.1, 1, (T, d // 128)).astype(np.float32)).to(dev)
    return torch.from_numpy(idx).to(dev), xq, xs


def _call_noalloc(dev, idx, E, xq, xs):
    """Raw C-ABI call with caller-allocated outputs."""
    T, K = idx.shape
    d = xq.shape[1]
    mt = _abi.moe_max_m_tiles(T, K, E, True)
    o = {
        "counts": torch.empty(E, dtype=torch.int32, device=dev),
        "offsets": torch.empty(E + 2, dtype=torch.int32, device=dev),
        "src_row": torch.empty(T * K, dtype=torch.int32, device=dev),
        "dst_of": torch.empty(T, K, dtype=torch.int32, device=dev),
        "xq_perm": torch.empty(T * K, d, dtype=torch.uint8, device=dev),
        "xs_perm": torch.empty(T * K, d // 128, dtype=torch.float32, device=dev),
        "tile_group": torch.empty(mt, dtype=torch.int32, device=dev),
        "tile_start": torch.empty(E + 2, dtype=torch.int32, device=dev),
        "n_tiles": torch.empty(1, dtype=torch.int32, device=dev),
    }
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = _abi.lib().moe_permute_noalloc(
        p(idx), T, K, E, 1, p(xq), p(xs), d, p(o["counts"]), p(o["offsets"]), p(o["src_row"]),
        p(o["dst_of"]), p(o["xq_perm"]), p(o["xs_perm"]), p(o["tile_group"]),
        p(o["tile_start"]), p(o["n_tiles"]), p(err),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, _abi.lib().moe_status_string(st)
    return o, err


@pytest.mark.parametrize("first,second", [((4096, 256, 8, 1024), (333, 64, 6, 512))])
def test_noalloc_matches_permute_twice(cuda_dev, first, second):
    for seed, (T, E, K, d) in enumerate([first, second]):
        idx, xq, xs = _inputs(cuda_dev, T, E, K, d, seed)
        got, err = _call_noalloc(cuda_dev, idx, E, xq, xs)
        ref = _abi.moe_permute(idx, E, xq, xs, True)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        for n in NAMES:
            assert torch.equal(got[n], ref[n]), n
        n_t = int(ref["n_tiles"].item())
        assert torch.equal(got["tile_group"][:n_t], ref["tile_group"][:n_t])


def test_noalloc_refuses_oversized_batch(cuda_dev):
    # ceil(131072/128) chunks x 512 experts = 524288 int32 > the 262144 available
    st = _abi.lib().moe_permute_noalloc(None, 131072, 8, 512, 1, None, None, 1024, None, None,
                                        None, None, None, None, None, None, None, None, None)
    assert st == 4  # MOE_ERR_UNSUPPORTED, refused before any launch
