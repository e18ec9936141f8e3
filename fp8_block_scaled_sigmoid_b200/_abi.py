"""ctypes binding of libmoefp8.so: argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors that already live on the GPU, passes their raw pointers and sizes,
and raises MoEError on a non-zero status.  Output tensors are allocated with
torch when the caller does not pass them (device memory is torch's job; all
arithmetic happens in the library's kernels).  There is no fallback: if the
library is missing or a CUDA device is absent the call fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoefp8.so")

_c = ctypes
_p = _c.c_void_p
_i = _c.c_int
_i64 = _c.c_int64
_sz = _c.c_size_t
_f = _c.c_float

_SIGS = {
    "moe_status_string": (_c.c_char_p, [_i]),
    "moe_abi_version": (_i, []),
    "fp8_quant_1x128": (_i, [_p, _i64, _i, _i, _p, _p, _p]),
    "fp8_quant_128x128": (_i, [_p, _i64, _i, _i, _p, _p, _p]),
    "fp8_quant_1x128_pow2": (_i, [_p, _i64, _i, _i, _p, _p, _p]),
    "fp8_quant_128x128_pow2": (_i, [_p, _i64, _i, _i, _p, _p, _p]),
    "moe_route_workspace_size": (_i, [_i, _i, _i, _c.POINTER(_sz)]),
    "moe_route": (_i, [_p, _i64, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _sz, _p,
                       _p]),
    "moe_max_m_tiles": (_i, [_i, _i, _i, _i]),
    "moe_permute_workspace_size": (_i, [_i, _i, _i, _c.POINTER(_sz)]),
    "moe_permute": (_i, [_p, _i, _i, _i, _i, _p, _p, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                         _p, _sz, _p, _p]),
    "moe_permute_noalloc": (_i, [_p, _i, _i, _i, _i, _p, _p, _i, _p, _p, _p, _p, _p, _p, _p,
                                 _p, _p, _p, _p]),
    "moe_tile_table": (_i, [_p, _i, _i, _p, _p, _p, _p, _p]),
    "moe_permute_index": (_i, [_p, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p, _p]),
    "fp8_quant_1x128_scatter": (_i, [_p, _i64, _i, _i, _p, _i, _i, _p, _p, _p, _p, _p]),
    "moe_segment_ids": (_i, [_p, _i, _i, _i64, _i64, _p, _p, _p]),
    "grouped_gemm_fp8_blockscaled": (_i, [_p, _p, _i64, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i,
                                          _i, _p, _p, _p, _p, _p, _p]),
    "grouped_gemm_fp8_pow2": (_i, [_p, _p, _i64, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i,
                                   _i, _p, _p, _p, _p, _p, _p]),
    "swiglu_quant": (_i, [_p, _i, _i, _p, _p, _p]),
    "swiglu_quant_pow2": (_i, [_p, _i, _i, _p, _p, _p]),
    "fp8_quant_1x128_f32": (_i, [_p, _i64, _i, _i, _i, _p, _p, _p]),
    "moe_combine_backward": (_i, [_p, _p, _p, _i, _i, _i, _p, _p, _p, _p]),
    "swiglu_backward": (_i, [_p, _p, _p, _i, _i, _p, _p, _p, _p, _p]),
    "fp8_quant_128x1_pow2": (_i, [_p, _i64, _p, _p, _p, _p, _i, _i, _p, _i64, _p, _p, _p]),
    "fp8_requant_128x1_pow2": (_i, [_p, _p, _i64, _p, _p, _p, _p, _i, _i, _p, _i64, _p, _p, _p]),
    "fp8_transpose_128x128": (_i, [_p, _p, _i, _i, _i, _p, _p, _p]),
    "moe_unpermute_add": (_i, [_p, _p, _p, _i, _i, _i, _p, _p]),
    "grouped_gemm_fp8_wgrad": (_i, [_p, _p, _p, _p, _i64, _i, _i, _p, _i, _p, _p, _p]),
    "moe_combine": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _p, _p]),
    "moe_bias_update": (_i, [_p, _i, _i64, _i, _f, _p, _p]),
    "moe_seq_balance_loss_workspace_size": (_i, [_i, _i, _i, _c.POINTER(_sz)]),
    "moe_seq_balance_loss": (_i, [_p, _i, _i, _i, _i, _f, _p, _p, _p, _p, _sz, _p]),
    "moe_fp8_mma_peak": (_i, [_i, _i, _i, _p, _p, _p]),
}

EP_F32 = 0
EP_SWIGLU_QUANT = 1


class _BalanceLoss(ctypes.Structure):
    """moe_balance_loss (include/moefp8.h)."""
    _fields_ = [("seq_len", _i), ("alpha", _f), ("acc", _p), ("cnt", _p), ("done", _p),
                ("loss", _p), ("f", _p), ("P", _p)]


class BalanceLossState:
    """Device buffers of the balance loss that moe_route computes in its
    selection pass, for T tokens in sequences of seq_len: the zeroed sums and
    counters (each call leaves them zero) and the outputs loss [T/seq_len],
    f and P [T/seq_len][E] (with_fp)."""

    def __init__(self, T, E, seq_len, alpha=1e-4, with_fp=False, device=None):
        n_seq = T // seq_len if seq_len > 0 else 0
        n = max(n_seq, 1)
        self.T, self.E, self.seq_len, self.alpha, self.n_seq = T, E, seq_len, alpha, n_seq
        self.acc = torch.zeros(n, E, dtype=torch.int64, device=device)
        self.cnt = torch.zeros(n, E, dtype=torch.int32, device=device)
        self.done = torch.zeros(n, dtype=torch.int32, device=device)
        self.loss = torch.zeros(n, dtype=torch.float32, device=device)
        self.f = torch.zeros(n, E, dtype=torch.float32, device=device) if with_fp else None
        self.P = torch.zeros(n, E, dtype=torch.float32, device=device) if with_fp else None
        self.c = _BalanceLoss(int(seq_len), float(alpha), _ptr(self.acc), _ptr(self.cnt),
                              _ptr(self.done), _ptr(self.loss), _ptr(self.f), _ptr(self.P))
DEVERR = {0: "none", 1: "bounded wait timed out", 2: "inconsistent segment table",
          3: "expert index out of range", 4: "a scale is not a power of two"}

_lib = None

# Kernels each entry point launches (for the benchmark's launch count).
LAUNCHES_PER_CALL = {"fp8_quant_1x128": 1, "fp8_quant_128x128": 1, "swiglu_quant": 1,
                     "swiglu_quant_pow2": 1,
                     "fp8_quant_1x128_pow2": 1, "fp8_quant_128x128_pow2": 1,
                     "grouped_gemm_fp8_pow2": 1, "fp8_quant_1x128_f32": 1,
                     "moe_combine_backward": 1, "swiglu_backward": 1, "fp8_quant_128x1_pow2": 1,
                     "fp8_requant_128x1_pow2": 1, "fp8_transpose_128x128": 1,
                     "moe_unpermute_add": 1, "grouped_gemm_fp8_wgrad": 1,
                     "moe_route": 2, "moe_permute": 3, "moe_permute_noalloc": 3,
                     "moe_permute_index": 2, "fp8_quant_1x128_scatter": 1,
                     "moe_tile_table": 1, "moe_segment_ids": 1,
                     "grouped_gemm_fp8_blockscaled": 1, "moe_combine": 1, "moe_bias_update": 1,
                     "moe_seq_balance_loss": 3, "moe_fp8_mma_peak": 1}
launch_count = 0


def _count(name: str) -> None:
    global launch_count
    launch_count += LAUNCHES_PER_CALL[name]


class MoEError(RuntimeError):
    pass


def lib() -> ctypes.CDLL:
    """Load libmoefp8.so (built in-tree by ``python -m fp8_block_scaled_sigmoid_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise MoEError(f"{LIB_PATH} is missing: build it with "
                           "`python -m fp8_block_scaled_sigmoid_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGS)


def _check(status: int, what: str) -> None:
    if status != 0:
        msg = lib().moe_status_string(status).decode()
        raise MoEError(f"{what}: status {status} ({msg})")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise MoEError("expected a CUDA tensor")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dev(t):
    return t.device


# ----------------------------------------------------------------- quant ---
def fp8_quant_1x128(x, q=None, scale=None, stream=None, pow2=False):
    """x bf16 [rows][cols] (row stride may exceed cols) -> (q uint8, scale fp32);
    pow2 rounds every scale up to a power of two."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    q = torch.empty(rows, cols, dtype=torch.uint8, device=_dev(x)) if q is None else q
    scale = torch.empty(rows, cols // 128, dtype=torch.float32, device=_dev(x)) if scale is None else scale
    name = "fp8_quant_1x128_pow2" if pow2 else "fp8_quant_1x128"
    _count(name)
    _check(getattr(lib(), name)(_ptr(x), x.stride(0), rows, cols, _ptr(q), _ptr(scale),
                                _stream(stream)), name)
    return q, scale


def fp8_quant_128x128(w, q=None, scale=None, stream=None, pow2=False):
    """w bf16 [rows][cols] or a stack [G][N][K] (N % 128 == 0) -> (q, scale)
    with scale [ceil(rows/128)][cols/128] (stack: [G][N/128][K/128]); pow2
    rounds every scale up to a power of two."""
    assert w.dtype == torch.bfloat16 and w.stride(-1) == 1
    shape = w.shape
    w2 = w.reshape(-1, shape[-1])
    rows, cols = w2.shape
    if w.dim() == 3:
        assert shape[1] % 128 == 0
        sshape = (shape[0], shape[1] // 128, cols // 128)
    else:
        sshape = ((rows + 127) // 128, cols // 128)
    q = torch.empty(shape, dtype=torch.uint8, device=_dev(w)) if q is None else q
    scale = torch.empty(sshape, dtype=torch.float32, device=_dev(w)) if scale is None else scale
    name = "fp8_quant_128x128_pow2" if pow2 else "fp8_quant_128x128"
    _count(name)
    _check(getattr(lib(), name)(_ptr(w2), w2.stride(0), rows, cols, _ptr(q), _ptr(scale),
                                _stream(stream)), name)
    return q, scale


def swiglu_quant(gu, I, h=None, h_scale=None, stream=None, pow2=False):
    rows = gu.shape[0]
    h = torch.empty(rows, I, dtype=torch.uint8, device=_dev(gu)) if h is None else h
    h_scale = torch.empty(rows, I // 128, dtype=torch.float32, device=_dev(gu)) if h_scale is None else h_scale
    name = "swiglu_quant_pow2" if pow2 else "swiglu_quant"
    _count(name)
    _check(getattr(lib(), name)(_ptr(gu), rows, I, _ptr(h), _ptr(h_scale), _stream(stream)), name)
    return h, h_scale


# ----------------------------------------------------------------- route ---
def moe_route_workspace_size(T, d, E) -> int:
    n = _sz(0)
    _check(lib().moe_route_workspace_size(T, d, E, ctypes.byref(n)), "moe_route_workspace_size")
    return n.value


def moe_route(u, centroids, bias, G, M, K, topk_idx=None, topk_gate=None, logits_out=None,
              ws=None, dev_err=None, stream=None, aux=None):
    """aux: a BalanceLossState for the same T, or None."""
    T, d = u.shape
    E = centroids.shape[0]
    dev = _dev(u)
    topk_idx = torch.empty(T, K, dtype=torch.int32, device=dev) if topk_idx is None else topk_idx
    topk_gate = torch.empty(T, K, dtype=torch.float32, device=dev) if topk_gate is None else topk_gate
    need = moe_route_workspace_size(T, d, E)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _count("moe_route")
    _check(lib().moe_route(_ptr(u), u.stride(0), _ptr(centroids), _ptr(bias), T, d, E, G, M, K,
                           _ptr(topk_idx), _ptr(topk_gate), _ptr(logits_out),
                           ctypes.addressof(aux.c) if aux is not None else None,
                           _ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_err),
                           _stream(stream)),
           "moe_route")
    return topk_idx, topk_gate


# --------------------------------------------------------------- permute ---
def moe_max_m_tiles(T, K, E, with_shared) -> int:
    return lib().moe_max_m_tiles(T, K, E, int(bool(with_shared)))


def moe_permute_workspace_size(T, K, E) -> int:
    n = _sz(0)
    _check(lib().moe_permute_workspace_size(T, K, E, ctypes.byref(n)), "moe_permute_workspace_size")
    return n.value


def moe_permute(topk_idx, E, xq, xscale, with_shared=True, out=None, ws=None, dev_err=None,
                stream=None):
    """Returns a dict of the outputs (allocated here unless ``out`` holds them).
    xq_perm needs T*K rows at least; for the layer the caller passes a buffer
    of T*K+T rows whose tail already holds xq."""
    T, K = topk_idx.shape
    d = xq.shape[1]
    dev = _dev(topk_idx)
    groups = E + (1 if with_shared else 0)
    o = {} if out is None else out
    mt = moe_max_m_tiles(T, K, E, with_shared)

    def get(name, shape, dtype):
        if name not in o:
            o[name] = torch.empty(shape, dtype=dtype, device=dev)
        return o[name]

    counts = get("counts", (E,), torch.int32)
    offsets = get("offsets", (groups + 1,), torch.int32)
    src_row = get("src_row", (T * K,), torch.int32)
    dst_of = get("dst_of", (T, K), torch.int32)
    xq_perm = get("xq_perm", (T * K, d), torch.uint8)
    xs_perm = get("xs_perm", (T * K, d // 128), torch.float32)
    tile_group = get("tile_group", (max(mt, 1),), torch.int32)
    tile_start = get("tile_start", (groups + 1,), torch.int32)
    n_tiles = get("n_tiles", (1,), torch.int32)
    need = moe_permute_workspace_size(T, K, E)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _count("moe_permute")
    _check(lib().moe_permute(_ptr(topk_idx), T, K, E, int(bool(with_shared)), _ptr(xq),
                             _ptr(xscale), d, _ptr(counts), _ptr(offsets), _ptr(src_row),
                             _ptr(dst_of), _ptr(xq_perm), _ptr(xs_perm), _ptr(tile_group),
                             _ptr(tile_start), _ptr(n_tiles), _ptr(ws),
                             ws.numel() * ws.element_size(), _ptr(dev_err), _stream(stream)),
           "moe_permute")
    o["max_tiles"] = mt
    return o


def moe_permute_index(topk_idx, E, with_shared=True, out=None, ws=None, dev_err=None,
                      stream=None):
    """moe_permute without the row gather: counts, offsets, src_row, dst_of
    and the tile table in a dict (allocated here unless ``out`` holds them)."""
    T, K = topk_idx.shape
    dev = _dev(topk_idx)
    groups = E + (1 if with_shared else 0)
    o = {} if out is None else out
    mt = moe_max_m_tiles(T, K, E, with_shared)

    def get(name, shape, dtype):
        if name not in o:
            o[name] = torch.empty(shape, dtype=dtype, device=dev)
        return o[name]

    counts = get("counts", (E,), torch.int32)
    offsets = get("offsets", (groups + 1,), torch.int32)
    src_row = get("src_row", (T * K,), torch.int32)
    dst_of = get("dst_of", (T, K), torch.int32)
    tile_group = get("tile_group", (max(mt, 1),), torch.int32)
    tile_start = get("tile_start", (groups + 1,), torch.int32)
    n_tiles = get("n_tiles", (1,), torch.int32)
    need = moe_permute_workspace_size(T, K, E)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _count("moe_permute_index")
    _check(lib().moe_permute_index(_ptr(topk_idx), T, K, E, int(bool(with_shared)),
                                   _ptr(counts), _ptr(offsets), _ptr(src_row), _ptr(dst_of),
                                   _ptr(tile_group), _ptr(tile_start), _ptr(n_tiles), _ptr(ws),
                                   ws.numel() * ws.element_size(), _ptr(dev_err),
                                   _stream(stream)), "moe_permute_index")
    o["max_tiles"] = mt
    return o


def fp8_quant_1x128_scatter(x, dst_of, q_perm, s_perm, q_tok=None, s_tok=None, pow2=False,
                            stream=None):
    """x bf16 [rows][cols] -> its 1x128 FP8 tiles at every dst_of[t][k] row of
    q_perm / s_perm, and (when given) in token order in q_tok / s_tok."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    K = dst_of.shape[1]
    _count("fp8_quant_1x128_scatter")
    _check(lib().fp8_quant_1x128_scatter(_ptr(x), x.stride(0), rows, cols, _ptr(dst_of), K,
                                         int(bool(pow2)), _ptr(q_tok), _ptr(s_tok), _ptr(q_perm),
                                         _ptr(s_perm), _stream(stream)), "fp8_quant_1x128_scatter")
    return q_perm, s_perm


def moe_permute_noalloc(topk_idx, E, xq, xscale, with_shared=True, out=None, dev_err=None,
                        stream=None):
    """moe_permute without a workspace argument: the library's fixed 1 MiB
    device scratch array is used instead (for callers that cannot allocate;
    calls must not overlap on the GPU).  Returns the same dict as moe_permute."""
    T, K = topk_idx.shape
    d = xq.shape[1]
    dev = _dev(topk_idx)
    groups = E + (1 if with_shared else 0)
    o = {} if out is None else out
    mt = moe_max_m_tiles(T, K, E, with_shared)

    def get(name, shape, dtype):
        if name not in o:
            o[name] = torch.empty(shape, dtype=dtype, device=dev)
        return o[name]

    counts = get("counts", (E,), torch.int32)
    offsets = get("offsets", (groups + 1,), torch.int32)
    src_row = get("src_row", (T * K,), torch.int32)
    dst_of = get("dst_of", (T, K), torch.int32)
    xq_perm = get("xq_perm", (T * K, d), torch.uint8)
    xs_perm = get("xs_perm", (T * K, d // 128), torch.float32)
    tile_group = get("tile_group", (max(mt, 1),), torch.int32)
    tile_start = get("tile_start", (groups + 1,), torch.int32)
    n_tiles = get("n_tiles", (1,), torch.int32)
    _count("moe_permute_noalloc")
    _check(lib().moe_permute_noalloc(_ptr(topk_idx), T, K, E, int(bool(with_shared)), _ptr(xq),
                                     _ptr(xscale), d, _ptr(counts), _ptr(offsets), _ptr(src_row),
                                     _ptr(dst_of), _ptr(xq_perm), _ptr(xs_perm),
                                     _ptr(tile_group), _ptr(tile_start), _ptr(n_tiles),
                                     _ptr(dev_err), _stream(stream)),
           "moe_permute_noalloc")
    o["max_tiles"] = mt
    return o


def moe_tile_table(offsets, max_tiles, tile_group=None, tile_start=None, n_tiles=None,
                   dev_err=None, stream=None):
    groups = offsets.numel() - 1
    dev = _dev(offsets)
    tile_group = torch.empty(max(max_tiles, 1), dtype=torch.int32, device=dev) if tile_group is None else tile_group
    tile_start = torch.empty(groups + 1, dtype=torch.int32, device=dev) if tile_start is None else tile_start
    n_tiles = torch.empty(1, dtype=torch.int32, device=dev) if n_tiles is None else n_tiles
    _count("moe_tile_table")
    _check(lib().moe_tile_table(_ptr(offsets), groups, max_tiles, _ptr(tile_group),
                                _ptr(tile_start), _ptr(n_tiles), _ptr(dev_err), _stream(stream)),
           "moe_tile_table")
    return tile_group, tile_start, n_tiles


def moe_segment_ids(counts, E, n_rows, ids=None, dev_err=None, stream=None, lead_rows=0):
    """counts int32 [sources][E] (or flat) -> ids int32 [n_rows]: the local
    expert of every row of a source-major, expert-sorted receive buffer; with
    lead_rows > 0 the first lead_rows rows are group 0 and the received rows
    after them get 1 + their expert."""
    c = counts.reshape(-1)
    ids = torch.empty(n_rows, dtype=torch.int32, device=_dev(counts)) if ids is None else ids
    _count("moe_segment_ids")
    _check(lib().moe_segment_ids(_ptr(c), c.numel(), E, lead_rows, n_rows, _ptr(ids),
                                 _ptr(dev_err), _stream(stream)), "moe_segment_ids")
    return ids


# ------------------------------------------------------------------ GEMM ---
def grouped_gemm_fp8_blockscaled(A, sa, B, sb, offsets, tile_group, tile_start, n_tiles,
                                 max_tiles, ep=EP_F32, D=None, d_scale=None, dev_err=None,
                                 stream=None, pow2=False, d_rows=None, sched=None):
    """A uint8 [rows][K], sa fp32 [rows][K/128], B uint8 [G][N][K], sb fp32
    [G][N/128][K/128].  ep=EP_F32 -> D fp32 [rows][N] (d_rows int32 [rows]
    optionally sends row j's output to D row d_rows[j]); ep=EP_SWIGLU_QUANT ->
    (sched: one device int32 -> dynamic work scheduling; the layer passes one)
    (h uint8 [rows][N/2], h_scale fp32 [rows][N/256]).  pow2 calls
    grouped_gemm_fp8_pow2 (every scale a power of two; the tensor core
    applies them)."""
    rows, K = A.shape
    G, N, _ = B.shape
    dev = _dev(A)
    if ep == EP_F32:
        D = torch.zeros(rows, N, dtype=torch.float32, device=dev) if D is None else D
    else:
        D = torch.empty(rows, N // 2, dtype=torch.uint8, device=dev) if D is None else D
        d_scale = torch.empty(rows, N // 256, dtype=torch.float32, device=dev) if d_scale is None else d_scale
    name = "grouped_gemm_fp8_pow2" if pow2 else "grouped_gemm_fp8_blockscaled"
    _count(name)
    _check(getattr(lib(), name)(_ptr(A), _ptr(sa), rows, _ptr(B), _ptr(sb), _ptr(offsets),
                                _ptr(tile_group), _ptr(tile_start), _ptr(n_tiles), max_tiles, G,
                                N, K, ep, _ptr(D), _ptr(d_scale), _ptr(d_rows), _ptr(sched),
                                _ptr(dev_err), _stream(stream)),
           name)
    return D if ep == EP_F32 else (D, d_scale)


# --------------------------------------------------------- combine / bias ---
def moe_combine(Y, dst_of, topk_gate, Y_shared, u, out=None, stream=None):
    T, d = u.shape
    K = dst_of.shape[1]
    out = torch.empty(T, d, dtype=torch.float32, device=_dev(u)) if out is None else out
    _count("moe_combine")
    _check(lib().moe_combine(_ptr(Y), _ptr(dst_of), _ptr(topk_gate), _ptr(Y_shared), _ptr(u),
                             T, K, d, _ptr(out), _stream(stream)), "moe_combine")
    return out


def moe_seq_balance_loss_ws(T, E, seq_len) -> int:
    n = _sz(0)
    _check(lib().moe_seq_balance_loss_workspace_size(T, E, seq_len, ctypes.byref(n)),
           "moe_seq_balance_loss_workspace_size")
    return n.value


def moe_seq_balance_loss(logits, K, seq_len, alpha=1e-4, with_fp=False, ws=None, stream=None):
    """Sequence-wise balance loss of logits fp32 [T][E] (moe_route's
    logits_out) per sequence of seq_len tokens.  Returns loss fp32 [T/seq_len],
    or (loss, f, P) with with_fp."""
    T, E = logits.shape
    dev = _dev(logits)
    n_seq = T // seq_len if seq_len > 0 else 0
    loss = torch.empty(max(n_seq, 1), dtype=torch.float32, device=dev)
    f = torch.empty(max(n_seq, 1), E, dtype=torch.float32, device=dev) if with_fp else None
    P = torch.empty(max(n_seq, 1), E, dtype=torch.float32, device=dev) if with_fp else None
    n = _sz(0)
    _check(lib().moe_seq_balance_loss_workspace_size(T, E, seq_len, ctypes.byref(n)),
           "moe_seq_balance_loss_workspace_size")
    if ws is None:
        ws = torch.empty(max(n.value, 16), dtype=torch.uint8, device=dev)
    _count("moe_seq_balance_loss")
    _check(lib().moe_seq_balance_loss(_ptr(logits), T, E, K, seq_len, float(alpha), _ptr(loss),
                                      _ptr(f), _ptr(P), _ptr(ws), ws.numel() * ws.element_size(),
                                      _stream(stream)), "moe_seq_balance_loss")
    loss = loss[:n_seq]
    if with_fp:
        return loss, f[:n_seq], P[:n_seq]
    return loss




def moe_bias_update(counts, T, K, gamma, bias, stream=None):
    if counts.dtype != torch.int32 or bias.dtype != torch.float32:
        raise MoEError("moe_bias_update: counts must be int32 and bias fp32")
    E = counts.numel()
    _count("moe_bias_update")
    _check(lib().moe_bias_update(_ptr(counts), E, T, K, float(gamma), _ptr(bias),
                                 _stream(stream)), "moe_bias_update")
    return bias


def moe_fp8_mma_peak(block_scaled, iters, ctas, sink, dev_err=None, stream=None):
    """Queue one FP8 MMA-loop launch (the caller times it); sink fp32 [ctas].
    Returns the launch's FLOP count."""
    _count("moe_fp8_mma_peak")
    _check(lib().moe_fp8_mma_peak(int(bool(block_scaled)), int(iters), int(ctas), _ptr(sink),
                                  _ptr(dev_err), _stream(stream)), "moe_fp8_mma_peak")
    return ctas * iters * 4 * (2 * 128 * 256 * 32)


def read_dev_err(dev_err) -> int:
    v = int(dev_err.item())
    return v


def raise_dev_err(dev_err) -> None:
    v = read_dev_err(dev_err)
    if v != 0:
        raise MoEError(f"device-side error {v}: {DEVERR.get(v, 'unknown')}")


# ------------------------------------------------------ backward (experts) ---
def fp8_quant_1x128_f32(x, pow2=False, q=None, scale=None, stream=None):
    """x fp32 [rows][cols] -> (q uint8, scale fp32 [rows][cols/128])."""
    assert x.dtype == torch.float32 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    q = torch.empty(rows, cols, dtype=torch.uint8, device=_dev(x)) if q is None else q
    scale = torch.empty(rows, cols // 128, dtype=torch.float32, device=_dev(x)) if scale is None else scale
    _count("fp8_quant_1x128_f32")
    _check(lib().fp8_quant_1x128_f32(_ptr(x), x.stride(0), rows, cols, int(bool(pow2)), _ptr(q),
                                     _ptr(scale), _stream(stream)), "fp8_quant_1x128_f32")
    return q, scale


def moe_combine_backward(dout, dst_of, topk_gate, dyq=None, dys=None, dy=None, want_dy=False,
                         stream=None):
    """dout fp32 [T][d] -> (dyq uint8 [T*K+T][d], dys [T*K+T][d/128], dy fp32 or None)."""
    T, d = dout.shape
    K = dst_of.shape[1]
    rows = T * K + T
    dev = _dev(dout)
    dyq = torch.empty(rows, d, dtype=torch.uint8, device=dev) if dyq is None else dyq
    dys = torch.empty(rows, d // 128, dtype=torch.float32, device=dev) if dys is None else dys
    if want_dy and dy is None:
        dy = torch.empty(rows, d, dtype=torch.float32, device=dev)
    _count("moe_combine_backward")
    _check(lib().moe_combine_backward(_ptr(dout), _ptr(dst_of), _ptr(topk_gate), T, K, d,
                                      _ptr(dyq), _ptr(dys), _ptr(dy), _stream(stream)),
           "moe_combine_backward")
    return dyq, dys, dy


def swiglu_backward(dh, guq, gus, dguq=None, dgus=None, dgu=None, h=None, want_fp32=False,
                    stream=None):
    """dh fp32 [rows][I], cached gu (uint8 [rows][2I], scales [rows][2I/128]) ->
    (dguq, dgus, dgu fp32 or None, h fp32 or None)."""
    rows, I = dh.shape
    dev = _dev(dh)
    dguq = torch.empty(rows, 2 * I, dtype=torch.uint8, device=dev) if dguq is None else dguq
    dgus = torch.empty(rows, 2 * I // 128, dtype=torch.float32, device=dev) if dgus is None else dgus
    if want_fp32:
        dgu = torch.empty(rows, 2 * I, dtype=torch.float32, device=dev) if dgu is None else dgu
        h = torch.empty(rows, I, dtype=torch.float32, device=dev) if h is None else h
    _count("swiglu_backward")
    _check(lib().swiglu_backward(_ptr(dh), _ptr(guq), _ptr(gus), rows, I, _ptr(dguq), _ptr(dgus),
                                 _ptr(dgu), _ptr(h), _stream(stream)), "swiglu_backward")
    return dguq, dgus, dgu, h


def wgrad_ld(max_tiles: int) -> int:
    """Row length (bytes) of a token-major Wgrad operand: 128 per tile, a
    multiple of 512."""
    return (128 * max_tiles + 511) // 512 * 512


def fp8_quant_128x1_pow2(src, offsets, tile_group, tile_start, n_tiles, max_tiles, src_scale=None,
                         qt=None, st=None, atoms=None, stream=None):
    """Token-major 128x1 re-quantisation.  src fp32 [rows][C] (or uint8 with
    src_scale [rows][C/128], the _requant form) -> (qt uint8 [C][ldt], st fp32
    [C][ldt/128], atoms uint8 [C/128][ldt/512][512])."""
    rows, C = src.shape
    ldt = wgrad_ld(max_tiles)
    dev = _dev(src)
    # columns past the last tile are never read (left unwritten)
    qt = torch.empty(C, ldt, dtype=torch.uint8, device=dev) if qt is None else qt
    st = torch.empty(C, ldt // 128, dtype=torch.float32, device=dev) if st is None else st
    atoms = torch.empty(C // 128, ldt // 512, 512, dtype=torch.uint8, device=dev) if atoms is None else atoms
    if src_scale is None:
        assert src.dtype == torch.float32
        _count("fp8_quant_128x1_pow2")
        _check(lib().fp8_quant_128x1_pow2(_ptr(src), src.stride(0), _ptr(offsets), _ptr(tile_group),
                                          _ptr(tile_start), _ptr(n_tiles), max_tiles, C, _ptr(qt),
                                          ldt, _ptr(st), _ptr(atoms), _stream(stream)),
               "fp8_quant_128x1_pow2")
    else:
        assert src.dtype == torch.uint8
        _count("fp8_requant_128x1_pow2")
        _check(lib().fp8_requant_128x1_pow2(_ptr(src), _ptr(src_scale), src.stride(0),
                                            _ptr(offsets), _ptr(tile_group), _ptr(tile_start),
                                            _ptr(n_tiles), max_tiles, C, _ptr(qt), ldt, _ptr(st),
                                            _ptr(atoms), _stream(stream)),
               "fp8_requant_128x1_pow2")
    return qt, st, atoms


def fp8_transpose_128x128(q, scale, qt=None, scale_t=None, stream=None):
    """[G][N][K] FP8 weights and [G][N/128][K/128] scales -> [G][K][N], [G][K/128][N/128]."""
    G, N, K = q.shape
    dev = _dev(q)
    qt = torch.empty(G, K, N, dtype=torch.uint8, device=dev) if qt is None else qt
    scale_t = torch.empty(G, K // 128, N // 128, dtype=torch.float32, device=dev) if scale_t is None else scale_t
    _count("fp8_transpose_128x128")
    _check(lib().fp8_transpose_128x128(_ptr(q), _ptr(scale), G, N, K, _ptr(qt), _ptr(scale_t),
                                       _stream(stream)), "fp8_transpose_128x128")
    return qt, scale_t


def moe_unpermute_add(dx, dst_of, dout, du=None, stream=None):
    """du[t] = dout[t] + dx[T*K + t] + sum_k dx[dst_of[t][k]]."""
    T, d = dout.shape
    K = dst_of.shape[1]
    du = torch.empty(T, d, dtype=torch.float32, device=_dev(dout)) if du is None else du
    _count("moe_unpermute_add")
    _check(lib().moe_unpermute_add(_ptr(dx), _ptr(dst_of), _ptr(dout), T, K, d, _ptr(du),
                                   _stream(stream)), "moe_unpermute_add")
    return du


def grouped_gemm_fp8_wgrad(At, a_atoms, Bt, b_atoms, tile_start, groups, dW=None, dev_err=None,
                           stream=None):
    """At uint8 [Ma][ldt], Bt uint8 [Nb][ldt] (token-major) -> dW fp32 [groups][Ma][Nb]."""
    Ma, ldt = At.shape
    Nb = Bt.shape[0]
    dW = torch.empty(groups, Ma, Nb, dtype=torch.float32, device=_dev(At)) if dW is None else dW
    _count("grouped_gemm_fp8_wgrad")
    _check(lib().grouped_gemm_fp8_wgrad(_ptr(At), _ptr(a_atoms), _ptr(Bt), _ptr(b_atoms), ldt, Ma,
                                        Nb, _ptr(tile_start), groups, _ptr(dW), _ptr(dev_err),
                                        _stream(stream)), "grouped_gemm_fp8_wgrad")
    return dW
