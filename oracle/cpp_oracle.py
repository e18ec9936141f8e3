"""ctypes front of the C++ oracle (moe_oracle_ref.cpp): single-threaded, fp64.

TEST INFRASTRUCTURE ONLY, like moe_oracle.py: only the tests, the smoke check
and the benchmark's CPU legs may import it.  The functions have the names and
the array conventions of moe_oracle.py, so every pin can run against both
oracles; all of the method's arithmetic happens in the C++ library, this file
only allocates numpy arrays and passes pointers (plus the integer bookkeeping
of segment offsets and tile tables, as in moe_oracle.py).

The library is compiled on first import when it is missing or older than its
source (g++, see build_oracle.py).
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build_oracle

E4M3_MAX = 448.0
TILE = 128

_L = None
_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float
_d = ctypes.c_double

_SIGS = {
    "orc_version": (_i, []),
    "orc_e4m3_decode": (None, [_p, _i64, _p]),
    "orc_e4m3_encode": (_i, [_p, _i64, _p]),
    "orc_pow2_ceil": (None, [_p, _i64, _p]),
    "orc_quant_1x128": (None, [_p, _i64, _i64, _i, _p, _p]),
    "orc_quant_128x128": (None, [_p, _i64, _i64, _i, _p, _p]),
    "orc_dequant": (None, [_p, _p, _i64, _i64, _i, _p]),
    "orc_router_logits": (None, [_p, _p, _i64, _i64, _i64, _p]),
    "orc_sigmoid": (None, [_p, _i64, _p]),
    "orc_route_select": (_i, [_p, _p, _i64, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p]),
    "orc_permute": (_i, [_p, _i64, _i, _i, _p, _p, _p, _p]),
    "orc_grouped_gemm": (None, [_p, _p, _i64, _p, _p, _i, _i64, _i64, _p, _p]),
    "orc_swiglu": (None, [_p, _i64, _i64, _p]),
    "orc_combine": (None, [_p, _p, _p, _p, _p, _i64, _i, _i64, _p]),
    "orc_bias_update": (None, [_p, _i, _i64, _i, _f, _p, _p]),
    "orc_seq_balance_loss": (_i, [_p, _i64, _i, _i, _i64, _d, _p, _p, _p, _p]),
}


def lib() -> ctypes.CDLL:
    global _L
    if _L is None:
        L = ctypes.CDLL(build_oracle.build())
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _L = L
    return _L


def _c(a, dtype):
    """C-contiguous array of the given dtype (a copy only when needed)."""
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data


# ------------------------------------------------------------------ E4M3 --
def e4m3_decode(codes) -> np.ndarray:
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_e4m3_decode(_ptr(c), c.size, _ptr(out))
    return out


def e4m3_encode(v) -> np.ndarray:
    x = _c(v, np.float64)
    out = np.empty(x.shape, np.uint8)
    if lib().orc_e4m3_encode(_ptr(x), x.size, _ptr(out)) != 0:
        raise ValueError("e4m3_encode: NaN input")
    return out


def pow2_ceil(s) -> np.ndarray:
    s64 = np.asarray(s, np.float64)
    if (s64 <= 0).any() or not np.isfinite(s64).all():
        raise ValueError("pow2_ceil: positive finite scales only")
    x = _c(s, np.float32)
    out = np.empty(x.shape, np.float32)
    lib().orc_pow2_ceil(_ptr(x), x.size, _ptr(out))
    return out


# ---------------------------------------------------------- quantisation --
def _quant_1x128(x, pow2):
    x = _c(x, np.float32)
    rows, cols = x.shape
    assert cols % TILE == 0
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows, cols // TILE), np.float32)
    lib().orc_quant_1x128(_ptr(x), rows, cols, int(pow2), _ptr(q), _ptr(s))
    return q, s


def _quant_128x128(w, pow2):
    w = _c(w, np.float32)
    rows, cols = w.shape
    assert cols % TILE == 0
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((-(-rows // TILE), cols // TILE), np.float32)
    lib().orc_quant_128x128(_ptr(w), rows, cols, int(pow2), _ptr(q), _ptr(s))
    return q, s


def quant_1x128(x):
    return _quant_1x128(x, False)


def quant_1x128_pow2(x):
    return _quant_1x128(x, True)


def quant_128x128(w):
    return _quant_128x128(w, False)


def quant_128x128_pow2(w):
    return _quant_128x128(w, True)


def _dequant(q, scale, block_rows):
    q = _c(q, np.uint8)
    scale = _c(scale, np.float32)
    rows, cols = q.shape
    out = np.empty((rows, cols), np.float64)
    lib().orc_dequant(_ptr(q), _ptr(scale), rows, cols, block_rows, _ptr(out))
    return out


def dequant_1x128(q, scale):
    return _dequant(q, scale, 1)


def dequant_128x128(q, scale):
    return _dequant(q, scale, TILE)


# ---------------------------------------------------------------- router --
def router_logits(u, centroids) -> np.ndarray:
    u = _c(u, np.float32)
    c = _c(centroids, np.float32)
    T, d = u.shape
    E = c.shape[0]
    z = np.empty((T, E), np.float64)
    lib().orc_router_logits(_ptr(u), _ptr(c), T, E, d, _ptr(z))
    return z


def sigmoid(z) -> np.ndarray:
    z = _c(z, np.float64)
    s = np.empty(z.shape, np.float64)
    lib().orc_sigmoid(_ptr(z), z.size, _ptr(s))
    return s


def route_select(z, bias, G: int, M: int, K: int, group_score: str = "biased"):
    z = _c(z, np.float64)
    T, E = z.shape
    b = _c(bias, np.float64)
    idx = np.empty((T, K), np.int32)
    gate = np.empty((T, K), np.float64)
    s = np.empty((T, E), np.float64)
    beta = np.empty((T, E), np.float64)
    km, gm, om = (np.empty(T, np.float64) for _ in range(3))
    st = lib().orc_route_select(_ptr(z), _ptr(b), T, E, G, M, K, int(group_score == "raw"),
                                _ptr(idx), _ptr(gate), _ptr(s), _ptr(beta), _ptr(km), _ptr(gm),
                                _ptr(om))
    if st != 0:
        raise AssertionError("route_select: inconsistent E, G, M, K")
    return idx, gate, {"k_margin": km, "g_margin": gm, "o_margin": om, "s": s, "beta": beta}


def route(u, centroids, bias, G, M, K, group_score="biased"):
    z = router_logits(u, centroids)
    idx, gate, info = route_select(z, bias, G, M, K, group_score)
    info["z"] = z
    return idx, gate, info


# ----------------------------------------------------------- permutation --
def permute(idx, E: int):
    idx = _c(idx, np.int32)
    T, K = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    src_row = np.empty(T * K, np.int32)
    dst_of = np.empty((T, K), np.int32)
    if lib().orc_permute(_ptr(idx), T, K, E, _ptr(counts), _ptr(offsets), _ptr(src_row),
                         _ptr(dst_of)) != 0:
        raise ValueError("permute: expert index out of range")
    return counts, offsets, src_row, dst_of


def segment_offsets_with_shared(offsets, T: int) -> np.ndarray:
    offsets = np.asarray(offsets, np.int64)
    return np.concatenate([offsets, [offsets[-1] + T]]).astype(np.int32)


def mtile_table(offsets, tile_m: int = TILE):
    offsets = np.asarray(offsets, np.int64)
    cnt = np.diff(offsets)
    mt = -(-cnt // tile_m)
    start = np.concatenate([[0], np.cumsum(mt)]).astype(np.int32)
    grp = np.repeat(np.arange(len(cnt)), mt).astype(np.int32)
    return grp, start


# ------------------------------------------------------------------ GEMM --
def grouped_gemm(aq, sa, bq, sb, offsets) -> np.ndarray:
    aq = _c(aq, np.uint8)
    sa = _c(sa, np.float32)
    bq = _c(bq, np.uint8)
    sb = _c(sb, np.float32)
    offs = _c(offsets, np.int32)
    rows, K = aq.shape
    groups, N, _ = bq.shape
    out = np.empty((rows, N), np.float64)
    lib().orc_grouped_gemm(_ptr(aq), _ptr(sa), rows, _ptr(bq), _ptr(sb), groups, N, K,
                           _ptr(offs), _ptr(out))
    return out


# ---------------------------------------------------------------- SwiGLU --
def swiglu(gu, I: int) -> np.ndarray:
    gu = _c(gu, np.float64)
    rows = gu.shape[0]
    assert gu.shape[1] == 2 * I and I % TILE == 0
    h = np.empty((rows, I), np.float64)
    lib().orc_swiglu(_ptr(gu), rows, I, _ptr(h))
    return h


def silu(x) -> np.ndarray:
    """SiLU through the SwiGLU kernel with up = 1 (one 128-wide block)."""
    x = np.asarray(x, np.float64)
    flat = x.reshape(-1)
    n = flat.size
    pad = -(-max(n, 1) // TILE) * TILE
    gu = np.zeros((pad // TILE, 2 * TILE), np.float64)
    g = np.zeros(pad)
    g[:n] = flat
    gu[:, :TILE] = g.reshape(-1, TILE)
    gu[:, TILE:] = 1.0
    return swiglu(gu, TILE).reshape(-1)[:n].reshape(x.shape)


def swiglu_quant(gu, I: int, pow2: bool = False):
    h = swiglu(gu, I).astype(np.float32)
    return _quant_1x128(h, pow2)


# --------------------------------------------------------------- combine --
def combine(Y, dst_of, gate, Y_shared, u) -> np.ndarray:
    Y = _c(Y, np.float64)
    dst = _c(dst_of, np.int32)
    g = _c(gate, np.float64)
    ys = None if Y_shared is None else _c(Y_shared, np.float64)
    u = _c(u, np.float64)
    T, K = dst.shape
    d = Y.shape[1]
    out = np.empty((T, d), np.float64)
    lib().orc_combine(_ptr(Y), _ptr(dst), _ptr(g), _ptr(ys), _ptr(u), T, K, d, _ptr(out))
    return out


# ----------------------------------------------------------- bias update --
def bias_update(counts, T: int, K: int, gamma: float, bias) -> np.ndarray:
    c = _c(counts, np.int32)
    b = _c(bias, np.float32)
    out = np.empty(b.shape, np.float32)
    lib().orc_bias_update(_ptr(c), c.size, T, K, float(np.float32(gamma)), _ptr(b), _ptr(out))
    return out


# ------------------------------------------------------------ balance loss --
def seq_balance_loss(z, K: int, seq_len: int, alpha: float = 1e-4):
    z = _c(z, np.float64)
    T, E = z.shape
    assert T % seq_len == 0 and 0 < K <= E
    n_seq = T // seq_len
    loss = np.empty(n_seq, np.float64)
    f = np.empty((n_seq, E), np.float64)
    P = np.empty((n_seq, E), np.float64)
    km = np.empty(T, np.float64)
    if lib().orc_seq_balance_loss(_ptr(z), T, E, K, seq_len, float(alpha), _ptr(loss), _ptr(f),
                                  _ptr(P), _ptr(km)) != 0:
        raise AssertionError("seq_balance_loss: inconsistent sizes")
    return loss, f, P, km


# ----------------------------------------------------------- whole layer --
def quantise_weights(w1, w2, pow2: bool = False):
    qf = quant_128x128_pow2 if pow2 else quant_128x128
    q1, s1 = zip(*[qf(w) for w in np.asarray(w1, np.float32)])
    q2, s2 = zip(*[qf(w) for w in np.asarray(w2, np.float32)])
    return np.stack(q1), np.stack(s1), np.stack(q2), np.stack(s2)


def moe_layer(u, centroids, bias, w1q, w1s, w2q, w2s, G, M, K, gamma,
              h_override=None, pow2: bool = False):
    """The layer composed from the steps above, as moe_oracle.moe_layer
    (without the backward's SwiGLU-input cache)."""
    u = np.asarray(u, np.float32)
    T, d = u.shape
    E = np.asarray(centroids).shape[0]
    I = np.asarray(w1q).shape[1] // 2
    idx, gate, rinfo = route(u, centroids, bias, G, M, K)
    xq_tok, xs_tok = _quant_1x128(u, pow2)
    counts, offsets, src_row, dst_of = permute(idx, E)
    pairs = T * K
    xq = np.concatenate([xq_tok[src_row], xq_tok])
    xs = np.concatenate([xs_tok[src_row], xs_tok])
    offs = segment_offsets_with_shared(offsets, T)
    gu = grouped_gemm(xq, xs, w1q, w1s, offs)
    hq, hs = swiglu_quant(gu, I, pow2) if h_override is None else h_override
    Y = grouped_gemm(hq, hs, w2q, w2s, offs)
    out = combine(Y[:pairs], dst_of, gate, Y[pairs:], u)
    new_bias = bias_update(counts, T, K, gamma, bias)
    return {"idx": idx, "gate": gate, "route": rinfo, "xq_tok": xq_tok, "xs_tok": xs_tok,
            "counts": counts, "offsets": offs, "src_row": src_row, "dst_of": dst_of,
            "xq": xq, "xs": xs, "gu": gu, "hq": hq, "hs": hs, "Y": Y, "out": out,
            "bias": new_bias}
