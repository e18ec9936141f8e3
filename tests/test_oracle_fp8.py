"""Pins of the oracle's E4M3 codec and online quantisation (CPU only).

The oracle is checked against things other than itself: the format's own
definition worked out by hand (tests/golden/e4m3_points.txt), brute-force
nearest-value search over the 254 finite codes, PyTorch's float8_e4m3fn cast
as an independent third opinion, and the closed-form properties the pages
state for the scale ("DeepSeek_V3_Report：Annotation", "Online Quantization":
the tile maximum maps to Q_max = 448).
"""
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as ONP

GOLD = os.path.join(os.path.dirname(__file__), "golden", "e4m3_points.txt")
FINITE_CODES = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)


def _finite_values():
    return ONP.e4m3_decode(FINITE_CODES)


def _nearest_code_bruteforce(v: float) -> int:
    """Nearest finite E4M3 value by exhaustive search; ties to the even code;
    magnitudes above 448 saturate."""
    vals = _finite_values()
    if abs(v) >= 448.0:
        return 0xFE if v < 0 else 0x7E
    dist = np.abs(vals - v)
    best = dist.min()
    cands = [int(c) for c, dd in zip(FINITE_CODES, dist) if dd == best]
    # equal magnitude +0/-0: keep the sign of v
    same_sign = [c for c in cands if ((c & 0x80) != 0) == bool(np.signbit(v))]
    cands = same_sign or cands
    even = [c for c in cands if (c & 1) == 0]
    return (even or cands)[0]


def test_golden_points(O):
    rows = []
    with open(GOLD) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            v, code = line.split()[:2]
            rows.append((float(v), int(code, 16)))
    vals = np.array([r[0] for r in rows])
    codes = O.e4m3_encode(vals)
    for (v, c), got in zip(rows, codes):
        assert got == c, (v, hex(c), hex(got))


def test_roundtrip_all_finite_codes(O):
    vals = O.e4m3_decode(FINITE_CODES)
    assert np.array_equal(O.e4m3_encode(vals), FINITE_CODES)
    assert np.isnan(O.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()
    pos = O.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)          # codes 0..0x7E are increasing
    assert pos[-1] == 448.0 and pos[1] == 2.0 ** -9


def test_encode_matches_bruteforce_nearest(O):
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.normal(0, 1, 400) * np.exp2(rng.integers(-12, 10, 400)),
        # exact midpoints between neighbours
        (O.e4m3_decode(FINITE_CODES[:-1]) + O.e4m3_decode(FINITE_CODES[1:]))[:120] / 2,
        [447.9, 448.1, 463.9, 464.0, 465.0, -500.0, 1e-12, -1e-12],
    ])
    got = O.e4m3_encode(v)
    want = np.array([_nearest_code_bruteforce(float(x)) for x in v], np.uint8)
    assert np.array_equal(got, want)


def test_encode_agrees_with_torch_float8_in_range(O):
    rng = np.random.default_rng(1)
    v = (rng.normal(0, 60, 20000)).astype(np.float32)
    v = v[np.abs(v) <= 448]
    ours = O.e4m3_encode(v)
    theirs = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_quant_1x128_properties(O):
    rng = np.random.default_rng(2)
    x = rng.normal(0, 1, (9, 512)).astype(np.float32)
    x[3, 130] = -50.0                           # an outlier in tile (3, 1)
    x[5, 256:384] = 0.0                         # an all-zero tile
    q, s = O.quant_1x128(x)
    assert q.shape == x.shape and s.shape == (9, 4) and s.dtype == np.float32
    tiles = np.abs(x.reshape(9, 4, 128))
    amax = tiles.max(axis=2)
    # scale is the fp32 dequantisation multiplier max(amax, eps)/448
    ref = np.maximum(amax, np.float32(1e-4)) / 448.0
    assert np.all(np.abs(s.astype(np.float64) - ref) <= ref * 2.0 ** -23)
    # the tile maximum lands on +-448 (code 0x7E / 0xFE)
    qt = q.reshape(9, 4, 128)
    for r in range(9):
        for j in range(4):
            if amax[r, j] == 0:
                assert np.all(qt[r, j] == 0)
                assert s[r, j] == np.float32(np.float32(1e-4) / np.float32(448.0))
                continue
            m = np.argmax(tiles[r, j])
            assert qt[r, j, m] in (0x7E, 0xFE)
    assert q[3, 130] == 0xFE
    # dequantisation error: at most half an E4M3 step of the scaled value
    deq = O.dequant_1x128(q, s)
    y = x / np.repeat(s, 128, axis=1).astype(np.float64)
    _, ex = np.frexp(np.abs(y))
    half_step = np.exp2(np.maximum(ex - 1, -6) - 4)
    assert np.all(np.abs(deq - x) <= half_step * np.repeat(s, 128, axis=1) * (1 + 1e-6))


def test_quant_1x128_bruteforce_codes(O):
    rng = np.random.default_rng(3)
    x = (rng.normal(0, 3, (2, 256)) * np.exp2(rng.integers(-6, 6, (2, 256)))).astype(np.float32)
    q, s = O.quant_1x128(x)
    for r in range(2):
        for c in range(256):
            y = np.float32(x[r, c]) / np.float32(s[r, c // 128])
            assert q[r, c] == _nearest_code_bruteforce(float(y))


def test_quant_128x128_blocks(O):
    rng = np.random.default_rng(4)
    w = rng.normal(0, 0.05, (200, 256)).astype(np.float32)   # ragged last row-block
    w[7, 200] = 3.0
    q, s = O.quant_128x128(w)
    assert s.shape == (2, 2)
    for i in range(2):
        for j in range(2):
            blk = w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            assert s[i, j] == np.float32(np.float32(np.abs(blk).max()) / np.float32(448))
    assert q[7, 200] == 0x7E
    # an element change inside block (1, 0) moves only that block's scale
    w2 = w.copy()
    w2[150, 5] = 9.0
    _, s2 = O.quant_128x128(w2)
    assert s2[1, 0] != s[1, 0] and s2[0, 0] == s[0, 0] and s2[1, 1] == s[1, 1] and s2[0, 1] == s[0, 1]
    # spot-check codes by brute force
    for (r, c) in [(0, 0), (7, 200), (130, 3), (199, 255), (64, 128)]:
        y = np.float32(w[r, c]) / np.float32(s[r // 128, c // 128])
        assert q[r, c] == _nearest_code_bruteforce(float(y))
    # dequantisation restores the block maximum exactly up to fp32 rounding
    deq = O.dequant_128x128(q, s)
    assert abs(deq[7, 200] - 3.0) <= 3.0 * 2.0 ** -22
