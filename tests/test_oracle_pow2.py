"""Pins of the oracle's power-of-two scale variant (CPU only).

"DeepSeek_V3_Report：Annotation", "Low-Precision Storage and Communication":
the activations quantised before the dispatch carry scaling factors that are
integral powers of 2.  The oracle reads this as the fp32 scale rounded up to
the next power of two.  The pins below use a brute-force search over powers
of two, a worked example by hand, the nearest-code search over all finite E4M3
values, and the reduction to the fp32-scale quantiser when amax/448 is
itself a power of two.
"""
import numpy as np

from oracle import moe_oracle as ONP

FINITE_CODES = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
FINITE_VALUES = ONP.e4m3_decode(FINITE_CODES)


def _nearest_code(v: float) -> int:
    """Nearest finite E4M3 value by exhaustive search, ties to the even code,
    the sign of v kept on zero."""
    dist = np.abs(FINITE_VALUES - v)
    cands = [int(c) for c, d in zip(FINITE_CODES, dist) if d == dist.min()]
    same = [c for c in cands if ((c & 0x80) != 0) == bool(np.signbit(v))]
    cands = same or cands
    even = [c for c in cands if (c & 1) == 0]
    return (even or cands)[0]


def _smallest_pow2_at_least(s: float) -> float:
    for k in range(-160, 130):
        if 2.0 ** k >= s:
            return 2.0 ** k
    raise AssertionError("out of range")


def test_pow2_ceil_bruteforce(O):
    rng = np.random.default_rng(11)
    s = np.exp2(rng.uniform(-30, 20, 400)).astype(np.float32)
    exact = np.exp2(np.arange(-30, 20)).astype(np.float32)
    above = np.nextafter(exact, np.float32(np.inf))
    below = np.nextafter(exact, np.float32(0))
    allv = np.concatenate([s, exact, above, below])
    got = O.pow2_ceil(allv)
    assert got.dtype == np.float32
    for v, g in zip(allv, got):
        assert float(g) == _smallest_pow2_at_least(float(v)), v
    # a power of two is its own ceiling; one ulp above it doubles
    assert np.array_equal(O.pow2_ceil(exact), exact)
    assert np.array_equal(O.pow2_ceil(above), 2 * exact)


def test_quant_1x128_pow2_worked_example(O):
    # amax 0.3: 0.3/448 = 6.70e-4 lies in (2^-11, 2^-10], so the scale is 2^-10;
    # 0.3 * 1024 = 307.2 lies between the E4M3 values 288 and 320 (step 32
    # in [256, 512)) and rounds to 320 = 1.25 * 2^8: exponent field 15,
    # mantissa 2, code 0x7A (0xFA for -0.3).  0.001 * 1024 = 1.024 rounds to
    # 1.0 (step 1/8 in [1, 2)): code 0x38.
    x = np.zeros((1, 128), np.float32)
    x[0, 0] = 0.3
    x[0, 1] = -0.3
    x[0, 2] = 0.001
    q, s = O.quant_1x128_pow2(x)
    assert s[0, 0] == np.float32(2.0 ** -10)
    assert q[0, 0] == 0x7A and q[0, 1] == 0xFA and q[0, 2] == 0x38
    assert np.all(q[0, 3:] == 0)


def test_quant_1x128_pow2_properties(O):
    rng = np.random.default_rng(12)
    x = (rng.normal(0, 1, (7, 384)) * np.exp2(rng.integers(-8, 8, (7, 1)))).astype(np.float32)
    x[2, 130] = -77.0
    x[4, 0:128] = 0.0                            # all-zero tile
    q, s = O.quant_1x128_pow2(x)
    assert q.shape == x.shape and s.shape == (7, 3) and s.dtype == np.float32
    amax = np.abs(x.reshape(7, 3, 128)).max(axis=2)
    lin = (np.maximum(amax, np.float32(1e-4)) / np.float32(448)).astype(np.float32)
    m, _ = np.frexp(s.astype(np.float64))
    assert np.all(m == 0.5)                      # powers of two
    assert np.all(s >= lin) and np.all(s < 2 * lin.astype(np.float64))
    assert s[4, 0] == np.float32(2.0 ** -22)     # 1e-4/448 = 2.23e-7 in (2^-23, 2^-22]
    # nothing saturates: |x / s| <= 448 and the tile maximum lands in [224, 448]
    y = x.astype(np.float64) / np.repeat(s, 128, axis=1)
    assert np.all(np.abs(y) <= 448.0)
    deq = O.e4m3_decode(q).reshape(7, 3, 128)
    big = np.abs(deq).max(axis=2)
    assert np.all((big >= 224.0) | (amax == 0))
    # the fp32 quotient is exact, so every code is the nearest E4M3 value of x/s
    for r in range(7):
        for c in range(0, 384, 5):
            yy = np.float32(x[r, c]) / s[r, c // 128]
            assert float(yy) == y[r, c]
            assert q[r, c] == _nearest_code(float(yy))


def test_pow2_reduces_to_fp32_scale_when_exact(O):
    # a tile whose amax/448 is a power of two gets the same scale and bytes
    rng = np.random.default_rng(13)
    x = rng.uniform(-1, 1, (3, 256)).astype(np.float32)
    x[0, 5] = 448.0 * 2.0 ** -3
    x[0, 200] = -448.0 * 2.0 ** 4
    x[1, 17] = 448.0
    x[1, 128:] *= np.float32(2.0 ** -10)
    x[1, 140] = 448.0 * 2.0 ** -9
    x[2, 3] = 448.0 * 2.0 ** 2
    x[2, 130] = 448.0
    q2, s2 = O.quant_1x128_pow2(x)
    q1, s1 = O.quant_1x128(x)
    assert np.array_equal(s1, s2) and np.array_equal(q1, q2)


def test_quant_128x128_pow2(O):
    rng = np.random.default_rng(14)
    w = rng.normal(0, 0.02, (200, 256)).astype(np.float32)   # ragged last row-block
    w[150, 200] = 0.9
    q, s = O.quant_128x128_pow2(w)
    assert s.shape == (2, 2)
    for i in range(2):
        for j in range(2):
            blk = w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            lin = float(np.float32(np.abs(blk).max()) / np.float32(448))
            assert float(s[i, j]) == _smallest_pow2_at_least(lin)
    # 0.9/448 = 2.0e-3 in (2^-9, 2^-8]: 0.9 * 256 = 230.4 lies between the
    # E4M3 values 224 and 240 (step 16 in [128, 256)) and rounds to 224 =
    # 1.75 * 2^7: exponent field 14, mantissa 6, code 0x76
    assert s[1, 1] == np.float32(2.0 ** -8) and q[150, 200] == 0x76
    for (r, c) in [(0, 0), (150, 200), (130, 3), (199, 255), (64, 128)]:
        yy = np.float32(w[r, c]) / s[r // 128, c // 128]
        assert q[r, c] == _nearest_code(float(yy))


def test_swiglu_quant_pow2(O):
    rng = np.random.default_rng(15)
    gu = rng.normal(0, 2, (5, 512)).astype(np.float32)
    hq, hs = O.swiglu_quant(gu, 256, pow2=True)
    h = O.swiglu(gu, 256).astype(np.float32)
    hq_ref, hs_ref = O.quant_1x128_pow2(h)
    assert np.array_equal(hq, hq_ref) and np.array_equal(hs, hs_ref)
    m, _ = np.frexp(hs.astype(np.float64))
    assert np.all(m == 0.5)
    # default path keeps the fp32 scales
    _, hs32 = O.swiglu_quant(gu, 256)
    assert not np.array_equal(hs32, hs)
