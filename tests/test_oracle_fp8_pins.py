"""Pins of the oracle's FP8 comparison format (E4M3 elements, one power-of-two scale per 32
elements along K, stored as an E8M0 code) against definitions restated here: the scale rule,
a brute-force signed E4M3 encoder, grid round trips, and exact rational GEMM sums."""
import math
from fractions import Fraction

import numpy as np
import pytest

from nvfp4_w4a4_moe_02_b200 import synthetic as syn


def e4m3_value(code: int) -> float:
    """Closed form of an E4M3 code (bias 7, subnormal step 2^-9, 0x7F / 0xFF are NaN)."""
    s = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 7
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1 + m / 8) * 2.0 ** (e - 7)


FINITE = [c for c in range(256) if (c & 0x7F) != 0x7F]


def brute_e4m3_signed(v: float) -> int:
    """Nearest finite E4M3 value, ties to the even code, |v| > 448 saturates, sign kept."""
    neg = math.copysign(1.0, v) < 0
    a = abs(v)
    if a >= 448.0:
        return 0xFE if neg else 0x7E
    best = None
    for c in range(0x7F):  # non-negative codes, ascending value
        d = abs(e4m3_value(c) - a)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1] | (0x80 if neg else 0)


def min_exponent(b: float) -> int:
    X = -127
    while X < 127 and math.ldexp(448.0, X) < b:
        X += 1
    return X


def test_scale_exponent_is_the_smallest_that_avoids_saturation(orc):
    rng = np.random.default_rng(1)
    bs = [0.0, 1.0, 448.0, 449.0, 2.0 ** -140, 3.0e38, 1e-30]
    bs += [float(np.float32(math.ldexp(448.0, k))) for k in range(-20, 20)]
    bs += [float(np.float32(math.ldexp(448.0, k) * (1 + 2.0 ** -23))) for k in range(-20, 20)]
    bs += list(np.exp(rng.uniform(-60, 60, 300)).astype(np.float32))
    for b in bs:
        X = orc.mx8_exponent(b)
        assert math.ldexp(448.0, X) >= b or X == 127
        assert X == -127 or math.ldexp(448.0, X - 1) < b
        assert X == min_exponent(float(np.float32(b)))


def test_signed_e4m3_encoder_matches_brute_force(orc):
    vals = [0.0, -0.0, 448.0, -448.0, 500.0, -1e9, 2.0 ** -10, -(2.0 ** -10), 2.0 ** -9 * 1.5]
    for c in FINITE:  # every value and the midpoints to its neighbours, +- one binary32 ulp
        v = e4m3_value(c)
        vals += [v, float(np.nextafter(np.float32(v), np.float32(np.inf))),
                 float(np.nextafter(np.float32(v), np.float32(-np.inf)))]
    pos = sorted(e4m3_value(c) for c in range(0x7F))
    for lo, hi in zip(pos, pos[1:]):
        mid = np.float32((lo + hi) / 2)
        vals += [float(mid), float(np.nextafter(mid, np.float32(0))), float(np.nextafter(mid, np.float32(1e9))),
                 -float(mid)]
    for v in vals:
        assert orc.e4m3_encode_signed(v) == brute_e4m3_signed(float(np.float32(v))), v
    for c in FINITE:
        assert orc.e4m3_decode_signed(c) == e4m3_value(c)


def test_quantize_matches_float32_numpy_steps(orc):
    rng = np.random.default_rng(3)
    rows, K = 6, 128
    x = syn.normal_bf16(3, 1, rows, K, 1.0, np.exp(3 * rng.standard_normal(K)))
    x[0, :32] = 0  # an all-zero block
    x[1, 5] = 0x8000  # a negative zero
    codes, S = orc.mx8_quantize(x)
    xf = syn.bf16_to_f32(x)
    for r in range(rows):
        for b in range(K // 32):
            blk = xf[r, 32 * b:32 * b + 32]
            X = min_exponent(float(np.max(np.abs(blk))))
            assert S[r, b] == X + 127
            v = blk * np.float32(math.ldexp(1.0, -X))  # binary32 RN multiply
            assert [brute_e4m3_signed(float(t)) for t in v] == codes[r, 32 * b:32 * b + 32].tolist(), (r, b)
    assert S[0, 0] == 0 and not codes[0, :32].any()
    assert codes[1, 5] == 0x80


def test_on_grid_values_round_trip_exactly(orc):
    rng = np.random.default_rng(4)
    rows, K = 4, 96
    X = rng.integers(-40, 40, (rows, K // 32))
    c = rng.choice(FINITE, (rows, K))
    c[:, ::32] = 0x7E  # each block holds +448: its scale exponent is exactly X
    vals = np.vectorize(e4m3_value)(c) * np.ldexp(1.0, np.repeat(X, 32, axis=1))
    x = orc.f64_to_bf16_array(vals)
    assert np.array_equal(syn.bf16_to_f32(x).astype(np.float64), vals)  # the grid is exact in bf16
    codes, S = orc.mx8_quantize(x)
    assert np.array_equal(S.astype(np.int64), X + 127)
    assert np.array_equal(orc.mx8_dequant(codes, S), vals)


def test_gemm_exact_vs_fraction_brute_force(orc):
    rng = np.random.default_rng(5)
    a = syn.normal_bf16(5, 1, 3, 64, 1.0, np.exp(2 * rng.standard_normal(64)))
    w = syn.normal_bf16(5, 2, 2, 64, 0.02)
    ac, aS = orc.mx8_quantize(a)
    wc, wS = orc.mx8_quantize(w)
    y, ad = orc.mx8_gemm(ac, aS, wc, wS)
    for m in range(3):
        for n in range(2):
            s = Fraction(0)
            sa = Fraction(0)
            for k in range(64):
                p = (Fraction(e4m3_value(int(ac[m, k]))) * 2 ** (int(aS[m, k // 32]) - 127) *
                     Fraction(e4m3_value(int(wc[n, k]))) * 2 ** (int(wS[n, k // 32]) - 127))
                s += p
                sa += abs(p)
            assert abs(Fraction(y[m, n]) - s) <= sa * Fraction(1, 2 ** 50)
            assert ad[m, n] == pytest.approx(float(sa), rel=1e-15)


def test_gemm_matches_dequantized_float_matmul(orc):
    a = syn.normal_bf16(6, 1, 16, 256, 1.0)
    w = syn.normal_bf16(6, 2, 24, 256, 0.02)
    ac, aS = orc.mx8_quantize(a)
    wc, wS = orc.mx8_quantize(w)
    y, ad = orc.mx8_gemm(ac, aS, wc, wS)
    ref = orc.mx8_dequant(ac, aS) @ orc.mx8_dequant(wc, wS).T
    assert np.all(np.abs(y - ref) <= 1e-12 * ad)
