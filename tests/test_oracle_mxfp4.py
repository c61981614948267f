"""Pins of the oracle's MXFP A8W4 reading (the "MXFP A8w4" row of the accuracy table in section 六
of "Qwen3-Next-80B-A3B-Instruct 在 AMCT 中的 MoE 混合注意力量化适配实战"), read as the OCP
Microscaling formats: MXFP8 activations and MXFP4 weights (blocks of 32 values along K, one E8M0
power-of-two scale per block, FP4 E2M1 elements, two per byte).

Each test checks the oracle against something other than itself: the E2M1 value table written out
by hand, the ml_dtypes package's own float4_e2m1fn type (decode and rounding), a brute-force
nearest-value search, the shared exponent recomputed with Python's math module, hand-built packed
bytes, and an exact-rational brute force of the GEMM.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import w8a8_oracle as O

# the eight non-negative E2M1 magnitudes, in code order 0..7
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def bits(v):
    return O.f32_to_bf16(np.asarray(v, np.float32))


def test_e2m1_decode_matches_the_format_table():
    codes = np.arange(16, dtype=np.uint8)
    got = O.e2m1_decode(codes)
    np.testing.assert_array_equal(got[:8], E2M1_TABLE)
    np.testing.assert_array_equal(got[8:], [-v for v in E2M1_TABLE])
    assert np.signbit(got[8])  # code 0x8 is -0
    # only the low nibble of a byte is a code
    np.testing.assert_array_equal(O.e2m1_decode(codes | 0xF0), got)


def test_e2m1_codec_matches_ml_dtypes():
    ml_dtypes = pytest.importorskip("ml_dtypes")
    codes = np.arange(16, dtype=np.uint8)
    theirs = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(O.e2m1_decode(codes), theirs)
    rng = np.random.default_rng(21)
    # every midpoint, points around them, and random values, inside and beyond the range
    # (fp32 values: ml_dtypes converts from fp32)
    mids = np.array([(a + b) / 2 for a, b in zip(E2M1_TABLE, E2M1_TABLE[1:])], np.float32)
    v = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(10)),
                        rng.uniform(-8, 8, 20000).astype(np.float32),
                        (rng.standard_normal(5000) * 0.3).astype(np.float32),
                        np.array([6.0, 6.5, 7.9, 100.0], np.float32)])
    v = np.concatenate([v, -v])
    ours = O.e2m1_decode(O.e2m1_encode(v.astype(np.float64)))
    ref = v.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(ours, ref)


def test_e2m1_encode_is_the_nearest_value_with_ties_to_even():
    rng = np.random.default_rng(4)
    v = np.concatenate([rng.uniform(0, 7, 4000), np.arange(0, 6.25, 0.125)])
    enc = O.e2m1_encode(v)
    table = np.array(E2M1_TABLE)
    for x, c in zip(v, enc):
        d = np.abs(table - min(x, 6.0))
        best = np.flatnonzero(d == d.min())
        # one nearest value, or a tie between two neighbours: the even code (mantissa bit 0) wins
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert c == want, (x, c, want)


def test_e2m1_encode_hand_cases():
    cases = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0, 5.5: 6.0, 6.0: 6.0,
             7.0: 6.0, 1.0e9: 6.0, 0.2: 0.0, 0.3: 0.5}
    for v, want in cases.items():
        for sgn in (1.0, -1.0):
            got = O.e2m1_decode(O.e2m1_encode(np.array([sgn * v])))[0]
            assert got == sgn * want, (sgn * v, got, sgn * want)
    assert O.e2m1_encode(np.array([-0.0]))[0] == 0x8
    assert O.e2m1_encode(np.array([-0.1]))[0] == 0x8  # a negative value rounding to zero keeps its sign


def test_mx4_shared_exponent_packing_and_saturation():
    rng = np.random.default_rng(8)
    R, K = 6, 128
    v = rng.standard_normal((R, K)) * np.exp2(rng.integers(-20, 20, (R, 1)))
    v[0, :32] = 0.0                                # an all-zero block
    v[1, :32] = np.tile([0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.5], 4)  # amax 6: E = 0, exact codes
    v[2, :32] = 1.0
    v[2, 5] = 7.5                                  # amax 7.5: E = 0, 7.5 clips to 6
    vb = bits(v)
    packed, scales = O.mx4_quantize_rows(vb)
    assert packed.shape == (R, K // 2) and scales.shape == (R, K // 32)
    vf = O.bf16_to_f32(vb).astype(np.float64)
    for r in range(R):
        for b in range(K // 32):
            amax = float(np.abs(vf[r, 32 * b:32 * b + 32]).max())
            e = -127 if amax == 0 else max(-127, min(127, math.frexp(amax)[1] - 1 - 2))
            assert scales[r, b] == e + 127, (r, b)
    assert scales[0, 0] == 0 and np.all(packed[0, :16] == 0)
    # row 1: codes 1, 2, 3, 4, 5, 6, 7, 9 repeating; the even element sits in the low nibble
    assert scales[1, 0] == 127
    np.testing.assert_array_equal(packed[1, :4], [0x21, 0x43, 0x65, 0x97])
    np.testing.assert_array_equal(O.mx4_dequantize(packed, scales)[1, :8], [0.5, 1, 1.5, 2, 3, 4, 6, -0.5])
    assert scales[2, 0] == 127 and O.mx4_dequantize(packed, scales)[2, 5] == 6.0


def test_mx4_dequantised_values_are_within_half_a_step():
    rng = np.random.default_rng(10)
    v = bits(rng.standard_normal((16, 256)) * 0.02)
    packed, scales = O.mx4_quantize_rows(v)
    d = O.mx4_dequantize(packed, scales)
    vf = O.bf16_to_f32(v).astype(np.float64)
    X = np.repeat(np.exp2(scales.astype(np.float64) - 127.0), 32, axis=1)
    r = vf / X
    clipped = np.abs(r) > 6.0
    # away from the clip: |error| <= half the local quantum (0.25 below 2, 0.5 in [2, 4), 1 in [4, 6])
    half_q = np.where(np.abs(r) < 2, 0.25, np.where(np.abs(r) < 4, 0.5, 1.0))
    assert np.all(np.abs(d - vf)[~clipped] <= (half_q * X)[~clipped])
    assert np.all(np.abs(d[clipped]) == 6.0 * X[clipped])


def test_linear_mxfp_a8w4_brute_force_exact():
    rng = np.random.default_rng(17)
    M, K, N = 3, 64, 4
    x = bits(rng.standard_normal((M, K)) * np.where(np.arange(K) == 5, 30.0, 1.0))
    w = bits(rng.standard_normal((N, K)) * 0.05)
    wp, ws = O.mx4_quantize_rows(w)
    out = O.linear_mxfp_a8w4(x, wp, ws)
    xc, xs = out["codes"], out["scales"]

    def e4m3(code, scale):  # exact rational value of an MXFP8 element
        c = int(code)
        sgn = -1 if c & 0x80 else 1
        e, m = (c >> 3) & 0xF, c & 7
        mag = Fraction(m, 8) * Fraction(1, 2 ** 6) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        return sgn * mag * Fraction(2) ** (int(scale) - 127)

    def e2m1(byte, k, scale):  # exact rational value of an MXFP4 element, read from its byte
        c = (int(byte) >> (4 * (k & 1))) & 0xF
        sgn = -1 if c & 0x8 else 1
        e, m = (c >> 1) & 3, c & 1
        mag = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
        return sgn * mag * Fraction(2) ** (int(scale) - 127)

    for t in range(M):
        for n in range(N):
            exact = sum(e4m3(xc[t, k], xs[t, k // 32]) * e2m1(wp[n, k // 2], k, ws[n, k // 32]) for k in range(K))
            assert float(exact) == out["y"][t, n]
    # the bound covers an fp32 summation in order followed by one bf16 rounding
    A = O.mx_dequantize(xc, xs).astype(np.float32)
    W = O.mx4_dequantize(wp, ws).astype(np.float32)
    acc = np.zeros((M, N), np.float32)
    for k in range(K):
        acc = (acc + A[:, k:k + 1] * W[:, k][None, :]).astype(np.float32)
    y_bf16 = O.bf16_to_f32(O.f32_to_bf16(acc)).astype(np.float64)
    assert np.all(np.abs(y_bf16 - out["y"]) <= out["bound"])
