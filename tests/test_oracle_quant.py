"""Pins for the oracle's quantisers, exponential and SiLU (CPU only).

Each check rests on something other than the oracle's own formula: the scheme the pages
state (tests/golden/quant_scheme.txt), closed forms, exact special cases, error bounds and
the C library's exponential.
"""
import math
import os
import struct

import numpy as np
import pytest

from oracle import w8a8_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = (s.strip() for s in line.split("=", 1))
            out[k] = v
    return out


def bf16(vals):
    return O.f32_to_bf16(np.asarray(vals, np.float32))


# ------------------------------------------------------------------ scheme from the pages
def test_scheme_constants_follow_the_pages():
    g = _golden("quant_scheme.txt")
    assert g["weights.symmetric"] == g["activations.symmetric"] == "true"
    assert O.Q_MAX_INT8 == 2 ** (int(g["weights.num_bits"]) - 1) - 1
    assert O.Q_MAX_INT8 == 2 ** (int(g["activations.num_bits"]) - 1) - 1
    assert O.Q_MAX_INT4 == 2 ** (int(g["w4.num_bits"]) - 1) - 1


def test_weight_scale_is_per_output_channel_and_static():
    g = _golden("quant_scheme.txt")
    assert g["weights.strategy"] == "channel" and g["weights.dynamic"] == "false"
    rng = np.random.default_rng(1)
    w = rng.standard_normal((3, 5, 64)).astype(np.float32)
    w[1, 2] *= 50  # one output channel much larger than the rest
    q, s = O.quantize_weight_per_channel(bf16(w))
    assert q.shape == (3, 5, 64) and s.shape == (3, 5)
    assert s[1, 2] > 20 * np.median(s)  # its own scale, nobody else's
    assert np.all(np.abs(q).max(axis=-1) == 127)  # every channel reaches the full range


def test_activation_scale_is_per_token():
    g = _golden("quant_scheme.txt")
    assert g["activations.strategy"] == "token" and g["activations.dynamic"] == "true"
    x = np.ones((4, 32), np.float32)
    x[2] *= 1024.0
    q, s = O.quant_act_per_token(bf16(x))
    assert s.shape == (4,)
    np.testing.assert_array_equal(q, np.full((4, 32), 127, np.int8))
    assert s[2] == s[0] * 1024  # scales follow each token, exact power-of-two ratio


def test_int4_group_size_and_twos_complement():
    g = _golden("quant_scheme.txt")
    group = int(g["w4.group_size"])
    assert g["w4.encoding"] == "twos_complement"
    # designed bytes: low nibble is the even code, high nibble the odd code
    packed = np.array([[0x9F, 0x07, 0x10, 0xE2]], np.uint8)
    np.testing.assert_array_equal(O.unpack_int4(packed)[0], [-1, -7, 7, 0, 0, 1, 2, -2])
    rng = np.random.default_rng(2)
    w = rng.standard_normal((6, 4 * group)).astype(np.float32)
    w[:, group:2 * group] *= 16  # second group much larger
    p, s = O.quantize_weight_int4_per_group(bf16(w), group)
    assert p.shape == (6, 2 * group) and s.shape == (6, 4)
    assert np.all(s[:, 1] > 8 * s[:, 0])
    codes = O.unpack_int4(p)
    assert codes.min() >= -7 and codes.max() <= 7
    for gi in range(4):  # each group reaches +-7 in every row
        assert np.all(np.abs(codes[:, gi * group:(gi + 1) * group]).max(axis=1) == 7)


# ------------------------------------------------------------------ exact special cases
def test_integer_rows_round_trip_exactly():
    rng = np.random.default_rng(3)
    v = rng.integers(-127, 128, size=(50, 96)).astype(np.float32)
    v[:, 7] = np.where(rng.random(50) < 0.5, 127, -127)  # amax = 127 in every row
    q, s = O.symmetric_quantize_rows(v, O.Q_MAX_INT8)
    np.testing.assert_array_equal(s, np.ones(50, np.float32))
    np.testing.assert_array_equal(q.astype(np.float32), v)


@pytest.mark.parametrize("m", [-20, -3, 0, 5, 40])
def test_power_of_two_scaling(m):
    rng = np.random.default_rng(4)
    v = rng.standard_normal((8, 64)).astype(np.float32)
    q0, s0 = O.symmetric_quantize_rows(v, O.Q_MAX_INT8)
    q1, s1 = O.symmetric_quantize_rows(v * np.float32(2.0 ** m), O.Q_MAX_INT8)
    np.testing.assert_array_equal(q0, q1)
    np.testing.assert_array_equal(s1, s0 * np.float32(2.0 ** m))


def test_round_half_to_even():
    v = np.array([[127, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, 126.5]], np.float32)
    q, s = O.symmetric_quantize_rows(v, O.Q_MAX_INT8)
    assert s[0] == 1.0
    np.testing.assert_array_equal(q[0], [127, 0, 2, 2, 0, -2, -2, 4, 126])


def test_zero_row_and_negation():
    v = np.zeros((2, 16), np.float32)
    v[1] = np.linspace(-3, 5, 16)
    q, s = O.symmetric_quantize_rows(v, O.Q_MAX_INT8)
    assert s[0] == 0 and not q[0].any()
    qn, sn = O.symmetric_quantize_rows(-v, O.Q_MAX_INT8)
    np.testing.assert_array_equal(qn, -q)
    np.testing.assert_array_equal(sn, s)


def test_error_bound_and_range():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal((200, 128)) * rng.lognormal(0, 3, (200, 1))).astype(np.float32)
    q, s = O.symmetric_quantize_rows(v, O.Q_MAX_INT8)
    assert q.min() >= -127 and q.max() <= 127
    err = np.abs(v.astype(np.float64) - q.astype(np.float64) * s[:, None])
    assert np.all(err <= s[:, None] * (0.5 + 1e-6))
    np.testing.assert_array_equal(np.abs(q).max(axis=1), 127)


def _f32(x):
    return struct.unpack("f", struct.pack("f", x))[0]


def test_brute_force_scalar_quantiser():
    """Scalar re-derivation with Python floats: fp32 divide = correctly rounded f64 divide
    rounded to fp32 (exact for one operation); round() is half-to-even."""
    rng = np.random.default_rng(6)
    v = (rng.standard_normal((6, 40)) * 3).astype(np.float32)
    q, s = O.symmetric_quantize_rows(v, O.Q_MAX_INT8)
    for r in range(v.shape[0]):
        amax = max(abs(float(a)) for a in v[r])
        sr = _f32(amax / 127.0)
        assert sr == s[r]
        for c in range(v.shape[1]):
            qc = max(-127, min(127, round(_f32(float(v[r, c]) / sr))))
            assert qc == q[r, c]


# ------------------------------------------------------------------ exponential and SiLU
def _ulp_dist(a, b):
    ia = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    ib = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(ia - ib)


def test_spec_exp_against_libm():
    x = np.linspace(-87.0, 88.0, 200001, dtype=np.float32)
    x = np.concatenate([x, np.linspace(-1, 1, 20001, dtype=np.float32)])
    got = O.spec_exp(x)
    ref = np.array([math.exp(float(t)) for t in x], np.float64).astype(np.float32)
    assert _ulp_dist(got, ref).max() <= 2


def test_spec_exp_special_values():
    assert O.spec_exp(np.float32(0.0)) == 1.0
    assert np.isinf(O.spec_exp(np.float32(88.5)))
    assert O.spec_exp(np.float32(-90.0)) == 0.0
    x = np.sort(np.random.default_rng(7).uniform(-80, 80, 50000).astype(np.float32))
    assert np.all(np.diff(O.spec_exp(x).astype(np.float64)) >= 0)  # monotone


def test_silu_closed_forms():
    assert O.silu(np.float32(0.0)) == 0.0
    g = np.array([20.0, 25.5, 64.0, 1e4], np.float32)
    np.testing.assert_array_equal(O.silu(g), g)  # exp(-g) below half an ulp of 1
    assert np.all(O.silu(-g) <= 0) and np.all(np.abs(O.silu(-g)) < 1e-6)
    x = np.linspace(-30, 30, 60001, dtype=np.float32)
    ref = np.array([t / (1.0 + math.exp(-t)) for t in x.astype(np.float64)]).astype(np.float32)
    assert _ulp_dist(O.silu(x), ref).max() <= 4
    # silu(g) - silu(-g) = g
    np.testing.assert_allclose(O.silu(x).astype(np.float64) - O.silu(-x), x, atol=1e-5, rtol=1e-6)


def test_bf16_rounding():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -20], np.float32)
    back = O.bf16_to_f32(O.f32_to_bf16(v))
    np.testing.assert_array_equal(back, [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 1.0 + 2 ** -7])


# ------------------------------------------------------------------ fused multiply-add
def round_f32_exact(fr):
    """Nearest fp32 (ties to even) of an exact rational, by integer arithmetic (normal range)."""
    from fractions import Fraction
    if fr == 0:
        return 0.0
    sign = -1.0 if fr < 0 else 1.0
    fr = abs(Fraction(fr))
    e = fr.numerator.bit_length() - fr.denominator.bit_length()
    if Fraction(2) ** e > fr:
        e -= 1
    if Fraction(2) ** (e + 1) <= fr:
        e += 1
    scaled = fr / Fraction(2) ** (e - 23)  # in [2^23, 2^24)
    q, rem = divmod(scaled.numerator, scaled.denominator)
    twice = 2 * rem
    if twice > scaled.denominator or (twice == scaled.denominator and q % 2 == 1):
        q += 1
    return sign * float(q) * 2.0 ** (e - 23)


def _fma_exact(a, b, c):
    from fractions import Fraction
    return round_f32_exact(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def test_fma32_matches_exact_rational_rounding():
    rng = np.random.default_rng(21)
    n = 3000
    a = (rng.standard_normal(n) * np.exp2(rng.integers(-20, 20, n))).astype(np.float32)
    b = (rng.standard_normal(n) * np.exp2(rng.integers(-20, 20, n))).astype(np.float32)
    c = (rng.standard_normal(n) * np.exp2(rng.integers(-40, 40, n))).astype(np.float32)
    # designed hard cases: c cancels a*b to within an ulp, and products landing on fp32 ties
    # and double-rounding traps: a*b + c lies 2^-40 below an fp32 midpoint whose lower
    # neighbour is odd, so rounding to float64 first lands on the midpoint and ties-to-even
    # would pick the wrong neighbour
    a2 = np.array([1 + 2 ** -23, 1 + 2 ** -12, 3.0, 1 + 2 ** -23, 0.1, 8 + 2 ** -20, -(8 + 2 ** -20)], np.float32)
    b2 = np.array([1 - 2 ** -23, 1 + 2 ** -12, 1 / 3, 1 + 2 ** -23, 10.0, 8 - 2 ** -20, 8 - 2 ** -20], np.float32)
    c2 = np.array([-1.0, -1.0, -1.0, 2 ** -47, -1.0, 2 ** 30 + 128, -(2 ** 30 + 128)], np.float32)
    a, b, c = np.concatenate([a, a2]), np.concatenate([b, b2]), np.concatenate([c, c2])
    got = O.fma32(a, b, c)
    want = np.array([_fma_exact(x, y, z) for x, y, z in zip(a, b, c)], np.float32)
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
    # it is genuinely fused: differs from the two-rounding result on the cancellation cases
    two_step = (a2 * b2).astype(np.float32) + c2
    assert np.any(O.fma32(a2, b2, c2) != two_step)
