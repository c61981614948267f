"""Pins of the oracle's MXFP8 A8W8 reading (the "MXFP A8w8" row of the accuracy table in section 六
of "Qwen3-Next-80B-A3B-Instruct 在 AMCT 中的 MoE 混合注意力量化适配实战"), read as the OCP
Microscaling FP8 format: blocks of 32 values along K, one E8M0 power-of-two scale per block, E4M3
elements.

Each test checks the oracle against something other than itself: torch's own float8_e4m3fn
type (decode of every byte, rounding of in-range values), hand-worked rounding cases, the shared
exponent recomputed with Python's math module, and an exact-rational brute force of the GEMM.
"""
import math
from fractions import Fraction

import numpy as np
import torch

from oracle import w8a8_oracle as O


def bits(v):
    return O.f32_to_bf16(np.asarray(v, np.float32))


def test_e4m3_decode_matches_torch_for_every_byte():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(codes)
    theirs = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = (codes & 0x7F) == 0x7F
    assert np.all(np.isnan(ours[nan])) and np.all(np.isnan(theirs[nan]))
    np.testing.assert_array_equal(ours[~nan], theirs[~nan])
    assert O.e4m3_decode(np.array([0x7E], np.uint8))[0] == 448.0
    assert O.e4m3_decode(np.array([0x01], np.uint8))[0] == 2.0 ** -9  # smallest subnormal


def test_e4m3_encode_round_trips_every_finite_value():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = O.e4m3_decode(codes)
    enc = O.e4m3_encode(vals)
    # +0 / -0 keep their sign bit; every other value returns its own byte
    np.testing.assert_array_equal(enc, codes)


def test_e4m3_encode_rounds_to_nearest_even_and_saturates():
    cases = {
        1.0625: 1.0,               # halfway between 1 (mantissa 0) and 1.125 (mantissa 1): even
        1.1875: 1.25,              # halfway between 1.125 and 1.25 (mantissa 2): even
        1.1: 1.125,
        2.0 ** -10: 0.0,           # half the smallest subnormal: to zero (even)
        3 * 2.0 ** -10: 2.0 ** -8,  # halfway between subnormals 1 and 2: even (2)
        0.0146484375: 0.015625,    # 15 * 2**-10, halfway between 7 * 2**-9 and 2**-6 (the first normal): even
        432.0: 448.0,              # halfway between 416 (mantissa 5) and 448 (mantissa 6): even
        440.0: 448.0,
        464.0: 448.0,              # above the largest value: saturates
        1.0e6: 448.0,
    }
    for v, want in cases.items():
        for sgn in (1.0, -1.0):
            got = O.e4m3_decode(O.e4m3_encode(np.array([sgn * v])))[0]
            assert got == sgn * want, (sgn * v, got, sgn * want)
    assert O.e4m3_encode(np.array([-0.0]))[0] == 0x80
    assert O.e4m3_encode(np.array([-1.0e-9]))[0] == 0x80  # a negative value rounding to zero keeps its sign


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(20000) * s for s in (2.0 ** -8, 0.01, 1.0, 30.0, 200.0)])
    v = v[np.abs(v) <= 448.0]
    ours = O.e4m3_decode(O.e4m3_encode(v))
    theirs = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, theirs)


def test_shared_exponent_and_saturation_of_the_largest_element():
    rng = np.random.default_rng(5)
    R, K = 6, 128
    v = rng.standard_normal((R, K)) * np.exp2(rng.integers(-20, 20, (R, 1)))
    v[0, :32] = 0.0                # an all-zero block
    v[1, :32] = 1.0                # amax exactly 1: E = -8, every element 256
    v[2, :32] = 0.5
    v[2, 5] = 1.9                  # 1.9 * 2**8 = 486.4: clips to 448
    vb = bits(v)
    codes, scales = O.mx_quantize_rows(vb)
    vf = O.bf16_to_f32(vb).astype(np.float64)
    for r in range(R):
        for b in range(K // 32):
            amax = float(np.abs(vf[r, 32 * b:32 * b + 32]).max())
            e = -127 if amax == 0 else max(-127, min(127, math.frexp(amax)[1] - 1 - 8))
            assert scales[r, b] == e + 127, (r, b)
    assert scales[0, 0] == 0 and np.all(codes[0, :32] == 0)
    assert scales[1, 0] == 127 - 8 and np.all(O.e4m3_decode(codes[1, :32]) == 256.0)
    assert O.e4m3_decode(codes[2, 5:6])[0] == 448.0
    assert O.e4m3_decode(codes[2, 0:1])[0] == 0.5 * 2.0 ** 8


def test_dequantised_values_are_within_half_an_e4m3_step():
    rng = np.random.default_rng(9)
    v = bits(rng.standard_normal((16, 256)) * 3.0)
    codes, scales = O.mx_quantize_rows(v)
    d = O.mx_dequantize(codes, scales)
    vf = O.bf16_to_f32(v).astype(np.float64)
    X = np.repeat(np.exp2(scales.astype(np.float64) - 127.0), 32, axis=1)
    r = vf / X
    clipped = np.abs(r) > 448.0
    # away from the clip: |error| <= half the local quantum 2**(floor(log2|r|) - 3), or 2**-10 below
    # the normal range, in units of X
    _, ex = np.frexp(np.where(np.abs(r) > 0, np.abs(r), 1.0))
    half_q = np.exp2(np.maximum(ex - 1, -6).astype(np.float64) - 4.0)
    assert np.all(np.abs(d - vf)[~clipped] <= (half_q * X)[~clipped])
    assert np.all(np.abs(d[clipped]) == 448.0 * X[clipped])


def test_linear_mxfp8_brute_force_exact():
    rng = np.random.default_rng(13)
    M, K, N = 3, 64, 4
    x = bits(rng.standard_normal((M, K)) * np.where(np.arange(K) == 9, 20.0, 1.0))
    w = bits(rng.standard_normal((N, K)) * 0.05)
    wc, ws = O.mx_quantize_rows(w)
    out = O.linear_mxfp8(x, wc, ws)
    xc, xs = out["codes"], out["scales"]

    def val(code, scale):  # exact rational value of one element
        c = int(code)
        sgn = -1 if c & 0x80 else 1
        e, m = (c >> 3) & 0xF, c & 7
        mag = Fraction(m, 8) * Fraction(1, 2 ** 6) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        return sgn * mag * Fraction(2) ** (int(scale) - 127)

    for t in range(M):
        for n in range(N):
            exact = sum(val(xc[t, k], xs[t, k // 32]) * val(wc[n, k], ws[n, k // 32]) for k in range(K))
            assert float(exact) == out["y"][t, n]
    # the bound covers an fp32 summation in order followed by one bf16 rounding
    A = O.mx_dequantize(xc, xs).astype(np.float32)
    W = O.mx_dequantize(wc, ws).astype(np.float32)
    acc = np.zeros((M, N), np.float32)
    for k in range(K):
        acc = (acc + A[:, k:k + 1] * W[:, k][None, :]).astype(np.float32)
    y_bf16 = O.bf16_to_f32(O.f32_to_bf16(acc)).astype(np.float64)
    assert np.all(np.abs(y_bf16 - out["y"]) <= out["bound"])
