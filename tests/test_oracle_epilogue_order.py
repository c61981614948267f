"""Pins of the oracle's epilogue arithmetic against exact rational restatements.

The pages fix the scales (per-token activation scale, per-output-channel weight scale; the
group_0 block of "Qwen3.6-35B-A3B-w8a8量化配置深度解读：config.json与recipe.yaml关键参数解析")
and that the k selected experts' outputs are weighted and summed ("Qwen3-30B-A3B-Instruct-2507-
quantized.w8a8", section 三 3.1), but not the order of the fp32 operations. The readings are:

* dequant: ((float)acc * s_row) * s_col, with the int32 -> fp32 conversion and each product
  rounded to nearest, ties to even;
* combine: acc = 0; acc = fma(w[t, j], o[t, j, n], acc) for j = 0 .. k-1; y = bf16(acc).

Each test restates the reading with Python's exact rationals (one explicit rounding per step,
by integer arithmetic) and checks the oracle bit for bit. It also checks that the plausible
mis-readings (a single fused scale, the other product order, two roundings per slot, the
reversed slot order, one rounding of the exact sum) give different bits on the same inputs,
so that the pin can tell them apart.
"""
from fractions import Fraction

import numpy as np

from oracle import w8a8_oracle as O


def round_exact(fr, mant_bits):
    """Nearest binary float with `mant_bits` significand bits (ties to even) of an exact
    rational, with the fp32 / bf16 exponent range (subnormals below 2^-126). Returns a Fraction."""
    fr = Fraction(fr)
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    if Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)  # subnormal range: fixed quantum 2^(-126 - (mant_bits - 1))
    quantum = Fraction(2) ** (e - (mant_bits - 1))
    q, rem = divmod(a / quantum, 1)
    q = int(q)
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and q % 2 == 1):
        q += 1
    out = q * quantum
    assert out < Fraction(2) ** 128, "overflow is outside these tests"
    return sign * out


def f32(fr):
    return round_exact(fr, 24)


def bf16(fr):
    return round_exact(fr, 8)  # bf16 keeps fp32's exponent range and 8 significand bits


def as_f32(fr) -> np.float32:
    return np.float32(float(fr))  # exact: fr is an fp32 value


def _scales(rng, n, spread):
    # amax / 127 style scales: fp32 quotients of bf16 maxima
    amax = O.bf16_to_f32(O.f32_to_bf16(np.abs(rng.standard_normal(n)).astype(np.float32) * spread + 1e-3))
    return (amax / np.float32(127.0)).astype(np.float32)


def test_dequant_is_two_rounded_products_in_token_then_channel_order():
    rng = np.random.default_rng(5)
    R, C = 24, 40
    # int32 accumulators up to 127*127*4096 (beyond 2^24, so the conversion itself rounds)
    acc = rng.integers(-(127 * 127 * 4096), 127 * 127 * 4096, (R, C)).astype(np.int32)
    acc[0, :8] = [2 ** 24 + 1, 2 ** 24 + 3, -(2 ** 25 + 2), 2 ** 25 + 6, 1, -1, 0, 127 * 127 * 4096 - 1]
    s_row = _scales(rng, R, 20.0)
    s_col = _scales(rng, C, 0.06)
    got = O.dequant(acc, s_row, s_col)
    want = np.empty((R, C), np.float32)
    alt_fused = np.empty((R, C), np.float32)
    alt_swapped = np.empty((R, C), np.float32)
    for r in range(R):
        for c in range(C):
            a = f32(int(acc[r, c]))  # int32 -> fp32, round to nearest even
            sr, sc = Fraction(float(s_row[r])), Fraction(float(s_col[c]))
            want[r, c] = as_f32(f32(f32(a * sr) * sc))
            alt_fused[r, c] = as_f32(f32(a * f32(sr * sc)))
            alt_swapped[r, c] = as_f32(f32(f32(a * sc) * sr))
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
    # the pin separates the reading from the plausible alternatives
    assert np.any(alt_fused.view(np.uint32) != want.view(np.uint32))
    assert np.any(alt_swapped.view(np.uint32) != want.view(np.uint32))
    # the int32 -> fp32 conversion rounds to nearest even (2^24 + 1 -> 2^24, 2^24 + 3 -> 2^24 + 4)
    assert float(f32(2 ** 24 + 1)) == 2.0 ** 24 and float(f32(2 ** 24 + 3)) == 2.0 ** 24 + 4


def test_dequant_inside_linear_w8a8():
    # the dense W8A8 linear applies the same dequant to its int32 GEMM, then rounds to bf16
    rng = np.random.default_rng(9)
    M, K, N = 5, 256, 7
    x = O.f32_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    w = O.f32_to_bf16((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    wq, sw = O.quantize_weight_per_channel(w)
    xq, sx = O.quant_act_per_token(x)
    y = O.linear_w8a8(x, wq, sw)
    for m in range(M):
        for n in range(N):
            acc = sum(int(xq[m, i]) * int(wq[n, i]) for i in range(K))
            v = bf16(f32(f32(f32(acc) * Fraction(float(sx[m]))) * Fraction(float(sw[n]))))
            assert O.bf16_to_f32(y[m:m + 1, n])[0] == float(v)


def _chain_exact(o, w, order, fused=True):
    """fp32 accumulator of the weighted sum over the slots in `order`; fused: one rounding per
    slot (an fma), else the product and the sum each rounded."""
    T, k, H = o.shape
    out = np.empty((T, H), np.float32)
    for t in range(T):
        for n in range(H):
            acc = Fraction(0)
            for j in order:
                prod = Fraction(float(w[t, j])) * Fraction(float(o[t, j, n]))
                acc = f32(prod + acc) if fused else f32(f32(prod) + acc)
            out[t, n] = as_f32(acc)
    return out


def _combine_inputs(rng, T, k, H):
    o_bits = O.f32_to_bf16((rng.standard_normal((T, k, H)) * np.exp2(rng.integers(-3, 4, (T, k, H)))).astype(
        np.float32))
    p = np.exp(rng.standard_normal((T, k)))
    w = (p / p.sum(1, keepdims=True)).astype(np.float32)
    return o_bits, w


def test_combine_accumulator_is_an_fma_chain_in_slot_order_from_zero():
    rng = np.random.default_rng(17)
    T, k, H = 6, 8, 48
    o_bits, w = _combine_inputs(rng, T, k, H)
    o = O.bf16_to_f32(o_bits)
    got = O.combine_acc(o_bits, w)
    want = _chain_exact(o, w, range(k))
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
    # alternatives that a different reading would produce differ on these inputs
    two_round = _chain_exact(o, w, range(k), fused=False)
    reverse = _chain_exact(o, w, range(k - 1, -1, -1))
    exact_sum = np.array([[as_f32(f32(sum(Fraction(float(w[t, j])) * Fraction(float(o[t, j, n]))
                                          for j in range(k)))) for n in range(H)] for t in range(T)], np.float32)
    for alt in (two_round, reverse, exact_sum):
        assert np.any(alt.view(np.uint32) != want.view(np.uint32))


def test_combine_output_is_the_accumulator_rounded_once_to_bf16():
    rng = np.random.default_rng(23)
    o_bits, w = _combine_inputs(rng, 5, 3, 64)
    acc = O.combine_acc(o_bits, w)
    y = O.bf16_to_f32(O.combine(o_bits, w))
    want = np.array([as_f32(bf16(Fraction(float(v)))) for v in acc.reshape(-1)], np.float32).reshape(acc.shape)
    np.testing.assert_array_equal(y.view(np.uint32), want.view(np.uint32))


def test_combine_with_three_slots_and_designed_cancellation():
    # k = 3: w0*o0 + w1*o1 cancels to about 2^-14 while neither product is an fp32 number, so
    # the result hangs on where the products are rounded and on the slot order:
    # fma chain 6.168336e-05, two roundings per slot 6.169081e-05, reversed order 6.168522e-05
    w = np.array([[float.fromhex("0x1.00003cp-1"), float.fromhex("0x1.00003p-2"), 0.25]], np.float32)
    o_vals = np.array([[[1.796875], [-3.59375], [2.0 ** -12]]], np.float32)
    o_bits = O.f32_to_bf16(o_vals)
    o = O.bf16_to_f32(o_bits)
    np.testing.assert_array_equal(o, o_vals)  # bf16 values
    got = O.combine_acc(o_bits, w)
    want = _chain_exact(o, w, range(3))
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
    assert _chain_exact(o, w, range(3), fused=False)[0, 0] != want[0, 0]
    assert _chain_exact(o, w, range(2, -1, -1))[0, 0] != want[0, 0]
