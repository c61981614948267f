"""Pins of the oracle's shared-expert path (the Qwen3-Next / Qwen3.6 MoE layers).

The pages fix that the shared expert is a dense path quantised W8A8 directly ("Qwen3-Next-80B-A3B-
Instruct 在 AMCT 中的 MoE 混合注意力量化适配实战", section 二 2.2) and that shared_expert_gate stays
bf16 (the ignore list of "Qwen3.6-35B-A3B-w8a8量化配置深度解读：config.json与recipe.yaml关键参数解析").
The combination y = routed + sigmoid(x . w_sg) * shared, with the shared output entering the
combine's fma chain after the k routed slots, is the reading the oracle states. Each test checks
it against a restatement that does not go through the oracle's vectorised helpers.
"""
from fractions import Fraction

import numpy as np

from oracle import w8a8_oracle as O
from tests.test_oracle_epilogue_order import as_f32, bf16, f32


def bits(v):
    return O.f32_to_bf16(np.asarray(v, np.float32))


def _shared_weights(rng, H, Is):
    wgu = bits(rng.standard_normal((2 * Is, H)) * 0.05)
    wd = bits(rng.standard_normal((H, Is)) * 0.05)
    gq, gs = O.quantize_weight_per_channel(wgu)
    dq, ds = O.quantize_weight_per_channel(wd)
    return gq, gs, dq, ds


def test_combine_with_shared_is_the_chain_then_one_more_fma():
    rng = np.random.default_rng(31)
    T, k, H = 4, 3, 40
    o_bits = bits(rng.standard_normal((T, k, H)))
    p = np.exp(rng.standard_normal((T, k)))
    w = (p / p.sum(1, keepdims=True)).astype(np.float32)
    o_s_bits = bits(rng.standard_normal((T, H)) * 4)
    g = rng.uniform(0, 1, T).astype(np.float32)
    got = O.combine_acc_with_shared(o_bits, w, o_s_bits, g)
    o, o_s = O.bf16_to_f32(o_bits), O.bf16_to_f32(o_s_bits)
    want = np.empty((T, H), np.float32)
    shared_first = np.empty((T, H), np.float32)
    for t in range(T):
        for n in range(H):
            acc = Fraction(0)
            for j in range(k):
                acc = f32(Fraction(float(w[t, j])) * Fraction(float(o[t, j, n])) + acc)
            acc = f32(Fraction(float(g[t])) * Fraction(float(o_s[t, n])) + acc)
            want[t, n] = as_f32(acc)
            acc = f32(Fraction(float(g[t])) * Fraction(float(o_s[t, n])))
            for j in range(k):
                acc = f32(Fraction(float(w[t, j])) * Fraction(float(o[t, j, n])) + acc)
            shared_first[t, n] = as_f32(acc)
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
    assert np.any(shared_first.view(np.uint32) != want.view(np.uint32))  # the order is pinned
    # the layer output is that accumulator rounded once to bf16
    y = O.bf16_to_f32(O.combine_with_shared(o_bits, w, o_s_bits, g))
    np.testing.assert_array_equal(y, O.bf16_to_f32(O.f32_to_bf16(want)))


def test_shared_gate_closed_forms():
    rng = np.random.default_rng(5)
    H = 64
    wsg = bits(rng.standard_normal(H) * 0.1)
    x = bits(rng.standard_normal((6, H)))
    g = O.shared_gate(x, wsg)
    assert O.shared_gate(np.zeros((2, H), np.uint16), wsg).tolist() == [0.5, 0.5]  # z = 0
    g_neg = O.shared_gate(x ^ np.uint16(0x8000), wsg)  # negated tokens: z -> -z
    np.testing.assert_allclose(g + g_neg, 1.0, rtol=0, atol=1e-15)
    z = O.bf16_to_f32(x).astype(np.float64) @ O.bf16_to_f32(wsg).astype(np.float64)
    np.testing.assert_allclose(g, 1.0 / (1.0 + np.exp(-z)), rtol=1e-15)
    big = bits(np.full((1, H), 8.0))
    assert O.shared_gate(big, bits(np.full(H, 1.0)))[0] == 1.0  # z = 512: saturates


def test_shared_expert_brute_force_tiny():
    """Integer GEMMs by Python ints, every fp32 step written out scalar by scalar."""
    rng = np.random.default_rng(11)
    T, H, Is = 3, 128, 32
    x = bits(rng.standard_normal((T, H)) * np.where(np.arange(H) == 7, 20.0, 1.0))
    gq, gs, dq, ds = _shared_weights(rng, H, Is)
    sh = O.shared_expert(x, gq, gs, dq, ds)
    xv = O.bf16_to_f32(x)
    for t in range(T):
        amax = max(abs(float(v)) for v in xv[t])
        sx = np.float32(np.float32(amax) / np.float32(127.0))
        xq = [int(np.clip(np.rint(np.float32(float(v)) / sx), -127, 127)) for v in xv[t]]
        assert xq == sh["xq"][t].tolist() and sx == sh["sx"][t]
        h = []
        for c in range(Is):
            ag = sum(xq[i] * int(gq[c, i]) for i in range(H))
            au = sum(xq[i] * int(gq[Is + c, i]) for i in range(H))
            gval = np.float32(np.float32(np.float32(ag) * sx) * gs[c])
            uval = np.float32(np.float32(np.float32(au) * sx) * gs[Is + c])
            silu = np.float32(gval / np.float32(np.float32(1.0) + O.spec_exp(np.float32(-gval))))
            h.append(O.f32_to_bf16(np.float32(silu * uval)))
        assert np.array_equal(np.array(h, np.uint16), sh["h"][t])
        hv = O.bf16_to_f32(np.array(h, np.uint16))
        sh_t = np.float32(np.float32(max(abs(float(v)) for v in hv)) / np.float32(127.0))
        hq = [int(np.clip(np.rint(np.float32(v) / sh_t), -127, 127)) if sh_t > 0 else 0 for v in hv]
        assert hq == sh["hq"][t].tolist() and sh_t == sh["s_h"][t]
        for n in range(H):
            a = sum(hq[i] * int(dq[n, i]) for i in range(Is))
            o = O.f32_to_bf16(np.float32(np.float32(np.float32(a) * sh_t) * ds[n]))
            assert o == sh["o"][t, n]


def test_layer_with_shared_expert_reduces_to_routed_when_the_gate_is_zero():
    rng = np.random.default_rng(2)
    T, H, E, k, I, Is = 6, 128, 4, 2, 64, 32
    x = bits(rng.standard_normal((T, H)))
    wg = bits(rng.standard_normal((E, H)) * 0.05)
    wgu = bits(rng.standard_normal((E, 2 * I, H)) * 0.05)
    wd = bits(rng.standard_normal((E, H, I)) * 0.05)
    q = O.quantize_experts(wgu, wd)
    sq = _shared_weights(rng, H, Is)
    wsg = bits(rng.standard_normal(H) * 0.05)
    full = O.moe_forward_shared(x, wg, None, *q, k, wsg, *sq)
    routed = O.moe_forward(x, wg, None, *q, k)
    zero = O.moe_forward_shared(x, wg, None, *q, k, wsg, *sq, gate=np.zeros(T, np.float32))
    np.testing.assert_array_equal(O.bf16_to_f32(zero["y"]), O.bf16_to_f32(routed["y"]))
    assert not np.array_equal(full["y"], routed["y"])
    # the shared output is that of one routed expert that every token selects with weight 1
    single = O.moe_forward(x, wg[:1], None, sq[0][None], sq[1][None], sq[2][None], sq[3][None], 1)
    np.testing.assert_array_equal(full["shared"]["o"], single["o"][:, 0])
