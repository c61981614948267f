"""Pins for the oracle's router, expert grouping, integer GEMM, MoE layer and dense linear.

Checks rest on closed forms, invariants, brute force on tiny inputs, the quantisation-off
error bound, and the sizes printed on the pages (tests/golden/model_sizes.txt).
"""
import math
import os

import numpy as np
import pytest

from oracle import w8a8_oracle as O
from w8a8_int8_quantized_act_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(vals):
    return O.f32_to_bf16(np.asarray(vals, np.float32))


def _golden(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = (s.strip() for s in line.split("=", 1))
            out[k] = float(v)
    return out


# ------------------------------------------------------------------ sizes from the pages
def test_workload_shapes_reproduce_page_sizes():
    g = _golden("model_sizes.txt")
    wl = synth.MOE_WORKLOADS["qwen3-30b-a3b-decode"]
    assert (wl.H, wl.E, wl.k) == (g["q30b.hidden"], g["q30b.experts"], g["q30b.top_k"])
    gate = wl.H * wl.E
    assert abs(gate - g["q30b.gate_params_per_layer"]) / gate < 0.02
    assert abs(gate * g["q30b.moe_layers"] - g["q30b.gate_params_all_layers"]) / 1.26e7 < 0.01
    assert gate * g["q30b.moe_layers"] * 2 < g["q30b.gate_bytes_bf16_max"]
    # expert intermediate size 768: 3 matrices of H x I per expert, ~600 M per layer
    experts = wl.E * 3 * wl.H * wl.I
    assert abs(experts - g["q30b.expert_params_per_layer"]) / experts < 0.01
    assert abs(wl.H * g["q30b.vocab"] - g["q30b.lm_head_params"]) / 3.1e8 < 0.01
    big = synth.MOE_WORKLOADS["qwen3-235b-a22b"]
    assert (big.H, big.E, big.k) == (g["q235b.hidden"], g["q235b.experts"], g["q235b.top_k"])
    assert abs(g["q235b.int8_bytes"] / g["q235b.bf16_bytes"] - 0.5) < 0.01


def test_int8_expert_storage_is_half_of_bf16():
    """int8 codes plus fp32 per-channel scales take about half the bf16 bytes."""
    wl = synth.MOE_WORKLOADS["tiny"]
    wgu = synth.expert_gate_up(2, wl.I, wl.H, 0)
    q, s = O.quantize_weight_per_channel(wgu)
    ratio = (q.nbytes + s.nbytes) / wgu.nbytes
    assert 0.5 <= ratio < 0.51


# ------------------------------------------------------------------ router
def _x_wg(T, H, E, seed=0):
    rng = np.random.default_rng(seed)
    return bf16(rng.standard_normal((T, H))), bf16(rng.standard_normal((E, H)) * 0.05)


@pytest.mark.parametrize("k,E", [(1, 4), (2, 8), (8, 128), (8, 16)])
def test_router_invariants(k, E):
    x, wg = _x_wg(40, 64, E)
    r = O.route(x, wg, None, k, True)
    np.testing.assert_allclose(r.probs.sum(axis=1), 1.0, atol=1e-12)
    np.testing.assert_allclose(r.weights.astype(np.float64).sum(axis=1), 1.0, atol=1e-6)
    assert r.ids.shape == (40, k)
    assert all(len(set(row)) == k for row in r.ids.tolist())
    assert r.ids.min() >= 0 and r.ids.max() < E
    sel = np.take_along_axis(r.probs, r.ids.astype(np.int64), axis=1)
    assert np.all(np.diff(sel, axis=1) <= 0)  # slots in descending probability
    # every unselected expert is no more likely than the k-th selected one
    mask = np.ones_like(r.probs, bool)
    np.put_along_axis(mask, r.ids.astype(np.int64), False, axis=1)
    assert np.all(np.where(mask, r.probs, -1).max(axis=1) <= sel[:, -1])


def test_router_uniform_scores_break_ties_to_lower_index():
    x = bf16(np.random.default_rng(0).standard_normal((5, 32)))
    wg = bf16(np.zeros((16, 32)))
    r = O.route(x, wg, None, 4, True)
    np.testing.assert_array_equal(r.ids, np.tile(np.arange(4), (5, 1)))
    np.testing.assert_array_equal(r.weights, np.full((5, 4), 0.25, np.float32))
    r = O.route(x, wg, None, 4, False)
    np.testing.assert_allclose(r.weights, 1 / 16, rtol=1e-7)


def test_router_k_equals_e_and_two_expert_sigmoid():
    x, wg = _x_wg(7, 16, 6, seed=3)
    r = O.route(x, wg, None, 6, False)
    assert sorted(r.ids[0].tolist()) == list(range(6))
    np.testing.assert_allclose(r.weights.sum(axis=1), 1.0, atol=1e-6)
    x, wg = _x_wg(9, 16, 2, seed=4)
    r = O.route(x, wg, None, 2, False)
    lx = O.bf16_to_f32(x).astype(np.float64) @ O.bf16_to_f32(wg).astype(np.float64).T
    for t in range(9):
        p0 = 1.0 / (1.0 + math.exp(lx[t, 1] - lx[t, 0]))
        top = 0 if p0 >= 0.5 else 1
        assert r.ids[t, 0] == top
        assert abs(r.weights[t, 0] - max(p0, 1 - p0)) < 1e-7


def test_router_bias_forces_hot_experts():
    x, wg = _x_wg(64, 32, 16, seed=5)
    b = np.zeros(16, np.float32)
    b[[3, 11]] = 50.0
    r = O.route(x, wg, b, 2, True)
    np.testing.assert_array_equal(np.sort(r.ids, axis=1), np.tile([3, 11], (64, 1)))


def test_router_reads_the_gate_unquantised():
    """Two experts whose gate rows differ by one bf16 step that per-channel int8 would
    erase: the router must still rank them by the exact bf16 logits."""
    H = 8
    x = np.zeros((1, H), np.float32)
    x[0, 0] = 1.0
    wg = np.zeros((2, H), np.float32)
    wg[0, 0], wg[1, 0] = 1.0, 1.0078125  # 1 + 2^-7, representable in bf16
    wg[:, 1] = 127.0  # per-channel scale 1 -> both would quantise to code 1
    q, s = O.quantize_weight_per_channel(bf16(wg))
    assert q[0, 0] == q[1, 0]
    r = O.route(bf16(x), bf16(wg), None, 1, True)
    assert r.ids[0, 0] == 1


def test_router_brute_force_tiny():
    x, wg = _x_wg(6, 8, 5, seed=6)
    r = O.route(x, wg, None, 3, True)
    xf, wf = O.bf16_to_f32(x), O.bf16_to_f32(wg)
    for t in range(6):
        logit = [sum(float(xf[t, h]) * float(wf[e, h]) for h in range(8)) for e in range(5)]
        m = max(logit)
        ex = [math.exp(v - m) for v in logit]
        p = [v / sum(ex) for v in ex]
        top = sorted(range(5), key=lambda e: (-p[e], e))[:3]
        assert r.ids[t].tolist() == top
        tot = sum(p[e] for e in top)
        np.testing.assert_allclose(r.weights[t], [p[e] / tot for e in top], rtol=1e-6)


# ------------------------------------------------------------------ grouping by expert
def test_group_by_expert_hand_example():
    ids = np.array([[2, 0], [0, 1], [2, 1]], np.int32)
    perm, off = O.group_by_expert(ids, 4)
    np.testing.assert_array_equal(perm, [1, 2, 3, 5, 0, 4])
    np.testing.assert_array_equal(off, [0, 2, 4, 6, 6])


def test_group_by_expert_invariants():
    rng = np.random.default_rng(8)
    T, k, E = 300, 4, 24
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    perm, off = O.group_by_expert(ids, E)
    np.testing.assert_array_equal(np.sort(perm), np.arange(T * k))
    flat = ids.reshape(-1)
    assert off[-1] == T * k and np.all(np.diff(off) == np.bincount(flat, minlength=E))
    for e in range(E):
        rows = perm[off[e]:off[e + 1]]
        assert np.all(flat[rows] == e)
        assert np.all(np.diff(rows // k) > 0)  # ordered by token


# ------------------------------------------------------------------ integer GEMM
def test_int_gemm_brute_force_and_extremes():
    rng = np.random.default_rng(9)
    a = rng.integers(-127, 128, (5, 33)).astype(np.int8)
    b = rng.integers(-127, 128, (7, 33)).astype(np.int8)
    acc = O.int_gemm(a, b)
    for i in range(5):
        for j in range(7):
            assert acc[i, j] == sum(int(a[i, t]) * int(b[j, t]) for t in range(33))
    K = 4096
    a = np.full((2, K), -127, np.int8)
    b = np.full((3, K), -127, np.int8)
    b[1] = 127
    acc = O.int_gemm(a, b)
    assert acc.dtype == np.int32
    np.testing.assert_array_equal(acc[:, 0], 16129 * K)
    np.testing.assert_array_equal(acc[:, 1], -16129 * K)


# ------------------------------------------------------------------ whole MoE layer
def _tiny_layer(T=24, H=128, E=6, k=2, I=64, seed=0, n_out=2):
    x = synth.activations(T, H, n_out, seed)
    wg = synth.router_weight(E, H, seed)
    wgu = synth.expert_gate_up(E, I, H, seed)
    wd = synth.expert_down(E, H, I, seed)
    return x, wg, wgu, wd


def _run(x, wg, wgu, wd, k, bias=None, **kw):
    return O.moe_forward(x, wg, bias, *O.quantize_experts(wgu, wd), k, **kw)


def test_zero_input_gives_zero_output():
    x, wg, wgu, wd = _tiny_layer()
    out = _run(np.zeros_like(x), wg, wgu, wd, 2)
    assert not O.bf16_to_f32(out["y"]).any()
    assert not out["hq"].any() and not out["s_h"].any()


@pytest.mark.parametrize("n_out,bound", [(0, 0.03), (2, 0.12)])
def test_quantisation_error_bound(n_out, bound):
    """Relative L2 distance to the unquantised float64 layer (same routing). A dropped
    scale, a wrong sign or a transposed operand gives errors of order 1."""
    x, wg, wgu, wd = _tiny_layer(n_out=n_out, seed=1)
    out = _run(x, wg, wgu, wd, 2)
    ref = O.moe_forward_float(x, wg, None, wgu, wd, 2, routing=(out["ids"], out["weights"]))
    y = O.bf16_to_f32(out["y"]).astype(np.float64)
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < bound, rel


def test_single_expert_reduces_to_dense_gated_mlp():
    x, wg, wgu, wd = _tiny_layer(E=1)
    out = _run(x, wg, wgu, wd, 1)
    np.testing.assert_array_equal(out["ids"], 0)
    np.testing.assert_array_equal(out["weights"], 1.0)
    np.testing.assert_array_equal(out["y"], out["o"][:, 0, :])  # 0 + 1*o == o exactly


def test_token_permutation_equivariance_and_batch_independence():
    x, wg, wgu, wd = _tiny_layer(seed=2)
    y = _run(x, wg, wgu, wd, 2)["y"]
    pi = np.random.default_rng(10).permutation(x.shape[0])
    np.testing.assert_array_equal(_run(x[pi], wg, wgu, wd, 2)["y"], y[pi])
    np.testing.assert_array_equal(_run(x[5:6], wg, wgu, wd, 2)["y"], y[5:6])


def test_expert_relabelling_invariance():
    x, wg, wgu, wd = _tiny_layer(seed=3)
    out = _run(x, wg, wgu, wd, 2)
    sig = np.random.default_rng(11).permutation(wg.shape[0])
    out2 = _run(x, wg[sig], wgu[sig], wd[sig], 2)
    np.testing.assert_array_equal(out2["y"], out["y"])
    np.testing.assert_array_equal(sig[out2["ids"]], out["ids"])


def test_down_weight_doubling_doubles_output_exactly():
    x, wg, wgu, wd = _tiny_layer(seed=4)
    y = O.bf16_to_f32(_run(x, wg, wgu, wd, 2)["y"])
    wd2 = bf16(O.bf16_to_f32(wd) * 2)
    y2 = O.bf16_to_f32(_run(x, wg, wgu, wd2, 2)["y"])
    np.testing.assert_array_equal(y2, 2 * y)


def test_injected_routing_matches_own_routing():
    x, wg, wgu, wd = _tiny_layer(seed=5)
    a = _run(x, wg, wgu, wd, 2)
    b = _run(x, wg, wgu, wd, 2, routing=(a["ids"], a["weights"]))
    for key in ("y", "o", "h", "hq", "s_h", "perm", "offsets"):
        np.testing.assert_array_equal(a[key], b[key])


def test_skewed_router_concentrates_tokens():
    x, wg, wgu, wd = _tiny_layer(T=64, E=16, seed=6)
    b = synth.router_bias(16, 0, n_hot=2)
    out = _run(x, wg, wgu, wd, 2, bias=b)
    hot = np.flatnonzero(b)
    counts = np.diff(out["offsets"])
    assert counts[hot].sum() > 0.6 * counts.sum()


def test_empty_batch():
    x, wg, wgu, wd = _tiny_layer()
    out = _run(x[:0], wg, wgu, wd, 2)
    assert out["y"].shape == (0, x.shape[1])


# ------------------------------------------------------------------ dense linear
def test_linear_error_bounds_and_scaling():
    rng = np.random.default_rng(12)
    M, K, N = 16, 512, 24
    x = bf16(rng.standard_normal((M, K)))
    w = bf16(rng.standard_normal((N, K)) * 0.02)
    ref = O.bf16_to_f32(x).astype(np.float64) @ O.bf16_to_f32(w).astype(np.float64).T
    q8, s8 = O.quantize_weight_per_channel(w)
    y8 = O.bf16_to_f32(O.linear_w8a8(x, q8, s8)).astype(np.float64)
    assert np.linalg.norm(y8 - ref) / np.linalg.norm(ref) < 0.02
    p4, s4 = O.quantize_weight_int4_per_group(w, 128)
    y4 = O.bf16_to_f32(O.linear_w4a8(x, p4, s4, 128)).astype(np.float64)
    assert np.linalg.norm(y4 - ref) / np.linalg.norm(ref) < 0.15
    p4b, s4b = O.quantize_weight_int4_per_group(bf16(O.bf16_to_f32(w) * 4), 128)
    np.testing.assert_array_equal(p4b, p4)
    np.testing.assert_array_equal(O.bf16_to_f32(O.linear_w4a8(x, p4b, s4b, 128)),
                                  4 * O.bf16_to_f32(O.linear_w4a8(x, p4, s4, 128)))


def test_w4a8_brute_force_tiny():
    """Per-group integer sums, scaled and added in group order, then the token scale."""
    rng = np.random.default_rng(13)
    M, K, N, G = 2, 256, 3, 128
    x = bf16(rng.standard_normal((M, K)))
    w = bf16(rng.standard_normal((N, K)) * 0.02)
    p, s = O.quantize_weight_int4_per_group(w, G)
    y = O.linear_w4a8(x, p, s, G)
    from fractions import Fraction

    from tests.test_oracle_quant import round_f32_exact

    xq, sx = O.quant_act_per_token(x)
    codes = O.unpack_int4(p)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for g in range(K // G):
                part = sum(int(xq[m, c]) * int(codes[n, c]) for c in range(g * G, (g + 1) * G))
                # one rounding per step: fp32(part), then fused part * s + acc
                acc = round_f32_exact(Fraction(float(np.float32(part))) * Fraction(float(s[n, g])) + Fraction(acc))
            assert O.f32_to_bf16(np.float32(acc) * sx[m]) == y[m, n]


def test_oracle_is_independent_of_the_library():
    src = open(O.__file__).read()
    assert "w8a8_int8_quantized_act_b200" not in src and "ctypes" not in src
