"""GPU parity: every stage of the CUDA path through the C ABI against the CPU oracle.

Integer codes, scales, int32 accumulators, perm/offsets and the bf16 intermediates (h, o)
and output y are compared bit for bit, the oracle being fed the GPU's routing; the routing
itself is compared with the oracle's router (identical expert sets wherever the k-th/(k+1)-th
probability gap exceeds 1e-4, weights within fp32 rounding); y is also checked end to end
against the oracle's own routing (max abs <= 2e-2, relative L2 <= 5e-3).
"""
import numpy as np
import pytest
import torch

from oracle import w8a8_oracle as O
from w8a8_int8_quantized_act_b200 import binding as B
from w8a8_int8_quantized_act_b200 import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from tests import gpu_common as G  # noqa: E402
else:  # pragma: no cover
    G = None


@pytest.fixture(autouse=True)
def _clean_status():
    yield
    if torch.cuda.is_available():
        B.w8a8_check_status()


# ------------------------------------------------------------------ exact int8 GEMM
@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (128, 128, 256), (300, 384, 2048), (1000, 256, 768),
                                   (77, 6144, 128), (129, 128, 128), (136, 640, 384), (4133, 512, 1024),
                                   (256, 6144, 2048)])
def test_gemm_s8s8s32_exact(M, N, K):
    rng = np.random.default_rng(M + N + K)
    a = rng.integers(-127, 128, (M, K)).astype(np.int8)
    b = rng.integers(-127, 128, (N, K)).astype(np.int8)
    c = B.w8a8_gemm_s8s8s32(G.to_dev(a), G.to_dev(b))
    np.testing.assert_array_equal(c.cpu().numpy(), O.int_gemm(a, b))


def test_gemm_s8s8s32_extremes():
    K = 4096
    a = np.full((130, K), -127, np.int8)
    b = np.full((128, K), -127, np.int8)
    b[::2] = 127
    c = B.w8a8_gemm_s8s8s32(G.to_dev(a), G.to_dev(b)).cpu().numpy()
    np.testing.assert_array_equal(c, O.int_gemm(a, b))


# ------------------------------------------------------------------ quantisers
@pytest.mark.parametrize("T,K", [(1, 128), (64, 256), (64, 2048), (300, 2048), (129, 4096), (8192, 2048)])
def test_quant_act_per_token_exact(T, K):
    x = synth.activations(T, K, max(1, K // 100), seed=T)
    x[min(3, T - 1)] = 0  # an all-zero token
    q, s = B.w8a8_quant_act_per_token(G.bf16_dev(x))
    oq, os_ = O.quant_act_per_token(x)
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy(), os_)


def test_quant_act_rounding_ties():
    # rows with amax 127: v/scale lands exactly on .5 for the designed entries
    v = np.zeros((2, 128), np.float32)
    v[:, 0] = 127
    v[0, 1:9] = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, -126.5]
    v[1, 1:3] = [3.5, -3.5]
    x = O.f32_to_bf16(v)
    q, s = B.w8a8_quant_act_per_token(G.bf16_dev(x))
    np.testing.assert_array_equal(q.cpu().numpy(), O.quant_act_per_token(x)[0])
    assert q.cpu().numpy()[0, 1:9].tolist() == [0, 2, 2, 0, -2, -2, 126, -126]


def test_quant_tiny_and_subnormal_rows():
    # Rows whose amax is so small that amax / 127 is a subnormal fp32 (its reciprocal overflows
    # to inf), rows of subnormal bf16 values, and rows at the edge of that range: the codes and
    # scales still follow the true divide bit for bit, for the activation and weight quantisers.
    rows = []
    for e_amax in (-124, -126, -121, -120):
        r = np.zeros(256, np.float32)
        r[0] = 2.0 ** e_amax
        r[1] = -(2.0 ** e_amax)
        r[2:40] = (np.arange(38) - 19) * 2.0 ** (e_amax - 6)  # small multiples, some subnormal bf16
        rows.append(r)
    sub = np.zeros(256, np.float32)
    sub[:64] = np.arange(1, 65) * 2.0 ** -133  # every value a subnormal bf16
    sub[64] = -(2.0 ** -127)
    rows.append(sub)
    x = O.f32_to_bf16(np.stack(rows))
    assert np.array_equal(O.bf16_to_f32(x), np.stack(rows))  # all exactly representable
    oq, os_ = O.quant_act_per_token(x)
    assert np.all(np.abs(oq[:4, :2]) == 127)
    q, s = B.w8a8_quant_act_per_token(G.bf16_dev(x))
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    wq, ws = B.w8a8_quantize_weight_per_channel(G.bf16_dev(x[None]))
    np.testing.assert_array_equal(wq.cpu().numpy()[0], oq)
    np.testing.assert_array_equal(ws.cpu().numpy()[0].view(np.uint32), os_.view(np.uint32))


def test_quant_act_empty():
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q, s = B.w8a8_quant_act_per_token(x)
    assert q.shape == (0, 256) and s.shape == (0,)


@pytest.mark.parametrize("G_,N,K", [(1, 4, 128), (8, 256, 128), (3, 1536, 2048), (2, 2048, 768)])
def test_quantize_weight_per_channel_exact(G_, N, K):
    w = synth.expert_gate_up(G_, N // 2, K, seed=K) if N % 2 == 0 else None
    w[0, 1] = 0  # an all-zero channel
    q, s = B.w8a8_quantize_weight_per_channel(G.bf16_dev(w))
    oq, os_ = O.quantize_weight_per_channel(w)
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy(), os_)


@pytest.mark.parametrize("N,K", [(4, 128), (6144, 2048), (130, 1024)])
def test_quantize_int4_exact(N, K):
    w = synth.dense_weight(N, K, seed=N)
    p, s = B.w8a8_quantize_weight_int4_per_group(G.bf16_dev(w), 128)
    op, os_ = O.quantize_weight_int4_per_group(w, 128)
    np.testing.assert_array_equal(p.cpu().numpy(), op)
    np.testing.assert_array_equal(s.cpu().numpy(), os_)


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("T,H,E,k,renorm,skew", [
    (64, 256, 8, 2, True, False), (64, 2048, 128, 8, True, False), (1, 2048, 128, 8, True, False),
    (300, 1024, 100, 6, False, False), (8192, 2048, 128, 8, True, True), (129, 4096, 128, 8, True, False),
    (50, 512, 16, 16, True, False), (40, 256, 256, 4, False, False), (33, 128, 1, 1, True, False),
    # tensor-core router with 32-token tiles (one wave), a ragged last tile, and at the 235B shape
    (1000, 2048, 128, 8, True, False), (4096, 4096, 128, 8, True, False)])
def test_route(T, H, E, k, renorm, skew):
    x = synth.activations(T, H, max(1, H // 100), seed=T)
    wg = synth.router_weight(E, H, seed=E)
    bias = synth.router_bias(E, 0, n_hot=min(8, E)) if skew else None
    ids, w, counts = B.w8a8_moe_route(G.bf16_dev(x), G.bf16_dev(wg), k, renorm,
                                      bias=G.to_dev(bias) if bias is not None else None)
    ids, w, counts = ids.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy()
    r = O.route(x, wg, bias, k, renorm)
    clear = r.gap > 1e-4
    np.testing.assert_array_equal(np.sort(ids[clear], 1), np.sort(r.ids[clear], 1))
    same = np.all(ids == r.ids, axis=1)
    assert same.mean() > 0.9
    G.check_topk_valid(ids, w, r, k, renorm)  # every token, near ties included
    np.testing.assert_array_equal(counts, np.bincount(ids.reshape(-1), minlength=E))


# ------------------------------------------------------------------ whole layer
def _full_check(run):
    wl = run.wl
    m = run.mid
    G.check_grouping(m["topk_ids"], m["perm"], m["offsets"], wl.E)
    tokens = np.arange(run.inp.x.shape[0])
    G.compare_tokens(run, tokens)
    clear = G.check_routing(run, m["topk_ids"], m["topk_w"])
    G.y_tolerance_check(run, tokens, clear)


def test_moe_tiny_all_stages():
    _full_check(G.run_moe(synth.MOE_WORKLOADS["tiny"]))


def test_moe_decode_all_tokens():
    _full_check(G.run_moe(synth.MOE_WORKLOADS["qwen3-30b-a3b-decode"]))


# I = 2176 (rows longer than 2048): h is requantised by a separate launch instead of inside gate_up
@pytest.mark.parametrize("T,E,k,I", [(1, 8, 2, 128), (129, 8, 2, 128), (37, 8, 8, 128), (200, 1, 1, 256),
                                     (70, 16, 4, 384), (40, 4, 2, 2176)])
def test_moe_edge_shapes(T, E, k, I):
    wl = synth.MoEWorkload("edge", T=T, H=256, E=E, k=k, I=I, n_outlier=2, seed=T)
    _full_check(G.run_moe(wl))


# The fused short-batch front end (one cooperative kernel, T <= 128, H <= 2048) at its extremes:
# a full 128-token chunk, 256 experts with k = 16, one token, hidden 2048 (the largest row held in
# registers). Routing against the oracle's router, every integer stage and y bit for bit.
@pytest.mark.parametrize("T,H,E,k,I", [(128, 2048, 128, 8, 128), (1, 2048, 256, 16, 128), (97, 1024, 64, 6, 256),
                                       (128, 128, 256, 1, 128)])
def test_moe_fused_front_end_shapes(T, H, E, k, I):
    wl = synth.MoEWorkload("front", T=T, H=H, E=E, k=k, I=I, n_outlier=2, seed=T + E)
    _full_check(G.run_moe(wl))


# Long token lists (the CTA-pair GEMMs): several 256-row blocks per expert with ragged tails,
# an odd number of 128-channel blocks in the down projection (H = 384), a single expert.
@pytest.mark.parametrize("T,H,E,k,I", [(600, 384, 4, 2, 256), (1031, 256, 8, 3, 128), (700, 512, 1, 1, 384),
                                       (2000, 640, 16, 4, 256), (600, 256, 4, 2, 2176), (1500, 256, 3, 2, 1024)])
def test_moe_long_token_lists(T, H, E, k, I):
    wl = synth.MoEWorkload("long", T=T, H=H, E=E, k=k, I=I, n_outlier=3, seed=T)
    run = G.run_moe(wl)
    assert np.diff(run.mid["offsets"]).max() > 256
    _full_check(run)


def test_moe_zero_tokens_and_empty_experts():
    wl = synth.MoEWorkload("empty-experts", T=100, H=256, E=16, k=2, I=128, n_outlier=2)
    bias = np.zeros(16, np.float32)
    bias[[2, 9, 11]] = 40.0  # every token picks two of three experts: 13 experts stay empty
    run = G.run_moe(wl, bias_override=bias)
    assert (np.diff(run.mid["offsets"]) == 0).sum() == 13
    _full_check(run)
    x0 = np.zeros_like(run.inp.x)
    run0 = G.run_moe(wl, x_override=x0)
    assert not O.bf16_to_f32(run0.y).any()
    e = synth.MoEWorkload("empty", T=0, H=256, E=8, k=2, I=128, n_outlier=0)
    run_e = G.run_moe(e)
    assert run_e.y.shape == (0, 256)


@pytest.mark.parametrize("name", ["qwen3-30b-a3b-prefill", "qwen3-30b-a3b-prefill-skewed", "qwen3-235b-a22b"])
def test_moe_full_size_sampled_tokens(name):
    wl = synth.MOE_WORKLOADS[name]
    run = G.run_moe(wl)
    m = run.mid
    G.check_grouping(m["topk_ids"], m["perm"], m["offsets"], wl.E)
    rng = np.random.default_rng(1)
    tokens = np.unique(np.concatenate([[0, wl.T - 1], rng.choice(wl.T, 14, replace=False)]))
    G.compare_tokens(run, tokens)
    clear = G.check_routing(run, m["topk_ids"], m["topk_w"], tokens)
    G.y_tolerance_check(run, tokens, clear)
    if wl.skewed:
        counts = np.diff(m["offsets"])
        hot = np.flatnonzero(run.inp.bias)
        assert counts[hot].min() > 4 * np.median(counts)


# ------------------------------------------------------------------ dense linear
@pytest.mark.parametrize("M,K,N", [(1, 128, 128), (200, 512, 384), (2048, 2048, 6144)])
def test_linear_w8a8_exact(M, K, N):
    x = synth.activations(M, K, max(1, K // 100), seed=M)
    w = synth.dense_weight(N, K, seed=N)
    q, s = B.w8a8_quantize_weight_per_channel(G.bf16_dev(w))
    y = B.w8a8_linear(G.bf16_dev(x), q, s, B.W8A8_W_INT8_PER_CHANNEL)
    oq, os_ = O.quantize_weight_per_channel(w)
    np.testing.assert_array_equal(G.host(y), O.linear_w8a8(x, oq, os_))


# (1000, 1024, 6144): 384 tiles, several per CTA, the last token tile ragged (104 rows), so the
# shared-memory output tile is handed between bulk stores and its store clips rows past M;
# (200, 512, 384): four groups, the scales of a channel in one 16-byte load and none read past the
# row; (300, 1152, 512): 9 groups, so the scales are read one by one; (257, 256, 256): a last
# token tile of one row.
@pytest.mark.parametrize("M,K,N", [(1, 128, 128), (200, 512, 384), (77, 1024, 256), (1000, 1024, 6144),
                                   (2048, 2048, 6144), (300, 1152, 512), (257, 256, 256), (600, 1024, 384)])
def test_linear_w4a8_exact(M, K, N):
    x = synth.activations(M, K, max(1, K // 100), seed=M + 1)
    w = synth.dense_weight(N, K, seed=N + 1)
    packed, s = B.w8a8_quantize_weight_int4_per_group(G.bf16_dev(w), 128)
    y = B.w8a8_linear(G.bf16_dev(x), packed, s, B.W8A8_W_INT4_PER_GROUP, 128)
    op, os_ = O.quantize_weight_int4_per_group(w, 128)
    np.testing.assert_array_equal(packed.cpu().numpy(), op)
    np.testing.assert_array_equal(G.host(y), O.linear_w4a8(x, op, os_, 128))


@pytest.mark.parametrize("fmt,M,K,N", [("int8", 77, 512, 384), ("int8", 300, 1024, 512), ("int4", 200, 512, 384),
                                       ("int4", 1000, 1024, 6144)])
def test_linear_prequant_matches_linear(fmt, M, K, N):
    # the GEMM-only entry on per-token codes gives exactly w8a8_linear's output
    x = synth.activations(M, K, max(1, K // 100), seed=M + 7)
    w = synth.dense_weight(N, K, seed=N + 7)
    if fmt == "int8":
        wq, sw = B.w8a8_quantize_weight_per_channel(G.bf16_dev(w))
        f, g = B.W8A8_W_INT8_PER_CHANNEL, 128
    else:
        wq, sw = B.w8a8_quantize_weight_int4_per_group(G.bf16_dev(w), 128)
        f, g = B.W8A8_W_INT4_PER_GROUP, 128
    xd = G.bf16_dev(x)
    y = B.w8a8_linear(xd, wq, sw, f, g)
    xq, sx = B.w8a8_quant_act_per_token(xd)
    y2 = B.w8a8_linear_prequant(xq, sx, wq, sw, f, g)
    np.testing.assert_array_equal(G.host(y2), G.host(y))


@pytest.mark.parametrize("M,N", [(130, 128), (520, 256)])
def test_linear_w4a8_extreme_codes(M, N):
    # every nibble pattern the quantiser can produce, including -7 and +7 everywhere
    K = 256
    x = O.f32_to_bf16(np.where(np.arange(M * K).reshape(M, K) % 3 == 0, -127.0, 127.0).astype(np.float32))
    wv = np.tile(np.array([7, -7, 1, -1, 0, 3, -3, 5], np.float32), (N, K // 8))
    w = O.f32_to_bf16(wv * np.float32(0.01))
    packed, s = B.w8a8_quantize_weight_int4_per_group(G.bf16_dev(w), 128)
    y = B.w8a8_linear(G.bf16_dev(x), packed, s, B.W8A8_W_INT4_PER_GROUP, 128)
    op, os_ = O.quantize_weight_int4_per_group(w, 128)
    np.testing.assert_array_equal(G.host(y), O.linear_w4a8(x, op, os_, 128))


@pytest.mark.parametrize("M", [96, 700])
def test_linear_w4a8_largest_group_sums(M):
    # every group partial at the largest magnitude the codes allow, 127 * 7 * 128, with both signs
    K, N = 384, 256
    sign = np.where(np.arange(M) % 2 == 1, -1.0, 1.0).astype(np.float32)
    x = O.f32_to_bf16(np.repeat((sign * (1.0 + 0.01 * np.arange(M)))[:, None], K, axis=1).astype(np.float32))
    w = O.f32_to_bf16(np.full((N, K), 0.07, np.float32) * np.where(np.arange(N) % 3 == 0, -1.0, 1.0)[:, None]
                      .astype(np.float32))
    packed, s = B.w8a8_quantize_weight_int4_per_group(G.bf16_dev(w), 128)
    op, os_ = O.quantize_weight_int4_per_group(w, 128)
    assert np.all((op == 0x77) | (op == 0x99))  # +7 and -7 in both nibbles
    y = B.w8a8_linear(G.bf16_dev(x), packed, s, B.W8A8_W_INT4_PER_GROUP, 128)
    np.testing.assert_array_equal(G.host(y), O.linear_w4a8(x, op, os_, 128))


# ------------------------------------------------------------------ hardware premise of the certified SiLU
def test_rcp_approx_within_two_ulp():
    # The gate_up epilogue of the CTA-pair GEMM accepts bf16(fl(fl(g * rcp.approx(d)) * u)) only
    # when its fp32 bits are more than 16 ulps from a bf16 rounding midpoint; the proof needs
    # rcp.approx within 2 ulps of the correctly rounded reciprocal. Every mantissa, three binades.
    for first in (0x3F800000, 0x5F800000, 0x1F800000):
        assert B.w8a8_debug_rcp_approx_ulp(first, 1 << 23) <= 2


def test_ex2_approx_within_three_ulp():
    # The same epilogue computes e^-g as ex2.approx of a split argument; its bound needs ex2.approx
    # within 3 ulps of 2^x. Every fp32 x with 2^-40 <= |x| < 126, both signs (the fast path only
    # takes |g| <= 64, i.e. |x| < 93).
    worst = 0
    for sign in (0, 0x80000000):
        for exp_field in range(127 - 40, 127 + 6):  # 2^-40 <= |x| < 64, whole binades
            worst = max(worst, B.w8a8_debug_ex2_approx_ulp(sign | (exp_field << 23), 1 << 23))
        first = sign | 0x42800000  # 64 <= |x| < 126
        worst = max(worst, B.w8a8_debug_ex2_approx_ulp(first, 0x42FC0000 - 0x42800000))
    assert worst <= 3, worst


# ------------------------------------------------------------------ failure detection
_LONG_GEMM = r"""
import numpy as np, torch
from w8a8_int8_quantized_act_b200 import binding as B
from oracle import w8a8_oracle as O
M, N, K = 32768, 16384, 2048  # about 55 tiles per CTA pair: the CTAs live far longer than 0.1 ms
g = torch.Generator(device="cuda").manual_seed(3)
a = torch.randint(-127, 128, (M, K), dtype=torch.int8, device="cuda", generator=g)
b = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda", generator=g)
c = torch.empty((M, N), dtype=torch.int32, device="cuda")
torch.cuda.synchronize()
s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
s.record()
B.w8a8_gemm_s8s8s32(a, b, c)
e.record()
B.w8a8_check_status()  # raises if any wait ran out
ms = s.elapsed_time(e)
rng = np.random.default_rng(0)
rows, cols = rng.integers(0, M, 64), rng.integers(0, N, 64)
ah, bh = a[torch.as_tensor(rows, device="cuda")].cpu().numpy(), b[torch.as_tensor(cols, device="cuda")].cpu().numpy()
want = O.int_gemm(ah, bh)
got = c[torch.as_tensor(rows, device="cuda")][:, torch.as_tensor(cols, device="cuda")].cpu().numpy()
assert np.array_equal(got, want)
print("LAUNCH_MS", ms)
"""


def test_wait_bound_is_per_wait_not_per_launch():
    # With every wait bounded at 0.1 ms, a healthy GEMM whose launch lasts several ms must finish
    # with W8A8_OK and exact results: each wait is short, only the CTAs live long. (The bound is
    # read once per process, so the GEMM runs in a child process with the variable set.)
    import os
    import subprocess
    import sys

    env = dict(os.environ, W8A8_WAIT_TIMEOUT_MS="0.1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env["PYTHONPATH"] = root + os.pathsep + env.get("PYTHONPATH", "")
    res = subprocess.run([sys.executable, "-c", _LONG_GEMM], env=env, cwd=root, capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    ms = float(res.stdout.split("LAUNCH_MS")[1].split()[0])
    assert ms > 0.5, ms  # the launch outlived the per-wait bound several times over


def test_bounded_wait_reports_timeout_and_context_survives():
    B.w8a8_debug_wait_timeout(2_000_000)  # 2 ms
    with pytest.raises(B.W8A8Error) as ei:
        B.w8a8_check_status()
    assert ei.value.status == B.W8A8_ERR_DEVICE
    B.w8a8_check_status()  # cleared
    x = synth.activations(8, 256, 2)
    q, s = B.w8a8_quant_act_per_token(G.bf16_dev(x))
    np.testing.assert_array_equal(q.cpu().numpy(), O.quant_act_per_token(x)[0])
