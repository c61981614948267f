"""GPU parity of the MXFP A8W4 path (w8a8_mxfp4_quantize, w8a8_mxfp_a8w4_linear) against the oracle.

The weight quantiser's packed E2M1 codes and E8M0 scales are compared bit for bit. The linear
multiplies MXFP8 token codes by MXFP4 weight codes on the block-scaled MMA and sums in fp32: every
element must lie within the oracle's bound of the exact sum ((K - 1) * 2^-24 * sum |products| for
an fp32 summation in any order, plus one bf16 rounding), and the relative L2 error must stay at the
bf16 rounding level. Both GEMM kernels are covered: one CTA per tile (at most 192 token rows, or N
not a multiple of 256) and CTA pairs.
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


def _edge_rows(rng, R, K):
    """bf16 rows whose blocks cover the MXFP4 quantiser's cases: zeros, subnormal and huge
    magnitudes, values that clip at 6 after scaling, exact ties of the E2M1 grid, negative zeros."""
    v = rng.standard_normal((R, K)) * np.exp2(rng.integers(-30, 30, (R, 1)))
    if R >= 7 and K >= 64:
        v[0, :32] = 0.0
        v[1, :32] = np.exp2(-130.0) * np.arange(1, 33)        # bf16 subnormals
        v[2, 32:64] = 3.0e38 * np.linspace(-1, 1, 32)          # near the bf16 maximum
        v[3, :32] = 1.0
        v[3, 7] = 1.875                                        # 1.875 * 2^2 = 7.5: clips to 6
        # amax 6 (E = 0): every midpoint of the E2M1 grid, both signs
        v[4, :32] = np.tile([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], 4) * np.repeat([1, -1, 1, -1], 8)
        v[5, :32] = 1e-30 * rng.standard_normal(32)
        v[5, 3] = -0.0
        v[6, :32] = -np.exp2(np.arange(32) - 16.0)             # powers of two, negative
    return O.f32_to_bf16(v.astype(np.float32))


@pytest.mark.parametrize("R,K", [(1, 32), (7, 64), (77, 256), (300, 2048), (6144, 2048)])
def test_mxfp4_quantize_exact(R, K):
    rng = np.random.default_rng(R + 2 * K)
    w = _edge_rows(rng, R, K)
    packed, scales = B.w8a8_mxfp4_quantize(G.bf16_dev(w))
    op, os_ = O.mx4_quantize_rows(w)
    np.testing.assert_array_equal(scales.cpu().numpy(), os_)
    np.testing.assert_array_equal(packed.cpu().numpy(), op)


@pytest.mark.parametrize("M,K,N", [(1, 128, 128), (77, 256, 384), (200, 512, 384), (257, 512, 256),
                                   (300, 1152, 512), (2048, 2048, 6144)])
def test_mxfp_a8w4_linear_within_the_summation_bound(M, K, N):
    x = synth.activations(M, K, max(1, K // 100), seed=M + 5)
    w = synth.dense_weight(N, K, seed=N + 5)
    wp, ws = B.w8a8_mxfp4_quantize(G.bf16_dev(w))
    owp, ows = O.mx4_quantize_rows(w)
    np.testing.assert_array_equal(wp.cpu().numpy(), owp)
    np.testing.assert_array_equal(ws.cpu().numpy(), ows)
    workspace = torch.empty(B.w8a8_mxfp8_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    y = B.w8a8_mxfp_a8w4_linear(G.bf16_dev(x), wp, ws, workspace=workspace)
    torch.cuda.synchronize()
    B.w8a8_check_status()
    ref = O.linear_mxfp_a8w4(x, owp, ows)
    inter = B.mxfp8_linear_intermediates(workspace, M, K)
    np.testing.assert_array_equal(inter["codes"].cpu().numpy(), ref["codes"])
    np.testing.assert_array_equal(inter["scales"].cpu().numpy(), ref["scales"])
    yg = O.bf16_to_f32(G.host(y)).astype(np.float64)
    err = np.abs(yg - ref["y"])
    assert np.all(err <= ref["bound"]), float((err - ref["bound"]).max())
    assert np.linalg.norm(yg - ref["y"]) <= 4e-3 * np.linalg.norm(ref["y"])
    # the GEMM-only entry on the same codes and scales gives the same bits
    y2 = B.w8a8_mxfp_a8w4_linear_prequant(inter["codes"].clone(), inter["scales"].clone(), wp, ws)
    np.testing.assert_array_equal(G.host(y2), G.host(y))


def test_mxfp_a8w4_linear_extreme_codes():
    # weights at the E2M1 extremes (every block holds +-6 and the smallest nonzero +-0.5) against
    # large activations: the largest products the MMA sums, checked against the exact sum
    M, K, N = 300, 512, 256
    rng = np.random.default_rng(11)
    w = rng.choice([6.0, -6.0, 0.5, -0.5, 0.0], size=(N, K)) * np.exp2(rng.integers(-8, 8, (N, 1)))
    w[:, ::32] = 6.0 * np.exp2(rng.integers(-8, 8, (N, 1)))  # amax of every block a grid point
    wb = O.f32_to_bf16(w.astype(np.float32))
    x = O.f32_to_bf16((rng.standard_normal((M, K)) * 100.0).astype(np.float32))
    wp, ws = B.w8a8_mxfp4_quantize(G.bf16_dev(wb))
    owp, ows = O.mx4_quantize_rows(wb)
    np.testing.assert_array_equal(wp.cpu().numpy(), owp)
    y = B.w8a8_mxfp_a8w4_linear(G.bf16_dev(x), wp, ws)
    torch.cuda.synchronize()
    B.w8a8_check_status()
    ref = O.linear_mxfp_a8w4(x, owp, ows)
    yg = O.bf16_to_f32(G.host(y)).astype(np.float64)
    assert np.all(np.abs(yg - ref["y"]) <= ref["bound"])


def test_mxfp_a8w4_linear_empty_batch():
    w = synth.dense_weight(128, 128, seed=2)
    wp, ws = B.w8a8_mxfp4_quantize(G.bf16_dev(w))
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    y = B.w8a8_mxfp_a8w4_linear(x, wp, ws)
    assert y.shape == (0, 128)
