"""GPU parity of the MXFP8 A8W8 path (w8a8_mxfp8_quantize, w8a8_mxfp8_linear) against the oracle.

The quantiser's E4M3 codes and E8M0 scales are compared bit for bit. The linear's result is the
block-scaled FP8 MMA's fp32 sum of the products, rounded to bf16: every element must lie within the
oracle's bound of the exact sum ((K - 1) * 2^-24 * sum |products| for an fp32 summation in any
order, plus one bf16 rounding), and the relative L2 error must stay at the bf16 rounding level.
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
    """bf16 rows whose blocks cover the quantiser's cases: zeros, subnormal and huge magnitudes,
    an outlier per block, exact powers of two, values that clip at 448 after scaling."""
    v = rng.standard_normal((R, K)) * np.exp2(rng.integers(-30, 30, (R, 1)))
    if R >= 6 and K >= 64:
        v[0, :32] = 0.0
        v[1, :32] = np.exp2(-130.0) * np.arange(1, 33)       # bf16 subnormals
        v[2, 32:64] = 3.0e38 * np.linspace(-1, 1, 32)         # near the bf16 maximum
        v[3, :32] = 1.0
        v[3, 7] = 1.9                                         # clips to 448 * 2^E
        v[4, :32] = -np.exp2(np.arange(32) - 16.0)            # powers of two, negative
        v[5, :32] = 1e-30 * rng.standard_normal(32)
        v[5, 3] = -0.0
    return O.f32_to_bf16(v.astype(np.float32))


@pytest.mark.parametrize("R,K", [(1, 32), (6, 64), (77, 256), (300, 2048), (6144, 2048)])
def test_mxfp8_quantize_exact(R, K):
    rng = np.random.default_rng(R + K)
    x = _edge_rows(rng, R, K)
    codes, scales = B.w8a8_mxfp8_quantize(G.bf16_dev(x))
    oc, os_ = O.mx_quantize_rows(x)
    np.testing.assert_array_equal(scales.cpu().numpy(), os_)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)


@pytest.mark.parametrize("M,K,N", [(1, 128, 128), (77, 256, 384), (300, 1152, 512), (2048, 2048, 6144)])
def test_mxfp8_linear_within_the_summation_bound(M, K, N):
    x = synth.activations(M, K, max(1, K // 100), seed=M + 3)
    w = synth.dense_weight(N, K, seed=N + 3)
    wc, ws = B.w8a8_mxfp8_quantize(G.bf16_dev(w))
    owc, ows = O.mx_quantize_rows(w)
    np.testing.assert_array_equal(wc.cpu().numpy(), owc)
    np.testing.assert_array_equal(ws.cpu().numpy(), ows)
    workspace = torch.empty(B.w8a8_mxfp8_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    y = B.w8a8_mxfp8_linear(G.bf16_dev(x), wc, ws, workspace=workspace)
    torch.cuda.synchronize()
    B.w8a8_check_status()
    ref = O.linear_mxfp8(x, owc, ows)
    inter = B.mxfp8_linear_intermediates(workspace, M, K)
    np.testing.assert_array_equal(inter["codes"].cpu().numpy(), ref["codes"])
    np.testing.assert_array_equal(inter["scales"].cpu().numpy(), ref["scales"])
    yg = O.bf16_to_f32(G.host(y)).astype(np.float64)
    err = np.abs(yg - ref["y"])
    assert np.all(err <= ref["bound"]), float((err - ref["bound"]).max())
    assert np.linalg.norm(yg - ref["y"]) <= 4e-3 * np.linalg.norm(ref["y"])
    # the GEMM-only entry on the same codes and scales gives the same bits
    y2 = B.w8a8_mxfp8_linear_prequant(inter["codes"].clone(), inter["scales"].clone(), wc, ws)
    np.testing.assert_array_equal(G.host(y2), G.host(y))


def test_mxfp8_linear_empty_batch():
    w = synth.dense_weight(128, 128, seed=1)
    wc, ws = B.w8a8_mxfp8_quantize(G.bf16_dev(w))
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    y = B.w8a8_mxfp8_linear(x, wc, ws)
    assert y.shape == (0, 128)
