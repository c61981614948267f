"""GPU parity of the MoE layer with a shared expert (w8a8_moe_forward_shared) against the oracle.

The routed part is checked as in the plain layer; the shared expert's codes, scales, h, hq and o
are compared bit for bit with the oracle's dense W8A8 gated MLP; its gate against the oracle's
float64 sigmoid (the GPU sums the gate logit in fp32); y bit for bit once the oracle is given the
GPU's routing and gate, and end to end within the layer's tolerance.
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


@pytest.mark.parametrize("T,H,E,k,I,Is", [(64, 256, 8, 2, 128, 128), (64, 2048, 128, 8, 768, 512),
                                          (300, 512, 16, 4, 256, 384), (1, 256, 8, 2, 128, 256)])
def test_moe_with_shared_expert(T, H, E, k, I, Is):
    wl = synth.MoEWorkload("shared", T=T, H=H, E=E, k=k, I=I, n_outlier=max(1, H // 100), seed=T + Is)
    inp = synth.moe_inputs(wl)
    wsg, sgu, sd = synth.shared_expert_weights(H, Is, wl.seed)
    x, wg = G.bf16_dev(inp.x), G.bf16_dev(inp.wg)
    wgu_q, s_gu = B.w8a8_quantize_weight_per_channel(G.bf16_dev(inp.wgu))
    wd_q, s_d = B.w8a8_quantize_weight_per_channel(G.bf16_dev(inp.wd))
    sgu_q, s_sgu = B.w8a8_quantize_weight_per_channel(G.bf16_dev(sgu[None]))
    sd_q, s_sd = B.w8a8_quantize_weight_per_channel(G.bf16_dev(sd[None]))
    ws = torch.empty(B.w8a8_moe_shared_workspace_size(T, H, E, k, I, Is), dtype=torch.uint8, device="cuda")
    y = B.w8a8_moe_forward_shared(x, wg, wgu_q, s_gu, wd_q, s_d, k, G.bf16_dev(wsg), sgu_q[0], s_sgu[0], sd_q[0],
                                  s_sd[0], workspace=ws)
    B.w8a8_check_status()
    m = B.moe_shared_intermediates(ws, T, H, E, k, I, Is)
    sh = {key: G.host(v) for key, v in m.pop("shared").items()}
    ids, w = G.host(m["topk_ids"]), G.host(m["topk_w"])
    # the shared expert (dense W8A8 gated MLP) bit for bit
    gq, gs = O.quantize_weight_per_channel(sgu)
    dq, ds = O.quantize_weight_per_channel(sd)
    ref = O.shared_expert(inp.x, gq, gs, dq, ds)
    for key in ("xq", "sx", "h", "s_h", "hq", "o"):
        np.testing.assert_array_equal(sh[key], ref[key], err_msg=key)
    # the gate: fp32 logit sum against float64
    g64 = O.shared_gate(inp.x, wsg)
    np.testing.assert_allclose(sh["gate"], g64, rtol=0, atol=2e-6)
    # the whole layer with the GPU's routing and gate fed in: y bit for bit
    rq = O.quantize_experts(inp.wgu, inp.wd)
    out = O.moe_forward_shared(inp.x, inp.wg, None, *rq, k, wsg, gq, gs, dq, ds, routing=(ids, w), gate=sh["gate"])
    np.testing.assert_array_equal(G.host(y), out["y"])
    np.testing.assert_array_equal(G.host(m["o"]).reshape(T, k, H), out["o"])
    # end to end against the oracle's own routing and gate, on tokens with an unambiguous top-k
    own = O.moe_forward_shared(inp.x, inp.wg, None, *rq, k, wsg, gq, gs, dq, ds)
    clear = own["routing"].gap > 1e-4
    yr = O.bf16_to_f32(own["y"][clear]).astype(np.float64)
    yg = O.bf16_to_f32(G.host(y)[clear]).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(yr), 2.0 ** -126))) - 7)
    assert np.all(np.abs(yg - yr) <= np.maximum(2e-2, ulp))
    assert np.linalg.norm(yg - yr) <= 5e-3 * max(np.linalg.norm(yr), 1e-30)
