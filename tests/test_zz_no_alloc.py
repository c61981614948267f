"""The allocation-free MoE forward (w8a8_moe_forward_noalloc) against the workspace one.

Callers that cannot allocate device memory (a serving hot path where cudaMalloc may stall
the device, a plugin whose host owns all device memory, a fixed memory budget) use the entry
point whose scratch is a buffer built into the library. This checks, through the C ABI, that
two calls in a row on different batches each give exactly the output of w8a8_moe_forward
(the same kernels run, so the bf16 results must be identical) and agree with the CPU oracle
within the layer's tolerance on their own, and that a shape whose scratch would not fit is
refused instead of run. The file name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

from oracle import w8a8_oracle as O
from w8a8_int8_quantized_act_b200 import binding as B
from w8a8_int8_quantized_act_b200 import synth

pytestmark = pytest.mark.gpu


def _dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).view(dtype).cuda()


@pytest.mark.parametrize("name", ["tiny", "qwen3-30b-a3b-decode"])
def test_noalloc_forward_matches_workspace_forward_twice(name):
    wl = synth.MOE_WORKLOADS[name]
    inp = synth.moe_inputs(wl)
    wg = _dev(inp.wg, torch.bfloat16)
    wgu_q, s_gu = B.w8a8_quantize_weight_per_channel(_dev(inp.wgu, torch.bfloat16))
    wd_q, s_d = B.w8a8_quantize_weight_per_channel(_dev(inp.wd, torch.bfloat16))
    from tests import gpu_common as G

    for call, seed in enumerate((11, 12)):  # two calls in a row, different batches
        x_host = synth.activations(wl.T, wl.H, wl.n_outlier, seed)
        x = _dev(x_host, torch.bfloat16)
        ref = B.w8a8_moe_forward(x, wg, wgu_q, s_gu, wd_q, s_d, wl.k, renorm=wl.renorm)
        got = B.w8a8_moe_forward_noalloc(x, wg, wgu_q, s_gu, wd_q, s_d, wl.k, renorm=wl.renorm)
        B.w8a8_check_status()
        a = ref.cpu().view(torch.int16).numpy()
        b = got.cpu().view(torch.int16).numpy()
        np.testing.assert_array_equal(b, a, err_msg=f"call {call}")
        # on its own against the oracle (its own routing): max abs <= 2e-2 and relative L2 <=
        # 5e-3 on every token whose top-k is unambiguous
        inp.x = x_host
        run = G.MoERun(wl, inp, b.view(np.uint16), {}, wgu_q, s_gu, wd_q, s_d)
        r = O.route(x_host, inp.wg, inp.bias, wl.k, wl.renorm)
        G.y_tolerance_check(run, np.arange(wl.T), r.gap > 1e-4)


def test_noalloc_refuses_shapes_beyond_its_buffer():
    wl = synth.MOE_WORKLOADS["qwen3-30b-a3b-prefill"]
    assert B.w8a8_moe_workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I) > B.NOALLOC_SCRATCH_BYTES
    x = torch.zeros((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros((wl.E, wl.H), dtype=torch.bfloat16, device="cuda")
    wgu = torch.zeros((wl.E, 2 * wl.I, wl.H), dtype=torch.int8, device="cuda")
    wd = torch.zeros((wl.E, wl.H, wl.I), dtype=torch.int8, device="cuda")
    s_gu = torch.zeros((wl.E, 2 * wl.I), dtype=torch.float32, device="cuda")
    s_d = torch.zeros((wl.E, wl.H), dtype=torch.float32, device="cuda")
    with pytest.raises(B.W8A8Error) as ei:
        B.w8a8_moe_forward_noalloc(x, wg, wgu, s_gu, wd, s_d, wl.k)
    assert ei.value.status == B.W8A8_ERR_UNSUPPORTED
