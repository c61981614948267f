"""GPU parity of the expert-parallel building blocks (w8a8_moe_route_group, w8a8_moe_experts,
w8a8_moe_combine_sorted) and of ep.ExpertParallelMoE on one GPU.

* W virtual ranks on one GPU, the exchanges done by slicing: every rank routes its own tokens,
  the rows for each destination are cut from the sources' sorted rows and concatenated in source
  order, each destination runs the expert FFN on (source, local expert) groups with its own half
  of the weights, the outputs go back and each source combines. y must equal the oracle's forward
  of all tokens given the GPU's routing, bit for bit, and the intermediates of every stage must
  equal those of the fused forward on the same rank's tokens.
* ExpertParallelMoE with a one-rank NCCL group (its all-to-alls are copies): y bit-exact against
  w8a8_moe_forward on the same tokens.
Runs on more GPUs than one are not part of this suite (the gloo tests on CPU cover the exchange
logic across ranks).
"""
import datetime

import numpy as np
import pytest
import torch

from oracle import w8a8_oracle as O
from w8a8_int8_quantized_act_b200 import binding as B
from w8a8_int8_quantized_act_b200 import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from tests import gpu_common as G  # noqa: E402


def _layer(T, H, E, k, I, seed):
    wl = synth.MoEWorkload("ep", T=T, H=H, E=E, k=k, I=I, n_outlier=3, seed=seed)
    inp = synth.moe_inputs(wl)
    wgu_q, s_gu = B.w8a8_quantize_weight_per_channel(G.bf16_dev(inp.wgu))
    wd_q, s_d = B.w8a8_quantize_weight_per_channel(G.bf16_dev(inp.wd))
    return wl, inp, wgu_q, s_gu, wd_q, s_d


@pytest.mark.parametrize("tokens,H,E,k,I", [((64, 64), 256, 8, 2, 128), ((600, 700), 512, 8, 2, 256),
                                            ((37, 300), 256, 16, 4, 128)])
def test_virtual_ranks_equal_the_forward(tokens, H, E, k, I):
    W = len(tokens)
    T = sum(tokens)
    wl, inp, wgu_q, s_gu, wd_q, s_d = _layer(T, H, E, k, I, seed=T + E)
    El = E // W
    wg = G.bf16_dev(inp.wg)
    starts = np.concatenate([[0], np.cumsum(tokens)])
    # 1. every rank routes and groups its own tokens
    routed = []
    for r in range(W):
        x_r = G.bf16_dev(inp.x[starts[r]:starts[r + 1]])
        ws = B.w8a8_moe_route_group(x_r, wg, E, k, True)
        v = B.moe_intermediates(ws, tokens[r], H, E, k, 128)
        A = tokens[r] * k
        routed.append(dict(offsets=v["offsets"].cpu().numpy().astype(np.int64), perm=v["perm"][:A].clone(),
                           w=v["topk_w"].clone(), ids=v["topk_ids"].clone(), xq=v["xq"][:A].clone(),
                           sx=v["sx_sorted"][:A].clone(), ws=ws))
        # the route_group stage is the fused forward's first two stages, bit for bit
        ws_f = torch.empty(B.w8a8_moe_workspace_size(tokens[r], H, E, k, I), dtype=torch.uint8, device="cuda")
        B.w8a8_moe_forward(x_r, wg, wgu_q, s_gu, wd_q, s_d, k, workspace=ws_f)
        vf = B.moe_intermediates(ws_f, tokens[r], H, E, k, I)
        for name in ("topk_ids", "topk_w", "offsets", "perm", "sx"):
            np.testing.assert_array_equal(G.host(v[name]), G.host(vf[name]))
        np.testing.assert_array_equal(G.host(v["xq"][:A]), G.host(vf["xq"][:A]))
    torch.cuda.synchronize()
    B.w8a8_check_status()
    # 2-4. dispatch by slicing, experts per destination, outputs back
    o_back = [torch.empty((tokens[r] * k, H), dtype=torch.bfloat16, device="cuda") for r in range(W)]
    for d in range(W):
        rows, scales, counts, where = [], [], [], []
        for s in range(W):
            off = routed[s]["offsets"]
            for e in range(El):
                r0, r1 = int(off[d * El + e]), int(off[d * El + e + 1])
                rows.append(routed[s]["xq"][r0:r1])
                scales.append(routed[s]["sx"][r0:r1])
                counts.append(r1 - r0)
                where.append((s, r0, r1))
        A_in = sum(counts)
        xq_in = torch.cat(rows) if A_in else torch.empty((0, H), dtype=torch.int8, device="cuda")
        sx_in = torch.cat(scales) if A_in else torch.empty((0,), dtype=torch.float32, device="cuda")
        offs = np.concatenate([[0], np.cumsum(counts)]).tolist()
        mine = slice(d * El, (d + 1) * El)
        if A_in:
            o_in = B.w8a8_moe_experts(xq_in, sx_in, offs, wgu_q[mine].contiguous(), s_gu[mine].contiguous(),
                                      wd_q[mine].contiguous(), s_d[mine].contiguous(), weight_groups=El)
            for (s, r0, r1), a0, a1 in zip(where, offs[:-1], offs[1:]):
                o_back[s][r0:r1] = o_in[a0:a1]
    # 5. combine on every source
    ys = [B.w8a8_moe_combine_sorted(o_back[r], routed[r]["perm"], routed[r]["w"], k) for r in range(W)]
    torch.cuda.synchronize()
    B.w8a8_check_status()
    # against the oracle given the GPU's routing
    ids = np.concatenate([G.host(rt["ids"]) for rt in routed])
    w = np.concatenate([G.host(rt["w"]) for rt in routed])
    oq_gu, os_gu, oq_d, os_d = O.quantize_experts(inp.wgu, inp.wd)
    ref = O.moe_forward(inp.x, inp.wg, None, oq_gu, os_gu, oq_d, os_d, k, routing=(ids, w))
    np.testing.assert_array_equal(np.concatenate([G.host(y) for y in ys]), ref["y"])


def test_experts_rejects_bad_offsets():
    H, I = 256, 128
    wgu = torch.zeros((2, 2 * I, H), dtype=torch.int8, device="cuda")
    s_gu = torch.ones((2, 2 * I), dtype=torch.float32, device="cuda")
    wd = torch.zeros((2, H, I), dtype=torch.int8, device="cuda")
    s_d = torch.ones((2, H), dtype=torch.float32, device="cuda")
    xq = torch.zeros((10, H), dtype=torch.int8, device="cuda")
    sx = torch.ones((10,), dtype=torch.float32, device="cuda")
    for offs in ([0, 6, 4, 10], [1, 5, 10], [0, 5, 9]):  # decreasing, not from 0, not ending at A
        with pytest.raises(B.W8A8Error):
            B.w8a8_moe_experts(xq, sx, offs, wgu, s_gu, wd, s_d, weight_groups=2, A=10)


def test_expert_parallel_one_rank_nccl():
    import torch.distributed as dist

    from w8a8_int8_quantized_act_b200.ep import ExpertParallelMoE

    T, H, E, k, I = 300, 512, 8, 2, 256
    wl, inp, wgu_q, s_gu, wd_q, s_d = _layer(T, H, E, k, I, seed=11)
    store = dist.HashStore()
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        x = G.bf16_dev(inp.x)
        wg = G.bf16_dev(inp.wg)
        layer = ExpertParallelMoE(wg, wgu_q, s_gu, wd_q, s_d, E, k)
        y = layer.forward(x)
        y_ref = B.w8a8_moe_forward(x, wg, wgu_q, s_gu, wd_q, s_d, k)
        torch.cuda.synchronize()
        B.w8a8_check_status()
        np.testing.assert_array_equal(G.host(y), G.host(y_ref))
    finally:
        dist.destroy_process_group()
