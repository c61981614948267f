"""Expert parallelism (w8a8_int8_quantized_act_b200/ep.py) across two and four ``gloo`` ranks on CPU.

The exchange logic of ExpertParallelMoE runs as it does on GPUs (all-to-alls of the counts, the
int8 rows, their fp32 scales and the bf16 outputs, the (source rank, local expert) groups of the
received rows); its three compute steps are given here by the oracle, so that the result can be
checked without a GPU. Each rank holds its share of the experts and its own tokens; y of every rank must
equal, bit for bit, the single-process oracle forward of all ranks' tokens with the same routing
("Qwen3-235B-A22B-quantized.w8a8" file-structure explainer: 128 experts, 8 per token, weights
sharded over cards; every step of the forward is row-wise, so the split changes no bit).
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

WORLD = 2  # the default; one case below runs four ranks


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bf16_tensor(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _bits(t):
    import torch
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class OracleSteps:
    """route_group / experts / combine of ep.ExpertParallelMoE, computed by the oracle on CPU."""

    def __init__(self, routing):
        self.routing = routing  # (ids [T, k], weights [T, k]) of this rank's tokens

    def route_group(self, x, wg, E, k, renorm, bias):
        import torch

        from oracle import w8a8_oracle as O
        from w8a8_int8_quantized_act_b200.ep import Routed

        ids, w = self.routing
        xq, sx = O.quant_act_per_token(_bits(x))
        perm, offsets = O.group_by_expert(ids, E)
        tok = perm // k
        return Routed(offsets=[int(v) for v in offsets], perm=torch.from_numpy(perm.astype(np.int32)),
                      topk_w=torch.from_numpy(np.asarray(w, np.float32)),
                      xq=torch.from_numpy(np.ascontiguousarray(xq[tok])),
                      sx=torch.from_numpy(np.ascontiguousarray(sx[tok])))

    def alloc_rows(self, A, H, device):
        import torch
        return torch.zeros((A, H), dtype=torch.int8)

    def experts(self, xq, sx, offsets, weights, weight_groups):
        from oracle import w8a8_oracle as O

        wgu_q, s_gu, wd_q, s_d = weights
        A = offsets[-1]
        xq = xq[:A].numpy()
        sx = sx.numpy()
        o = np.zeros((A, xq.shape[1]), np.uint16)
        for g in range(len(offsets) - 1):
            r0, r1 = offsets[g], offsets[g + 1]
            if r1 == r0:
                continue
            e = g % weight_groups
            h = O.gated_activation(O.int_gemm(xq[r0:r1], wgu_q[e]), sx[r0:r1], s_gu[e])
            hq, s_h = O.symmetric_quantize_rows(O.bf16_to_f32(h), O.Q_MAX_INT8)
            o[r0:r1] = O.f32_to_bf16(O.dequant(O.int_gemm(hq, wd_q[e]), s_h, s_d[e]))
        return _bf16_tensor(o)

    def combine(self, o_sorted, perm, topk_w, k):
        from oracle import w8a8_oracle as O

        o = _bits(o_sorted)
        A, H = o.shape
        slots = np.zeros_like(o)
        slots[perm.numpy()] = o
        return _bf16_tensor(O.combine(slots.reshape(A // k, k, H), topk_w.numpy()))


def _worker(rank, world, port, root, tokens, k, E=8):
    if root not in sys.path:
        sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist

    from oracle import w8a8_oracle as O
    from w8a8_int8_quantized_act_b200 import synth
    from w8a8_int8_quantized_act_b200.ep import ExpertParallelMoE

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = synth.MoEWorkload("ep", T=sum(tokens), H=256, E=E, k=k, I=128, n_outlier=2, seed=5)
        inp = synth.moe_inputs(wl)
        wgu_q, s_gu, wd_q, s_d = O.quantize_experts(inp.wgu, inp.wd)
        # every rank builds the same global batch and takes its own slice of tokens
        x_all = inp.x
        t0 = sum(tokens[:rank])
        x_r = x_all[t0:t0 + tokens[rank]]
        full = O.moe_forward(x_all, inp.wg, None, wgu_q, s_gu, wd_q, s_d, k, True)
        ids, w = full["ids"], full["weights"]
        El = wl.E // world
        mine = slice(rank * El, (rank + 1) * El)
        layer = ExpertParallelMoE(_bf16_tensor(inp.wg), wgu_q[mine], s_gu[mine], wd_q[mine], s_d[mine], wl.E, k,
                                  steps=OracleSteps((ids[t0:t0 + tokens[rank]], w[t0:t0 + tokens[rank]])))
        y = layer.forward(_bf16_tensor(x_r))
        assert y.shape == (tokens[rank], wl.H)
        np.testing.assert_array_equal(_bits(y), full["y"][t0:t0 + tokens[rank]])
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("tokens,k", [((64, 64), 2), ((40, 0), 2), ((23, 57), 4)])
def test_expert_parallel_two_gloo_ranks(tokens, k):
    import torch.multiprocessing as mp

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    mp.start_processes(_worker, args=(WORLD, _free_port(), root, tokens, k), nprocs=WORLD, join=True,
                       start_method="spawn")


def test_expert_parallel_four_gloo_ranks():
    # four sources per destination, uneven token counts and one rank without tokens: the
    # (source, local expert) groups of the received rows in source-major order
    import torch.multiprocessing as mp

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    tokens = (31, 0, 70, 16)
    mp.start_processes(_worker, args=(4, _free_port(), root, tokens, 3, 16), nprocs=4, join=True,
                       start_method="spawn")


def test_expert_parallel_rejects_uneven_split():
    import torch
    import torch.distributed as dist

    from w8a8_int8_quantized_act_b200.ep import ExpertParallelMoE

    store = dist.HashStore()
    dist.init_process_group("gloo", store=store, rank=0, world_size=1)
    try:
        w = np.zeros((2, 256, 256), np.int8)
        with pytest.raises(ValueError):
            ExpertParallelMoE(torch.zeros((8, 256)), w, None, w, None, E=8, k=2)  # 2 local experts, not 8
    finally:
        dist.destroy_process_group()
