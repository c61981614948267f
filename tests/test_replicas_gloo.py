"""Multi-rank host logic of the replica layout, on CPU with two ``gloo`` ranks.

The layer shards by tokens with no exchange step: routing, activation quantisation, the
expert FFN and the combine are all per token ("Qwen3-30B-A3B-Instruct-2507-quantized.w8a8"
explainer, section 二: token-granular dynamic activation scales; section 三 3.1: each
token's router scores and top-8 choice). These tests check, across two real processes:

* the benchmark's max-over-ranks timing reduction and whole-job rate;
* that each rank draws its own, distinct batch;
* that the oracle's forward of the two ranks' batches, computed on their own ranks and
  gathered, equals the forward of the concatenated batch: nothing crosses between tokens,
  so replicas need no collective on the data path.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

WORLD = 2


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(wl):
    """Quantised weights of a workload's layer, built from the seeded generators."""
    from oracle import w8a8_oracle as O
    from w8a8_int8_quantized_act_b200 import synth

    inp = synth.moe_inputs(wl)
    wgu_q, s_gu, wd_q, s_d = O.quantize_experts(inp.wgu, inp.wd)
    return inp, wgu_q, s_gu, wd_q, s_d


def _worker(rank, world, port, root):
    if root not in sys.path:
        sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist

    import bench
    from oracle import w8a8_oracle as O
    from w8a8_int8_quantized_act_b200 import synth

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # 1. timing: element-wise max over ranks, whatever rank holds it
        local = [10.0 + rank, 7.0 - 3.0 * rank]
        got = bench.max_over_ranks(dist, local)
        assert got == [10.0 + (world - 1), 7.0], got
        rate = bench.whole_job_rate(world, 64, 100, got[0])
        assert rate == pytest.approx(world * 64 * 100 / (got[0] / 1e3))

        # 2. each rank's own batch of the layer
        wl = synth.MOE_WORKLOADS["tiny"]
        inp, wgu_q, s_gu, wd_q, s_d = _layer(wl)
        x_r = synth.activations(wl.T, wl.H, wl.n_outlier, bench.rank_seed(wl.seed, rank))
        out = O.moe_forward(x_r, inp.wg, inp.bias, wgu_q, s_gu, wd_q, s_d, wl.k, wl.renorm)

        def gather(a):
            t = torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).copy())
            parts = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(parts, t)
            return [p.numpy().view(a.dtype).reshape(a.shape) for p in parts]

        xs = gather(x_r)
        ys = gather(out["y"])
        ids = gather(out["ids"])
        ws = gather(out["weights"])
        if rank == 0:
            for r in range(1, world):
                assert not np.array_equal(xs[0], xs[r]), "ranks drew the same batch"
            x_all = np.concatenate(xs)
            full = O.moe_forward(x_all, inp.wg, inp.bias, wgu_q, s_gu, wd_q, s_d, wl.k, wl.renorm)
            # routing: the same experts per token; weights up to the float64 logit rounding
            # of a different batch size in the BLAS call
            np.testing.assert_array_equal(full["ids"], np.concatenate(ids))
            np.testing.assert_allclose(full["weights"], np.concatenate(ws), rtol=1e-6, atol=1e-7)
            # every later stage given the same routing: bit-exact, token by token
            fed = O.moe_forward(x_all, inp.wg, inp.bias, wgu_q, s_gu, wd_q, s_d, wl.k, wl.renorm,
                                routing=(np.concatenate(ids), np.concatenate(ws)))
            np.testing.assert_array_equal(fed["y"], np.concatenate(ys))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_two_gloo_ranks():
    import torch.multiprocessing as mp

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    mp.start_processes(_worker, args=(WORLD, _free_port(), root), nprocs=WORLD, join=True,
                       start_method="spawn")


def test_max_over_ranks_single_process():
    import bench

    assert bench.max_over_ranks(None, [3.5, 1.25]) == [3.5, 1.25]
    assert bench.rank_seed(7, 0) == 7 and bench.rank_seed(7, 3) != bench.rank_seed(7, 0)
