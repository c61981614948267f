"""Expert-parallel W8A8 MoE forward over torch.distributed (one process per GPU).

Rank r of W holds the experts [r E/W, (r+1) E/W) and routes its own tokens. The forward is the
single-GPU one cut at its two exchange points ("Qwen3-235B-A22B-quantized.w8a8" file-structure
explainer: 128 experts, 8 per token, weights sharded so that several cards serve the model):

  1. route_group: router, top-k, grouping of the local assignments by global expert and the
     per-token int8 rows (sorted, so the rows for each destination rank are consecutive);
  2. dispatch: the per-(destination, local expert) row counts, then the int8 rows and their fp32
     scales, by all-to-all;
  3. experts: the grouped gate_up / requantisation / down on the received rows, given as groups
     of (source rank, local expert), source-major (regrouped by expert inside the call, the
     outputs written back in received order);
  4. return: the bf16 expert outputs, by all-to-all in the reverse direction;
  5. combine: the outputs back in slot order and the ordered fma chain over the k slots.

Every step is row-wise, so y equals the single-GPU forward of the same tokens bit for bit. The
exchanges are NCCL all-to-alls between the GPUs (int8 rows and fp32 scales out, bf16 rows back);
received rows land in local device memory before any kernel reads them. The compute steps are the
library's CUDA kernels (binding.w8a8_moe_route_group / w8a8_moe_experts / w8a8_moe_combine_sorted);
the class takes them as an object so that the exchange logic can also run under another
implementation of the same three steps.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class Routed:
    """Output of the route_group step on a rank's T tokens (A = T * k assignments)."""

    offsets: list          # host ints [E+1]: sorted rows of each global expert
    perm: torch.Tensor     # [A] int32: sorted row -> slot t*k + j
    topk_w: torch.Tensor   # [T, k] fp32
    xq: torch.Tensor       # [A, H] int8 rows in sorted order
    sx: torch.Tensor       # [A] fp32 per-row (token) scales in sorted order


class GpuSteps:
    """The three compute steps on this library's kernels (device tensors)."""

    def __init__(self, binding):
        self.B = binding

    def route_group(self, x, wg, E: int, k: int, renorm: bool, bias) -> Routed:
        B = self.B
        T, H = x.shape
        if T == 0:
            dev = x.device
            return Routed(offsets=[0] * (E + 1), perm=torch.empty((0,), dtype=torch.int32, device=dev),
                          topk_w=torch.empty((0, k), dtype=torch.float32, device=dev),
                          xq=torch.empty((0, H), dtype=torch.int8, device=dev),
                          sx=torch.empty((0,), dtype=torch.float32, device=dev))
        ws = B.w8a8_moe_route_group(x, wg, E, k, renorm, bias=bias)
        v = B.moe_intermediates(ws, T, H, E, k, 128)
        A = T * k
        return Routed(offsets=[int(o) for o in v["offsets"].cpu().tolist()], perm=v["perm"],
                      topk_w=v["topk_w"], xq=v["xq"][:A], sx=v["sx_sorted"][:A])

    def alloc_rows(self, A: int, H: int, device) -> torch.Tensor:
        return torch.empty((A, H), dtype=torch.int8, device=device)

    def experts(self, xq, sx, offsets: list, weights, weight_groups: int) -> torch.Tensor:
        wgu, s_gu, wd, s_d = weights
        return self.B.w8a8_moe_experts(xq, sx, offsets, wgu, s_gu, wd, s_d, weight_groups=weight_groups)

    def combine(self, o_sorted, perm, topk_w, k: int) -> torch.Tensor:
        return self.B.w8a8_moe_combine_sorted(o_sorted, perm, topk_w, k)


class ExpertParallelMoE:
    """One MoE layer with its experts split evenly over the ranks of `group`.

    wg [E, H] bf16 (replicated), local expert weights wgu [E/W, 2I, H] int8, s_gu [E/W, 2I],
    wd [E/W, H, I] int8, s_d [E/W, H]; forward(x [T_local, H] bf16) -> y [T_local, H] bf16.
    Every rank takes the same collective steps in the same order (the counts, then rows and
    scales out, then rows back), also when it has no tokens. A rank that raises between the
    exchanges leaves the others in their next all-to-all until the process group's timeout ends it
    with an error, so give the group a short timeout.
    """

    def __init__(self, wg, wgu, s_gu, wd, s_d, E: int, k: int, renorm: bool = True, bias=None, group=None,
                 steps=None):
        self.group = group
        self.W = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.W:
            raise ValueError(f"{E} experts do not split evenly over {self.W} ranks")
        self.E, self.k, self.renorm, self.bias = E, k, renorm, bias
        self.El = E // self.W
        if wgu.shape[0] != self.El or wd.shape[0] != self.El:
            raise ValueError(f"expected {self.El} local experts per rank")
        self.wg = wg
        self.weights = (wgu, s_gu, wd, s_d)
        if steps is None:
            from . import binding
            steps = GpuSteps(binding)
        self.steps = steps

    def _a2a(self, out, inp, out_splits, in_splits):
        dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def forward(self, x):
        W, El, k = self.W, self.El, self.k
        T, H = x.shape
        dev = x.device
        r = self.steps.route_group(x, self.wg, self.E, k, self.renorm, self.bias)
        # rows for (destination rank d, its local expert e): consecutive in global expert order
        send_counts = [r.offsets[d * El + e + 1] - r.offsets[d * El + e] for d in range(W) for e in range(El)]
        send_rows = [sum(send_counts[d * El:(d + 1) * El]) for d in range(W)]
        counts_out = torch.tensor(send_counts, dtype=torch.int64, device=dev)
        counts_in = torch.empty_like(counts_out)
        self._a2a(counts_in, counts_out, [El] * W, [El] * W)
        recv_counts = [int(c) for c in counts_in.cpu().tolist()]  # [W * El], source-major
        recv_rows = [sum(recv_counts[s * El:(s + 1) * El]) for s in range(W)]
        A_in = sum(recv_rows)

        xq_in = self.steps.alloc_rows(A_in, H, dev)
        sx_in = torch.empty((A_in,), dtype=torch.float32, device=dev)
        self._a2a(xq_in[:A_in], r.xq.contiguous(), recv_rows, send_rows)
        self._a2a(sx_in, r.sx.contiguous(), recv_rows, send_rows)

        # groups (source s, local expert e), source-major; group s*El + e uses local expert e
        offs = [0]
        for c in recv_counts:
            offs.append(offs[-1] + c)
        if A_in > 0:
            o_in = self.steps.experts(xq_in, sx_in, offs, self.weights, El)
        else:
            o_in = torch.empty((0, H), dtype=torch.bfloat16, device=dev)

        o_back = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
        self._a2a(o_back, o_in.contiguous(), send_rows, recv_rows)
        if T == 0:
            return torch.empty((0, H), dtype=torch.bfloat16, device=dev)
        return self.steps.combine(o_back, r.perm, r.topk_w, k)
