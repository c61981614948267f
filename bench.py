"""Benchmark of the W8A8 MoE expert-FFN layer forward on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

A step is one whole forward (router, grouping + quantisation, gate_up GEMM with the fused
dequant and SiLU * up, requantisation of h, down GEMM, combine) over one batch of synthetic
tokens. The
headline workload is the largest single-GPU layer: the Qwen3-235B-A22B shaped MoE layer (4096
tokens, hidden 4096, 128 experts, top-8, intermediate 1536). With no --workload the same line
also carries the other workloads as sub-results (the Qwen3-30B-A3B decode, prefill and skewed
prefill layers, the dense W4A8 linear and the dense W8A8 linears), each with its own timing,
roofline, end-to-end figure and CPU-oracle baseline. --workload NAME times one workload alone.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier and a device
synchronisation on both sides, timed with CUDA events on the launching stream; the maximum
over ranks is reported. Every step streams more than the 126 MB L2 (the touched experts'
weights of the MoE layers, 32 rotating weight copies for the dense linears), so no step is
served from L2 by the previous one.

Multi-GPU (torchrun): replicas. Every rank holds the full layer and runs its own batch of the
same size; nothing is exchanged on the data path (tokens are independent), so scaling is weak.
Only the headline workload is timed with more than one rank.

--impl reference times the CPU oracle on this host on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W8A8 MoE layer tokens/s on 1 B200; INT8 TOPS and HBM GB/s vs peak"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet dense INT8 tensor throughput (the 9 POPS figure NVIDIA quotes is with 2:4
# sparsity); fractions are also given against 2 x the measured bf16 GEMM rate (the nominal
# int8:bf16 ratio applied to this machine's measured peak)
INT8_DATASHEET_TOPS = 4500.0  # B200 dense int8 (and fp8)

HEADLINE = "qwen3-235b-a22b"
SUB_MOE = ("qwen3-30b-a3b-decode", "qwen3-30b-a3b-prefill", "qwen3-30b-a3b-prefill-skewed",
           "qwen3-30b-a3b-prefill-shared")
SUB_LINEAR = ("qwen3-1.7b-mlp-w4a8", "qwen3-1.7b-mlp-w8a8", "qwen3-30b-a3b-q-proj-w8a8",
              "qwen3-30b-a3b-k-proj-w8a8", "qwen3-30b-a3b-o-proj-w8a8", "qwen3-1.7b-mlp-mxfp8",
              "qwen3-1.7b-mlp-mxfp-a8w4")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, help="time one workload alone (default: headline + sub-results)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=0)
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                break
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------------------- CPU oracle leg
def cpu_oracle_rate(wl, n_tokens: int, min_seconds: float = 10.0, max_seconds: float = 30.0):
    """Times the oracle (as it stands) on `n_tokens` tokens of the MoE workload; tokens/s."""
    from oracle import w8a8_oracle as O
    from w8a8_int8_quantized_act_b200 import synth

    x = synth.activations(wl.T, wl.H, wl.n_outlier, wl.seed)[:n_tokens]
    wg = synth.router_weight(wl.E, wl.H, wl.seed)
    bias = synth.router_bias(wl.E, wl.seed) if wl.skewed else None
    r = O.route(x, wg, bias, wl.k, wl.renorm)
    touched = np.unique(r.ids)
    gq, gs = O.quantize_weight_per_channel(synth.expert_gate_up(wl.E, wl.I, wl.H, wl.seed, experts=touched))
    dq, ds = O.quantize_weight_per_channel(synth.expert_down(wl.E, wl.H, wl.I, wl.seed, experts=touched))
    d = lambda a: {int(e): a[i] for i, e in enumerate(touched)}  # noqa: E731
    wgu_q, s_gu, wd_q, s_d = d(gq), d(gs), d(dq), d(ds)
    if wl.shared_I:
        wsg, sgu, sd = synth.shared_expert_weights(wl.H, wl.shared_I, wl.seed)
        shared = (wsg, *O.quantize_weight_per_channel(sgu), *O.quantize_weight_per_channel(sd))
        fwd = lambda: O.moe_forward_shared(x, wg, bias, wgu_q, s_gu, wd_q, s_d, wl.k, *shared, renorm=wl.renorm)  # noqa: E731
    else:
        fwd = lambda: O.moe_forward(x, wg, bias, wgu_q, s_gu, wd_q, s_d, wl.k, wl.renorm)  # noqa: E731
    t0 = time.perf_counter()
    reps = 0
    while True:
        fwd()
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or (reps >= 1 and el * (reps + 1) / reps > max_seconds):
            break
    return n_tokens * reps / el, reps, el


def cpu_oracle_linear_rate(wl, n_tokens: int, min_seconds: float = 5.0, max_seconds: float = 15.0):
    """Times the oracle's dense linear (as it stands) on `n_tokens` rows of the workload; tokens/s."""
    from oracle import w8a8_oracle as O
    from w8a8_int8_quantized_act_b200 import synth

    x = synth.activations(wl.M, wl.K, wl.n_outlier, wl.seed)[:n_tokens]
    w = synth.dense_weight(wl.N, wl.K, wl.seed)
    if wl.fmt == "int4":
        packed, sw = O.quantize_weight_int4_per_group(w, wl.group)
        fwd = lambda: O.linear_w4a8(x, packed, sw, wl.group)  # noqa: E731
    elif wl.fmt == "mxfp8":
        wc, ws = O.mx_quantize_rows(w)
        fwd = lambda: O.linear_mxfp8(x, wc, ws)  # noqa: E731
    elif wl.fmt == "mxfp_a8w4":
        wp, ws = O.mx4_quantize_rows(w)
        fwd = lambda: O.linear_mxfp_a8w4(x, wp, ws)  # noqa: E731
    else:
        wq, sw = O.quantize_weight_per_channel(w)
        fwd = lambda: O.linear_w8a8(x, wq, sw)  # noqa: E731
    t0 = time.perf_counter()
    reps = 0
    while True:
        fwd()
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or (reps >= 1 and el * (reps + 1) / reps > max_seconds):
            break
    return n_tokens * reps / el, reps, el


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def default_sample_tokens(wl) -> int:
    return min(wl.T, 16)


# ---------------------------------------------------------------------------- algorithmic work
def algorithmic(wl, counts: np.ndarray):
    """Algorithmic ops and bytes of one layer forward, and of its gate_up and down launches.

    Bytes are what the method must move: the touched experts' int8 weights and fp32 scales, x
    in and y out, the bf16 router weight. The implementation's own intermediates (token codes,
    h, o) are not counted."""
    touched = int((counts > 0).sum())
    A = wl.T * wl.k
    ops = 2 * A * (2 * wl.I * wl.H + wl.H * wl.I) + 2 * wl.T * wl.H * wl.E
    w_bytes = touched * (3 * wl.I * wl.H + 4 * (2 * wl.I + wl.H))
    io_bytes = 2 * wl.T * wl.H * 2 + 2 * wl.E * wl.H
    if wl.shared_I:  # the shared expert on every token, its weights and its bf16 gate
        ops += 2 * wl.T * 3 * wl.shared_I * wl.H + 2 * wl.T * wl.H
        w_bytes += 3 * wl.shared_I * wl.H + 4 * (2 * wl.shared_I + wl.H) + 2 * wl.H
    gate_up_bytes = touched * (2 * wl.I * wl.H + 4 * 2 * wl.I)
    down_bytes = touched * (wl.H * wl.I + 4 * wl.H)
    return dict(ops=ops, bytes=w_bytes + io_bytes, touched=touched, gate_up_bytes=gate_up_bytes,
                down_bytes=down_bytes, gate_up_ops=2 * A * 2 * wl.I * wl.H, down_ops=2 * A * wl.H * wl.I)


def moe_launches(wl) -> int:
    """Kernels of this library one forward launches (memsets not counted): the fused front end
    for T <= 128 and H <= 2048, else the router (two kernels for T <= 512) and the grouping;
    then gate_up, the requantisation of h, down and the combine."""
    if wl.T <= 128 and wl.H <= 2048:
        front = 1
    elif wl.T <= 512:
        front = 3
    else:
        front = 2
    small = wl.T * wl.k <= 32 * wl.E
    routed = front + (3 if (small and wl.I <= 1024) else 4)  # requantisation inside the short-batch down GEMM
    return routed + (5 if wl.shared_I else 0)  # shared expert: gate, quantise, gate_up, requantise, down


# ---------------------------------------------------------------------------- native arm
def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's own token batch: the replicas run independent batches of the same layer."""
    return seed + rank


def max_over_ranks(dist, values, device=None):
    """Element-wise maximum over ranks of per-rank timings: the slowest rank sets the job's time."""
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_rate(world: int, units_per_rank_step: int, steps: int, ms: float) -> float:
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    return world * units_per_rank_step * steps / (ms / 1e3)


class MoELayer:
    """One layer's device weights (quantised by the library), shared by workloads of one shape."""

    def __init__(self, wl, dev):
        import torch

        from w8a8_int8_quantized_act_b200 import binding as B
        from w8a8_int8_quantized_act_b200 import synth

        self.key = (wl.H, wl.E, wl.I, wl.seed, wl.shared_I)
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev)  # noqa: E731
        self.wg = bf(synth.router_weight(wl.E, wl.H, wl.seed))
        self.wgu_q, self.s_gu = B.w8a8_quantize_weight_per_channel(bf(synth.expert_gate_up(wl.E, wl.I, wl.H,
                                                                                            wl.seed)))
        self.wd_q, self.s_d = B.w8a8_quantize_weight_per_channel(bf(synth.expert_down(wl.E, wl.H, wl.I, wl.seed)))
        self.shared = None
        if wl.shared_I:
            wsg, sgu, sd = synth.shared_expert_weights(wl.H, wl.shared_I, wl.seed)
            gq, gs = B.w8a8_quantize_weight_per_channel(bf(sgu[None]))
            dq, ds = B.w8a8_quantize_weight_per_channel(bf(sd[None]))
            self.shared = (bf(wsg), gq[0], gs[0], dq[0], ds[0])
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def run_moe(args, wl, layer, rank, dist, dev):
    import torch

    from w8a8_int8_quantized_act_b200 import binding as B
    from w8a8_int8_quantized_act_b200 import synth

    local = dev.index
    # every rank: its own batch of wl.T tokens (seeded by rank), the full layer's weights
    x_host = synth.activations(wl.T, wl.H, wl.n_outlier, rank_seed(wl.seed, rank))
    x = torch.from_numpy(x_host).view(torch.bfloat16).to(dev)
    bias = torch.from_numpy(synth.router_bias(wl.E, wl.seed)).to(dev) if wl.skewed else None
    wg, wgu_q, s_gu, wd_q, s_d = layer.wg, layer.wgu_q, layer.s_gu, layer.wd_q, layer.s_d
    sh = layer.shared
    ws_bytes = (B.w8a8_moe_shared_workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I, wl.shared_I) if sh is not None
                else B.w8a8_moe_workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def forward(xd, yd, st=None):
        if sh is None:
            B.w8a8_moe_forward(xd, wg, wgu_q, s_gu, wd_q, s_d, wl.k, renorm=wl.renorm, bias=bias, workspace=ws, y=yd,
                               stream=st)
        else:
            B.w8a8_moe_forward_shared(xd, wg, wgu_q, s_gu, wd_q, s_d, wl.k, *sh, renorm=wl.renorm, bias=bias,
                                      workspace=ws, y=yd, stream=st)

    def step():
        forward(x, y)

    for _ in range(args.warmup):
        step()
    B.w8a8_check_status()
    counts = np.diff(B.moe_intermediates(ws, wl.T, wl.H, wl.E, wl.k, wl.I)["offsets"].cpu().numpy())

    # ---- timed region (the figure reported): K replays of the forward captured in a CUDA graph
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    graph.replay()
    torch.cuda.synchronize()
    B.w8a8_check_status()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for _ in range(args.steps):
            graph.replay()
        stop.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    B.w8a8_check_status()
    ms = start.elapsed_time(stop)

    # ---- second pass: K direct calls recording events at the stage boundaries, for the
    # per-kernel durations (the dominant kernel's roofline figure comes from here); with a shared
    # expert this pass times the routed layer alone (the same routed kernels)
    nst = 7
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(args.steps)]
    for row in ev:  # torch creates the CUDA event on its first record
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    for i in range(args.steps):
        B.w8a8_moe_forward_profiled(x, wg, wgu_q, s_gu, wd_q, s_d, wl.k, ev[i], renorm=wl.renorm, bias=bias,
                                    workspace=ws, y=y)
    torch.cuda.synchronize()
    B.w8a8_check_status()
    stage_ms = np.zeros(nst - 1)
    for i in range(args.steps):
        for s_ in range(nst - 1):
            stage_ms[s_] += ev[i][s_].elapsed_time(ev[i][s_ + 1])
    stage_ms /= args.steps
    del graph

    # ---- end to end through the public API with host buffers (copies inside the timed region)
    x_pin = torch.from_numpy(x_host).view(torch.bfloat16).pin_memory()
    e2e_steps = max(1, min(args.steps, 500))

    def run_e2e(xd, yd, st):
        forward(xd, yd, st)

    pipelined_e2e(3, x_pin, (wl.T, wl.H), run_e2e, dev)  # warm-up
    if dist is not None:
        dist.barrier()
    e2e_ms = pipelined_e2e(e2e_steps, x_pin, (wl.T, wl.H), run_e2e, dev)
    B.w8a8_check_status()

    ms, e2e_ms = max_over_ranks(dist, [ms, e2e_ms], dev)
    del ws, y, x
    return dict(ms=ms, e2e_ms=e2e_ms, e2e_steps=e2e_steps, stage_ms=stage_ms, counts=counts,
                clocks=clk.summary(), h2d=wl.T * wl.H * 2, d2h=wl.T * wl.H * 2)


E2E_OVERLAP = "double-buffered: copy-in of step i+1 and copy-out of step i-1 overlap step i's compute"


def pipelined_e2e(n, x_pin, y_shape, run, dev):
    """Times n steps end to end with host buffers and returns the elapsed ms. Every step copies
    its input from pinned host memory, runs the forward through the public API and copies its
    result back into pinned host memory, all inside the timed region. As in a serving loop, two
    device buffers per side and three streams (copy in, compute, copy out) let the copies of the
    neighbouring steps overlap a step's compute; buffer reuse is ordered by events.
    run(x_dev, y_dev, stream) enqueues one forward on `stream`."""
    import torch

    h2d, comp, d2h = (torch.cuda.Stream(dev) for _ in range(3))
    xs = [torch.empty(x_pin.shape, dtype=x_pin.dtype, device=dev) for _ in range(2)]
    ys = [torch.empty(y_shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    y_pins = [torch.empty(y_shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d_done, comp_done, d2h_done = [], [], []
    cur = torch.cuda.current_stream(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(cur)
    for st in (h2d, comp, d2h):
        st.wait_event(start)
    for i in range(n):
        b = i % 2
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(comp_done[i - 2])  # step i - 2 has read xs[b]
            xs[b].copy_(x_pin, non_blocking=True)
            h2d_done.append(torch.cuda.Event())
            h2d_done[i].record(h2d)
        with torch.cuda.stream(comp):
            comp.wait_event(h2d_done[i])
            if i >= 2:
                comp.wait_event(d2h_done[i - 2])  # step i - 2's result has left ys[b]
            run(xs[b], ys[b], comp)
            comp_done.append(torch.cuda.Event())
            comp_done[i].record(comp)
        with torch.cuda.stream(d2h):
            d2h.wait_event(comp_done[i])
            y_pins[b].copy_(ys[b], non_blocking=True)
            d2h_done.append(torch.cuda.Event())
            d2h_done[i].record(d2h)
    cur.wait_event(d2h_done[n - 1])
    end.record(cur)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def run_linear(args, wl, rank, dist, dev):
    """Dense W4A8 / W8A8 linear (x [M, K] bf16 -> y [M, N] bf16) through w8a8_linear."""
    import torch

    from w8a8_int8_quantized_act_b200 import binding as B
    from w8a8_int8_quantized_act_b200 import synth

    local = dev.index
    x_host = synth.activations(wl.M, wl.K, wl.n_outlier, rank_seed(wl.seed, rank))
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev)  # noqa: E731
    x = bf(x_host)
    w = bf(synth.dense_weight(wl.N, wl.K, wl.seed))
    mx = wl.fmt in ("mxfp8", "mxfp_a8w4")
    if wl.fmt == "int4":
        wq, sw = B.w8a8_quantize_weight_int4_per_group(w, wl.group)
        fmt, group = B.W8A8_W_INT4_PER_GROUP, wl.group
    elif wl.fmt == "mxfp8":
        wq, sw = B.w8a8_mxfp8_quantize(w)  # E4M3 codes [N, K], E8M0 scales [N, K/32]
        fmt, group = None, 32
    elif wl.fmt == "mxfp_a8w4":
        wq, sw = B.w8a8_mxfp4_quantize(w)  # packed E2M1 codes [N, K/2], E8M0 scales [N, K/32]
        fmt, group = None, 32
    else:
        wq, sw = B.w8a8_quantize_weight_per_channel(w)
        fmt, group = B.W8A8_W_INT8_PER_CHANNEL, 128
    del w
    ws_bytes = (B.w8a8_mxfp8_linear_workspace_size(wl.M, wl.K, wl.N) if mx
                else B.w8a8_linear_workspace_size(wl.M, wl.K, wl.N, fmt, group))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def linear(xd, pk, s_, wsp, yd, st=None):
        if wl.fmt == "mxfp8":
            B.w8a8_mxfp8_linear(xd, pk, s_, workspace=wsp, y=yd, stream=st)
        elif wl.fmt == "mxfp_a8w4":
            B.w8a8_mxfp_a8w4_linear(xd, pk, s_, workspace=wsp, y=yd, stream=st)
        else:
            B.w8a8_linear(xd, pk, s_, fmt, group, workspace=wsp, y=yd, stream=st)

    y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device=dev)
    # rotate over weight copies (more than the L2 together) so every step reads its weights from HBM
    n_copies = max(2, min(32, -(-256 * 2 ** 20 // (wq.numel() * wq.element_size()))))
    copies = [(wq, sw)] + [(wq.clone(), sw.clone()) for _ in range(n_copies - 1)]
    stream = torch.cuda.current_stream()

    def step(i):
        pk, s_ = copies[i % len(copies)]
        linear(x, pk, s_, ws, y)

    for i in range(args.warmup):
        step(i)
    B.w8a8_check_status()
    graphs = []
    for i in range(len(copies)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(i)
        graphs.append(g)
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(args.steps):
            graphs[i % len(graphs)].replay()
        stop.record(stream)
        torch.cuda.synchronize()
    B.w8a8_check_status()
    ms = start.elapsed_time(stop)
    # the GEMM launch alone (the dominant kernel): the quantised activations are made once, then
    # K GEMM launches are timed with events on the launching stream
    if mx:
        gemm_ms = time_mxfp8_gemm(B, x, copies, wl, args.steps, stream)
    else:
        gemm_ms = time_linear_gemm(B, x, copies, fmt, group, wl, args.steps, stream)
    # end to end with host buffers (copies inside the timed region)
    x_pin = torch.from_numpy(x_host).view(torch.bfloat16).pin_memory()
    n_e2e = max(1, min(args.steps, 200))
    e2e_ws = torch.empty_like(ws)  # the e2e forwards run on their own stream
    e2e_i = [0]

    def run_e2e(xd, yd, st):
        pk, s_ = copies[e2e_i[0] % len(copies)]
        e2e_i[0] += 1
        linear(xd, pk, s_, e2e_ws, yd, st)

    pipelined_e2e(3, x_pin, (wl.M, wl.N), run_e2e, dev)  # warm-up
    if dist is not None:
        dist.barrier()
    e2e_ms = pipelined_e2e(n_e2e, x_pin, (wl.M, wl.N), run_e2e, dev)
    B.w8a8_check_status()
    ms, e2e_ms = max_over_ranks(dist, [ms, e2e_ms], dev)
    return dict(ms=ms, e2e_ms=e2e_ms, e2e_steps=n_e2e, gemm_ms=gemm_ms, clocks=clk.summary(),
                h2d=wl.M * wl.K * 2, d2h=wl.M * wl.N * 2,
                weight_bytes=wq.numel() * wq.element_size() + sw.numel() * sw.element_size())


def time_mxfp8_gemm(B, x, copies, wl, steps, stream):
    """Mean duration (ms) of the MX linear's GEMM launch alone: x is quantised to MXFP8 once,
    then K launches of w8a8_mxfp8_linear_prequant (or w8a8_mxfp_a8w4_linear_prequant) over the
    rotating weight copies are timed with CUDA events on `stream`."""
    import torch

    gemm = B.w8a8_mxfp_a8w4_linear_prequant if wl.fmt == "mxfp_a8w4" else B.w8a8_mxfp8_linear_prequant
    xc, xs = B.w8a8_mxfp8_quantize(x)
    y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device=x.device)
    for i in range(3):
        pk, s_ = copies[i % len(copies)]
        gemm(xc, xs, pk, s_, y=y)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(steps):
        pk, s_ = copies[i % len(copies)]
        gemm(xc, xs, pk, s_, y=y)
    e1.record(stream)
    torch.cuda.synchronize()
    B.w8a8_check_status()
    return e0.elapsed_time(e1) / steps


def time_linear_gemm(B, x, copies, fmt, group, wl, steps, stream):
    """Mean duration (ms) of the linear's GEMM launch alone: the activations are quantised once,
    then K launches of w8a8_linear_prequant are timed with CUDA events on `stream`."""
    import torch

    xq, sx = B.w8a8_quant_act_per_token(x)
    y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device=x.device)
    for i in range(3):
        pk, s_ = copies[i % len(copies)]
        B.w8a8_linear_prequant(xq, sx, pk, s_, fmt, group, y=y)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(steps):
        pk, s_ = copies[i % len(copies)]
        B.w8a8_linear_prequant(xq, sx, pk, s_, fmt, group, y=y)
    e1.record(stream)
    torch.cuda.synchronize()
    B.w8a8_check_status()
    return e0.elapsed_time(e1) / steps


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the dominant kernel,
# from one ncu capture of that workload, with the sha1 of the CUDA sources the kernel is built from;
# reported only while those sources are unchanged (null otherwise: the counters no longer describe
# the kernel). Keys: workload name.
MEASURED_TRAFFIC = {
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum on the gate_up launch of the
    # Qwen3-235B-A22B-shaped layer (1 pass, full workload): 1906.3 MB read + 97.3 MB written
    "qwen3-235b-a22b": (1_906_306_560 + 97_287_424, "43cc740bc128bff5c184ea5be0154d9b92498849"),
    # the same two metrics on the gate_up launch of the 30B-shaped layers: decode (T = 64)
    # 392.0 MB read + 3.9 MB written; prefill (T = 8192) 538.7 MB read + 88.7 MB written
    "qwen3-30b-a3b-decode": (391_971_072 + 3_937_280, "43cc740bc128bff5c184ea5be0154d9b92498849"),
    "qwen3-30b-a3b-prefill": (538_654_208 + 88_660_224, "43cc740bc128bff5c184ea5be0154d9b92498849"),
    # the W4A8 GEMM launch of the 2048 x 2048 -> 6144 linear: 10.9 MB read (weights, scales, token
    # codes once), nothing written back to DRAM within the launch (the 25 MB output stays in L2)
    "qwen3-1.7b-mlp-w4a8": (10_932_992 + 0, "3d048a51e1c8030a8b0a8441792e2ca2d2309450"),
    # the block-scaled MXFP8 GEMM launch (CTA pairs) of the same shape: 17.3 MB read (FP8 weights
    # and scales, token codes and scales, each once), nothing written back within the launch
    "qwen3-1.7b-mlp-mxfp8": (17_344_256 + 0, "6f75f15e5f7becc17f8027677e0192c83257eacd"),
    # the MXFP A8W4 GEMM launch of the same shape: 11.1 MB read (6.3 MB of packed E2M1 weights, their
    # scales, the token codes and scales, each once), nothing written back within the launch
    "qwen3-1.7b-mlp-mxfp-a8w4": (11_052_544 + 0, "6f75f15e5f7becc17f8027677e0192c83257eacd"),
}
TRAFFIC_SOURCES = {  # device-code files each dominant kernel is built from
    "gate_up": ("gemm.cuh", "gemm_pair.cuh", "numerics.cuh", "ptx.cuh", "routing.cuh"),
    "w4a8": ("gemm.cuh", "gemm_w4a8.cuh", "numerics.cuh", "ptx.cuh", "routing.cuh"),
    "w8a8": ("gemm.cuh", "gemm_pair.cuh", "numerics.cuh", "ptx.cuh", "routing.cuh"),
    "mxfp8": ("elementwise.cuh", "gemm.cuh", "mxfp8.cuh", "numerics.cuh", "ptx.cuh", "routing.cuh"),
}


def csrc_sha1(kind: str) -> str:
    import hashlib
    d = os.path.join(ROOT, "w8a8_int8_quantized_act_b200", "csrc")
    h = hashlib.sha1()
    for name in sorted(TRAFFIC_SOURCES[kind]):
        path = os.path.join(d, name)
        if os.path.exists(path):
            with open(path, "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()


def measured_traffic(workload: str, kind: str):
    entry = MEASURED_TRAFFIC.get(workload)
    if entry is None or entry[1] != csrc_sha1(kind):
        return None
    return entry[0]


def tensor_fracs(ops: float, seconds: float, peaks) -> dict:
    tops = ops / seconds / 1e12
    derived = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    return {"tops": tops, "frac_of_2x_measured_bf16": tops / derived, "peak_2x_measured_bf16": derived,
            "frac_of_datasheet": tops / INT8_DATASHEET_TOPS, "peak_datasheet": INT8_DATASHEET_TOPS}


def roofline_entry(ops: float, nbytes: float, seconds: float, peaks, peak_kind, traffic, kernel: str) -> dict:
    """Roofline of one kernel launch: bound by whichever of its tensor time (at 2 x the measured
    bf16 rate) and its HBM time (at the measured copy bandwidth) is longer."""
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tf = tensor_fracs(ops, seconds, peaks)
    t_ops = ops / (tf["peak_2x_measured_bf16"] * 1e12)
    t_bytes = nbytes / (hbm * 1e9)
    gbs = nbytes / seconds / 1e9
    if t_ops >= t_bytes:
        roof = {"bound": "tensor", "achieved": tf["tops"], "peak": tf["peak_2x_measured_bf16"], "unit": "TOPS",
                "frac": tf["frac_of_2x_measured_bf16"],
                "peak_source": f"{peak_kind} bf16 TFLOP/s x 2 (nominal int8 or fp8 : bf16 ratio)"}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                "peak_source": f"{peak_kind} HBM copy GB/s"}
    roof.update({"traffic": traffic, "traffic_unit": "bytes per launch", "kernel": kernel,
                 "alg_ops": ops, "alg_bytes": nbytes, "launch_ms": seconds * 1e3,
                 "tensor": tf, "hbm": {"gbs": gbs, "frac": gbs / hbm, "peak": hbm}})
    return roof


def moe_result(wl, res, K, world, peaks, peak_kind):
    ms_step = res["ms"] / K
    alg = algorithmic(wl, res["counts"])
    st = dict(zip(("router", "group_quant", "gate_up", "requant", "down", "combine"), res["stage_ms"].tolist()))
    gu_s = st["gate_up"] / 1e3
    roof = roofline_entry(alg["gate_up_ops"], alg["gate_up_bytes"], gu_s, peaks, peak_kind,
                          measured_traffic(wl.name, "gate_up"),
                          "gate_up grouped INT8 GEMM (tcgen05 kind::i8) with the dequant + SiLU*up epilogue")
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    t = ms_step / 1e3
    layer_tf = tensor_fracs(alg["ops"], t, peaks)
    t_ops = alg["ops"] / (layer_tf["peak_2x_measured_bf16"] * 1e12)
    t_bytes = alg["bytes"] / (hbm * 1e9)
    return {
        "value": whole_job_rate(world, wl.T, K, res["ms"]), "unit": UNIT, "ms_per_step": ms_step,
        "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I,
                   "skewed_router": wl.skewed, "shared_expert_I": wl.shared_I, "tokens_per_step_per_gpu": wl.T},
        "roofline": roof,
        "layer": {"tops": layer_tf["tops"], "gbs": alg["bytes"] / t / 1e9, "hbm_frac": alg["bytes"] / t / 1e9 / hbm,
                  "tensor_frac_of_2x_measured_bf16": layer_tf["frac_of_2x_measured_bf16"],
                  "tensor_frac_of_datasheet": layer_tf["frac_of_datasheet"],
                  "roofline_frac": max(t_ops, t_bytes) / t,
                  "roofline_bound": "tensor" if t_ops >= t_bytes else "hbm",
                  "alg_bytes": alg["bytes"], "alg_ops": alg["ops"], "touched_experts": alg["touched"]},
        "stage_ms": st,
        "e2e": {"value": whole_job_rate(world, wl.T, res["e2e_steps"], res["e2e_ms"]), "unit": UNIT,
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"], "overlap": E2E_OVERLAP},
        "gpu_launches": moe_launches(wl) * K,
        "clocks": res["clocks"],
    }


def linear_result(wl, res, K, world, peaks, peak_kind):
    ms_step = res["ms"] / K
    ops = 2.0 * wl.M * wl.N * wl.K
    nbytes = res["weight_bytes"] + wl.M * wl.K * 2 + wl.M * wl.N * 2
    if wl.fmt in ("mxfp8", "mxfp_a8w4"):
        a8w4 = wl.fmt == "mxfp_a8w4"
        kernel = ("MXFP A8W4 GEMM (tcgen05 kind::mxf8f6f4 block-scaled MMA, E2M1 weights x E4M3 tokens, "
                  "E8M0 scales in TMEM)" if a8w4 else
                  "MXFP8 GEMM (tcgen05 kind::mxf8f6f4 block-scaled FP8 MMA, E8M0 scales in TMEM)")
        roof = roofline_entry(ops, nbytes, res["gemm_ms"] / 1e3, peaks, peak_kind,
                              measured_traffic(wl.name, "mxfp8"), kernel)
        step_tf = tensor_fracs(ops, ms_step / 1e3, peaks)
        return {
            "value": whole_job_rate(world, wl.M, K, res["ms"]), "unit": UNIT, "ms_per_step": ms_step,
            "config": {"workload": wl.name, "M": wl.M, "K": wl.K, "N": wl.N,
                       "weights": "mxfp4 e2m1 + e8m0" if a8w4 else "mxfp8 e4m3 + e8m0", "block": 32},
            "roofline": roof,
            "step": {"tops": step_tf["tops"], "tensor_frac_of_2x_measured_bf16": step_tf["frac_of_2x_measured_bf16"],
                     "tensor_frac_of_datasheet": step_tf["frac_of_datasheet"],
                     "note": "step = MXFP8 quantisation of x + block-scaled GEMM"},
            "e2e": {"value": whole_job_rate(world, wl.M, res["e2e_steps"], res["e2e_ms"]), "unit": UNIT,
                    "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"], "overlap": E2E_OVERLAP},
            "gpu_launches": 2 * K,
            "clocks": res["clocks"],
        }
    kind = "w4a8" if wl.fmt == "int4" else "w8a8"
    kernel = ("W4A8 GEMM (tcgen05 kind::i8, int4 unpacked to int8 in shared memory, per-group fp32 scaling)"
              if wl.fmt == "int4" else "W8A8 GEMM (tcgen05 kind::i8, per-token x per-channel dequant epilogue)")
    roof = roofline_entry(ops, nbytes, res["gemm_ms"] / 1e3, peaks, peak_kind, measured_traffic(wl.name, kind), kernel)
    step_tf = tensor_fracs(ops, ms_step / 1e3, peaks)
    return {
        "value": whole_job_rate(world, wl.M, K, res["ms"]), "unit": UNIT, "ms_per_step": ms_step,
        "config": {"workload": wl.name, "M": wl.M, "K": wl.K, "N": wl.N, "weights": wl.fmt,
                   "group": wl.group if wl.fmt == "int4" else None},
        "roofline": roof,
        "step": {"tops": step_tf["tops"], "tensor_frac_of_2x_measured_bf16": step_tf["frac_of_2x_measured_bf16"],
                 "tensor_frac_of_datasheet": step_tf["frac_of_datasheet"],
                 "note": "step = per-token activation quantisation + GEMM"},
        "e2e": {"value": whole_job_rate(world, wl.M, res["e2e_steps"], res["e2e_ms"]), "unit": UNIT,
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"], "overlap": E2E_OVERLAP},
        "gpu_launches": 2 * K,
        "clocks": res["clocks"],
    }


def moe_cpu_baseline(wl, sample, min_s, max_s):
    rate, reps, el = cpu_oracle_rate(wl, sample, min_s, max_s)
    return {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{sample} of the workload's {wl.T} tokens per oracle forward, {reps} forwards in {el:.1f} s"}


def linear_cpu_baseline(wl, sample, min_s, max_s):
    rate, reps, el = cpu_oracle_linear_rate(wl, sample, min_s, max_s)
    return {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{sample} of the workload's {wl.M} rows per oracle call, {reps} calls in {el:.1f} s"}


def int8_gemm_probe(dev, steps=20, n=8192):
    """Rate of this library's plain int8 GEMM (w8a8_gemm_s8s8s32) on an n x n x n problem: the
    build's own measured tcgen05 kind::i8 throughput, for context next to the peaks."""
    import torch

    from w8a8_int8_quantized_act_b200 import binding as B

    g = torch.Generator(device=dev).manual_seed(0)
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
    c = torch.empty((n, n), dtype=torch.int32, device=dev)
    for _ in range(3):
        B.w8a8_gemm_s8s8s32(a, b, c)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        B.w8a8_gemm_s8s8s32(a, b, c)
    e1.record()
    torch.cuda.synchronize()
    B.w8a8_check_status()
    ms = e0.elapsed_time(e1) / steps
    del a, b, c
    torch.cuda.empty_cache()
    return {"shape": [n, n, n], "ms": ms, "tops": 2.0 * n ** 3 / (ms / 1e3) / 1e12}


def top_line(metric_res, name, args, world):
    out = {"metric": METRIC, "value": metric_res["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": metric_res["ms_per_step"], "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic"}
    cfg = dict(metric_res["config"])
    cfg.update({"parallelism": f"replicas x{world}",
                "l2": "inputs larger than L2: each step streams more than 126 MB of int8 weights",
                "timing": "CUDA graph of one step, replayed K times; stage / GEMM times from a second pass"})
    out["config"] = cfg
    for key in ("roofline", "layer", "step", "stage_ms", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        if key in metric_res:
            out[key] = metric_res[key]
    return out


def init_dist(world):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist_mod

    dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return dist_mod


def main():
    args = parse()
    from w8a8_int8_quantized_act_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    peaks, peak_kind = load_peaks()
    name = args.workload or HEADLINE
    single = args.workload is not None

    if args.impl == "reference":
        if rank != 0:
            return
        if name in synth.LINEAR_WORKLOADS:
            wl = synth.LINEAR_WORKLOADS[name]
            sample = args.cpu_sample_tokens or 16
            base = linear_cpu_baseline(wl, sample, min(30.0, 2.0 * max(1, args.steps)), 120.0)
            cfg = {"workload": wl.name, "M": wl.M, "K": wl.K, "N": wl.N, "weights": wl.fmt}
        else:
            wl = synth.MOE_WORKLOADS[name]
            sample = args.cpu_sample_tokens or default_sample_tokens(wl)
            base = moe_cpu_baseline(wl, sample, min(30.0, 2.0 * max(1, args.steps)), 120.0)
            cfg = {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I}
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": base["value"], "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32/f64 (CPU oracle)", "data": "synthetic", "config": cfg,
            "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    import torch

    from w8a8_int8_quantized_act_b200 import binding as B

    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B.lib()
    dist = init_dist(world)
    K = args.steps

    def run_one(wname, layer_cache):
        if wname in synth.LINEAR_WORKLOADS:
            wl = synth.LINEAR_WORKLOADS[wname]
            res = run_linear(args, wl, rank, dist, dev)
            return wl, linear_result(wl, res, K, world, peaks, peak_kind)
        wl = synth.MOE_WORKLOADS[wname]
        key = (wl.H, wl.E, wl.I, wl.seed, wl.shared_I)
        if layer_cache.get("key") != key:
            layer_cache.clear()
            torch.cuda.empty_cache()
            layer_cache["key"], layer_cache["layer"] = key, MoELayer(wl, dev)
        res = run_moe(args, wl, layer_cache["layer"], rank, dist, dev)
        return wl, moe_result(wl, res, K, world, peaks, peak_kind)

    cache = {}
    wl, head = run_one(name, cache)
    subs = {}
    probe = None
    if not single and world == 1:
        for wname in SUB_MOE + SUB_LINEAR:
            _, subs[wname] = run_one(wname, cache)
        cache.clear()
        torch.cuda.empty_cache()
        probe = int8_gemm_probe(dev)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    if not args.no_cpu_baseline and world == 1:
        if name in synth.LINEAR_WORKLOADS:
            head["cpu_baseline"] = linear_cpu_baseline(wl, args.cpu_sample_tokens or 16, 10.0, 30.0)
        else:
            head["cpu_baseline"] = moe_cpu_baseline(wl, args.cpu_sample_tokens or default_sample_tokens(wl), 10.0,
                                                    30.0)
        for wname, sub in subs.items():
            if wname in synth.LINEAR_WORKLOADS:
                sub["cpu_baseline"] = linear_cpu_baseline(synth.LINEAR_WORKLOADS[wname], 16, 4.0, 12.0)
            else:
                swl = synth.MOE_WORKLOADS[wname]
                sub["cpu_baseline"] = moe_cpu_baseline(swl, default_sample_tokens(swl), 4.0, 12.0)
    out = top_line(head, name, args, world)
    if name in synth.LINEAR_WORKLOADS:
        out["dtype"] = {"int4": "int8 (int4 weights unpacked to int8)", "int8": "int8",
                        "mxfp8": "mxfp8 (e4m3 elements, e8m0 scales per 32)",
                        "mxfp_a8w4": "mxfp8 x mxfp4 (e4m3 tokens, e2m1 weights, e8m0 scales per 32)"}[wl.fmt]
    if subs:
        out["sub_results"] = subs
    if probe is not None:
        out["int8_gemm_probe"] = probe
    print(json.dumps(out))


if __name__ == "__main__":
    main()
