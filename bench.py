"""Benchmark of the W8A8 MoE expert-FFN layer forward on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

A step is one whole forward (router, grouping + quantisation, gate_up GEMM, requantisation,
down GEMM, combine) over one batch of synthetic tokens. Default workload: the Qwen3-30B-A3B
shaped decode layer (64 tokens, hidden 2048, 128 experts, top-8, intermediate 768).

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier and a device
synchronisation on both sides, timed with CUDA events on the launching stream; the maximum
over ranks is reported. Each step streams the touched experts' weights (about 597 MB for the
decode layer), more than the 126 MB L2, so no step is served from L2 by the previous one.

Multi-GPU (torchrun): replicas. Every rank holds the full layer and runs its own batch of the
same size; nothing is exchanged on the data path (tokens are independent), so scaling is weak.

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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="qwen3-30b-a3b-decode")
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

    def __init__(self, index: int, period_s: float = 0.02):
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
    """Times the oracle (as it stands) on `n_tokens` tokens of the workload; tokens/s."""
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
    t0 = time.perf_counter()
    reps = 0
    while True:
        O.moe_forward(x, wg, bias, wgu_q, s_gu, wd_q, s_d, wl.k, wl.renorm)
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
    """Algorithmic ops and bytes of one layer forward, and bytes of the gate_up launch."""
    touched = int((counts > 0).sum())
    A = wl.T * wl.k
    ops = 2 * A * (2 * wl.I * wl.H + wl.H * wl.I) + 2 * wl.T * wl.H * wl.E
    w_bytes = touched * (3 * wl.I * wl.H + 4 * (2 * wl.I + wl.H))
    io_bytes = 2 * wl.T * wl.H * 2 + 2 * wl.E * wl.H
    gate_up_bytes = touched * (2 * wl.I * wl.H + 4 * 2 * wl.I) + A * wl.H + A * wl.I * 2
    down_bytes = touched * (wl.H * wl.I + 4 * wl.H) + A * wl.I + A * wl.H * 2
    return dict(ops=ops, bytes=w_bytes + io_bytes, touched=touched, gate_up_bytes=gate_up_bytes,
                down_bytes=down_bytes, gate_up_ops=2 * A * 2 * wl.I * wl.H, down_ops=2 * A * wl.H * wl.I)


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


def run_native(args, wl, rank, world, dist):
    import torch

    from w8a8_int8_quantized_act_b200 import binding as B
    from w8a8_int8_quantized_act_b200 import synth

    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B.lib()
    # every rank: its own batch of wl.T tokens (seeded by rank), the full layer's weights
    x_host = synth.activations(wl.T, wl.H, wl.n_outlier, rank_seed(wl.seed, rank))
    inp = synth.moe_inputs(wl)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev)  # noqa: E731
    x = bf(x_host)
    wg = bf(inp.wg)
    bias = torch.from_numpy(inp.bias).to(dev) if inp.bias is not None else None
    wgu_q, s_gu = B.w8a8_quantize_weight_per_channel(bf(inp.wgu))
    wd_q, s_d = B.w8a8_quantize_weight_per_channel(bf(inp.wd))
    del inp
    torch.cuda.empty_cache()
    ws = torch.empty(B.w8a8_moe_workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I), dtype=torch.uint8, device=dev)
    y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        B.w8a8_moe_forward(x, wg, wgu_q, s_gu, wd_q, s_d, wl.k, renorm=wl.renorm, bias=bias, workspace=ws, y=y)

    for _ in range(args.warmup):
        step()
    B.w8a8_check_status()
    counts = np.diff(B.moe_intermediates(ws, wl.T, wl.H, wl.E, wl.k, wl.I)["offsets"].cpu().numpy())

    # ---- timed region 1 (the headline): K replays of the forward captured in a CUDA graph
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
        for i in range(args.steps):
            graph.replay()
        stop.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    B.w8a8_check_status()
    ms = start.elapsed_time(stop)

    # ---- timed region 2: K direct calls recording events at the stage boundaries, for the
    # per-kernel durations (the dominant kernel's roofline figure comes from here)
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
        B.w8a8_moe_forward(xd, wg, wgu_q, s_gu, wd_q, s_d, wl.k, renorm=wl.renorm, bias=bias, workspace=ws, y=yd,
                           stream=st)

    pipelined_e2e(3, x_pin, (wl.T, wl.H), run_e2e, dev)  # warm-up
    if dist is not None:
        dist.barrier()
    e2e_ms = pipelined_e2e(e2e_steps, x_pin, (wl.T, wl.H), run_e2e, dev)
    B.w8a8_check_status()

    ms, e2e_ms = max_over_ranks(dist, [ms, e2e_ms], dev)
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



def run_linear(args, wl, rank, dist):
    """Dense W4A8 linear (x [M, K] bf16 -> y [M, N] bf16) through w8a8_linear."""
    import torch

    from w8a8_int8_quantized_act_b200 import binding as B
    from w8a8_int8_quantized_act_b200 import synth

    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B.lib()
    x_host = synth.activations(wl.M, wl.K, wl.n_outlier, rank_seed(wl.seed, rank))
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev)  # noqa: E731
    x = bf(x_host)
    packed, sw = B.w8a8_quantize_weight_int4_per_group(bf(synth.dense_weight(wl.N, wl.K, wl.seed)), wl.group)
    fmt = B.W8A8_W_INT4_PER_GROUP
    ws = torch.empty(B.w8a8_linear_workspace_size(wl.M, wl.K, wl.N, fmt, wl.group), dtype=torch.uint8, device=dev)
    y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device=dev)
    # rotate over weight copies so every step reads its weights from HBM, not from L2
    copies = [(packed, sw)] + [(packed.clone(), sw.clone()) for _ in range(31)]
    stream = torch.cuda.current_stream()

    def step(i):
        pk, s_ = copies[i % len(copies)]
        B.w8a8_linear(x, pk, s_, fmt, wl.group, workspace=ws, y=y)

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
    # the GEMM alone (dominant kernel): the quantisation is a separate entry point
    xq, sx = B.w8a8_quant_act_per_token(x)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    direct_ms = e0.elapsed_time(e1)
    # end to end with host buffers (copies inside the timed region)
    x_pin = torch.from_numpy(x_host).view(torch.bfloat16).pin_memory()
    n_e2e = max(1, min(args.steps, 200))
    e2e_ws = torch.empty_like(ws)  # the e2e forwards run on their own stream
    e2e_i = [0]

    def run_e2e(xd, yd, st):
        pk, s_ = copies[e2e_i[0] % len(copies)]
        e2e_i[0] += 1
        B.w8a8_linear(xd, pk, s_, fmt, wl.group, workspace=e2e_ws, y=yd, stream=st)

    pipelined_e2e(3, x_pin, (wl.M, wl.N), run_e2e, dev)  # warm-up
    if dist is not None:
        dist.barrier()
    e2e_ms = pipelined_e2e(n_e2e, x_pin, (wl.M, wl.N), run_e2e, dev)
    B.w8a8_check_status()
    ms, e2e_ms = max_over_ranks(dist, [ms, e2e_ms], dev)
    return dict(ms=ms, e2e_ms=e2e_ms, e2e_steps=n_e2e, direct_ms=direct_ms, clocks=clk.summary(),
                h2d=wl.M * wl.K * 2, d2h=wl.M * wl.N * 2)


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one gate_up launch, from one ncu
# capture of the bench's own workload, with the sha1 of the CUDA sources the gate_up GEMMs are built
# from (every csrc file but those holding only other kernels: the quantisation / grouping / combine
# kernels, the fused short-batch front end and the dense W4A8 GEMM); reported only while those
# sources are unchanged (null otherwise, since the counters no longer describe the kernel).
GATE_UP_TRAFFIC = {
    "qwen3-30b-a3b-decode": (391_960_576 + 5_193_216, "3f41d6b0e52cfb0ce400f8b802937efd3d00cde6"),
    "qwen3-30b-a3b-prefill": (541_549_568 + 90_793_984, "3f41d6b0e52cfb0ce400f8b802937efd3d00cde6"),
}


def csrc_sha1():
    import hashlib
    d = os.path.join(os.path.dirname(os.path.abspath(__file__)), "w8a8_int8_quantized_act_b200", "csrc")
    h = hashlib.sha1()
    for name in sorted(os.listdir(d)):
        if name in ("elementwise.cuh", "front.cuh", "gemm_w4a8.cuh"):
            continue
        with open(os.path.join(d, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(workload):
    entry = GATE_UP_TRAFFIC.get(workload)
    if entry is None or entry[1] != csrc_sha1():
        return None
    return entry[0]


def main_linear(args, wl, world, rank, peaks, peak_kind):
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod

        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    res = run_linear(args, wl, rank, dist)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    K = args.steps
    ms_step = res["ms"] / K
    ops = 2.0 * wl.M * wl.N * wl.K
    int8_peak = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = ops / (ms_step / 1e3) / 1e12
    out = {
        "metric": METRIC, "value": whole_job_rate(world, wl.M, K, res["ms"]), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8 (int4 weights unpacked to int8)", "data": "synthetic",
        "config": {"workload": wl.name, "M": wl.M, "K": wl.K, "N": wl.N, "group": wl.group,
                   "parallelism": f"replicas x{world}",
                   "l2": "32 rotating weight copies (201 MB > L2): each step reads its weights from HBM",
                   "timing": "CUDA graphs of quantise + GEMM, replayed K times"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": int8_peak, "unit": "TOPS",
                     "frac": achieved / int8_peak, "traffic": None,
                     "kernel": "w4a8_gemm_kernel (tcgen05 kind::i8, int4 unpacked in shared memory) + x quantisation",
                     "peak_source": f"{peak_kind} bf16 TFLOP/s x 2 (nominal int8:bf16 ratio)"},
        "direct_call_ms_per_step": res["direct_ms"] / K,
        "e2e": {"value": whole_job_rate(world, wl.M, res["e2e_steps"], res["e2e_ms"]), "unit": UNIT,
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"], "overlap": E2E_OVERLAP},
        "gpu_launches": 2 * K, "clocks": res["clocks"],
    }
    print(json.dumps(out))


def main():
    args = parse()
    from w8a8_int8_quantized_act_b200 import synth

    if args.workload in synth.LINEAR_WORKLOADS:
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        peaks, peak_kind = load_peaks()
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the CPU-oracle reference arm covers the MoE "
                              "workloads; run it with the default workload"}))
            return
        return main_linear(args, synth.LINEAR_WORKLOADS[args.workload], world, rank, peaks, peak_kind)
    wl = synth.MOE_WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    peaks, peak_kind = load_peaks()
    sample = args.cpu_sample_tokens or default_sample_tokens(wl)

    if args.impl == "reference":
        if rank != 0:
            return
        rate, reps, el = cpu_oracle_rate(wl, sample, min_seconds=min(30.0, 2.0 * max(1, args.steps)),
                                         max_seconds=120.0)
        cores = blas_threads()
        samp = f"{sample} of the workload's {wl.T} tokens per step, {reps} oracle forwards in {el:.1f} s"
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32/f64 (CPU oracle)", "data": "synthetic",
            "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I},
            "cpu_baseline": {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": samp},
            "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod

        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    res = run_native(args, wl, rank, world, dist)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return

    K = args.steps
    ms_step = res["ms"] / K
    value = whole_job_rate(world, wl.T, K, res["ms"])
    e2e_value = whole_job_rate(world, wl.T, res["e2e_steps"], res["e2e_ms"])
    alg = algorithmic(wl, res["counts"])
    st = dict(zip(("router", "group_quant", "gate_up", "requant", "down", "combine"), res["stage_ms"].tolist()))
    # dominant kernel: the gate_up GEMM (largest share of every step)
    prefill_like = wl.T * wl.k >= 4096
    gu_s = st["gate_up"] / 1e3
    if prefill_like:
        int8_peak = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        achieved = alg["gate_up_ops"] / gu_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": int8_peak, "unit": "TOPS",
                "frac": achieved / int8_peak, "traffic": measured_traffic(wl.name), "traffic_unit": "bytes per launch",
                "kernel": "gate_up grouped INT8 GEMM (tcgen05 kind::i8)",
                "peak_source": f"{peak_kind} bf16 TFLOP/s x 2 (nominal int8:bf16 ratio)"}
    else:
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        achieved = alg["gate_up_bytes"] / gu_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": measured_traffic(wl.name), "traffic_unit": "bytes per launch",
                "kernel": "gate_up grouped INT8 GEMM (tcgen05 kind::i8)",
                "peak_source": f"{peak_kind} HBM copy GB/s"}
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I,
                   "tokens_per_step_per_gpu": wl.T, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: each step streams the touched experts' int8 weights",
                   "timing": "CUDA graph of one forward, replayed K times; stage times from a second pass"},
        "roofline": roof,
        "layer": {"tops": alg["ops"] / (ms_step / 1e3) / 1e12, "gbs": alg["bytes"] / (ms_step / 1e3) / 1e9,
                  "hbm_frac": alg["bytes"] / (ms_step / 1e3) / 1e9 / float(peaks.get("hbm_gbs", 6650.0)),
                  "alg_bytes": alg["bytes"], "alg_ops": alg["ops"], "touched_experts": alg["touched"]},
        "stage_ms": st,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"], "overlap": E2E_OVERLAP},
        "gpu_launches": (5 if (wl.T <= 128 and wl.H <= 2048) else (7 if wl.T <= 512 else 6)) * K,
        "clocks": res["clocks"],
    }
    if not args.no_cpu_baseline:
        rate, reps, el = cpu_oracle_rate(wl, sample)
        out["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                               "sample": f"{sample} tokens of the workload per oracle forward, {reps} forwards "
                                         f"in {el:.1f} s"}
    print(json.dumps(out))


if __name__ == "__main__":
    main()
