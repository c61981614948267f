"""Seeded synthetic inputs for the W8A8 MoE expert-FFN forward and the dense W4A8 linear.

This module only draws random numbers and names the workloads. It holds none of the
method's arithmetic: no quantisation, no routing, no GEMM. Both the CUDA path (through
the C ABI) and the CPU oracle consume the exact same bytes produced here.

Recipe (the same for every workload):

* Every tensor is drawn in fp32 from a counter-based Philox stream keyed by
  ``(seed, tensor kind, chunk)`` and rounded to bf16 (round-to-nearest-even). Because the
  key names the chunk, any single expert's weights can be regenerated on its own, which
  lets the oracle rebuild only the experts a sampled token touches.
* Activations ``x ~ N(0, 1)``; a fixed set of outlier hidden channels, chosen without
  replacement, is multiplied by 20 (about 1% of the hidden size, as the 30B workload
  states; 2 channels for the tiny layer).
* Router weight ``W_gate ~ N(0, 0.02)`` with shape ``[E, H]`` (nn.Linear layout), kept bf16.
* Expert weights ``N(0, 0.02)``: packed ``gate_up`` ``[E, 2I, H]`` (rows ``0..I-1`` are
  gate_proj, rows ``I..2I-1`` are up_proj, the packed layout of the AMCT Qwen3-Next case
  study, section 2.2) and ``down`` ``[E, H, I]``.
* Skewed router: a bias of +2 on 8 experts drawn without replacement, 0 elsewhere.
* Dense linears (W4A8 and W8A8): ``W ~ N(0, 0.02)`` with shape ``[N, K]``, activations as
  above.
* Shared expert: gate ``w_sg [H]``, packed gate|up ``[2Is, H]`` and down ``[H, Is]``, all
  ``N(0, 0.02)``.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

# Tensor-kind stream ids (part of the Philox key).
_X, _OUTLIER, _WG, _BIAS, _WGU, _WD, _WDENSE, _WSG, _WSGU, _WSD = 1, 2, 3, 4, 5, 6, 7, 8, 9, 10
_ROWS_PER_CHUNK = 256


@dataclass(frozen=True)
class MoEWorkload:
    """Shapes of one MoE layer workload: T tokens, hidden H, E experts, top-k, intermediate I."""

    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    n_outlier: int
    skewed: bool = False
    renorm: bool = True
    seed: int = 0
    shared_I: int = 0  # intermediate size of a shared expert (0: none)

    @property
    def A(self) -> int:
        """Number of (token, expert) assignments."""
        return self.T * self.k


@dataclass(frozen=True)
class LinearWorkload:
    """Dense linear workload: x [M, K] times W [N, K]^T; weights int4 in groups of ``group``
    along K (``fmt`` "int4"), int8 per output channel (``fmt`` "int8"), MXFP8 with both
    operands in blocks of 32 along K (``fmt`` "mxfp8"), or MXFP8 activations with MXFP4 weights
    (``fmt`` "mxfp_a8w4")."""

    name: str
    M: int
    K: int
    N: int
    group: int
    n_outlier: int
    seed: int = 0
    fmt: str = "int4"


MOE_WORKLOADS = {
    w.name: w
    for w in (
        MoEWorkload("tiny", T=64, H=256, E=8, k=2, I=128, n_outlier=2),
        MoEWorkload("qwen3-30b-a3b-decode", T=64, H=2048, E=128, k=8, I=768, n_outlier=20),
        MoEWorkload("qwen3-30b-a3b-prefill", T=8192, H=2048, E=128, k=8, I=768, n_outlier=20),
        MoEWorkload("qwen3-30b-a3b-prefill-skewed", T=8192, H=2048, E=128, k=8, I=768,
                    n_outlier=20, skewed=True),
        MoEWorkload("qwen3-235b-a22b", T=4096, H=4096, E=128, k=8, I=1536, n_outlier=41),
        # the 30B-shaped prefill layer with one shared expert as wide as a routed one (the
        # shared-expert path of the Qwen3-Next / Qwen3.6 layers on a supported expert count)
        MoEWorkload("qwen3-30b-a3b-prefill-shared", T=8192, H=2048, E=128, k=8, I=768, n_outlier=20,
                    shared_I=768),
    )
}

LINEAR_WORKLOADS = {
    w.name: w
    for w in (
        LinearWorkload("qwen3-1.7b-mlp-w4a8", M=2048, K=2048, N=6144, group=128, n_outlier=20),
        # the same MLP shape with int8 per-channel weights, and the Qwen3-30B-A3B attention
        # projections (hidden 2048, 32 query heads and 4 key/value heads of 128): q_proj
        # 2048 -> 4096, k_proj / v_proj 2048 -> 512, o_proj 4096 -> 2048
        LinearWorkload("qwen3-1.7b-mlp-w8a8", M=2048, K=2048, N=6144, group=0, n_outlier=20, fmt="int8"),
        LinearWorkload("qwen3-30b-a3b-q-proj-w8a8", M=2048, K=2048, N=4096, group=0, n_outlier=20, fmt="int8"),
        LinearWorkload("qwen3-30b-a3b-k-proj-w8a8", M=2048, K=2048, N=512, group=0, n_outlier=20, fmt="int8"),
        LinearWorkload("qwen3-30b-a3b-o-proj-w8a8", M=2048, K=4096, N=2048, group=0, n_outlier=41, fmt="int8"),
        # the MLP shape in MXFP8 A8W8 (E4M3 elements, one E8M0 scale per 32 values along K)
        LinearWorkload("qwen3-1.7b-mlp-mxfp8", M=2048, K=2048, N=6144, group=32, n_outlier=20, fmt="mxfp8"),
        # and in MXFP A8W4 (MXFP8 activations, E2M1 weights with one E8M0 scale per 32 values)
        LinearWorkload("qwen3-1.7b-mlp-mxfp-a8w4", M=2048, K=2048, N=6144, group=32, n_outlier=20,
                       fmt="mxfp_a8w4"),
    )
}


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _rng(seed: int, kind: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[int(seed), int(kind) << 32 | int(chunk)]))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (torch's conversion)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _normal_bf16(seed: int, kind: int, chunk: int, shape, std: float) -> np.ndarray:
    a = _rng(seed, kind, chunk).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return to_bf16_bits(a)


def _parallel(fn, items):
    items = list(items)
    if len(items) <= 1:
        return [fn(i) for i in items]
    with ThreadPoolExecutor(min(_threads(), len(items))) as ex:
        return list(ex.map(fn, items))


def outlier_channels(H: int, n_outlier: int, seed: int = 0) -> np.ndarray:
    """Hidden channels scaled by 20, drawn without replacement."""
    return np.sort(_rng(seed, _OUTLIER, 0).permutation(H)[:n_outlier])


def activations(T: int, H: int, n_outlier: int, seed: int = 0) -> np.ndarray:
    """x [T, H] as bf16 bits: N(0,1) with ``n_outlier`` channels multiplied by 20."""
    cols = outlier_channels(H, n_outlier, seed)
    nchunk = max(1, -(-T // _ROWS_PER_CHUNK))

    def one(c):
        r0, r1 = c * _ROWS_PER_CHUNK, min(T, (c + 1) * _ROWS_PER_CHUNK)
        a = _rng(seed, _X, c).standard_normal((r1 - r0, H), dtype=np.float32)
        a[:, cols] *= np.float32(20.0)
        return to_bf16_bits(a)

    if T == 0:
        return np.zeros((0, H), np.uint16)
    return np.concatenate(_parallel(one, range(nchunk)), axis=0)


def router_weight(E: int, H: int, seed: int = 0) -> np.ndarray:
    """W_gate [E, H] as bf16 bits, N(0, 0.02)."""
    return _normal_bf16(seed, _WG, 0, (E, H), 0.02)


def router_bias(E: int, seed: int = 0, n_hot: int = 8, value: float = 2.0) -> np.ndarray:
    """fp32 [E]: +value on n_hot experts drawn without replacement, 0 elsewhere."""
    b = np.zeros(E, np.float32)
    b[_rng(seed, _BIAS, 0).permutation(E)[:n_hot]] = np.float32(value)
    return b


def expert_gate_up(E: int, I: int, H: int, seed: int = 0, experts=None) -> np.ndarray:
    """Packed gate_up [len(experts), 2I, H] as bf16 bits (gate rows first, then up rows)."""
    ids = range(E) if experts is None else [int(e) for e in experts]
    parts = _parallel(lambda e: _normal_bf16(seed, _WGU, e, (2 * I, H), 0.02), ids)
    return np.stack(parts) if parts else np.zeros((0, 2 * I, H), np.uint16)


def expert_down(E: int, H: int, I: int, seed: int = 0, experts=None) -> np.ndarray:
    """down [len(experts), H, I] as bf16 bits."""
    ids = range(E) if experts is None else [int(e) for e in experts]
    parts = _parallel(lambda e: _normal_bf16(seed, _WD, e, (H, I), 0.02), ids)
    return np.stack(parts) if parts else np.zeros((0, H, I), np.uint16)


def shared_expert_weights(H: int, Is: int, seed: int = 0):
    """Shared expert of a layer as bf16 bits: gate w_sg [H] (shared_expert_gate, N(0, 0.02)),
    packed gate|up [2Is, H] and down [H, Is], N(0, 0.02)."""
    return (_normal_bf16(seed, _WSG, 0, (H,), 0.02), _normal_bf16(seed, _WSGU, 0, (2 * Is, H), 0.02),
            _normal_bf16(seed, _WSD, 0, (H, Is), 0.02))


def dense_weight(N: int, K: int, seed: int = 0) -> np.ndarray:
    """Dense W [N, K] as bf16 bits, N(0, 0.02)."""
    nchunk = max(1, -(-N // _ROWS_PER_CHUNK))

    def one(c):
        r0, r1 = c * _ROWS_PER_CHUNK, min(N, (c + 1) * _ROWS_PER_CHUNK)
        return _normal_bf16(seed, _WDENSE, c, (r1 - r0, K), 0.02)

    return np.concatenate(_parallel(one, range(nchunk)), axis=0)


@dataclass
class MoEInputs:
    """Host copies (bf16 bit patterns as uint16) of one MoE workload's inputs."""

    wl: MoEWorkload
    x: np.ndarray
    wg: np.ndarray
    bias: np.ndarray | None
    wgu: np.ndarray | None = field(default=None, repr=False)
    wd: np.ndarray | None = field(default=None, repr=False)


def moe_inputs(wl: MoEWorkload, with_experts: bool = True) -> MoEInputs:
    """Generate every input of ``wl``; expert weights can be skipped (and drawn per expert)."""
    x = activations(wl.T, wl.H, wl.n_outlier, wl.seed)
    wg = router_weight(wl.E, wl.H, wl.seed)
    bias = router_bias(wl.E, wl.seed) if wl.skewed else None
    wgu = expert_gate_up(wl.E, wl.I, wl.H, wl.seed) if with_experts else None
    wd = expert_down(wl.E, wl.H, wl.I, wl.seed) if with_experts else None
    return MoEInputs(wl, x, wg, bias, wgu, wd)
