"""CPU oracle for the W8A8 INT8 MoE expert-FFN forward and the dense W8A8/W4A8/MXFP linears.

TEST INFRASTRUCTURE. This module is the slow, plain statement of what the GPU path must
compute. Only the test-suite, the smoke check and the CPU-baseline leg of the benchmark
may import it; the library itself never does, and there is no CPU fallback through it.
It shares no code, constant table or helper with the CUDA sources.

Sources (page title, then the section or block on that page):

* "Qwen3-30B-A3B-Instruct-2507-quantized.w8a8" explainer (lqnn.cn): section 二 (the
  quantization_config fields: int8 weights, channel granularity, symmetric min-max
  observer, static; int8 activations, token granularity, dynamic) and section 三 3.1
  (mlp.gate maps the hidden state to 128 expert scores, softmax, then top-8; the gate
  is not quantized).
* "Qwen3.6-35B-A3B-w8a8量化配置深度解读：config.json与recipe.yaml关键参数解析":
  the ``group_0`` block (weights: num_bits 8, strategy channel, symmetric, dynamic false,
  observer memoryless_minmax; input_activations: num_bits 8, strategy token, symmetric,
  dynamic true) and the recipe's ignore list (``re:.*mlp.gate$``).
* "Qwen3-1.7B-W4A8-V1" explainer: section "4bit 权重" (group_size 128, 4-bit two's
  complement packed weights) and section "8bit 激活" (per-token dynamic activation scale).
* "Qwen3-235B-A22B-quantized.w8a8" file-structure explainer: the model table (128
  experts, 8 per token) and the shard contents (gate_proj / up_proj / down_proj INT8,
  mlp.gate bf16).
* "Qwen3-Next-80B-A3B-Instruct 在 AMCT 中的 MoE 混合注意力量化适配实战", section 二 2.2:
  the packed expert layout (gate_proj and up_proj concatenated along the output feature
  dimension into gate_up_proj; down_proj separate).

Readings where the pages are silent (each one is fixed identically on the GPU side):

* Scale = amax / q_max with q_max = 2**(bits-1) - 1 (127 for int8, 7 for int4); code =
  clamp(round_half_even(v / scale), -q_max, q_max), all in IEEE fp32 with a true divide.
  A row whose amax is 0 gets scale 0 and all-zero codes.
* Router logits and softmax are exact-ish (float64 here); top-k takes the k largest
  probabilities, equal values resolved to the lower expert index, slot order descending;
  the k weights are renormalised to sum to 1 when ``renorm`` is set (Qwen3-MoE default).
* The gated activation is SiLU(gate) * up (the pages name gate/up/down projections but not
  the function). SiLU uses ``spec_exp``, an exponential defined below step by step so that
  both sides produce the same bits; its polynomial is evaluated with fused multiply-adds.
* Dequantisation is ((float)acc * s_token) * s_channel, two fp32 round-to-nearest products.
* h is rounded to bf16 before its per-row requantisation; o is rounded to bf16.
* Combine: acc = 0; for j in 0..k-1: acc = fma(w[t,j], o[t,j,n], acc) (one fp32 rounding
  per step); y = bf16(acc).
* W4A8: y = bf16(acc_f * s_token) where acc_f = fma((float)acc_g, s_w[n, g], acc_f) over the
  K-groups g in order.
* fma(a, b, c) is the fp32 fused multiply-add: a*b + c rounded once. numpy has none, so
  ``fma32`` computes it exactly from float64 arithmetic (see there).
* Shared expert (the Qwen3-Next / Qwen3.6 layers): the shared expert is a dense gated MLP
  quantised W8A8 like the routed experts (the AMCT Qwen3-Next page, section 二 2.2: the shared
  expert is a dense activated path, quantised directly); its gate ``shared_expert_gate`` is a
  bf16 Linear [H] -> 1 kept out of quantisation (the ignore list of the Qwen3.6-35B-A3B recipe).
  The pages do not give the combination: it is read as y = routed + sigmoid(x . w_sg) * shared,
  the shared output entering the combine's fma chain after the k routed slots with weight
  g = sigmoid(z), z the gate logit (float64 here), sigmoid(z) = 1 / (1 + exp(-z)).
* MXFP8 A8W8 (the AMCT Qwen3-Next page, section 六, names "MXFP A8w8" and nothing more): the OCP
  Microscaling FP8 format, blocks of 32 values along K with one E8M0 power-of-two scale and E4M3
  elements; E = floor(log2 amax) - 8, elements rounded to nearest even and saturated at 448. The
  layer's product is the exact sum of the dequantised products; the GPU's fp32 sum of the same
  products is checked within the summation bound (see ``linear_mxfp8``).
* MXFP A8W4 (the same table's "MXFP A8w4" row): MXFP8 activations as above and MXFP4 weights, the
  OCP format with E2M1 elements: E = floor(log2 amax) - 2, elements rounded to nearest even and
  saturated at 6, two codes per byte with the even element in the low nibble (see
  ``mx4_quantize_rows``).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

# num_bits: 8, symmetric: true  ->  codes in [-(2**7 - 1), 2**7 - 1].
Q_MAX_INT8 = np.float32(127.0)
# 4-bit two's-complement weights, symmetric (offset 0)  ->  codes in [-7, 7].
Q_MAX_INT4 = np.float32(7.0)

F32 = np.float32


# --------------------------------------------------------------------------------------
# bf16 <-> fp32
# --------------------------------------------------------------------------------------
def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) to fp32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16(v: np.ndarray) -> np.ndarray:
    """fp32 values to bf16 bit patterns, round to nearest, ties to even (finite inputs)."""
    b = np.asarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))
    return (b >> np.uint64(16)).astype(np.uint16)


def fma32(a, b, c) -> np.ndarray:
    """fp32 fused multiply-add round(a*b + c), computed exactly from float64 arithmetic.

    a*b of two fp32 values is exact in float64. The sum with c is taken in float64 and then
    made "round to odd" (Boldo & Melquiond, 2008): when the float64 sum s is inexact (its
    TwoSum error is non-zero) and its last bit is even, s moves one ulp toward the error.
    Rounding that round-to-odd float64 to fp32 gives the correctly rounded result, because
    float64's 53 bits exceed fp32's 24 by more than the 2 bits the theorem needs.
    """
    a = np.asarray(a, np.float32).astype(np.float64)
    b = np.asarray(b, np.float32).astype(np.float64)
    c = np.asarray(c, np.float32).astype(np.float64)
    p = a * b
    s = p + c
    bb = s - p
    err = (p - (s - bb)) + (c - bb)
    even = (np.asarray(s).view(np.int64) & 1) == 0
    toward = np.where(err > 0, np.inf, -np.inf)
    s = np.where((err != 0) & even, np.nextafter(s, toward), s)
    return np.asarray(s).astype(np.float32)


# --------------------------------------------------------------------------------------
# Symmetric min-max quantisation (one scale per row)
# --------------------------------------------------------------------------------------
def symmetric_quantize_rows(v: np.ndarray, q_max: np.float32):
    """Quantise each row of fp32 ``v`` with its own symmetric scale.

    scale[r] = max_k |v[r, k]| / q_max (fp32 divide); code = clamp(rint(v / scale)).
    Follows the "symmetric", "minmax observer" fields of the group_0 block
    (Qwen3.6-35B-A3B-w8a8 config page) with the round-half-even reading.
    """
    v = np.asarray(v, dtype=np.float32)
    amax = np.max(np.abs(v), axis=-1) if v.shape[-1] else np.zeros(v.shape[:-1], np.float32)
    scale = (amax / q_max).astype(np.float32)
    q = np.zeros(v.shape, np.float32)
    nz = scale > 0
    if np.any(nz):
        q[nz] = np.rint(v[nz] / scale[nz][..., None])
    q = np.clip(q, -q_max, q_max)
    return q.astype(np.int8), scale


def quantize_weight_per_channel(w_bits: np.ndarray):
    """Static per-output-channel int8 weights: w [..., N, K] bf16 -> q int8, scale fp32 [..., N].

    Weights: num_bits 8, strategy "channel", symmetric, dynamic false (group_0 block of the
    Qwen3.6-35B-A3B-w8a8 config page; section 二 of the Qwen3-30B-A3B-2507 w8a8 page).
    One output channel is one row of the nn.Linear weight [out, in].
    """
    return symmetric_quantize_rows(bf16_to_f32(w_bits), Q_MAX_INT8)


def quant_act_per_token(x_bits: np.ndarray):
    """Dynamic per-token int8 activations: x [T, K] bf16 -> q int8 [T, K], scale fp32 [T].

    input_activations: num_bits 8, strategy "token", dynamic true, symmetric (group_0 block
    of the Qwen3.6-35B-A3B-w8a8 config page; "8bit 激活" section of the Qwen3-1.7B-W4A8 page:
    each token's scale is computed online).
    """
    return symmetric_quantize_rows(bf16_to_f32(x_bits), Q_MAX_INT8)


def quantize_weight_int4_per_group(w_bits: np.ndarray, group: int = 128):
    """Symmetric int4 weights with one scale per ``group`` consecutive K values.

    w [N, K] bf16 -> packed uint8 [N, K/2] and scale fp32 [N, K/group]. Codes are 4-bit
    two's complement in [-7, 7]; byte i of a row holds code 2i in its low nibble and code
    2i+1 in its high nibble ("4bit 权重" section of the Qwen3-1.7B-W4A8 page: group_size
    128, two's-complement packing).
    """
    w = bf16_to_f32(w_bits)
    N, K = w.shape
    if K % group or group % 2:
        raise ValueError("K must be a multiple of the (even) group size")
    q, s = symmetric_quantize_rows(w.reshape(N, K // group, group), Q_MAX_INT4)
    q = q.reshape(N, K).astype(np.int16)
    lo = q[:, 0::2] & 0xF
    hi = q[:, 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8), s


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """Inverse of the packing above: uint8 [N, K/2] -> int8 codes [N, K] (sign-extended)."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((p.shape[0], p.shape[1] * 2), np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


# --------------------------------------------------------------------------------------
# Exact integer GEMM
# --------------------------------------------------------------------------------------
def int_gemm(a_q: np.ndarray, b_q: np.ndarray) -> np.ndarray:
    """acc[r, n] = sum_k a[r, k] * b[n, k] exactly, as int32.

    The products of int8 codes are summed in float64: every partial sum is an integer of
    magnitude at most 127*127*K < 2**53, so any summation order is exact. The result must
    fit int32 (|acc| <= 16129*K), which holds for K < 133143.
    """
    acc = np.asarray(a_q, np.float64) @ np.asarray(b_q, np.float64).T
    if acc.size and np.max(np.abs(acc)) >= 2.0**31:
        raise OverflowError("int32 accumulator overflow")
    return acc.astype(np.int64).astype(np.int32)


# --------------------------------------------------------------------------------------
# The exponential used by SiLU
# --------------------------------------------------------------------------------------
LOG2E = np.float32(1.4426950408889634)
# ln 2 split Cody-Waite style: the high part has 15 significant bits, so n * LN2_HI is exact
# for |n| < 2**8, and the low part carries the rest of ln 2.
LN2_HI = np.float32(0.693145751953125)
LN2_LO = np.float32(0.6931471805599453 - 0.693145751953125)
# Taylor coefficients 1/i!, i = 0..7, rounded to fp32.
TAYLOR = [np.float32(1.0 / f) for f in (1, 1, 2, 6, 24, 120, 720, 5040)]
EXP_HI = np.float32(88.0)
EXP_LO = np.float32(-87.0)


def spec_exp(x: np.ndarray) -> np.ndarray:
    """exp(x) in fp32 by Cody-Waite range reduction and a degree-7 Taylor polynomial.

    n = rint(x * log2(e)) (fp32 product); r = fma(-n, LN2_LO, fma(-n, LN2_HI, x));
    p = sum_{i<=7} r^i / i! by Horner with fused multiply-adds, p = fma(p, r, 1/i!);
    result = p * 2^n (exact scaling). x > 88 gives +inf, x < -87 gives 0. Error is within a
    few ulp of the true exponential.
    """
    x = np.asarray(x, dtype=np.float32)
    xc = np.clip(x, EXP_LO, EXP_HI)
    n = np.rint(xc * LOG2E).astype(np.float32)
    r = fma32(-n, LN2_LO, fma32(-n, LN2_HI, xc))
    p = np.full(x.shape, TAYLOR[7], np.float32)
    for c in TAYLOR[6::-1]:
        p = fma32(p, r, c)
    two_n = ((n.astype(np.int32) + 127).astype(np.uint32) << np.uint32(23)).view(np.float32)
    out = p * two_n
    out = np.where(x > EXP_HI, np.float32(np.inf), out)
    out = np.where(x < EXP_LO, np.float32(0.0), out)
    return out.astype(np.float32)


def silu(g: np.ndarray) -> np.ndarray:
    """SiLU(g) = g / (1 + exp(-g)) in fp32 with ``spec_exp`` and a true divide."""
    g = np.asarray(g, dtype=np.float32)
    with np.errstate(over="ignore"):
        d = np.float32(1.0) + spec_exp(-g)
    return (g / d).astype(np.float32)


# --------------------------------------------------------------------------------------
# Router: bf16 gate GEMM, softmax, top-k (never quantised)
# --------------------------------------------------------------------------------------
@dataclass
class Routing:
    logits: np.ndarray  # float64 [T, E]
    probs: np.ndarray  # float64 [T, E]
    ids: np.ndarray  # int32 [T, k], slot order = descending probability
    weights: np.ndarray  # float32 [T, k]
    gap: np.ndarray  # float64 [T]: p_(k) - p_(k+1) (inf when k == E)


def route(x_bits, wg_bits, bias=None, k: int = 8, renorm: bool = True) -> Routing:
    """mlp.gate in bf16 (never quantised), softmax over experts, top-k selection.

    Section 三 3.1 of the Qwen3-30B-A3B-2507 w8a8 page: the gate maps the hidden state to one
    score per expert, a softmax follows and the top-8 experts take part in the forward; the
    recipe's ignore list keeps ``mlp.gate`` out of quantisation. ``bias`` (optional) is added
    to the logits; it only serves the skewed-routing stress workload.
    """
    x = bf16_to_f32(x_bits).astype(np.float64)
    wg = bf16_to_f32(wg_bits).astype(np.float64)
    logits = x @ wg.T
    if bias is not None:
        logits = logits + np.asarray(bias, np.float64)[None, :]
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    if T == 0:
        z = np.zeros((0, k))
        return Routing(logits, logits.copy(), z.astype(np.int32), z.astype(np.float32), np.zeros(0))
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    probs = e / e.sum(axis=1, keepdims=True)
    order = np.argsort(-probs, axis=1, kind="stable")  # equal values keep index order
    ids = order[:, :k]
    sel = np.take_along_axis(probs, ids, axis=1)
    w = sel / sel.sum(axis=1, keepdims=True) if renorm else sel
    srt = np.take_along_axis(probs, order, axis=1)
    gap = srt[:, k - 1] - srt[:, k] if k < E else np.full(T, np.inf)
    return Routing(logits, probs, ids.astype(np.int32), w.astype(np.float32), gap)


# --------------------------------------------------------------------------------------
# Grouping assignments by expert
# --------------------------------------------------------------------------------------
def group_by_expert(ids: np.ndarray, E: int):
    """Stable counting sort of the T*k assignments by expert.

    Assignment a = t*k + j goes to expert ids[t, j]. Returns perm [A] (perm[r] = the
    assignment placed at sorted row r; rows of one expert are ordered by token) and
    offsets [E+1] (rows of expert e are offsets[e] .. offsets[e+1]-1).
    """
    flat = np.asarray(ids, np.int64).reshape(-1)
    perm = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E) if flat.size else np.zeros(E, np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    return perm.astype(np.int32), offsets.astype(np.int64)


# --------------------------------------------------------------------------------------
# Epilogues
# --------------------------------------------------------------------------------------
def dequant(acc: np.ndarray, s_row: np.ndarray, s_col: np.ndarray) -> np.ndarray:
    """((float)acc * s_row) * s_col, each product rounded to fp32."""
    a = np.asarray(acc, np.int32).astype(np.float32)
    return (a * np.asarray(s_row, np.float32)[:, None]) * np.asarray(s_col, np.float32)[None, :]


def gated_activation(acc_gu: np.ndarray, s_row: np.ndarray, s_gu: np.ndarray) -> np.ndarray:
    """h = bf16(SiLU(gate) * up) from the int32 gate_up accumulators of one expert.

    Columns 0..I-1 of the packed gate_up output are gate_proj, I..2I-1 are up_proj (AMCT
    Qwen3-Next page, section 二 2.2: gate and up concatenated along the feature dimension).
    """
    I = acc_gu.shape[1] // 2
    g = dequant(acc_gu[:, :I], s_row, s_gu[:I])
    u = dequant(acc_gu[:, I:], s_row, s_gu[I:])
    return f32_to_bf16(silu(g) * u)


def combine_acc(o_bits: np.ndarray, w: np.ndarray) -> np.ndarray:
    """The fp32 accumulator of the weighted combine: acc = 0, then for j = 0 .. k-1 in slot
    order acc = fma(w[t, j], o[t, j], acc), one rounding per slot."""
    o = bf16_to_f32(o_bits)
    T, k, H = o.shape
    acc = np.zeros((T, H), np.float32)
    w = np.asarray(w, np.float32)
    for j in range(k):
        acc = fma32(np.broadcast_to(w[:, j:j + 1], (T, H)), o[:, j, :], acc)
    return acc


def combine_acc_with_shared(o_bits: np.ndarray, w: np.ndarray, o_shared_bits: np.ndarray, g: np.ndarray
                            ) -> np.ndarray:
    """The combine's fp32 accumulator extended by the shared expert: acc over the k routed slots
    as in ``combine_acc``, then acc = fma(g[t], o_shared[t], acc), one rounding."""
    acc = combine_acc(o_bits, w)
    o_s = bf16_to_f32(o_shared_bits)
    g = np.asarray(g, np.float32)
    return fma32(np.broadcast_to(g[:, None], o_s.shape), o_s, acc)


def combine_with_shared(o_bits: np.ndarray, w: np.ndarray, o_shared_bits: np.ndarray, g: np.ndarray) -> np.ndarray:
    """y[t] = bf16(``combine_acc_with_shared``)."""
    return f32_to_bf16(combine_acc_with_shared(o_bits, w, o_shared_bits, g))


def combine(o_bits: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y[t] = bf16(sum_j w[t, j] * o[t, j]): the fma chain of ``combine_acc``, rounded to bf16.

    Section 三 3.1 of the Qwen3-30B-A3B-2507 w8a8 page: the selected experts' outputs are
    weighted by the router and summed."""
    return f32_to_bf16(combine_acc(o_bits, w))


# --------------------------------------------------------------------------------------
# The MoE expert-FFN layer
# --------------------------------------------------------------------------------------
def quantize_experts(wgu_bits, wd_bits):
    """Offline weight preparation of every expert (per-channel int8)."""
    wgu_q, s_gu = quantize_weight_per_channel(wgu_bits)
    wd_q, s_d = quantize_weight_per_channel(wd_bits)
    return wgu_q, s_gu, wd_q, s_d


def moe_forward(x_bits, wg_bits, bias, wgu_q, s_gu, wd_q, s_d, k: int, renorm: bool = True,
                routing: tuple | None = None) -> dict:
    """W8A8 MoE expert-FFN forward of one Qwen3-MoE layer.

    Steps: route (bf16, never quantised) -> per-token int8 quantisation of x -> per expert,
    int32 GEMM with the packed int8 gate_up weight -> dequant, SiLU(gate)*up, bf16 h ->
    per-row int8 requantisation of h -> int32 GEMM with the int8 down weight -> dequant to
    bf16 o -> weighted combine to bf16 y.

    ``wgu_q[e]``, ``s_gu[e]``, ``wd_q[e]``, ``s_d[e]`` are read only for experts that
    receive tokens, so dicts holding just those experts work. ``routing = (ids, weights)``
    replaces the oracle's own router (the GPU's routing can be fed in to compare every
    later stage exactly). Per-assignment results are returned in slot order [T, k, ...].
    """
    x_bits = np.asarray(x_bits, np.uint16)
    T, H = x_bits.shape
    E = np.asarray(wg_bits).shape[0]
    if routing is None:
        r = route(x_bits, wg_bits, bias, k, renorm)
        ids, w = r.ids, r.weights
    else:
        r = None
        ids = np.asarray(routing[0], np.int32)
        w = np.asarray(routing[1], np.float32)
    xq, sx = quant_act_per_token(x_bits)
    perm, offsets = group_by_expert(ids, E)

    first = None
    A = T * k
    h = hq = o = s_h = None
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        slots = perm[r0:r1]  # assignment ids t*k + j
        tok = slots // k
        acc_gu = int_gemm(xq[tok], wgu_q[e])
        h_e = gated_activation(acc_gu, sx[tok], s_gu[e])
        hq_e, s_h_e = symmetric_quantize_rows(bf16_to_f32(h_e), Q_MAX_INT8)
        acc_d = int_gemm(hq_e, wd_q[e])
        o_e = f32_to_bf16(dequant(acc_d, s_h_e, s_d[e]))
        if first is None:
            first = True
            I = h_e.shape[1]
            h = np.zeros((A, I), np.uint16)
            hq = np.zeros((A, I), np.int8)
            s_h = np.zeros(A, np.float32)
            o = np.zeros((A, H), np.uint16)
        h[slots], hq[slots], s_h[slots], o[slots] = h_e, hq_e, s_h_e, o_e
    if o is None:  # no assignments at all (T == 0)
        o = np.zeros((A, H), np.uint16)
    y = combine(o.reshape(T, k, H), w)
    out = dict(ids=ids, weights=w, xq=xq, sx=sx, perm=perm, offsets=offsets, y=y,
               o=o.reshape(T, k, H))
    if h is not None:
        I = h.shape[1]
        out.update(h=h.reshape(T, k, I), hq=hq.reshape(T, k, I), s_h=s_h.reshape(T, k))
    if r is not None:
        out["routing"] = r
    return out


def shared_gate(x_bits, wsg_bits) -> np.ndarray:
    """g[t] = sigmoid(x[t] . w_sg) in float64: the bf16 shared_expert_gate, never quantised
    (ignore list of the Qwen3.6-35B-A3B recipe)."""
    z = bf16_to_f32(x_bits).astype(np.float64) @ bf16_to_f32(wsg_bits).astype(np.float64).reshape(-1)
    return 1.0 / (1.0 + np.exp(-z))


def shared_expert(x_bits, wgu_q, s_gu, wd_q, s_d) -> dict:
    """The shared expert as a dense W8A8 gated MLP (every token): per-token int8 x, int32 GEMM
    with the packed gate|up weight, dequant, SiLU(gate) * up -> bf16 h, per-row requantisation,
    int32 GEMM with the down weight, dequant -> bf16 o. The same arithmetic as one routed expert
    that every token selects."""
    xq, sx = quant_act_per_token(np.asarray(x_bits, np.uint16))
    h = gated_activation(int_gemm(xq, wgu_q), sx, s_gu)
    hq, s_h = symmetric_quantize_rows(bf16_to_f32(h), Q_MAX_INT8)
    o = f32_to_bf16(dequant(int_gemm(hq, wd_q), s_h, s_d))
    return dict(xq=xq, sx=sx, h=h, hq=hq, s_h=s_h, o=o)


def moe_forward_shared(x_bits, wg_bits, bias, wgu_q, s_gu, wd_q, s_d, k: int, wsg_bits, sh_gu_q, sh_s_gu, sh_d_q,
                       sh_s_d, renorm: bool = True, routing: tuple | None = None, gate: np.ndarray | None = None
                       ) -> dict:
    """MoE layer with a shared expert: the routed forward of ``moe_forward``, the shared expert on
    every token, and y = bf16(fma(g, o_shared, routed fma chain)). ``gate`` replaces the oracle's
    own float64 sigmoid gate (the GPU's fp32 gate can be fed in, like the routing)."""
    out = moe_forward(x_bits, wg_bits, bias, wgu_q, s_gu, wd_q, s_d, k, renorm, routing)
    sh = shared_expert(x_bits, sh_gu_q, sh_s_gu, sh_d_q, sh_s_d)
    g64 = shared_gate(x_bits, wsg_bits)
    g = np.asarray(g64 if gate is None else gate, np.float32)
    out.update(shared=sh, gate=g64, y=combine_with_shared(out["o"], out["weights"], sh["o"], g))
    return out


def moe_forward_float(x_bits, wg_bits, bias, wgu_bits, wd_bits, k: int, renorm: bool = True,
                      routing: tuple | None = None) -> np.ndarray:
    """The same layer with quantisation switched off, in float64 (bf16 inputs, exact SiLU).

    Serves only to bound the error that W8A8 quantisation adds (the quant-off check of the
    AMCT Qwen3-Next page, sections 四 and 五).
    """
    x = bf16_to_f32(x_bits).astype(np.float64)
    T, H = x.shape
    if routing is None:
        r = route(x_bits, wg_bits, bias, k, renorm)
        ids, w = r.ids, r.weights.astype(np.float64)
    else:
        ids, w = np.asarray(routing[0]), np.asarray(routing[1], np.float64)
    y = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            wgu = bf16_to_f32(wgu_bits[e]).astype(np.float64)
            wd = bf16_to_f32(wd_bits[e]).astype(np.float64)
            gu = wgu @ x[t]
            I = gu.shape[0] // 2
            g, u = gu[:I], gu[I:]
            hh = g / (1.0 + np.exp(-g)) * u
            y[t] += w[t, j] * (wd @ hh)
    return y


# --------------------------------------------------------------------------------------
# Dense linear (W8A8 per-channel, W4A8 per-group)
# --------------------------------------------------------------------------------------
def linear_w8a8(x_bits, w_q, s_w) -> np.ndarray:
    """y = bf16(((float)(xq . w_q^T) * s_x) * s_w) with per-token x and per-channel w."""
    xq, sx = quant_act_per_token(x_bits)
    return f32_to_bf16(dequant(int_gemm(xq, w_q), sx, s_w))


def linear_w4a8(x_bits, packed, s_w, group: int = 128) -> np.ndarray:
    """Dense W4A8 linear: per-token int8 x, int4 per-group w.

    acc_g = int32 sum over the g-th group of K; acc_f = fma((float)acc_g, s_w[n, g], acc_f)
    over the groups in order, from 0; y = bf16(acc_f * s_x[t]).
    """
    xq, sx = quant_act_per_token(x_bits)
    wq = unpack_int4(packed)
    M, K = xq.shape
    N = wq.shape[0]
    acc_f = np.zeros((M, N), np.float32)
    s_w = np.asarray(s_w, np.float32)
    for g in range(K // group):
        ks = slice(g * group, (g + 1) * group)
        acc_g = int_gemm(xq[:, ks], wq[:, ks]).astype(np.float32)
        acc_f = fma32(acc_g, np.broadcast_to(s_w[None, :, g], acc_g.shape), acc_f)
    return f32_to_bf16(acc_f * sx[:, None])


# --------------------------------------------------------------------------------------
# MXFP8 A8W8 (the "MXFP A8w8" row of the accuracy table, section 六 of the AMCT Qwen3-Next page)
# --------------------------------------------------------------------------------------
# The page names the format only. It is read as the OCP Microscaling (MX) FP8 format: blocks of
# 32 consecutive values along K share one power-of-two scale X = 2**E stored as an E8M0 byte
# (E + 127), and every element is an FP8 E4M3 value (1 sign, 4 exponent bits with bias 7, 3
# mantissa bits; exponent field 0 holds the subnormals m/8 * 2**-6; 0x7F and 0xFF are NaN; no
# infinities; the largest magnitude is 1.75 * 2**8 = 448). Activations are quantised per token
# (dynamic), weights per output channel (static), both along K.
#   E = floor(log2(max |v| over the block)) - 8, clamped to [-127, 127] (8 is the exponent of
#       E4M3's largest binade); a block of zeros takes E = -127;
#   P = E4M3(v / 2**E), rounded to nearest with ties to even, magnitudes above 448 saturating
#       to 448 (the largest element of a block lands in [256, 512), so values in (448, 512) clip);
#       the sign of a value that rounds to zero is kept.
# The product of the layer is y[t, n] = sum_k (P_x[t,k] X_x[t,k/32]) (P_w[n,k] X_w[n,k/32]) in
# exact arithmetic; a tensor core sums it in fp32 in an order of its own, so the GPU result is
# checked against this exact value within the fp32 summation bound (``linear_mxfp8``).
MX_BLOCK = 32
E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """float64 value of each E4M3 byte (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    return np.where((c & 0x7F) == 0x7F, np.nan, sign * mag)


# non-negative finite E4M3 values in increasing order, with their codes
_E4M3_POS_CODES = np.arange(0x7F, dtype=np.uint8)
_E4M3_POS_VALUES = e4m3_decode(_E4M3_POS_CODES)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """E4M3 byte of each finite float64 value: nearest representable magnitude, ties to the even
    mantissa, saturating at 448; negative values (and -0) carry the sign bit."""
    v = np.asarray(v, np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    # the quantum of the binade that holds a: 2**(e - 3) for e = floor(log2 a) >= -6, and the
    # subnormal quantum 2**-9 below 2**-6
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(ex - 1, -6)
    q = np.exp2(e.astype(np.float64) - 3.0)
    n = np.rint(a / q)                        # a / q is exact; rint rounds halves to even
    mag = np.minimum(n * q, E4M3_MAX)         # n = 16 is the first value of the next binade
    idx = np.searchsorted(_E4M3_POS_VALUES, mag)
    assert np.all(_E4M3_POS_VALUES[idx] == mag)
    code = _E4M3_POS_CODES[idx]
    return np.where(np.signbit(v), code | np.uint8(0x80), code).astype(np.uint8)


def mx_quantize_rows(v_bits: np.ndarray):
    """MXFP8 codes [R, K] (uint8, E4M3) and scales [R, K/32] (uint8, E8M0) of bf16 rows."""
    v = bf16_to_f32(v_bits).astype(np.float64)
    R, K = v.shape
    assert K % MX_BLOCK == 0
    blocks = v.reshape(R, K // MX_BLOCK, MX_BLOCK)
    amax = np.abs(blocks).max(axis=2)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))      # amax in [2**(ex-1), 2**ex)
    E = np.where(amax > 0, ex - 1 - 8, -127)
    E = np.clip(E, -127, 127)
    codes = e4m3_encode(blocks / np.exp2(E.astype(np.float64))[:, :, None])
    return codes.reshape(R, K), (E + 127).astype(np.uint8)


def mx_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """float64 values P * 2**(scale - 127) of MXFP8 rows."""
    R, K = codes.shape
    p = e4m3_decode(codes).reshape(R, K // MX_BLOCK, MX_BLOCK)
    x = np.exp2(np.asarray(scales, np.float64) - 127.0)
    return (p * x[:, :, None]).reshape(R, K)


def linear_mxfp8(x_bits, w_codes, w_scales) -> dict:
    """Dense MXFP8 A8W8 linear: x quantised per token to MXFP8, then y = A . W^T exactly.

    Returns the token codes and scales, y (float64, the exact sum of the dequantised products
    up to float64 rounding) and ``bound``: the largest |y_gpu - y| a bf16 result of an fp32
    summation of the same products in any order can show, (K - 1) * 2**-24 * S (fp32
    summation) plus 2**-8 times the fp32 result's magnitude (one bf16 rounding), with
    S = sum_k |A[t,k] W[n,k]|."""
    xc, xs = mx_quantize_rows(x_bits)
    A = mx_dequantize(xc, xs)
    W = mx_dequantize(w_codes, w_scales)
    y = A @ W.T
    K = A.shape[1]
    S = np.abs(A) @ np.abs(W).T
    summ = (K - 1) * 2.0 ** -24 * S
    bound = summ + 2.0 ** -8 * (np.abs(y) + summ)
    return dict(codes=xc, scales=xs, y=y, bound=bound)


# --------------------------------------------------------------------------------------
# MXFP A8W4 (the "MXFP A8w4" row of the same accuracy table): MXFP8 activations, MXFP4 weights
# --------------------------------------------------------------------------------------
# Read, like the A8W8 row, as the OCP Microscaling formats: the activations exactly as above
# (MXFP8, E4M3 elements), the weights as MXFP4: blocks of 32 consecutive values along K with one
# E8M0 scale X = 2**E and FP4 E2M1 elements (1 sign, 2 exponent bits with bias 1, 1 mantissa bit;
# exponent field 0 holds the subnormal 0.5; the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6; no
# infinities or NaNs).
#   E = floor(log2(max |v| over the block)) - 2 (2 is the exponent of E2M1's largest binade),
#       clamped to [-127, 127]; a block of zeros takes E = -127;
#   P = E2M1(v / 2**E), rounded to nearest with ties to the even mantissa, magnitudes above 6
#       saturating to 6 (the block's largest element lands in [4, 8), so values in (6, 8) clip);
#       the sign of a value that rounds to zero is kept (code 0x8).
# Storage: two codes per byte, element 2i in the low nibble of byte i and element 2i + 1 in the
# high nibble (a weight row of K values takes K / 2 bytes).
# The product is y[t, n] = sum_k (P_x[t,k] X_x[t,k/32]) (P_w[n,k] X_w[n,k/32]), exact here, checked
# on the GPU within the same fp32 summation bound as the A8W8 product.
E2M1_MAX = 6.0


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """float64 value of each E2M1 code (the low four bits of each byte)."""
    c = np.asarray(codes, np.uint8).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = (c & 1).astype(np.float64)
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2(e.astype(np.float64) - 1.0))
    return sign * mag


# non-negative E2M1 values in increasing order; the code of each is its index
_E2M1_POS_VALUES = e2m1_decode(np.arange(8, dtype=np.uint8))


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """E2M1 code (0..15) of each finite float64 value: nearest representable magnitude, ties to the
    even mantissa, saturating at 6; negative values (and -0) carry the sign bit 0x8."""
    v = np.asarray(v, np.float64)
    a = np.minimum(np.abs(v), E2M1_MAX)
    # the quantum of the binade that holds a: 2**(e - 1) for e = floor(log2 a) >= 0; below 1 the
    # subnormal quantum 0.5, the same as that of [1, 2)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(ex - 1, 0)
    q = np.exp2(e.astype(np.float64) - 1.0)
    n = np.rint(a / q)                        # a / q is exact; rint rounds halves to even
    mag = np.minimum(n * q, E2M1_MAX)
    idx = np.searchsorted(_E2M1_POS_VALUES, mag)
    assert np.all(_E2M1_POS_VALUES[idx] == mag)
    code = idx.astype(np.uint8)
    return np.where(np.signbit(v), code | np.uint8(0x8), code).astype(np.uint8)


def mx4_quantize_rows(v_bits: np.ndarray):
    """MXFP4 weights of bf16 rows: packed E2M1 codes [R, K/2] (uint8) and E8M0 scales [R, K/32]."""
    v = bf16_to_f32(v_bits).astype(np.float64)
    R, K = v.shape
    assert K % MX_BLOCK == 0
    blocks = v.reshape(R, K // MX_BLOCK, MX_BLOCK)
    amax = np.abs(blocks).max(axis=2)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))      # amax in [2**(ex-1), 2**ex)
    E = np.where(amax > 0, ex - 1 - 2, -127)
    E = np.clip(E, -127, 127)
    codes = e2m1_encode(blocks / np.exp2(E.astype(np.float64))[:, :, None]).reshape(R, K)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, (E + 127).astype(np.uint8)


def mx4_unpack(packed: np.ndarray) -> np.ndarray:
    """E2M1 codes [R, K] of packed MXFP4 rows [R, K/2]."""
    p = np.asarray(packed, np.uint8)
    codes = np.empty((p.shape[0], 2 * p.shape[1]), np.uint8)
    codes[:, 0::2] = p & 0xF
    codes[:, 1::2] = p >> 4
    return codes


def mx4_dequantize(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """float64 values P * 2**(scale - 127) of packed MXFP4 rows."""
    codes = mx4_unpack(packed)
    R, K = codes.shape
    p = e2m1_decode(codes).reshape(R, K // MX_BLOCK, MX_BLOCK)
    x = np.exp2(np.asarray(scales, np.float64) - 127.0)
    return (p * x[:, :, None]).reshape(R, K)


def linear_mxfp_a8w4(x_bits, w_packed, w_scales) -> dict:
    """Dense MXFP A8W4 linear: x quantised per token to MXFP8, the weights in MXFP4, then
    y = A . W^T exactly; returns the same fields as ``linear_mxfp8`` (token codes and scales, y,
    and the bound of an fp32 summation in any order followed by one bf16 rounding)."""
    xc, xs = mx_quantize_rows(x_bits)
    A = mx_dequantize(xc, xs)
    W = mx4_dequantize(w_packed, w_scales)
    y = A @ W.T
    K = A.shape[1]
    S = np.abs(A) @ np.abs(W).T
    summ = (K - 1) * 2.0 ** -24 * S
    bound = summ + 2.0 ** -8 * (np.abs(y) + summ)
    return dict(codes=xc, scales=xs, y=y, bound=bound)
