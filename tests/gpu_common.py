"""Helpers shared by the GPU parity tests: upload synthetic inputs, run the C ABI, and turn
device results into host arrays the oracle can be compared with."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from oracle import w8a8_oracle as O
from w8a8_int8_quantized_act_b200 import binding as B
from w8a8_int8_quantized_act_b200 import synth


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(a: np.ndarray) -> torch.Tensor:
    return to_dev(a, torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns on the host."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return bits(t)
    return t.detach().cpu().numpy()


@dataclass
class MoERun:
    wl: synth.MoEWorkload
    inp: synth.MoEInputs
    y: np.ndarray
    mid: dict  # host copies of the workspace intermediates
    wgu_q: torch.Tensor
    s_gu: torch.Tensor
    wd_q: torch.Tensor
    s_d: torch.Tensor


def run_moe(wl: synth.MoEWorkload, x_override: np.ndarray | None = None, bias_override=None) -> MoERun:
    inp = synth.moe_inputs(wl)
    if x_override is not None:
        inp.x = x_override
    if bias_override is not None:
        inp.bias = bias_override
    x = bf16_dev(inp.x)
    wg = bf16_dev(inp.wg)
    bias = to_dev(inp.bias) if inp.bias is not None else None
    wgu_q, s_gu = B.w8a8_quantize_weight_per_channel(bf16_dev(inp.wgu))
    wd_q, s_d = B.w8a8_quantize_weight_per_channel(bf16_dev(inp.wd))
    T = inp.x.shape[0]
    ws = torch.empty(max(1, B.w8a8_moe_workspace_size(T, wl.H, wl.E, wl.k, wl.I)), dtype=torch.uint8,
                     device="cuda")
    y = B.w8a8_moe_forward(x, wg, wgu_q, s_gu, wd_q, s_d, wl.k, renorm=wl.renorm, bias=bias, workspace=ws)
    B.w8a8_check_status()
    mid = {k: host(v) for k, v in B.moe_intermediates(ws, T, wl.H, wl.E, wl.k, wl.I).items()} if T else {}
    return MoERun(wl, inp, host(y), mid, wgu_q, s_gu, wd_q, s_d)


def sorted_rows_of_tokens(perm: np.ndarray, k: int, tokens: np.ndarray) -> np.ndarray:
    """Sorted-row index of every (token, slot) of `tokens`, shape [len(tokens), k]."""
    row_of = np.empty_like(perm)
    row_of[perm] = np.arange(perm.size, dtype=perm.dtype)
    slots = tokens[:, None] * k + np.arange(k)[None, :]
    return row_of[slots]


def check_grouping(ids: np.ndarray, perm: np.ndarray, offsets: np.ndarray, E: int):
    """perm/offsets must equal the stable grouping of the given routing (exact)."""
    ref_perm, ref_off = O.group_by_expert(ids, E)
    np.testing.assert_array_equal(offsets.astype(np.int64), ref_off)
    np.testing.assert_array_equal(perm, ref_perm)


def check_topk_valid(ids: np.ndarray, w: np.ndarray, r, k: int, renorm: bool, tol: float = 1e-4):
    """Every token's routing is a valid top-k of the oracle's probabilities, near ties included.

    Several expert sets are correct where the k-th and (k+1)-th probabilities lie within `tol`
    of each other, so for every token this checks what is unique: the k ids are distinct and in
    range; each chosen expert has p >= p_(k) - tol and each rejected one p <= p_(k+1) + tol; the
    weights equal the oracle's probabilities of the chosen experts (renormalised over them when
    `renorm`), rtol 2e-4 / atol 2e-6; and the slots are in descending order of weight."""
    T, E = r.probs.shape
    assert ids.shape == (T, k) and w.shape == (T, k)
    assert np.all((ids >= 0) & (ids < E))
    srt = -np.sort(-r.probs, axis=1)
    pk = srt[:, k - 1]
    pk1 = srt[:, k] if k < E else np.full(T, -np.inf)
    for t in range(T):
        chosen = ids[t]
        assert len(set(chosen.tolist())) == k, (t, chosen)
        p = r.probs[t]
        assert np.all(p[chosen] >= pk[t] - tol), (t, chosen)
        rejected = np.setdiff1d(np.arange(E), chosen)
        if rejected.size:
            assert p[rejected].max() <= pk1[t] + tol, (t, chosen)
        ref = p[chosen] / p[chosen].sum() if renorm else p[chosen]
        np.testing.assert_allclose(w[t], ref, rtol=2e-4, atol=2e-6, err_msg=f"token {t}")
        assert np.all(np.diff(w[t]) <= 2e-6), (t, w[t])


def check_routing(run: MoERun, ids: np.ndarray, w: np.ndarray, tokens: np.ndarray | None = None,
                  gap: float = 1e-4):
    """Expert sets equal wherever the k-th/(k+1)-th probability gap exceeds `gap`; every token,
    near ties included, a valid top-k with the oracle's weights (check_topk_valid). Returns the
    mask of tokens whose routing is unambiguous."""
    wl = run.wl
    x = run.inp.x if tokens is None else run.inp.x[tokens]
    r = O.route(x, run.inp.wg, run.inp.bias, wl.k, wl.renorm)
    clear = r.gap > gap
    gi, gw = (ids, w) if tokens is None else (ids[tokens], w[tokens])
    np.testing.assert_array_equal(np.sort(gi[clear], 1), np.sort(r.ids[clear], 1))
    same = np.all(gi == r.ids, axis=1)
    assert same.mean() > 0.9
    check_topk_valid(gi, gw, r, wl.k, wl.renorm, gap)
    return clear


def oracle_on_tokens(run: MoERun, tokens: np.ndarray):
    """Oracle forward of the sampled tokens with the GPU's routing; weights of the touched
    experts are regenerated and quantised by the oracle itself."""
    wl = run.wl
    ids = run.mid["topk_ids"][tokens]
    w = run.mid["topk_w"][tokens]
    touched = np.unique(ids)
    wgu = synth.expert_gate_up(wl.E, wl.I, wl.H, wl.seed, experts=touched)
    wd = synth.expert_down(wl.E, wl.H, wl.I, wl.seed, experts=touched)
    gq, gs = O.quantize_weight_per_channel(wgu)
    dq, ds = O.quantize_weight_per_channel(wd)
    wgu_q = {int(e): gq[i] for i, e in enumerate(touched)}
    s_gu = {int(e): gs[i] for i, e in enumerate(touched)}
    wd_q = {int(e): dq[i] for i, e in enumerate(touched)}
    s_d = {int(e): ds[i] for i, e in enumerate(touched)}
    out = O.moe_forward(run.inp.x[tokens], run.inp.wg, run.inp.bias, wgu_q, s_gu, wd_q, s_d, wl.k, wl.renorm,
                        routing=(ids, w))
    return out, touched, (gq, gs, dq, ds)


def compare_tokens(run: MoERun, tokens: np.ndarray):
    """Bit-exact comparison of every per-token and per-assignment result for `tokens`."""
    wl = run.wl
    out, touched, (gq, gs, dq, ds) = oracle_on_tokens(run, tokens)
    # weight quantisation of the touched experts
    e_idx = torch.as_tensor(touched, device="cuda")
    np.testing.assert_array_equal(run.wgu_q[e_idx].cpu().numpy(), gq)
    np.testing.assert_array_equal(run.s_gu[e_idx].cpu().numpy(), gs)
    np.testing.assert_array_equal(run.wd_q[e_idx].cpu().numpy(), dq)
    np.testing.assert_array_equal(run.s_d[e_idx].cpu().numpy(), ds)
    m = run.mid
    rows = sorted_rows_of_tokens(m["perm"], wl.k, tokens)  # [n, k]
    np.testing.assert_array_equal(m["sx"][tokens], out["sx"])
    for j in range(wl.k):
        np.testing.assert_array_equal(m["xq"][rows[:, j]], out["xq"])
        np.testing.assert_array_equal(m["sx_sorted"][rows[:, j]], out["sx"])
        np.testing.assert_array_equal(m["h"][rows[:, j]], out["h"][:, j])
        np.testing.assert_array_equal(m["s_h"][rows[:, j]], out["s_h"][:, j])
        np.testing.assert_array_equal(m["hq"][rows[:, j]], out["hq"][:, j])
    o_gpu = m["o"].reshape(-1, wl.k, wl.H)[tokens]
    np.testing.assert_array_equal(o_gpu, out["o"])
    np.testing.assert_array_equal(run.y[tokens], out["y"])
    return out


def y_tolerance_check(run: MoERun, tokens: np.ndarray, clear: np.ndarray):
    """End to end against the oracle's own routing: max abs <= 2e-2, rel-L2 <= 5e-3 on tokens
    whose routing is unambiguous."""
    wl = run.wl
    sel = tokens[clear]
    touched = None
    r = O.route(run.inp.x[sel], run.inp.wg, run.inp.bias, wl.k, wl.renorm)
    touched = np.unique(r.ids)
    wgu = synth.expert_gate_up(wl.E, wl.I, wl.H, wl.seed, experts=touched)
    wd = synth.expert_down(wl.E, wl.H, wl.I, wl.seed, experts=touched)
    gq, gs = O.quantize_weight_per_channel(wgu)
    dq, ds = O.quantize_weight_per_channel(wd)
    d = lambda a: {int(e): a[i] for i, e in enumerate(touched)}  # noqa: E731
    ref = O.moe_forward(run.inp.x[sel], run.inp.wg, run.inp.bias, d(gq), d(gs), d(dq), d(ds), wl.k, wl.renorm)
    yr = O.bf16_to_f32(ref["y"]).astype(np.float64)
    yg = O.bf16_to_f32(run.y[sel]).astype(np.float64)
    err = np.abs(yg - yr)
    rel = np.linalg.norm(yg - yr) / max(np.linalg.norm(yr), 1e-30)
    # 2e-2 wherever a bf16 ulp is finer than that (|y| < 4); above, one rounding flip of
    # the bf16 output is one ulp (2**-5 at |y| in [4, 8)), so exactly one ulp is allowed there
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(yr), 2.0 ** -126))) - 7)
    tol = np.maximum(2e-2, ulp)
    assert np.all(err <= tol), (err.max(), yr.flat[np.argmax(err - tol)])
    assert (err > 2e-2).mean() <= 1e-4, (err > 2e-2).sum()
    assert rel <= 5e-3, rel
