"""The routing validity check used by the GPU parity tests, exercised on the CPU: it accepts the
oracle's own routing and a valid alternative at a near tie, and rejects an invalid top-k."""
import numpy as np
import pytest

from oracle import w8a8_oracle as O
from tests.gpu_common import check_topk_valid


def _route(seed=0, T=40, H=256, E=16, k=4):
    rng = np.random.default_rng(seed)
    x = O.f32_to_bf16(rng.standard_normal((T, H)).astype(np.float32))
    wg = O.f32_to_bf16((rng.standard_normal((E, H)) * 0.02).astype(np.float32))
    return O.route(x, wg, None, k, True), k


def test_accepts_the_oracle_routing():
    r, k = _route()
    check_topk_valid(r.ids, r.weights, r, k, True)


def test_accepts_either_expert_at_a_near_tie():
    r, k = _route()
    t = int(np.argmin(r.gap))
    # swap the k-th expert for the (k+1)-th: valid exactly when the gap is within the tolerance
    order = np.argsort(-r.probs[t], kind="stable")
    ids = r.ids.copy()
    ids[t, k - 1] = order[k]
    p = r.probs[t, ids[t]]
    w = r.weights.copy()
    w[t] = (p / p.sum()).astype(np.float32)
    tol = r.gap[t] + 1e-12
    check_topk_valid(ids, w, r, k, True, tol=tol)
    with pytest.raises(AssertionError):
        check_topk_valid(ids, w, r, k, True, tol=r.gap[t] / 2)


def test_rejects_a_wrong_expert_duplicates_and_wrong_weights():
    r, k = _route()
    order = np.argsort(-r.probs[0], kind="stable")
    bad = r.ids.copy()
    bad[0, 0] = order[-1]  # the least likely expert
    with pytest.raises(AssertionError):
        check_topk_valid(bad, r.weights, r, k, True)
    dup = r.ids.copy()
    dup[1, 1] = dup[1, 0]
    with pytest.raises(AssertionError):
        check_topk_valid(dup, r.weights, r, k, True)
    w = r.weights.copy()
    w[2, 0] *= 1.01
    with pytest.raises(AssertionError):
        check_topk_valid(r.ids, w, r, k, True)
