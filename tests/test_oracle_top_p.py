"""Pins of the oracle's adaptive expert top-p routing (CPU).

The pages name the knob ("colibri解説", section 速度を稼ぐ実用ノブ: --topp 0.7,
adaptive expert top-p) but not its rule; the oracle reads it as: among the k
selected experts, order by routing share pi_j = s_j / sum s (descending, lower
expert first on ties), keep the shortest prefix whose cumulative share reaches
p, renormalise the kept weights to the routed scale, mark dropped slots -1.
Each pin below is an independent statement of that rule (a hand-worked case,
the p >= 1 limit, brute force over subsets, invariants, the dense-gating form
of the layer).
"""
import itertools

import numpy as np
import pytest

import inputs
import oracle


def _onehot_router(logits, H=64):
    """Router whose scores for x = e_0 are exactly the given logits."""
    E = len(logits)
    w = np.zeros((E, H), np.float32)
    w[:, 0] = np.asarray(logits, np.float32)
    x = np.zeros((1, H), np.float32)
    x[0, 0] = 1.0
    return x, w


def _logit(s):
    s = np.asarray(s, np.float64)
    return np.log(s / (1 - s))


def test_hand_worked_cut():
    # s = (0.2, 0.8, 0.4, 0.6): shares 0.1, 0.4, 0.2, 0.3.  The bias puts expert 0
    # first in the selection order although its share is the smallest.
    s = np.array([0.2, 0.8, 0.4, 0.6])
    x, w_router = _onehot_router(_logit(s))
    bias = np.array([1.0, 0.0, 0.0, 0.0], np.float32)
    sig = 1 / (1 + np.exp(-w_router[:, 0].astype(np.float64)))  # the fp32 logits' sigmoids
    idx, w = oracle.route(x, w_router, bias, 4, 2.5)
    assert idx[0].tolist() == [0, 1, 3, 2]  # c = s + b descending
    # p = 0.3: the largest share (0.4, expert 1) already reaches it
    idx, w = oracle.route_top_p(x, w_router, bias, 4, 2.5, 0.3)
    assert idx[0].tolist() == [-1, 1, -1, -1]
    np.testing.assert_allclose(w[0], [0, 2.5, 0, 0], rtol=1e-14)
    # p = 0.65: 0.4 + 0.3 reaches it -> experts 1 and 3, weights renormalised over them
    idx, w = oracle.route_top_p(x, w_router, bias, 4, 2.5, 0.65)
    assert idx[0].tolist() == [-1, 1, 3, -1]
    np.testing.assert_allclose(w[0], [0, 2.5 * sig[1] / (sig[1] + sig[3]), 2.5 * sig[3] / (sig[1] + sig[3]), 0],
                               rtol=1e-14)
    # p = 0.85: 0.4 + 0.3 + 0.2 -> expert 0 (share 0.1) is the only one dropped
    idx, w = oracle.route_top_p(x, w_router, bias, 4, 2.5, 0.85)
    assert idx[0].tolist() == [-1, 1, 3, 2]


@pytest.mark.parametrize("p", [1.0, 1.5])
def test_p_at_least_one_is_plain_top_k(p):
    c = inputs.CONFIGS[0]
    d = inputs.tiny_layer(0)
    a_idx, a_w = oracle.route(d["x"], d["w_router"], d["sel_bias"], c.k, c.routed_scale)
    b_idx, b_w = oracle.route_top_p(d["x"], d["w_router"], d["sel_bias"], c.k, c.routed_scale, p)
    assert np.array_equal(a_idx, b_idx)
    np.testing.assert_array_equal(a_w, b_w)


def test_cut_is_the_best_smallest_subset_brute_force():
    """Among all subsets of the selected experts whose share reaches p, the kept
    set has the fewest experts and, for that size, the largest share."""
    rng = np.random.default_rng(3)
    for trial in range(200):
        E, k = 12, 5
        x = rng.standard_normal((1, 64)).astype(np.float32)
        w_router = (rng.standard_normal((E, 64)) * 0.3).astype(np.float32)
        bias = (rng.standard_normal(E) * 0.05).astype(np.float32)
        p = float(rng.uniform(0.05, 0.99))
        idx, _, (_, sig, _) = oracle.route(x, w_router, bias, k, 2.5, True)
        sel = idx[0]
        share = sig[0, sel] / sig[0, sel].sum()
        best_size, best_share = None, None
        for m in range(1, k + 1):
            ok = [sum(share[list(c)]) for c in itertools.combinations(range(k), m)
                  if sum(share[list(c)]) >= p - 1e-12]
            if ok:
                best_size, best_share = m, max(ok)
                break
        if best_size is None:
            best_size, best_share = k, 1.0
        pidx, pw = oracle.route_top_p(x, w_router, bias, k, 2.5, p)
        kept = pidx[0] >= 0
        assert kept.sum() == best_size, trial
        assert abs(share[kept].sum() - best_share) < 1e-12, trial
        assert np.array_equal(pidx[0][kept], sel[kept])  # kept slots keep their expert
        np.testing.assert_allclose(pw[0].sum(), 2.5, rtol=1e-12)
        assert np.all(pw[0][~kept] == 0) and np.all(pw[0][kept] > 0)


def test_larger_p_keeps_a_superset():
    c = inputs.CONFIGS[0]
    d = inputs.tiny_layer(0)
    prev = None
    for p in (0.1, 0.3, 0.5, 0.7, 0.9, 1.0):
        idx, _ = oracle.route_top_p(d["x"], d["w_router"], d["sel_bias"], c.k, c.routed_scale, p)
        kept = idx >= 0
        assert kept.sum(axis=1).min() >= 1
        if prev is not None:
            assert np.all(kept | ~prev)  # nothing kept at a smaller p is dropped at a larger one
        prev = kept


def test_layer_is_the_dense_gating_sum_over_kept_experts():
    c = inputs.CONFIGS[0]
    d = inputs.tiny_layer(0)
    x = d["x"][:2]
    idx, w, out = oracle.moe_layer_top_p(x, c.H, c.F, c.E, c.k, c.routed_scale, 0.5, d["w_router"],
                                         d["sel_bias"], d["experts"])
    for t in range(x.shape[0]):
        ref = oracle.expert_ffn(x[t], c.H, c.F, d["experts"][c.E]).copy()
        for e in range(c.E):
            g = w[t][idx[t] == e].sum()
            if g:
                ref += g * oracle.expert_ffn(x[t], c.H, c.F, d["experts"][e])
        np.testing.assert_allclose(out[t], ref, rtol=1e-12, atol=1e-12)
    # p = 1: the plain layer
    a = oracle.moe_layer(x, c.H, c.F, c.E, c.k, c.routed_scale, d["w_router"], d["sel_bias"], d["experts"])
    b = oracle.moe_layer_top_p(x, c.H, c.F, c.E, c.k, c.routed_scale, 1.0, d["w_router"], d["sel_bias"],
                               d["experts"])
    np.testing.assert_array_equal(a[2], b[2])
