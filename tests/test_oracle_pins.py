"""Pins of the CPU oracle to facts outside itself (CPU only).

The colibri pages print no worked example of the router, the nibble packing or a
layer output, so each part of the oracle is pinned to: hand-worked values of the
storage format, textbook library routines (numpy matmul, numpy stable argsort,
scipy's logistic function), brute force over all subsets, closed forms, and
invariants of the definition.  Each pin is chosen so that a plausible slip in the
oracle (nibble order, sign extension, group index, biased weights, a missing
shared expert, an unstable sort) fails it.
"""
import itertools
import math

import numpy as np
import pytest
from scipy.special import expit

import oracle
from inputs import pack_int4


# ---------------------------------------------------------------------------
# storage format: hand-worked bytes

def _row_bytes(K, pairs):
    """One row of K int4 values as bytes, with selected bytes set by hand."""
    q = np.zeros((1, K // 2), np.uint8)
    for pos, byte in pairs.items():
        q[0, pos] = byte
    return q


def test_nibble_hand_examples():
    # 0x8F: low nibble 0xF = -1 (k even), high nibble 0x8 = -8 (k odd)
    # 0x70: low 0x0 = 0, high 0x7 = 7;  0x08: low 0x8 = -8, high 0x0 = 0
    # 0x12: low 2, high 1
    q = _row_bytes(64, {0: 0x8F, 1: 0x70, 2: 0x08, 31: 0x12})
    s = np.array([[0.5]], np.float32)
    W = oracle.dequant(q, s, 1, 64)
    assert W[0, 0] == -0.5 and W[0, 1] == -4.0
    assert W[0, 2] == 0.0 and W[0, 3] == 3.5
    assert W[0, 4] == -4.0 and W[0, 5] == 0.0
    assert W[0, 62] == 1.0 and W[0, 63] == 0.5
    assert np.all(W[0, 6:62] == 0.0)


def test_group_index_hand_example():
    # K = 128: k 0..63 use scale 0, k 64..127 use scale 1.
    # byte 31 holds k = 62, 63; byte 32 holds k = 64, 65.
    q = _row_bytes(128, {31: 0x77, 32: 0x77})
    s = np.array([[0.5, 0.25]], np.float32)
    W = oracle.dequant(q, s, 1, 128)
    assert W[0, 62] == 3.5 and W[0, 63] == 3.5
    assert W[0, 64] == 1.75 and W[0, 65] == 1.75


def test_three_by_128_hand_matrix():
    # row 0: every byte 0x21 -> (1, 2) repeating, scales (1, 2)
    # row 1: every byte 0xF8 -> (-8, -1) repeating, scales (0.5, 0.125)
    # row 2: byte j = 0x0j for j < 8 else 0 -> k = 2j gets j, scale (3, 3)
    q = np.zeros((3, 64), np.uint8)
    q[0, :] = 0x21
    q[1, :] = 0xF8
    for j in range(8):
        q[2, j] = j
    s = np.array([[1.0, 2.0], [0.5, 0.125], [3.0, 3.0]], np.float32)
    W = oracle.dequant(q, s, 3, 128)
    exp0 = np.array([1, 2] * 32 + [2, 4] * 32, np.float64)
    exp1 = np.array([-4.0, -0.5] * 32 + [-1.0, -0.125] * 32)
    exp2 = np.zeros(128)
    for j in range(8):
        exp2[2 * j] = 3.0 * j
    assert np.array_equal(W[0], exp0)
    assert np.array_equal(W[1], exp1)
    assert np.array_equal(W[2], exp2)
    # the element accessor agrees with the dense copy
    for (n, kk) in [(0, 0), (0, 127), (1, 64), (2, 14)]:
        assert oracle.weight(q, s, 128, n, kk) == W[n, kk]


def test_dequant_matches_packed_integers():
    # The test encodes random integers (inverse direction); the oracle decodes.
    rng = np.random.default_rng(1)
    for N, K in [(3, 64), (5, 128), (7, 256)]:
        qi = rng.integers(-8, 8, size=(N, K))
        s = rng.uniform(0.1, 2.0, size=(N, K // 64)).astype(np.float32)
        W = oracle.dequant(pack_int4(qi), s, N, K)
        ref = qi * np.repeat(s.astype(np.float64), 64, axis=1)
        assert np.array_equal(W, ref)


def test_matvec_matches_numpy_matmul():
    rng = np.random.default_rng(2)
    for N, K in [(64, 64), (128, 64), (64, 128), (96, 192)]:
        qi = rng.integers(-8, 8, size=(N, K))
        s = rng.uniform(0.001, 0.01, size=(N, K // 64)).astype(np.float32)
        x = rng.standard_normal(K)
        y = oracle.matvec(pack_int4(qi), s, N, K, x)
        ref = np.matmul(qi * np.repeat(s.astype(np.float64), 64, axis=1), x)
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------------------
# router

def _router_case(seed, T=5, H=128, E=16):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H)).astype(np.float32)
    w = (rng.standard_normal((E, H)) * 0.1).astype(np.float32)
    b = (rng.standard_normal(E) * 0.05).astype(np.float32)
    return x, w, b


def test_route_scores_match_library_routines():
    x, w, b = _router_case(3)
    idx, wt, (l, s, c) = oracle.route(x, w, b, 4, 2.5, want_scores=True)
    ref_l = np.matmul(x.astype(np.float64), w.astype(np.float64).T)
    np.testing.assert_allclose(l, ref_l, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s, expit(ref_l), rtol=1e-13, atol=0)
    np.testing.assert_allclose(c, expit(ref_l) + b.astype(np.float64), rtol=1e-13, atol=1e-15)


def test_route_invariants():
    x, w, b = _router_case(4, T=9, E=32)
    k, alpha = 8, 2.5
    idx, wt, (l, s, c) = oracle.route(x, w, b, k, alpha, want_scores=True)
    for t in range(x.shape[0]):
        assert len(set(idx[t].tolist())) == k
        assert idx[t].min() >= 0 and idx[t].max() < 32
        assert abs(wt[t].sum() - alpha) < 1e-12
        assert np.all(wt[t] > 0)
        # descending biased score order
        assert np.all(np.diff(c[t, idx[t]]) <= 0)
        # weights are the unbiased sigmoids renormalised over the selection
        np.testing.assert_allclose(wt[t], alpha * s[t, idx[t]] / s[t, idx[t]].sum(), rtol=1e-14)


def test_route_zero_bias_is_argsort_of_logits():
    x, w, _ = _router_case(5, T=6, E=24)
    idx, _ = oracle.route(x, w, np.zeros(24, np.float32), 6, 1.0)
    ref = np.argsort(-np.matmul(x.astype(np.float64), w.astype(np.float64).T), axis=1,
                     kind="stable")[:, :6]
    assert np.array_equal(idx, ref)


def test_route_constant_bias_shift_changes_nothing():
    x, w, b = _router_case(6)
    i1, w1 = oracle.route(x, w, b, 4, 2.5)
    i2, w2 = oracle.route(x, w, (b.astype(np.float64) + 0.25).astype(np.float32), 4, 2.5)
    assert np.array_equal(i1, i2)
    np.testing.assert_allclose(w1, w2, rtol=1e-14)


def test_route_bias_forces_selection_without_weighting():
    x, w, b = _router_case(7, T=4, E=16)
    b = np.zeros(16, np.float32)
    b[11] = 10.0
    idx, wt, (l, s, c) = oracle.route(x, w, b, 3, 2.5, want_scores=True)
    assert np.all(idx[:, 0] == 11)
    for t in range(4):
        # expert 11's weight uses its sigmoid, not sigmoid + 10
        assert abs(wt[t, 0] - 2.5 * s[t, 11] / s[t, idx[t]].sum()) < 1e-14
        assert wt[t, 0] < 2.5


def test_route_zero_logits_closed_form():
    # W_r = 0: every sigmoid is 1/2, selection follows the bias, weights alpha/k.
    x = np.ones((2, 64), np.float32)
    w = np.zeros((8, 64), np.float32)
    b = np.array([0.1, 0.7, 0.3, 0.5, 0.2, 0.6, 0.0, 0.4], np.float32)
    idx, wt = oracle.route(x, w, b, 3, 2.5)
    assert idx.tolist() == [[1, 5, 3]] * 2
    np.testing.assert_array_equal(wt, np.full((2, 3), 2.5 / 3))


def test_route_ties_go_to_lower_index():
    x = np.ones((1, 64), np.float32)
    w = np.zeros((6, 64), np.float32)
    b = np.array([0.25, 0.5, 0.5, 0.25, 0.5, 0.0], np.float32)  # exact in fp32
    idx, _ = oracle.route(x, w, b, 4, 1.0)
    assert idx.tolist() == [[1, 2, 4, 0]]


def test_route_brute_force_subsets():
    # E = 8, k = 2: the selected set maximises the sum of biased scores over all
    # C(8,2) subsets (top-k of distinct scores), weights per the definition.
    x, w, b = _router_case(8, T=7, H=64, E=8)
    idx, wt, (l, s, c) = oracle.route(x, w, b, 2, 2.5, want_scores=True)
    for t in range(7):
        ct = expit(np.matmul(w.astype(np.float64), x[t].astype(np.float64))) + b.astype(np.float64)
        best = max(itertools.combinations(range(8), 2), key=lambda S: sum(ct[i] for i in S))
        assert sorted(idx[t].tolist()) == sorted(best)
        st = expit(np.matmul(w.astype(np.float64), x[t].astype(np.float64)))
        ref_w = {e: 2.5 * st[e] / sum(st[i] for i in best) for e in best}
        for j in range(2):
            assert abs(wt[t, j] - ref_w[idx[t, j]]) < 1e-13


# ---------------------------------------------------------------------------
# union

def _union_check(idx, E):
    u = oracle.union(idx, E)
    T, k = idx.shape
    flat = idx.ravel()
    assert u["count"].sum() == T * k
    assert np.array_equal(u["count"], np.bincount(flat, minlength=E))
    assert np.array_equal(u["offset"], np.concatenate([[0], np.cumsum(u["count"])]))
    act = np.unique(flat)
    assert u["n_active"] == len(act)
    assert np.array_equal(u["active"][: len(act)], act)
    assert np.all(u["active"][len(act):] == -1)
    assert np.array_equal(np.sort(u["perm"]), np.arange(T * k))
    assert np.array_equal(u["perm"], np.argsort(flat, kind="stable"))
    assert np.all(np.diff(flat[u["perm"]]) >= 0)
    assert np.array_equal(u["inv_perm"][u["perm"]], np.arange(T * k))
    return u


def test_union_small_hand_case():
    idx = np.array([[3, 1], [1, 0], [3, 2]], np.int32)
    u = _union_check(idx, 5)
    assert u["count"].tolist() == [1, 2, 1, 2, 0]
    assert u["perm"].tolist() == [3, 1, 2, 5, 0, 4]
    assert u["active"].tolist() == [0, 1, 2, 3, -1]


@pytest.mark.parametrize("T,k,E", [(1, 8, 256), (4, 8, 256), (64, 8, 256), (33, 3, 7), (512, 8, 64)])
def test_union_random(T, k, E):
    rng = np.random.default_rng(T * 1000 + E)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    _union_check(idx, E)


def test_union_one_expert_gets_every_token():
    idx = np.array([[5, t % 5] for t in range(17)], np.int32)
    u = _union_check(idx, 6)
    assert u["count"][5] == 17


# ---------------------------------------------------------------------------
# expert FFN

def _pack_expert(G, U, D, sg, su, sd):
    return dict(gate_q=pack_int4(G), gate_s=sg, up_q=pack_int4(U), up_s=su,
                down_q=pack_int4(D), down_s=sd)


def test_expert_identity_closed_form():
    # Wg = Wu = Wd = I (H = F = 64, scale 1): y = silu(x) * x elementwise.
    I = np.eye(64, dtype=np.int64)
    one = np.ones((64, 1), np.float32)
    ex = _pack_expert(I, I, I, one, one, one)
    x = np.linspace(-3.0, 3.0, 64)
    x[10] = 0.0
    x[20] = math.log(3.0)           # sigmoid(ln 3) = 3/4
    y, h = oracle.expert_ffn(x, 64, 64, ex, want_h=True)
    assert y[10] == 0.0
    assert abs(y[20] - 0.75 * math.log(3.0) ** 2) < 1e-15
    np.testing.assert_allclose(y, x * x * expit(x), rtol=1e-14, atol=1e-16)
    np.testing.assert_array_equal(y, h)


def test_expert_brute_force_numpy():
    rng = np.random.default_rng(9)
    for H, F in [(64, 64), (128, 64), (64, 128), (192, 128)]:
        G = rng.integers(-8, 8, (F, H)); U = rng.integers(-8, 8, (F, H)); D = rng.integers(-8, 8, (H, F))
        sg = rng.uniform(0.005, 0.02, (F, H // 64)).astype(np.float32)
        su = rng.uniform(0.005, 0.02, (F, H // 64)).astype(np.float32)
        sd = rng.uniform(0.005, 0.02, (H, F // 64)).astype(np.float32)
        x = rng.standard_normal(H)
        y = oracle.expert_ffn(x, H, F, _pack_expert(G, U, D, sg, su, sd))
        Wg = G * np.repeat(sg.astype(np.float64), 64, 1)
        Wu = U * np.repeat(su.astype(np.float64), 64, 1)
        Wd = D * np.repeat(sd.astype(np.float64), 64, 1)
        g = Wg @ x
        ref = Wd @ (g * expit(g) * (Wu @ x))
        np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-14)


# ---------------------------------------------------------------------------
# whole layer

def _tiny_random_layer(seed, H=64, F=64, E=6, T=5):
    rng = np.random.default_rng(seed)
    experts = {}
    for e in range(E + 1):
        experts[e] = _pack_expert(rng.integers(-8, 8, (F, H)), rng.integers(-8, 8, (F, H)),
                                  rng.integers(-8, 8, (H, F)),
                                  rng.uniform(0.01, 0.03, (F, H // 64)).astype(np.float32),
                                  rng.uniform(0.01, 0.03, (F, H // 64)).astype(np.float32),
                                  rng.uniform(0.01, 0.03, (H, F // 64)).astype(np.float32))
    w = (rng.standard_normal((E, H)) * 0.2).astype(np.float32)
    b = (rng.standard_normal(E) * 0.05).astype(np.float32)
    x = rng.standard_normal((T, H)).astype(np.float32)
    return x, w, b, experts


def test_layer_dense_gating_identity():
    H = F = 64; E = 6; k = 3
    x, w, b, ex = _tiny_random_layer(10, H, F, E)
    idx, wt, out = oracle.moe_layer(x, H, F, E, k, 2.5, w, b, ex)
    for t in range(x.shape[0]):
        gate = np.zeros(E)
        gate[idx[t]] = wt[t]
        dense = sum(gate[e] * oracle.expert_ffn(x[t], H, F, ex[e]) for e in range(E))
        dense = dense + oracle.expert_ffn(x[t], H, F, ex[E])
        np.testing.assert_allclose(out[t], dense, rtol=1e-12, atol=1e-14)


def test_layer_batch_independence():
    H = F = 64; E = 6; k = 2
    x, w, b, ex = _tiny_random_layer(11, H, F, E, T=4)
    _, _, out = oracle.moe_layer(x, H, F, E, k, 2.5, w, b, ex)
    for t in range(4):
        _, _, o1 = oracle.moe_layer(x[t:t + 1], H, F, E, k, 2.5, w, b, ex)
        np.testing.assert_array_equal(out[t], o1[0])


def test_layer_relabelling_invariance():
    H = F = 64; E = 6; k = 3
    x, w, b, ex = _tiny_random_layer(12, H, F, E)
    _, _, out = oracle.moe_layer(x, H, F, E, k, 2.5, w, b, ex)
    pi = np.random.default_rng(0).permutation(E)
    ex2 = {e: ex[pi[e]] for e in range(E)}
    ex2[E] = ex[E]
    _, _, out2 = oracle.moe_layer(x, H, F, E, k, 2.5, w[pi], b[pi], ex2)
    np.testing.assert_allclose(out, out2, rtol=1e-12, atol=1e-14)


def test_layer_zero_scale_leaves_shared_expert():
    H = F = 64; E = 6; k = 3
    x, w, b, ex = _tiny_random_layer(13, H, F, E)
    _, _, out = oracle.moe_layer(x, H, F, E, k, 0.0, w, b, ex)
    for t in range(x.shape[0]):
        np.testing.assert_allclose(out[t], oracle.expert_ffn(x[t], H, F, ex[E]), rtol=1e-13)


def test_layer_linear_in_down_scales():
    H = F = 64; E = 6; k = 3
    x, w, b, ex = _tiny_random_layer(14, H, F, E)
    _, _, out = oracle.moe_layer(x, H, F, E, k, 2.5, w, b, ex)
    ex2 = {e: dict(v, down_s=(v["down_s"] * 2).astype(np.float32)) for e, v in ex.items()}
    _, _, out2 = oracle.moe_layer(x, H, F, E, k, 2.5, w, b, ex2)
    np.testing.assert_allclose(out2, 2 * out, rtol=1e-13, atol=1e-15)


def test_layer_missing_needed_expert_is_an_error():
    H = F = 64; E = 6; k = 3
    x, w, b, ex = _tiny_random_layer(15, H, F, E)
    idx, _ = oracle.route(x, w, b, k, 2.5)
    partial = {e: v for e, v in ex.items() if e != idx[0, 0]}
    with pytest.raises(ValueError):
        oracle.moe_layer(x, H, F, E, k, 2.5, w, b, partial)
