"""Pins of the oracle's integer-activation variant (CPU).

The pages name an integer dot-product kernel that multiplies int8 activations
with packed int4 weights ("Colibri 完全ガイド", section コア技術のハイライト, row
整数ドット積カーネル; the IDOT switch in the same page's environment table) but
print no quantisation rule.  The oracle reads it as symmetric int8 per block of
32 values (scale = max|x| / 127, code = rint(x * 127 / max|x|), fp32) applied
to both expert inputs, x before gate/up and h before down.  Each pin below
states a consequence of that rule independently of its code: a hand-worked
block, the extreme code, the rounding bound, exactness on the grid, power-of-two
and sign symmetry, zero and non-finite blocks, and the layer as a composition
of the already pinned plain functions.
"""
import numpy as np
import pytest

import inputs
import oracle


def test_hand_worked_block():
    # max |x| = 2.54, so 127 / max = 50 and the scale is 0.02:
    #  2.54 -> 127, -1.0 -> -50, 0.5 -> 25, 0.02 -> 1, 0.013 -> 0.65 -> 1, 0.009 -> 0.45 -> 0
    x = np.zeros(32, np.float32)
    x[:6] = [2.54, -1.0, 0.5, 0.02, 0.013, 0.009]
    codes, scales = oracle.quant_i8(x)
    assert codes[:6].tolist() == [127, -50, 25, 1, 1, 0]
    assert not codes[6:].any()
    assert scales.shape == (1,)
    assert abs(float(scales[0]) - 0.02) < 1e-8


def test_extreme_code_and_rounding_bound():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 32 * 7)) * rng.uniform(1e-3, 1e3, (64, 1))).astype(np.float32)
    codes, scales = oracle.quant_i8(x)
    blocks = x.reshape(64, 7, 32)
    c = codes.reshape(64, 7, 32).astype(np.int64)
    assert np.abs(c).max() <= 127
    # the largest magnitude of every block lands on +-127 with the sign of the value
    top = np.abs(blocks).argmax(axis=2)
    picked = np.take_along_axis(c, top[..., None], 2)[..., 0]
    vals = np.take_along_axis(blocks, top[..., None], 2)[..., 0]
    assert (picked == 127 * np.sign(vals)).all()
    # every value is within half a step (plus fp32 slack) of its reconstruction
    s = scales.astype(np.float64)[..., None]
    err = np.abs(c * s - blocks.astype(np.float64))
    assert (err <= 0.5 * s * (1 + 1e-5)).all()


def test_on_grid_values_are_exact():
    # x = code * 2^-6 with a block maximum of 127: the scale is exactly 2^-6 and the codes come back
    rng = np.random.default_rng(6)
    code = rng.integers(-127, 128, (16, 32))
    code[:, 3] = 127
    x = (code * 2.0 ** -6).astype(np.float32)
    c, s = oracle.quant_i8(x)
    np.testing.assert_array_equal(c, code)
    np.testing.assert_array_equal(s, np.full((16, 1), 2.0 ** -6, np.float32))


@pytest.mark.parametrize("j", [-20, -3, 5, 40])
def test_power_of_two_and_sign_symmetry(j):
    rng = np.random.default_rng(7)
    x = rng.standard_normal(32 * 5).astype(np.float32)
    c0, s0 = oracle.quant_i8(x)
    c1, s1 = oracle.quant_i8((x * np.float32(2.0 ** j)).astype(np.float32))
    np.testing.assert_array_equal(c1, c0)
    np.testing.assert_array_equal(s1, (s0 * np.float32(2.0 ** j)).astype(np.float32))
    c2, s2 = oracle.quant_i8(-x)
    np.testing.assert_array_equal(c2, -c0)
    np.testing.assert_array_equal(s2, s0)


def test_zero_and_non_finite_blocks():
    x = np.zeros(96, np.float32)
    x[32] = np.inf
    x[64:96] = 1.0
    c, s = oracle.quant_i8(x)
    assert not c[:64].any()
    assert s[0] == 0.0 and np.isnan(s[1])
    assert (c[64:] == 127).all() and s[2] == np.float32(1.0) / np.float32(127.0)


def _hat(v):
    c, s = oracle.quant_i8(np.asarray(v, np.float32))
    return c.astype(np.float64) * np.repeat(s.astype(np.float64), 32)


def test_layer_is_the_composition_of_pinned_parts():
    # out = sum_j w_j Wd_j q(h_j) + Wd_E q(h_E),  h_j = silu(Wg_j q(x)) * (Wu_j q(x)) rounded to fp32:
    # built from the plain (pinned) route, expert_ffn's h, matvec and quant_i8
    c = inputs.CONFIGS[0]
    d = inputs.tiny_layer(0)
    x = d["x"][:3]
    idx, w, out = oracle.moe_layer_i8(x, c.H, c.F, c.E, c.k, c.routed_scale, d["w_router"], d["sel_bias"],
                                      d["experts"])
    idx0, w0 = oracle.route(x, d["w_router"], d["sel_bias"], c.k, c.routed_scale)
    np.testing.assert_array_equal(idx, idx0)
    np.testing.assert_array_equal(w, w0)
    for t in range(x.shape[0]):
        xh = _hat(x[t])
        ref = np.zeros(c.H)
        for j in range(c.k + 1):
            e = int(idx[t, j]) if j < c.k else c.E
            wt = w[t, j] if j < c.k else 1.0
            ex = d["experts"][e]
            _, h = oracle.expert_ffn(xh, c.H, c.F, ex, want_h=True)
            ref += wt * oracle.matvec(ex["down_q"], ex["down_s"], c.H, c.F, _hat(h.astype(np.float32)))
        np.testing.assert_allclose(out[t], ref, rtol=1e-12, atol=1e-12)


def test_layer_is_close_to_the_plain_layer():
    # int8 activations move each input by at most half a step (1/254 of its block maximum)
    c = inputs.CONFIGS[0]
    d = inputs.tiny_layer(1)
    x = d["x"][:4]
    _, _, a = oracle.moe_layer(x, c.H, c.F, c.E, c.k, c.routed_scale, d["w_router"], d["sel_bias"], d["experts"])
    _, _, b = oracle.moe_layer_i8(x, c.H, c.F, c.E, c.k, c.routed_scale, d["w_router"], d["sel_bias"],
                                  d["experts"])
    rel = np.abs(a - b).max(axis=1) / np.abs(a).max(axis=1)
    assert (rel < 3e-2).all() and (rel > 0).all()
