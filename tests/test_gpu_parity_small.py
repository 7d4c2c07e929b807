"""GPU parity against the oracle on small layers (the tiny workload and edge cases).

Routing indices, the union and the permutation must match bit for bit; routing
weights within fp32 rounding; the layer output within the fp32-accumulate
tolerance (per-token inf-norm relative error <= 2e-3).
"""
import numpy as np
import pytest

import inputs
import oracle
import _support as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    import int4_routed_expert_bias_b200 as coli
    torch.cuda.init()
    return coli, torch


def _random_experts(rng, H, F, E):
    ex = {}
    for e in range(E + 1):
        d = {}
        for name, N, K in (("gate", F, H), ("up", F, H), ("down", H, F)):
            q, s = inputs.quantise_gs64(rng.standard_normal((N, K)) * 0.02)
            d[name + "_q"], d[name + "_s"] = q, s
        ex[e] = d
    return ex


def _run_layer(env, c, w_router, sel_bias, experts, x, out_dtype=None):
    coli, torch = env
    L = S.upload_layer(coli, torch, c, w_router, sel_bias, inputs.stack_experts(experts, c.E))
    T = x.shape[0]
    xd = S.to_device_x(x, torch)
    od = torch.bfloat16 if (out_dtype or c.out_dtype) == "bf16" else torch.float32
    out = torch.full((T, c.H), float("nan"), dtype=od, device="cuda")
    ws = torch.empty(max(coli.moe_workspace_size(L, T), 1), dtype=torch.uint8, device="cuda")
    idx = torch.full((T, c.k), -1, dtype=torch.int32, device="cuda")
    w = torch.empty((T, c.k), dtype=torch.float32, device="cuda")
    coli.moe_forward(L, xd, out, ws, idx, w)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy(), S.output_to_f64(out, torch)


def _tie_free_tiny():
    c = inputs.CONFIGS[0]
    d = inputs.tiny_layer(0)
    x = d["x"].copy()
    for sub in range(1, 50):
        _, _, (_, _, biased) = oracle.route(x, d["w_router"], d["sel_bias"], c.k, c.routed_scale, True)
        bad = S.near_ties(biased, c.k)
        if len(bad) == 0:
            break
        for t in bad:
            x[t] = inputs.tiny_redraw(int(t), sub)
    return c, d, x


def test_tiny_layer_matches_oracle(env):
    c, d, x = _tie_free_tiny()
    idx, w, out = _run_layer(env, c, d["w_router"], d["sel_bias"], d["experts"], x)
    ridx, rw, rout = oracle.moe_layer(x, c.H, c.F, c.E, c.k, c.routed_scale, d["w_router"], d["sel_bias"],
                                      d["experts"])
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6, atol=0)
    err = S.rel_inf_err(out, rout)
    assert err <= S.TOL_DECODE, err
    assert err <= 1e-4  # fp32 accumulation of int4 x fp32 stays far inside the bound


def test_tiny_router_and_union_entry_points(env):
    coli, torch = env
    c, d, x = _tie_free_tiny()
    ridx, rw = oracle.route(x, d["w_router"], d["sel_bias"], c.k, c.routed_scale)
    idx = torch.empty((c.T, c.k), dtype=torch.int32, device="cuda")
    w = torch.empty((c.T, c.k), dtype=torch.float32, device="cuda")
    coli.router_topk(torch.from_numpy(x).cuda(), torch.from_numpy(d["w_router"]).cuda(),
                     torch.from_numpy(d["sel_bias"]).cuda(), c.k, c.routed_scale, idx, w)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=2e-6)
    _check_union(env, ridx, c.E)


def _check_union(env, idx_np, E):
    coli, torch = env
    T, k = idx_np.shape
    ref = oracle.union(idx_np, E)
    i32 = dict(dtype=torch.int32, device="cuda")
    count, offset, active = torch.full((E,), -7, **i32), torch.full((E + 1,), -7, **i32), torch.full((E,), -7, **i32)
    n_active = torch.full((1,), -7, **i32)
    perm, inv = torch.full((max(T * k, 1),), -7, **i32), torch.full((max(T * k, 1),), -7, **i32)
    coli.expert_union(torch.from_numpy(idx_np).cuda() if T else torch.empty((0, k), **i32), E,
                      count, offset, active, n_active, perm, inv)
    torch.cuda.synchronize()
    assert np.array_equal(count.cpu().numpy(), ref["count"])
    assert np.array_equal(offset.cpu().numpy(), ref["offset"])
    assert np.array_equal(active.cpu().numpy(), ref["active"])
    assert int(n_active.item()) == ref["n_active"]
    if T:
        assert np.array_equal(perm.cpu().numpy(), ref["perm"])
        assert np.array_equal(inv.cpu().numpy(), ref["inv_perm"])


@pytest.mark.parametrize("T,k,E", [(1, 8, 256), (4, 8, 256), (64, 8, 256), (33, 3, 7), (4096, 8, 256),
                                   (200, 32, 1024), (5000, 1, 1), (0, 8, 256)])
def test_union_matches_oracle(env, T, k, E):
    rng = np.random.default_rng(T + 7 * E)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32) \
        if T else np.zeros((0, k), np.int32)
    _check_union(env, idx.reshape(T, k), E)


def test_union_one_hot_expert(env):
    # expert 3 is chosen by every token; the second slot cycles over 0..2
    idx = np.array([[3, t % 3] for t in range(2000)], np.int32)
    _check_union(env, idx, 4)


@pytest.mark.parametrize("T", [1, 2, 5, 7, 33, 64, 130])
def test_ragged_batches(env, T):
    """Token counts that leave partial token groups and partial warps."""
    c = inputs.Config(0, "ragged", 256, 128, 16, 4, T, "f32", "f32", 1)
    rng = np.random.default_rng(100 + T)
    ex = _random_experts(rng, c.H, c.F, c.E)
    w_router = (rng.standard_normal((c.E, c.H)) * 0.05).astype(np.float32)
    sel_bias = (rng.standard_normal(c.E) * 0.02).astype(np.float32)
    x = rng.standard_normal((T, c.H)).astype(np.float32)
    for sub in range(100):
        _, _, (_, _, biased) = oracle.route(x, w_router, sel_bias, c.k, c.routed_scale, True)
        bad = S.near_ties(biased, c.k)
        if len(bad) == 0:
            break
        x[bad] = rng.standard_normal((len(bad), c.H)).astype(np.float32)
    idx, w, out = _run_layer(env, c, w_router, sel_bias, ex, x)
    ridx, rw, rout = oracle.moe_layer(x, c.H, c.F, c.E, c.k, c.routed_scale, w_router, sel_bias, ex)
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6)
    # ffn 128 is not a multiple of 256: every batch, 130 tokens included, runs on CUDA cores in fp32
    coli, torch = env
    L = S.upload_layer(coli, torch, c, w_router, sel_bias, inputs.stack_experts(ex, c.E))
    assert coli.moe_path(L, T) == ("single" if T == 1 else "decode" if T <= 64 else "wide")
    S.check_output(out, rout, S.TOL_DECODE, f"ragged T={T}")


@pytest.mark.parametrize("T", [65, 130])
def test_just_above_the_decode_batch_limit_takes_the_tensor_cores(env, T):
    """65 and 130 tokens at hidden and ffn multiples of 256 run the tcgen05 prefill path."""
    coli, torch = env
    c = inputs.Config(0, "ragged-tc", 256, 256, 16, 4, T, "f32", "f32", 1)
    rng = np.random.default_rng(300 + T)
    ex = _random_experts(rng, c.H, c.F, c.E)
    w_router = (rng.standard_normal((c.E, c.H)) * 0.05).astype(np.float32)
    sel_bias = (rng.standard_normal(c.E) * 0.02).astype(np.float32)
    x = rng.standard_normal((T, c.H)).astype(np.float32)
    for _ in range(100):
        _, _, (_, _, biased) = oracle.route(x, w_router, sel_bias, c.k, c.routed_scale, True)
        bad = S.near_ties(biased, c.k)
        if len(bad) == 0:
            break
        x[bad] = rng.standard_normal((len(bad), c.H)).astype(np.float32)
    L = S.upload_layer(coli, torch, c, w_router, sel_bias, inputs.stack_experts(ex, c.E))
    assert coli.moe_path(L, T) == "prefill"
    idx, w, out = _run_layer(env, c, w_router, sel_bias, ex, x)
    ridx, rw, rout = oracle.moe_layer(x, c.H, c.F, c.E, c.k, c.routed_scale, w_router, sel_bias, ex)
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6)
    S.check_output(out, rout, S.TOL_PREFILL, f"tensor-core T={T}")


def test_smallest_shapes_bf16_in_bf16_out(env):
    c = inputs.Config(0, "min", 64, 64, 2, 1, 3, "bf16", "bf16", 1)
    rng = np.random.default_rng(5)
    ex = _random_experts(rng, 64, 64, 2)
    w_router = np.array([[0.05] * 64, [-0.05] * 64], np.float32)
    sel_bias = np.zeros(2, np.float32)
    x = inputs.to_bf16_bits(rng.standard_normal((3, 64)).astype(np.float32))
    idx, w, out = _run_layer(env, c, w_router, sel_bias, ex, x)
    ridx, rw, rout = oracle.moe_layer(x, 64, 64, 2, 1, c.routed_scale, w_router, sel_bias, ex)
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6)
    # bf16 output: one rounding of the fp32 result (2^-9 relative) dominates
    assert S.rel_inf_err(out, rout) <= 1e-2


def test_exact_ties_go_to_lower_index(env):
    """Router weights zero: every sigmoid is exactly 1/2 and the bias (exact in
    fp32) decides; equal biases must resolve to the lower expert index."""
    coli, torch = env
    H, E, k = 64, 8, 4
    w_router = np.zeros((E, H), np.float32)
    sel_bias = np.array([0.25, 0.5, 0.5, 0.25, 0.5, 0.0, 0.125, 0.5], np.float32)
    x = np.ones((3, H), np.float32)
    ridx, rw = oracle.route(x, w_router, sel_bias, k, 2.5)
    assert ridx[0].tolist() == [1, 2, 4, 7]
    idx = torch.empty((3, k), dtype=torch.int32, device="cuda")
    w = torch.empty((3, k), dtype=torch.float32, device="cuda")
    coli.router_topk(torch.from_numpy(x).cuda(), torch.from_numpy(w_router).cuda(),
                     torch.from_numpy(sel_bias).cuda(), k, 2.5, idx, w)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.array_equal(w.cpu().numpy(), np.full((3, k), 2.5 / 4, np.float32))
    # the layer path routes the same way
    c = inputs.Config(0, "ties", H, 64, E, k, 3, "f32", "f32", 1)
    ex = _random_experts(np.random.default_rng(1), H, 64, E)
    lidx, lw, out = _run_layer(env, c, w_router, sel_bias, ex, x)
    assert np.array_equal(lidx, ridx)
    _, _, rout = oracle.moe_layer(x, H, 64, E, k, 2.5, w_router, sel_bias, ex)
    assert S.rel_inf_err(out, rout) <= S.TOL_DECODE


def test_degenerate_batches(env):
    """All tokens identical (union = k experts); one expert forced on every
    token by its bias; routed scale 0 leaves only the shared expert."""
    c = inputs.Config(0, "degenerate", 128, 64, 12, 3, 9, "f32", "f32", 1)
    rng = np.random.default_rng(9)
    ex = _random_experts(rng, c.H, c.F, c.E)
    w_router = (rng.standard_normal((c.E, c.H)) * 0.05).astype(np.float32)
    sel_bias = np.zeros(c.E, np.float32)
    x1 = rng.standard_normal((1, c.H)).astype(np.float32)
    x = np.repeat(x1, c.T, axis=0)
    idx, w, out = _run_layer(env, c, w_router, sel_bias, ex, x)
    ridx, rw, rout = oracle.moe_layer(x, c.H, c.F, c.E, c.k, c.routed_scale, w_router, sel_bias, ex)
    assert np.array_equal(idx, ridx) and len(np.unique(idx)) == c.k
    assert S.rel_inf_err(out, rout) <= S.TOL_DECODE
    assert np.array_equal(out, np.repeat(out[:1], c.T, axis=0))  # same token, same bits

    sel_bias[5] = 10.0
    x = rng.standard_normal((c.T, c.H)).astype(np.float32)
    idx, w, out = _run_layer(env, c, w_router, sel_bias, ex, x)
    ridx, rw, rout = oracle.moe_layer(x, c.H, c.F, c.E, c.k, c.routed_scale, w_router, sel_bias, ex)
    assert np.all(idx[:, 0] == 5) and np.array_equal(idx, ridx)
    assert S.rel_inf_err(out, rout) <= S.TOL_DECODE

    c0 = inputs.Config(0, "alpha0", 128, 64, 12, 3, 9, "f32", "f32", 1, routed_scale=0.0)
    idx, w, out = _run_layer(env, c0, w_router, sel_bias, ex, x)
    _, _, rout = oracle.moe_layer(x, c.H, c.F, c.E, c.k, 0.0, w_router, sel_bias, ex)
    assert np.all(w == 0)
    assert S.rel_inf_err(out, rout) <= S.TOL_DECODE


def test_empty_batch_launches_nothing(env):
    coli, torch = env
    c = inputs.Config(0, "empty", 64, 64, 2, 1, 0, "f32", "f32", 1)
    ex = _random_experts(np.random.default_rng(2), 64, 64, 2)
    L = S.upload_layer(coli, torch, c, np.zeros((2, 64), np.float32), np.zeros(2, np.float32),
                       inputs.stack_experts(ex, 2))
    x = torch.empty((0, 64), dtype=torch.float32, device="cuda")
    out = torch.empty((0, 64), dtype=torch.float32, device="cuda")
    ws = torch.empty(1, dtype=torch.uint8, device="cuda")
    coli.moe_forward(L, x, out, ws)
    torch.cuda.synchronize()
