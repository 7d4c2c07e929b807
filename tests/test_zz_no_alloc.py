"""The allocation-free entry point coli_moe_forward_noalloc (GPU).

It serves callers that cannot give the library a workspace: cudaMalloc and
cudaFree synchronise the device, so a decode loop that must not stall cannot
call them, and a host framework that owns every device allocation may forbid
the library to allocate at all.  The entry point uses a scratch array compiled
into the library instead.  Checked here through the C ABI: two calls in a row
give the same routing and, within the tests' tolerance, the same output as
coli_moe_forward with a caller workspace; a batch too large for the static
scratch is refused before anything is launched.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import inputs

pytestmark = pytest.mark.gpu

TOL = 2e-3  # per-token inf-norm relative error, as in the other parity tests


def _rel_inf_err(y, ref):
    return float((np.abs(y - ref).max(axis=1) / np.abs(ref).max(axis=1)).max())


def _tie_free(rng, T, H, w_router, sel_bias, k, alpha, bf16=False):
    """Activations whose top-(k+1) biased router scores differ by >= 1e-4 (the
    oracle's routing is then the only correct one)."""
    import oracle
    x = rng.standard_normal((T, H)).astype(np.float32)
    for _ in range(100):
        xs = inputs.to_bf16_bits(x) if bf16 else x
        _, _, (_, _, b) = oracle.route(xs, w_router, sel_bias, k, alpha, True)
        top = -np.sort(-b, axis=1)[:, : k + 1]
        bad = np.nonzero((np.diff(-top, axis=1) < 1e-4).any(axis=1))[0]
        if len(bad) == 0:
            return xs
        x[bad] = rng.standard_normal((len(bad), H)).astype(np.float32)
    raise RuntimeError("could not draw tie-free activations")


@pytest.fixture(scope="module")
def env():
    import torch
    import int4_routed_expert_bias_b200 as coli
    torch.cuda.set_device(0)
    c = inputs.CONFIGS[0]
    d = inputs.tiny_layer(0)
    st = inputs.stack_experts(d["experts"], c.E)
    dev = {n: torch.from_numpy(a).cuda() for n, a in st.items()}
    layer = coli.Layer(c.H, c.F, c.E, c.k, c.routed_scale, torch.from_numpy(d["w_router"]).cuda(),
                       torch.from_numpy(d["sel_bias"]).cuda(), dev["gate_q"], dev["gate_s"], dev["up_q"],
                       dev["up_s"], dev["down_q"], dev["down_s"])
    return coli, torch, c, layer


def _noalloc(coli, torch, layer, x, out, idx, w):
    st = coli.lib().coli_moe_forward_noalloc(layer.ref, x.data_ptr(), coli.F32, x.shape[0], out.data_ptr(),
                                             coli.F32, idx.data_ptr(), w.data_ptr(),
                                             torch.cuda.current_stream().cuda_stream)
    return st


def test_two_calls_match_the_workspace_entry_point(env):
    import oracle
    coli, torch, c, layer = env
    d = inputs.tiny_layer(0)
    rng = np.random.default_rng(77)
    for T in (4, 7):  # two calls in a row through the same static scratch
        x = torch.from_numpy(_tie_free(rng, T, c.H, d["w_router"], d["sel_bias"], c.k, c.routed_scale)).cuda()
        ref = torch.empty((T, c.H), dtype=torch.float32, device="cuda")
        ridx = torch.empty((T, c.k), dtype=torch.int32, device="cuda")
        rw = torch.empty((T, c.k), dtype=torch.float32, device="cuda")
        ws = torch.empty(coli.moe_workspace_size(layer, T), dtype=torch.uint8, device="cuda")
        coli.moe_forward(layer, x, ref, ws, ridx, rw)
        out = torch.full((T, c.H), float("nan"), dtype=torch.float32, device="cuda")
        idx = torch.full((T, c.k), -1, dtype=torch.int32, device="cuda")
        w = torch.empty((T, c.k), dtype=torch.float32, device="cuda")
        assert _noalloc(coli, torch, layer, x, out, idx, w) == 0, coli.last_error()
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), ridx.cpu().numpy())
        np.testing.assert_allclose(w.cpu().numpy(), rw.cpu().numpy(), rtol=2e-6)
        y = out.cpu().numpy().astype(np.float64)
        err = _rel_inf_err(y, ref.cpu().numpy().astype(np.float64))
        assert err <= TOL, err
        _, _, rout = oracle.moe_layer(x.cpu().numpy(), c.H, c.F, c.E, c.k, c.routed_scale, d["w_router"],
                                      d["sel_bias"], d["experts"])
        assert _rel_inf_err(y, rout) <= TOL


@pytest.fixture(scope="module")
def full_layer():
    """The full expert shape (hidden 6144, ffn 2048, 256 routed + 1 shared), on the device."""
    import torch
    import int4_routed_expert_bias_b200 as coli
    c = inputs.CONFIGS[3]
    bufs = inputs.device_layer_tensors(torch, c, 5, 0)
    w_router, sel_bias = inputs.router_params(c, 5, 0)
    layer = coli.Layer(c.H, c.F, c.E, c.k, c.routed_scale, torch.from_numpy(w_router).cuda(),
                       torch.from_numpy(sel_bias).cuda(), bufs["gate_q"], bufs["gate_s"], bufs["up_q"],
                       bufs["up_s"], bufs["down_q"], bufs["down_s"])
    yield coli, torch, c, layer, w_router, sel_bias
    del layer, bufs
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T,xdt", [(1, "f32"), (1, "bf16"), (28, "bf16")])
def test_full_shape_matches_the_workspace_call_and_the_oracle(full_layer, T, xdt):
    """One decode token (the one-token chain) in fp32 and bf16, and 28 tokens, the
    largest batch the 8 MiB scratch takes at this shape; two calls in a row."""
    import oracle
    coli, torch, c, layer, w_router, sel_bias = full_layer
    assert coli.moe_workspace_size(layer, T) <= 8 << 20
    rng = np.random.default_rng(1000 + T)
    xs = _tie_free(rng, T, c.H, w_router, sel_bias, c.k, c.routed_scale, xdt == "bf16")
    x = torch.from_numpy(xs.view(np.int16)).cuda().view(torch.bfloat16) if xdt == "bf16" else \
        torch.from_numpy(xs).cuda()
    ref = torch.empty((T, c.H), dtype=torch.float32, device="cuda")
    ridx = torch.empty((T, c.k), dtype=torch.int32, device="cuda")
    rw = torch.empty((T, c.k), dtype=torch.float32, device="cuda")
    ws = torch.empty(coli.moe_workspace_size(layer, T), dtype=torch.uint8, device="cuda")
    coli.moe_forward(layer, x, ref, ws, ridx, rw)
    for _ in range(2):
        out = torch.full((T, c.H), float("nan"), dtype=torch.float32, device="cuda")
        idx = torch.full((T, c.k), -1, dtype=torch.int32, device="cuda")
        w = torch.empty((T, c.k), dtype=torch.float32, device="cuda")
        st = coli.lib().coli_moe_forward_noalloc(layer.ref, x.data_ptr(), coli.BF16 if xdt == "bf16" else coli.F32,
                                                  T, out.data_ptr(), coli.F32, idx.data_ptr(), w.data_ptr(),
                                                  torch.cuda.current_stream().cuda_stream)
        assert st == 0, coli.last_error()
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), ridx.cpu().numpy())
        np.testing.assert_allclose(w.cpu().numpy(), rw.cpu().numpy(), rtol=2e-6)
        y = out.cpu().numpy().astype(np.float64)
        assert _rel_inf_err(y, ref.cpu().numpy().astype(np.float64)) <= TOL
    # and against the oracle, on up to 4 tokens (the oracle's f64 loops are slow at this shape)
    toks = np.unique(np.array([0, T // 3, (2 * T) // 3, T - 1]))
    oidx, _ = oracle.route(xs, w_router, sel_bias, c.k, c.routed_scale)
    assert np.array_equal(idx.cpu().numpy(), oidx)
    need = set(oidx[toks].ravel().tolist()) | {c.E}
    experts = {e: inputs.gen_expert_host(c, 5, 0, e) for e in need}
    _, _, rout = oracle.moe_layer(xs[toks], c.H, c.F, c.E, c.k, c.routed_scale, w_router, sel_bias, experts)
    assert _rel_inf_err(y[toks], rout) <= TOL


def test_batch_beyond_the_static_scratch_is_refused(env):
    coli, torch, c, layer = env
    limit = 8 << 20  # COLI_NOALLOC_SCRATCH_BYTES
    T = 1
    while coli.moe_workspace_size(layer, T) <= limit:
        T *= 2
    x = torch.zeros((T, c.H), dtype=torch.float32, device="cuda")
    out = torch.full((T, c.H), 7.0, dtype=torch.float32, device="cuda")
    idx = torch.zeros((T, c.k), dtype=torch.int32, device="cuda")
    w = torch.zeros((T, c.k), dtype=torch.float32, device="cuda")
    assert _noalloc(coli, torch, layer, x, out, idx, w) == 3  # COLI_ERR_WORKSPACE
    assert "static scratch" in coli.last_error()
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was launched
