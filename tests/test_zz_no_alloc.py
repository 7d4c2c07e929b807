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
    coli, torch, c, layer = env
    rng = np.random.default_rng(77)
    for T in (4, 7):  # two calls in a row through the same static scratch
        x = torch.from_numpy(rng.standard_normal((T, c.H)).astype(np.float32)).cuda()
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
        err = _rel_inf_err(out.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64))
        assert err <= TOL, err


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
