"""The kernels' bounded waits, made to run out on purpose (GPU).

Every wait inside a launch (the decode kernel's grid barriers, the prefill
GEMMs' pipeline waits) gives up after a time limit, records a non-zero status
word in the workspace and lets the kernel finish.  The test hook
coli_debug_set_wait_ns shortens the limit to a microsecond so that the waits
run out; the call must still return and complete, its status word must say so,
and the next call with the normal limit must match the oracle again.  No fault,
trap or endless wait is involved: a timed-out wait only stops waiting.
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
    yield coli, torch
    coli.debug_set_wait_ns(0)


def _experts(rng, H, F, E):
    ex = {}
    for e in range(E + 1):
        ex[e] = {}
        for name, N, K in (("gate", F, H), ("up", F, H), ("down", H, F)):
            q, s = inputs.quantise_gs64(rng.standard_normal((N, K)) * 0.02)
            ex[e][name + "_q"], ex[e][name + "_s"] = q, s
    return ex


@pytest.mark.parametrize("H,F,E,k,T,path,code", [
    (1024, 512, 64, 8, 4, "decode", 2),     # grid barriers of the fused decode kernel
    (1024, 512, 64, 8, 1, "single", 2),
    (256, 256, 16, 4, 100, "prefill", 1),   # mbarrier waits of the tcgen05 GEMMs
])
def test_waits_that_run_out_are_reported_and_the_next_call_is_right(env, H, F, E, k, T, path, code):
    coli, torch = env
    rng = np.random.default_rng(H + T)
    ex = _experts(rng, H, F, E)
    w_router = (rng.standard_normal((E, H)) * 0.05).astype(np.float32)
    sel_bias = (rng.standard_normal(E) * 0.02).astype(np.float32)
    c = inputs.Config(0, "waits", H, F, E, k, T, "f32", "f32", 1)
    x = rng.standard_normal((T, H)).astype(np.float32)
    for _ in range(100):
        _, _, (_, _, biased) = oracle.route(x, w_router, sel_bias, k, c.routed_scale, True)
        bad = S.near_ties(biased, k)
        if len(bad) == 0:
            break
        x[bad] = rng.standard_normal((len(bad), H)).astype(np.float32)
    L = S.upload_layer(coli, torch, c, w_router, sel_bias, inputs.stack_experts(ex, E))
    assert coli.moe_path(L, T) == path
    xd = torch.from_numpy(x).cuda()
    out = torch.empty((T, H), dtype=torch.float32, device="cuda")
    ws = torch.zeros(coli.moe_workspace_size(L, T), dtype=torch.uint8, device="cuda")
    off = coli.moe_status_word_offset(L, T)
    word = lambda: int(ws[off:off + 4].view(torch.int32).item())

    coli.debug_set_wait_ns(1000)  # 1 us: the waits run out
    try:
        coli.moe_forward(L, xd, out, ws)  # returns normally
        torch.cuda.synchronize()          # and the launch completes
    finally:
        coli.debug_set_wait_ns(0)
    assert word() == code

    out.fill_(float("nan"))
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    coli.moe_forward(L, xd, out, ws, idx)
    torch.cuda.synchronize()
    assert word() == 0
    ridx, _, rout = oracle.moe_layer(x, H, F, E, k, c.routed_scale, w_router, sel_bias, ex)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    S.check_output(S.output_to_f64(out, torch), rout, S.TOL_PREFILL if T > 64 else S.TOL_DECODE,
                   f"after a timed-out {path} call")
