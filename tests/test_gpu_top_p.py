"""GPU parity of adaptive expert top-p routing (layer.top_p) against the oracle.

Reading of the pages' --topp knob ("colibri解説", section 速度を稼ぐ実用ノブ): of
the k selected experts, ranked by share s_j / sum s, keep the shortest prefix
whose cumulative share reaches p and renormalise the kept weights; dropped
slots are index -1 with weight 0.  Every kernel chain (one token, the fused
decode kernel, the tensor-core prefill, the CUDA-core expert phases) is
checked: routing bit-exact (dropped slots included), weights within fp32
rounding, layer output within the chain's tolerance.  Inputs keep every score
gap and every cumulative share at least 1e-4 away from a tie or from p, so the
f64 oracle and the fp32 kernels take the same decisions.
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


def _experts(rng, H, F, E):
    ex = {}
    for e in range(E + 1):
        ex[e] = {}
        for name, N, K in (("gate", F, H), ("up", F, H), ("down", H, F)):
            q, s = inputs.quantise_gs64(rng.standard_normal((N, K)) * 0.02)
            ex[e][name + "_q"], ex[e][name + "_s"] = q, s
    return ex


@pytest.mark.parametrize("H,F,E,k,T,p,path", [
    (1024, 512, 64, 8, 1, 0.7, "single"),
    (1024, 512, 64, 8, 4, 0.7, "decode"),
    (1024, 512, 64, 8, 33, 0.5, "decode"),
    (256, 256, 16, 4, 300, 0.7, "prefill"),
    (256, 128, 16, 4, 130, 0.6, "wide"),
])
def test_top_p_layer_matches_oracle(env, H, F, E, k, T, p, path):
    coli, torch = env
    rng = np.random.default_rng(7 * T + H)
    ex = _experts(rng, H, F, E)
    w_router = (rng.standard_normal((E, H)) * 0.05).astype(np.float32)
    sel_bias = (rng.standard_normal(E) * 0.02).astype(np.float32)
    c = inputs.Config(0, "top-p", H, F, E, k, T, "f32", "f32", 1)
    x = rng.standard_normal((T, H)).astype(np.float32)
    for _ in range(200):
        _, _, (_, _, biased) = oracle.route(x, w_router, sel_bias, k, c.routed_scale, True)
        bad = np.union1d(S.near_ties(biased, k), S.near_top_p_boundary(x, w_router, sel_bias, k, c.routed_scale, p))
        if len(bad) == 0:
            break
        x[bad] = rng.standard_normal((len(bad), H)).astype(np.float32)
    else:
        raise RuntimeError("could not draw decision-free activations")
    stacked = inputs.stack_experts(ex, E)
    dev = {n: torch.from_numpy(a).cuda() for n, a in stacked.items()}
    L = coli.Layer(H, F, E, k, c.routed_scale, torch.from_numpy(w_router).cuda(), torch.from_numpy(sel_bias).cuda(),
                   dev["gate_q"], dev["gate_s"], dev["up_q"], dev["up_s"], dev["down_q"], dev["down_s"], top_p=p)
    assert coli.moe_path(L, T) == path
    out = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(coli.moe_workspace_size(L, T), dtype=torch.uint8, device="cuda")
    idx = torch.full((T, k), 99, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), 99.0, dtype=torch.float32, device="cuda")
    coli.moe_forward(L, torch.from_numpy(x).cuda(), out, ws, idx, w)
    torch.cuda.synchronize()
    ridx, rw, rout = oracle.moe_layer_top_p(x, H, F, E, k, c.routed_scale, p, w_router, sel_bias, ex)
    idx, w = idx.cpu().numpy(), w.cpu().numpy()
    assert np.array_equal(idx, ridx)
    assert (ridx < 0).any(), "the cut should drop some experts"
    assert np.all(w[ridx < 0] == 0)
    np.testing.assert_allclose(w, rw, rtol=2e-6, atol=0)
    S.check_output(S.output_to_f64(out, torch), rout, S.TOL_PREFILL if path == "prefill" else S.TOL_DECODE,
                   f"top-p {p} {path} T={T}")


def test_top_p_one_is_plain_top_k(env):
    coli, torch = env
    c = inputs.CONFIGS[0]
    d = inputs.tiny_layer(0)
    x = d["x"].copy()
    st = inputs.stack_experts(d["experts"], c.E)
    dev = {n: torch.from_numpy(a).cuda() for n, a in st.items()}
    outs = []
    for p in (0.0, 1.0):
        L = coli.Layer(c.H, c.F, c.E, c.k, c.routed_scale, torch.from_numpy(d["w_router"]).cuda(),
                       torch.from_numpy(d["sel_bias"]).cuda(), dev["gate_q"], dev["gate_s"], dev["up_q"],
                       dev["up_s"], dev["down_q"], dev["down_s"], top_p=p)
        out = torch.empty((c.T, c.H), dtype=torch.float32, device="cuda")
        ws = torch.empty(coli.moe_workspace_size(L, c.T), dtype=torch.uint8, device="cuda")
        coli.moe_forward(L, torch.from_numpy(x).cuda(), out, ws)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])
