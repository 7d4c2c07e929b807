"""GPU parity at the full layer shape (H 6144, F 2048, 256 routed experts + 1
shared, top-8), through the same entry point and launch path the benchmark
times, for the four full-size workloads (decode-1, verify-4, decode-64,
prefill-4096).

Routing and the union are compared for every token.  The layer output is
compared for every token of the decode batches (1, 4 and 64 tokens) and, for
the 4096-token prefill, for tokens chosen so that every tile the tensor-core
GEMMs compute is checked: one token from each 192-pair token tile of the shared
expert, the first and last pair of 16 routed experts, and the first and last
token (the oracle computes tokens independently: a T-token call equals T
one-token calls).
"""
import numpy as np
import pytest

import inputs
import oracle
import _support as S

pytestmark = pytest.mark.gpu

SEED = 20261202
LAYER = 0


@pytest.fixture(scope="module")
def full():
    import torch
    import int4_routed_expert_bias_b200 as coli
    c = inputs.CONFIGS[1]
    bufs = S.device_layer_generated(coli, torch, c, SEED, LAYER)
    torch.cuda.synchronize()
    cache = {}

    def host_expert(e):
        if e not in cache:
            cache[e] = inputs.gen_expert_host(c, SEED, LAYER, e)
        return cache[e]

    yield coli, torch, bufs, host_expert
    del bufs
    torch.cuda.empty_cache()


def _layer(coli, torch, c, bufs, w_router, sel_bias):
    return coli.Layer(c.H, c.F, c.E, c.k, c.routed_scale, torch.from_numpy(w_router).cuda(),
                      torch.from_numpy(sel_bias).cuda(), bufs["gate_q"], bufs["gate_s"], bufs["up_q"],
                      bufs["up_s"], bufs["down_q"], bufs["down_s"])


def test_device_generator_matches_host(full):
    coli, torch, bufs, host_expert = full
    for e in (0, 17, 256):
        h = host_expert(e)
        for n in ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s"):
            assert np.array_equal(bufs[n][e].cpu().numpy(), h[n]), (e, n)


PF_TILE = 192  # token-tile width of the prefill GEMMs (pairs of one expert per tile)


def prefill_tokens(ridx, u, T, k, rng, n_experts=16):
    """Tokens whose outputs cover every shared-expert token tile and both ends
    of the token tiles of n_experts routed experts, plus tokens 0 and T-1."""
    toks = {0, T - 1}
    for b in range(0, T, PF_TILE):
        toks.add(int(rng.integers(b, min(b + PF_TILE, T))))
    active = u["active"][: u["n_active"]]
    for e in rng.choice(active, size=min(n_experts, len(active)), replace=False):
        first, last = u["offset"][e], u["offset"][e + 1] - 1
        toks.add(int(u["perm"][first]) // k)
        toks.add(int(u["perm"][last]) // k)
    return np.array(sorted(toks))


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_full_size_layer_matches_oracle(full, cfg):
    coli, torch, bufs, host_expert = full
    c = inputs.CONFIGS[cfg]
    w_router, sel_bias = inputs.router_params(c, SEED, LAYER)
    x, _ = S.x_without_ties(c, SEED, 0, LAYER, w_router, sel_bias)
    L = _layer(coli, torch, c, bufs, w_router, sel_bias)
    T = c.T
    xd = S.to_device_x(x, torch)
    out = torch.empty((T, c.H), dtype=torch.bfloat16 if c.out_dtype == "bf16" else torch.float32,
                      device="cuda")
    ws = torch.empty(coli.moe_workspace_size(L, T), dtype=torch.uint8, device="cuda")
    idx = torch.empty((T, c.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, c.k), dtype=torch.float32, device="cuda")
    coli.moe_forward(L, xd, out, ws, idx, w)
    torch.cuda.synchronize()
    idx, w = idx.cpu().numpy(), w.cpu().numpy()
    out = S.output_to_f64(out, torch)

    # routing and union: every token, bit-exact
    ridx, rw = oracle.route(x, w_router, sel_bias, c.k, c.routed_scale)
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6)
    u = oracle.union(ridx, c.E)
    if cfg == 2:
        assert 8 <= u["n_active"] <= 32
    if cfg == 3:
        assert u["count"].max() > 8  # the Zipf bias makes hot experts

    # outputs: every token of a decode batch; the tile-covering sample of the prefill batch
    assert coli.moe_path(L, T) == {1: "single", 2: "decode", 3: "decode", 4: "prefill"}[cfg]
    rng = np.random.default_rng(cfg)
    tokens = np.arange(T) if T <= 64 else prefill_tokens(ridx, u, T, c.k, rng)
    assert tokens[-1] == T - 1
    need = set(ridx[tokens].ravel().tolist()) | {c.E}
    experts = {e: host_expert(e) for e in need}
    _, _, rout = oracle.moe_layer(x[tokens], c.H, c.F, c.E, c.k, c.routed_scale, w_router, sel_bias, experts)
    tol = S.TOL_PREFILL if T > 64 else S.TOL_DECODE
    S.check_output(out[tokens], rout, tol, f"{c.name} ({len(tokens)} of {T} tokens)")


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_full_size_int8_activations_match_oracle(full, cfg):
    """The integer-activation variant (layer.act_int8) at the full shape, every
    token: routing bit-exact, output against the oracle's int8-activation layer
    within the decode tolerance (the quantisation is reproduced exactly; an h
    value within fp32 rounding of a code boundary may take the other code,
    which moves the output by about 0.03 / sqrt(F) of its norm)."""
    coli, torch, bufs, host_expert = full
    c = inputs.CONFIGS[cfg]
    w_router, sel_bias = inputs.router_params(c, SEED, LAYER)
    x, _ = S.x_without_ties(c, SEED, 1, LAYER, w_router, sel_bias)
    L = coli.Layer(c.H, c.F, c.E, c.k, c.routed_scale, torch.from_numpy(w_router).cuda(),
                   torch.from_numpy(sel_bias).cuda(), bufs["gate_q"], bufs["gate_s"], bufs["up_q"],
                   bufs["up_s"], bufs["down_q"], bufs["down_s"], act_int8=True)
    T = c.T
    out = torch.empty((T, c.H), dtype=torch.bfloat16 if c.out_dtype == "bf16" else torch.float32,
                      device="cuda")
    ws = torch.empty(coli.moe_workspace_size(L, T), dtype=torch.uint8, device="cuda")
    idx = torch.empty((T, c.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, c.k), dtype=torch.float32, device="cuda")
    coli.moe_forward(L, S.to_device_x(x, torch), out, ws, idx, w)
    torch.cuda.synchronize()
    ridx, rw = oracle.route(x, w_router, sel_bias, c.k, c.routed_scale)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    need = set(ridx.ravel().tolist()) | {c.E}
    experts = {e: host_expert(e) for e in need}
    _, _, rout = oracle.moe_layer_i8(x, c.H, c.F, c.E, c.k, c.routed_scale, w_router, sel_bias, experts)
    S.check_output(S.output_to_f64(out, torch), rout, S.TOL_DECODE, f"{c.name} int8 activations")
