"""GPU parity of the integer-activation variant (layer.act_int8) against the
oracle at small shapes: one token, the fused decode kernel's 4- and 33-token
batches, fp32 and bf16 activations, and a block of zeros and a block of tiny
values in x.

Reading of the pages' integer dot-product kernel ("Colibri 完全ガイド", section
コア技術のハイライト, row 整数ドット積カーネル: int8 activations times packed int4
weights): symmetric int8 per 32 values, scale max/127, codes rounded to
nearest even in fp32, for x before gate/up and for h before down; the route is
the plain one.  The oracle reproduces the quantisation, so the output is held
to the decode tolerance (an h value within fp32 rounding of a code boundary may
take the other code; that moves the output by about 0.03 / sqrt(F) of its
norm).
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


@pytest.mark.parametrize("H,F,E,k,T,xdt,path", [
    (1024, 512, 64, 8, 1, "f32", "single"),
    (1024, 512, 64, 8, 1, "bf16", "single"),
    (1024, 512, 64, 8, 4, "f32", "decode"),
    (1024, 512, 64, 8, 33, "bf16", "decode"),
])
def test_int8_activation_layer_matches_oracle(env, H, F, E, k, T, xdt, path):
    coli, torch = env
    rng = np.random.default_rng(11 * T + H + (xdt == "bf16"))
    ex = _experts(rng, H, F, E)
    w_router = (rng.standard_normal((E, H)) * 0.05).astype(np.float32)
    sel_bias = (rng.standard_normal(E) * 0.02).astype(np.float32)
    x32 = rng.standard_normal((T, H)).astype(np.float32)
    x32[0, 64:96] = 0.0    # an all-zero block
    x32[0, 128:160] *= 1e-30  # a block of tiny values (quantised like any other)
    for _ in range(200):
        x = inputs.to_bf16_bits(x32) if xdt == "bf16" else x32
        _, _, (_, _, biased) = oracle.route(x, w_router, sel_bias, k, 2.5, True)
        bad = S.near_ties(biased, k)
        if len(bad) == 0:
            break
        x32[bad] = rng.standard_normal((len(bad), H)).astype(np.float32)
    else:
        raise RuntimeError("could not draw tie-free activations")
    stacked = inputs.stack_experts(ex, E)
    dev = {n: torch.from_numpy(a).cuda() for n, a in stacked.items()}
    L = coli.Layer(H, F, E, k, 2.5, torch.from_numpy(w_router).cuda(), torch.from_numpy(sel_bias).cuda(),
                   dev["gate_q"], dev["gate_s"], dev["up_q"], dev["up_s"], dev["down_q"], dev["down_s"],
                   act_int8=True)
    assert coli.moe_path(L, T) == path
    out = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(coli.moe_workspace_size(L, T), dtype=torch.uint8, device="cuda")
    idx = torch.full((T, k), 99, dtype=torch.int32, device="cuda")
    coli.moe_forward(L, S.to_device_x(x, torch), out, ws, idx)
    torch.cuda.synchronize()
    ridx, _, rout = oracle.moe_layer_i8(x, H, F, E, k, 2.5, w_router, sel_bias, ex)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    S.check_output(out.cpu().numpy(), rout, S.TOL_DECODE, f"int8 activations T={T} {xdt}")
    # the variant differs from the default layer by the quantisation, well above the parity tolerance
    _, _, plain = oracle.moe_layer(x, H, F, E, k, 2.5, w_router, sel_bias, ex)
    assert S.rel_inf_err(rout, plain) > 10 * S.rel_inf_err(out.cpu().numpy(), rout)
