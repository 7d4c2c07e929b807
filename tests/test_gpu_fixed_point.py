"""GPU parity of the decode kernel's fixed-point activation staging at its edges
(small shapes, against the oracle's f64 layer).

The fused decode kernel multiplies int4 weights with activations held as fixed
point per block of 32 values over a power-of-two block scale: 21 bits for fp32
activations, 14 bits plus sign for bf16 ones (and the SwiGLU output h of the
same call alike).  Blocks whose largest magnitude is below 2^-100 contribute
nothing.  These cases put a block of zeros, a block of values near 1e-30 and
one near 1e-33 (either side of that cut-off), a block with one value 50 times
its neighbours' scale and a block spanning twenty
binary orders into x, for one token, one group of 2, 3 or 4 tokens, 5 tokens
(a full group and one of a single token) and 33 tokens, in fp32 and bf16, with every one-token and several-token stream
shape the kernel has (four rows per step; two for several fp32 tokens).  The
output is held to the decode tolerance and the routing must be exact.
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


@pytest.mark.parametrize("T,xdt,path", [(1, "f32", "single"), (1, "bf16", "single"), (2, "bf16", "decode"),
                                        (3, "bf16", "decode"), (4, "f32", "decode"), (4, "bf16", "decode"),
                                        (5, "bf16", "decode"), (33, "f32", "decode"), (33, "bf16", "decode")])
def test_edge_blocks_match_the_oracle(env, T, xdt, path):
    coli, torch = env
    H, F, E, k = 1024, 512, 64, 8
    rng = np.random.default_rng(700 + 3 * T + (xdt == "bf16"))
    ex = _experts(rng, H, F, E)
    w_router = (rng.standard_normal((E, H)) * 0.05).astype(np.float32)
    sel_bias = (rng.standard_normal(E) * 0.02).astype(np.float32)
    x32 = rng.standard_normal((T, H)).astype(np.float32)

    def edges(x):
        x[:, 64:96] = 0.0                                   # a block of zeros
        x[:, 128:160] *= 1e-30                              # a block of tiny values (above 2^-100: quantised)
        x[:, 320:352] *= 1e-33                              # a block below the 2^-100 cut-off (contributes 0)
        x[:, 192] = 50.0                                    # one value far above its block's others
        x[:, 256:288] *= np.float32(2.0) ** -np.arange(0, 20, 20 / 32, dtype=np.float32)  # 20 binary orders

    edges(x32)
    for _ in range(200):
        x = inputs.to_bf16_bits(x32) if xdt == "bf16" else x32
        _, _, (_, _, biased) = oracle.route(x, w_router, sel_bias, k, 2.5, True)
        bad = S.near_ties(biased, k)
        if len(bad) == 0:
            break
        x32[bad] = rng.standard_normal((len(bad), H)).astype(np.float32)
        edges(x32)
    else:
        raise RuntimeError("could not draw tie-free activations")
    stacked = inputs.stack_experts(ex, E)
    dev = {n: torch.from_numpy(a).cuda() for n, a in stacked.items()}
    L = coli.Layer(H, F, E, k, 2.5, torch.from_numpy(w_router).cuda(), torch.from_numpy(sel_bias).cuda(),
                   dev["gate_q"], dev["gate_s"], dev["up_q"], dev["up_s"], dev["down_q"], dev["down_s"])
    assert coli.moe_path(L, T) == path
    out = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(coli.moe_workspace_size(L, T), dtype=torch.uint8, device="cuda")
    idx = torch.full((T, k), 99, dtype=torch.int32, device="cuda")
    coli.moe_forward(L, S.to_device_x(x, torch), out, ws, idx)
    torch.cuda.synchronize()
    ridx, _, rout = oracle.moe_layer(x, H, F, E, k, 2.5, w_router, sel_bias, ex)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    S.check_output(out.cpu().numpy(), rout, S.TOL_DECODE, f"fixed-point edges T={T} {xdt}")
