"""The host-buffer entry point coli_moe_forward_host (GPU).

One C-ABI call copies the activations in from pinned host memory, runs the
layer and copies the output back to pinned host memory, all on the caller's
stream.  Checked here: the host output equals, bit for bit, what
coli_moe_forward writes from the same device input (the same kernels run),
and it matches the oracle within the path's tolerance; one-token,
several-token and (100 tokens) tensor-core batches, fp32 and bf16
activations, fp32 and bf16 outputs, several calls in a row on one set of
buffers.
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
    torch.cuda.set_device(0)
    c = inputs.CONFIGS[0]
    d = inputs.tiny_layer(0)
    st = inputs.stack_experts(d["experts"], c.E)
    dev = {n: torch.from_numpy(a).cuda() for n, a in st.items()}
    layer = coli.Layer(c.H, c.F, c.E, c.k, c.routed_scale, torch.from_numpy(d["w_router"]).cuda(),
                       torch.from_numpy(d["sel_bias"]).cuda(), dev["gate_q"], dev["gate_s"], dev["up_q"],
                       dev["up_s"], dev["down_q"], dev["down_s"])
    return coli, torch, c, d, layer


def _draw(rng, T, c, d, bf16):
    """Activations with a score gap of at least 1e-4 around every token's top-k."""
    x = rng.standard_normal((T, c.H)).astype(np.float32)
    for _ in range(100):
        xs = inputs.to_bf16_bits(x) if bf16 else x
        _, _, (_, _, b) = oracle.route(xs, d["w_router"], d["sel_bias"], c.k, c.routed_scale, True)
        top = -np.sort(-b, axis=1)[:, : c.k + 1]
        bad = np.nonzero((np.diff(-top, axis=1) < 1e-4).any(axis=1))[0]
        if len(bad) == 0:
            return xs
        x[bad] = rng.standard_normal((len(bad), c.H)).astype(np.float32)
    raise RuntimeError("could not draw tie-free activations")


@pytest.mark.parametrize("T,xdt,odt", [(1, "f32", "f32"), (4, "f32", "bf16"), (4, "bf16", "f32"),
                                       (33, "bf16", "bf16"), (100, "bf16", "bf16")])
def test_host_call_matches_the_device_call_and_the_oracle(env, T, xdt, odt):
    coli, torch, c, d, layer = env
    rng = np.random.default_rng(500 + T)
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}
    x_dev = torch.empty((T, c.H), dtype=tdt[xdt], device="cuda")
    out_dev = torch.empty((T, c.H), dtype=tdt[odt], device="cuda")
    x_host = torch.empty((T, c.H), dtype=tdt[xdt]).pin_memory()
    out_host = torch.empty((T, c.H), dtype=tdt[odt]).pin_memory()
    ws = torch.empty(coli.moe_workspace_size(layer, T), dtype=torch.uint8, device="cuda")
    for _ in range(3):  # calls in a row on the same buffers, each with new activations
        xs = _draw(rng, T, c, d, xdt == "bf16")
        src = torch.from_numpy(xs.view(np.int16) if xdt == "bf16" else xs)
        x_host.view(torch.int16 if xdt == "bf16" else torch.float32).copy_(src)
        out_host.fill_(float("nan"))
        coli.moe_forward_host(layer, x_host, x_dev, out_host, out_dev, ws)
        torch.cuda.synchronize()
        # the same device input through the device-pointer call
        ref = torch.empty_like(out_dev)
        coli.moe_forward(layer, x_dev, ref, ws)
        torch.cuda.synchronize()
        got = out_host.view(torch.int16 if odt == "bf16" else torch.int32).numpy()
        want = ref.cpu().view(torch.int16 if odt == "bf16" else torch.int32).numpy()
        assert np.array_equal(got, want)
        _, _, rout = oracle.moe_layer(xs, c.H, c.F, c.E, c.k, c.routed_scale, d["w_router"], d["sel_bias"],
                                      d["experts"])
        y = out_host.float().numpy().astype(np.float64)
        # a bf16 output adds its own rounding (2^-9); above 64 tokens the tensor-core path's bf16 operands
        tol = S.TOL_DECODE if odt == "f32" and T <= 64 else S.TOL_PREFILL
        S.check_output(y, rout, tol, f"host call T={T} x {xdt} out {odt}")
