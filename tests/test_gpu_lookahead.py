"""Router-lookahead prefetch (layer.prefetch_next; GPU).

A one-token call that names the next layer asks the L2 cache for that layer's
router and shared expert while it routes its own token.  The prefetch is a
hint: the call's results must not change.  Checked here on two layers that
name each other (a cycle, as in a stack of layers replayed in order): routing
and output equal, bit for bit, those of the same calls without the field, and
the output matches the oracle; batches of several tokens ignore the field.
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
    layers, data = [], []
    for seed in (0, 1):
        d = inputs.tiny_layer(seed)
        st = inputs.stack_experts(d["experts"], c.E)
        dev = {n: torch.from_numpy(a).cuda() for n, a in st.items()}
        layers.append(coli.Layer(c.H, c.F, c.E, c.k, c.routed_scale, torch.from_numpy(d["w_router"]).cuda(),
                                 torch.from_numpy(d["sel_bias"]).cuda(), dev["gate_q"], dev["gate_s"],
                                 dev["up_q"], dev["up_s"], dev["down_q"], dev["down_s"]))
        data.append((d, dev))
    return coli, torch, c, layers, data


def _call(coli, torch, c, layer, x):
    T = x.shape[0]
    out = torch.full((T, c.H), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((T, c.k), -1, dtype=torch.int32, device="cuda")
    w = torch.empty((T, c.k), dtype=torch.float32, device="cuda")
    ws = torch.empty(coli.moe_workspace_size(layer, T), dtype=torch.uint8, device="cuda")
    coli.moe_forward(layer, x, out, ws, idx, w)
    torch.cuda.synchronize()
    return out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T", [1, 4])
def test_prefetch_changes_no_result(env, T):
    coli, torch, c, layers, data = env
    rng = np.random.default_rng(900 + T)
    xs = [rng.standard_normal((T, c.H)).astype(np.float32) for _ in range(4)]
    plain = []
    for i, x in enumerate(xs):
        plain.append(_call(coli, torch, c, layers[i % 2], torch.from_numpy(x).cuda()))
    layers[0].set_prefetch_next(layers[1])
    layers[1].set_prefetch_next(layers[0])
    try:
        for i, x in enumerate(xs):
            y, idx, w = _call(coli, torch, c, layers[i % 2], torch.from_numpy(x).cuda())
            assert np.array_equal(y.view(np.int32), plain[i][0].view(np.int32))
            assert np.array_equal(idx, plain[i][1])
            assert np.array_equal(w.view(np.int32), plain[i][2].view(np.int32))
            d = data[i % 2][0]
            ridx, _ = oracle.route(x, d["w_router"], d["sel_bias"], c.k, c.routed_scale)
            if np.array_equal(idx, ridx):  # a token without a score gap may route either way
                _, _, rout = oracle.moe_layer(x, c.H, c.F, c.E, c.k, c.routed_scale, d["w_router"],
                                              d["sel_bias"], d["experts"])
                S.check_output(y.astype(np.float64), rout, S.TOL_DECODE, f"lookahead T={T} call {i}")
    finally:
        layers[0].set_prefetch_next(None)
        layers[1].set_prefetch_next(None)
