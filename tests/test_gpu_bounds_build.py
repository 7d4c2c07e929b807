"""The bounds-checked build (libcoli_bounds.so, COLI_DEBUG_BOUNDS) on the GPU.

In that build the kernels check the indices they compute from data (the
routing's experts, union positions, output rows) before using them; a failed
check records status 4 in the call's status word and skips or redirects the
access instead of trapping.  Run in a child process that loads that library
(COLI_LIB=bounds): the tiny layer on the fused decode kernel (4 tokens and one
token) and a small prefill must give status 0 and match the oracle.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

CHILD = r"""
import sys
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import numpy as np, torch
import inputs, oracle, _support as S
import int4_routed_expert_bias_b200 as coli
assert coli.LIB_PATH.endswith("libcoli_bounds.so"), coli.LIB_PATH
torch.cuda.set_device(0)
def experts(rng, H, F, E):
    ex = {}
    for e in range(E + 1):
        ex[e] = {}
        for name, N, K in (("gate", F, H), ("up", F, H), ("down", H, F)):
            q, s = inputs.quantise_gs64(rng.standard_normal((N, K)) * 0.02)
            ex[e][name + "_q"], ex[e][name + "_s"] = q, s
    return ex
for H, F, E, k, T in ((1024, 512, 64, 8, 4), (1024, 512, 64, 8, 1), (256, 256, 16, 4, 100)):
    rng = np.random.default_rng(H + T)
    ex = experts(rng, H, F, E)
    wr = (rng.standard_normal((E, H)) * 0.05).astype(np.float32)
    sb = (rng.standard_normal(E) * 0.02).astype(np.float32)
    c = inputs.Config(0, "bounds", H, F, E, k, T, "f32", "f32", 1)
    x = rng.standard_normal((T, H)).astype(np.float32)
    for _ in range(100):
        _, _, (_, _, b) = oracle.route(x, wr, sb, k, c.routed_scale, True)
        bad = S.near_ties(b, k)
        if len(bad) == 0:
            break
        x[bad] = rng.standard_normal((len(bad), H)).astype(np.float32)
    L = S.upload_layer(coli, torch, c, wr, sb, inputs.stack_experts(ex, E))
    out = torch.empty((T, H), dtype=torch.float32, device="cuda")
    ws = torch.zeros(coli.moe_workspace_size(L, T), dtype=torch.uint8, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    coli.moe_forward(L, torch.from_numpy(x).cuda(), out, ws, idx)
    torch.cuda.synchronize()
    off = coli.moe_status_word_offset(L, T)
    word = int(ws[off:off + 4].view(torch.int32).item())
    assert word == 0, (T, word)
    ridx, _, rout = oracle.moe_layer(x, H, F, E, k, c.routed_scale, wr, sb, ex)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    S.check_output(S.output_to_f64(out, torch), rout, S.TOL_PREFILL if T > 64 else S.TOL_DECODE,
                   f"bounds build, {coli.moe_path(L, T)} T={T}")
print("bounds build ok")
"""


def test_bounds_checked_build_runs_clean_and_matches_the_oracle():
    lib = os.path.join(ROOT, "int4_routed_expert_bias_b200", "libcoli_bounds.so")
    if not os.path.exists(lib):
        sys.path.insert(0, ROOT)
        from int4_routed_expert_bias_b200 import _build
        _build.build(bounds=True)
    env = dict(os.environ, COLI_LIB="bounds")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + CHILD], env=env, capture_output=True,
                       text=True, timeout=600)
    print(r.stdout[-2000:])
    assert r.returncode == 0, r.stderr[-3000:]
    assert "bounds build ok" in r.stdout
