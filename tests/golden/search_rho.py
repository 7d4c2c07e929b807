"""Seeded search for the verify-batch correlation rho (4 tokens: 1 verified + 3 drafts).

Draft token t is x_t = sqrt(rho) z0 + sqrt(1 - rho) z_t with z ~ N(0, 1).  For
each candidate rho this routes many batches through the oracle router (only
oracle/ and the input generator are used) and reports the mean fraction of a
draft's experts that token 0 also selects, and the batch-union size U.  The
value kept in inputs.VERIFY_RHO is the one whose mean overlap is closest to
60 % with mean U inside [16, 24].

    python tests/golden/search_rho.py
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))

import inputs  # noqa: E402
import oracle  # noqa: E402


def measure(rho, batches=64, seed=7):
    c = inputs.CONFIGS[2]
    w, b = inputs.router_params(c, seed, 0)
    rng = np.random.default_rng(seed)
    ov, us = [], []
    for _ in range(batches):
        z0 = rng.standard_normal(c.H)
        x = [z0] + [np.sqrt(rho) * z0 + np.sqrt(1 - rho) * rng.standard_normal(c.H) for _ in range(3)]
        x = inputs.to_bf16_bits(np.array(x, np.float32))
        idx, _ = oracle.route(x, w, b, c.k, c.routed_scale)
        s0 = set(idx[0].tolist())
        ov.append(np.mean([len(s0 & set(idx[t].tolist())) / c.k for t in range(1, 4)]))
        us.append(len(np.unique(idx)))
    return float(np.mean(ov)), float(np.mean(us)), int(np.min(us)), int(np.max(us))


if __name__ == "__main__":
    for rho in (0.70, 0.75, 0.78, 0.79, 0.80, 0.81, 0.82, 0.85, 0.90):
        o, u, lo, hi = measure(rho)
        print(f"rho {rho:.2f}: mean overlap {o:.3f}, mean U {u:.1f} (min {lo}, max {hi})")
