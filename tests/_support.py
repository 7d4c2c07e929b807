"""Shared helpers of the parity tests: device upload, near-tie redraws, error metrics.

The oracle side and the CUDA side get the same stored inputs from the input
generator (inputs/); nothing here computes any part of the layer.
"""
import numpy as np

import inputs
import oracle

GAP = 1e-4        # minimum gap between adjacent top-(k+1) biased scores (exact routing)
TOL_DECODE = 2e-3  # per-token inf-norm relative error, fp32-accumulate path
TOL_PREFILL = 1e-2  # bf16 tensor-core path


def rel_inf_err(y, ref):
    """Per-token inf-norm relative error max_t |y_t - r_t|_inf / |r_t|_inf."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.abs(y - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    return float((num / den).max())


def big_element_err(y, ref):
    """Largest element-wise relative error over the elements that carry the
    output: |r| > 0.1 * |r_t|_inf of their token (near-zero elements are
    ill-conditioned for a relative measure)."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    big = np.abs(ref) > 0.1 * np.abs(ref).max(axis=-1, keepdims=True)
    return float((np.abs(y - ref)[big] / np.abs(ref)[big]).max())


def check_output(y, ref, tol, label=""):
    """Assert the layer-output bound (per-token inf-norm relative error <= tol)
    and the element-wise bound it implies on large elements (<= 10 tol); print
    both with the largest absolute error.  Returns the inf-norm error."""
    inf = rel_inf_err(y, ref)
    elem = big_element_err(y, ref)
    mabs = float(np.abs(np.asarray(y, np.float64) - ref).max())
    print(f"{label}: inf-norm rel err {inf:.3e}, element rel err (|r| > 0.1 max) {elem:.3e}, "
          f"max abs err {mabs:.3e} (tol {tol:g})")
    assert inf <= tol, (label, inf)
    assert elem <= 10 * tol, (label, elem)
    return inf


def near_ties(biased, k):
    """Tokens whose top-(k+1) biased scores have an adjacent gap below GAP."""
    top = -np.sort(-biased, axis=1)[:, : k + 1]
    return np.nonzero((np.diff(-top, axis=1) < GAP).any(axis=1))[0]


def x_without_ties(c, seed, step, layer, w_router, sel_bias, max_redraws=50):
    """Activations for (c, seed, step, layer), redrawing tokens with near-tied scores.
    Returns (x, subseeds)."""
    sub = np.zeros(c.T, np.int64)
    check = np.arange(c.T)
    for _ in range(max_redraws):
        x = inputs.activations(c, seed, step, layer, sub)
        _, _, (_, _, biased) = oracle.route(x[check], w_router, sel_bias, c.k, c.routed_scale,
                                            want_scores=True)
        bad = check[near_ties(biased, c.k)]
        if len(bad) == 0:
            return x, sub
        sub[bad] += 1
        # a redraw of token 0 of the verify batch moves every draft token
        check = np.arange(c.T) if (c.cfg == 2 and 0 in bad) else bad
    raise RuntimeError("could not draw tie-free activations")


def to_device_x(x, torch):
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(x).cuda()


def upload_layer(coli, torch, c, w_router, sel_bias, experts_stacked):
    dev = {n: torch.from_numpy(np.ascontiguousarray(a)).cuda() for n, a in experts_stacked.items()}
    return coli.Layer(c.H, c.F, c.E, c.k, c.routed_scale,
                      torch.from_numpy(w_router).cuda(), torch.from_numpy(sel_bias).cuda(),
                      dev["gate_q"], dev["gate_s"], dev["up_q"], dev["up_s"], dev["down_q"], dev["down_s"])


def device_layer_generated(coli, torch, c, seed, layer):
    """Full-size layer: expert weights generated on the device."""
    return inputs.device_layer_tensors(torch, c, seed, layer)


def output_to_f64(out, torch):
    if out.dtype == torch.bfloat16:
        return out.float().cpu().numpy().astype(np.float64)
    return out.cpu().numpy().astype(np.float64)


def near_top_p_boundary(x, w_router, sel_bias, k, alpha, top_p, gap=GAP):
    """Tokens where some prefix of the selected experts' routing shares (largest
    first) sums to within `gap` of top_p: the cut there is decided by rounding,
    and the oracle (f64) and the kernels (fp32) may cut differently."""
    idx, _, (_, sig, _) = oracle.route(x, w_router, sel_bias, k, alpha, want_scores=True)
    bad = []
    for t in range(idx.shape[0]):
        s = sig[t, idx[t]]
        order = np.lexsort((idx[t], -s))  # share descending, lower expert first
        cum = np.cumsum(s[order] / s.sum())
        if np.any(np.abs(cum - top_p) < gap):
            bad.append(t)
    return np.array(bad, np.int64)
