"""Shared helpers of the GPU parity tests: seeded cases, oracle calls, errors."""
import numpy as np

from edge_aware_graph_b200 import inputs as I

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def rel_err(gpu, ref) -> float:
    """max |gpu - ref| / max |ref| over one tensor (the parity measure)."""
    g = gpu.detach().float().cpu().numpy().astype(np.float64) if hasattr(gpu, "detach") else np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    if scale == 0:
        return float(np.abs(g).max())
    return float(np.abs(g - ref).max() / scale)


def _half_ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    """Half a unit in the last place of the storage dtype at each value of x."""
    bits = 8 if dtype == "bf16" else 24              # significand bits incl. the implicit one
    ax = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - bits), 0.0)


def increment_err(gpu_out, base, ref_out, dtype: str) -> float:
    """Error of a residual output's increment, on the increment's own scale.

    A residual output (X' = X + ..., E' = E + ..., dE = dE' + ..., dX = dX' + ...)
    is compared as out - base against the oracle's out - base, relative to
    max |oracle increment|, so that a small update is not hidden under the
    scale of the input it is added to.  The GPU output is stored in `dtype`
    (round to nearest): its unrounded increment lies within half an ulp of
    the stored output, so that half ulp (the storage rounding, not arithmetic
    of the layer) is allowed on top of the parity tolerance."""
    g = gpu_out.detach().float().cpu().numpy().astype(np.float64) if hasattr(gpu_out, "detach") else np.asarray(gpu_out, np.float64)
    b = base.detach().float().cpu().numpy().astype(np.float64) if hasattr(base, "detach") else np.asarray(base, np.float64)
    inc_ref = np.asarray(ref_out, np.float64) - b
    scale = np.abs(inc_ref).max()
    dev = np.maximum(np.abs((g - b) - inc_ref) - _half_ulp(g, dtype), 0.0)
    if scale == 0:
        return float(dev.max())
    return float(dev.max() / scale)


def custom_case(B, n, dx, de, dy, H, dh, dtype, seed, mask="random", with_grads=True):
    """Dense-family case of arbitrary dims with a chosen mask pattern.

    mask: "prefix" (random real counts), "random" (non-prefix, includes one
    fully masked graph and one single-node graph when B >= 3), "blocks" (node
    spans that leave whole 32-column chunks and 8-row blocks without a valid
    pair between live ones, an empty graph, a single-node graph), "full".
    """
    p = I.Preset("custom", seed, dtype, B=B, n=n, dx=dx, de=de, dy=dy, H=H, dh=dh, family="dense",
                 training=with_grads, n_real=(n,))
    d = I.draw_inputs(p, with_grads=with_grads)
    rng = np.random.default_rng(seed + 99)
    if mask == "random":
        M = (rng.random((B, n)) < 0.7).astype(np.uint8)
        M[:, 0] = 1
        if B >= 3:
            M[1] = 0
            M[2] = 0
            M[2, n // 2] = 1
    elif mask == "blocks":
        M = np.zeros((B, n), np.uint8)
        for b in range(B):
            spans = ([(0, 20), (70, 90), (n - 10, n)], [(40, 50)], [], [(n // 2, n // 2 + 1)])[b % 4]
            for lo, hi in spans:
                M[b, lo:min(hi, n)] = 1
    elif mask == "prefix":
        nr = rng.integers(1, n + 1, size=B)
        M = (np.arange(n)[None] < nr[:, None]).astype(np.uint8)
    else:
        M = np.ones((B, n), np.uint8)
    d["M"] = M
    return p, d, I.draw_weights(p)


def oracle_forward(oracle, p, d, W, want_attention=False):
    return oracle.forward(dict(H=p.H, dh=p.dh), d["X"], d["E"], d["y"], d["M"], W, want_attention=want_attention)


def oracle_backward(oracle, p, d, W):
    return oracle.backward(dict(H=p.H, dh=p.dh), d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"])
