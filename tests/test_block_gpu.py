"""GPU parity of the graph-transformer block around the layer
(eaga_block_forward / eaga_block_backward) against the block oracle
(oracle/block.py on top of the layer oracle), element by element at the bf16
parity tolerance, and of a two-block stack.

The FFN's relu takes a decision per hidden unit and row: h > 0 or not.  In
bf16 arithmetic the block's inputs X', E' are the layer's bf16 outputs and
Za is rounded to bf16 for the products, so a pre-activation within about
2^-7 of its scale of zero can take the other side than in the fp64 oracle,
and the gradients behind the gate (dW1, db1 and, through dZa, dX', dE' and
everything of the layer's backward) then differ by that row's whole term:
the oracle alone moves dW1 by 14-27% when its X', E' are rounded to bf16.
So, as for any decision floating point takes, both sides must take it alike:
  - the margin cases set each b1 column's sign and size from the oracle's own
    pre-activations so that every gate has a margin far above bf16 rounding,
    and then every output and gradient is compared at the bf16 tolerance;
  - the random-weight cases compare every output the gates cannot move
    (forward, dW2, db2, the second LayerNorm's gradients) at the tolerance,
    and dW1, db1 within the tolerance plus the sum of the terms of the gates
    whose pre-activation lies inside the rounding band (either side valid).

Cases span several 4 x 32 pair tiles with a ragged tail (n = 30, 96, 100,
192, 288, 544), masks with empty and single-node graphs, tiles without a valid
pair between live ones, and the smallest graph (n = 2)."""
import numpy as np
import pytest
import torch

from edge_aware_graph_b200 import eaga
from edge_aware_graph_b200 import inputs as I
from edge_aware_graph_b200.buffers import BlockBuffers
from oracle import block as OB

from harness import TOL, custom_case, rel_err

pytestmark = pytest.mark.gpu


def _margin_block_weights(p, d, W, Wb, X=None, E=None, y=None):
    """Wb with each sub-block's b1 replaced so that every row's pre-activation
    Za W1 + b1 keeps the sign s_f = (-1)^f with a margin of 10% of its
    largest magnitude plus 0.1, computed from the oracle's own Za."""
    dims = dict(H=p.H, dh=p.dh)
    import oracle as O
    lay = O.forward(dims, d["X"] if X is None else X, d["E"] if E is None else E,
                    d["y"] if y is None else y, d["M"], W)
    _, cache = OB.block_tail_forward(lay["Xout"], lay["Eout"], d["y"] if y is None else y, d["M"], Wb)
    out = dict(Wb)
    for s in ("x", "e", "y"):
        Za = cache[s]["Za"].reshape(-1, cache[s]["Za"].shape[-1])
        q = np.abs(Za @ np.asarray(Wb[f"{s}_W1"], np.float64)).max(axis=0)
        sign = np.where(np.arange(q.size) % 2 == 0, 1.0, -1.0)
        out[f"{s}_b1"] = I.to_storage(sign * (1.1 * q + 0.1), p.dtype)
    return out


def _run(B, n, mask, seed, dx=256, margins=True):
    p, d, W = custom_case(B, n, dx, 64, 64, 8, 32, "bf16", seed=seed, mask=mask)
    Wb = I.draw_block_weights(p)
    if margins:
        Wb = _margin_block_weights(p, d, W, Wb)
    dyo = I.draw_block_upstream(p)
    buf = BlockBuffers(B, n, dx, 64, 64, 8, 32, dtype="bf16", backward=True)
    buf.load_inputs(d, W)
    buf.load_block(Wb, dyo)
    buf.block_forward()
    buf.block_backward()
    torch.cuda.synchronize()
    assert eaga.get_device_status(buf.bws_bwd) == 0
    return p, d, W, Wb, dyo, buf


def _errs(pairs):
    errs = {k: rel_err(g, r) for k, (g, r) in pairs.items()}
    bad = {k: v for k, v in errs.items() if not v <= TOL["bf16"]}
    return errs, bad


CASES = [
    (2, 64, "random", 11),      # planar-sized graphs
    (4, 192, "prefix", 12),     # SBM-sized graphs
    (4, 96, "blocks", 13),      # tiles without a valid pair between live ones, an empty graph
    (3, 30, "random", 14),      # n < 32: one partial column tile, an empty and a single-node graph
    (1, 288, "prefix", 15),     # 9 column tiles, 72 row tiles
    (2, 100, "random", 16),     # ragged rows and columns
    (3, 2, "full", 17),         # the smallest graph
    (1, 544, "random", 18),     # the layer's columns over clusters of 4 CTAs under the block
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-n{c[1]}-{c[2]}")
def test_block_matches_oracle(case):
    """Margin weights: every output and gradient at the bf16 tolerance."""
    B, n, mask, seed = case
    p, d, W, Wb, dyo, buf = _run(B, n, mask, seed)
    dims = dict(H=p.H, dh=p.dh)
    fwd = OB.block_forward(dims, d["X"], d["E"], d["y"], d["M"], W, Wb, storage=p.dtype)
    errs, bad = _errs({"Xmid": (buf.Xmid, fwd["Xmid"]), "Emid": (buf.Emid, fwd["Emid"]),
                       "Xout": (buf.Xout, fwd["Xout"]), "Eout": (buf.Eout, fwd["Eout"]),
                       "yout": (buf.yout, fwd["yout"])})
    assert not bad, f"forward: {bad} (all: {errs})"
    # padding of the block's outputs is exactly zero
    M = torch.from_numpy(d["M"].astype(bool)).cuda()
    assert torch.all(buf.Xout[~M] == 0)
    valid = M[:, :, None] & M[:, None, :]
    assert torch.all(buf.Eout[~valid] == 0)

    g = OB.block_backward(dims, d["X"], d["E"], d["y"], d["M"], W, Wb, d["dXout"], d["dEout"], dyo,
                          storage=p.dtype)
    pairs = {"dEmid": (buf.dEmid, g["dEmid"]), "dX": (buf.dX, g["dX"]), "dE": (buf.dE, g["dE"]),
             "dy": (buf.dy, g["dy"])}
    pairs.update({"d" + k: (buf.dW[k], g["d" + k]) for k in I.WEIGHT_NAMES})
    pairs.update({"d" + k: (buf.dWb[k], g["d" + k]) for k in I.BLOCK_WEIGHT_NAMES})
    errs, bad = _errs(pairs)
    assert not bad, f"backward: {bad} (all: {errs})"


def _gate_bounds(Z, P, dZo, cache):
    """Per-entry bounds of dW1 and db1 over the gates inside the rounding band:
    the sum of |Za_pc dh_pf| (and |dh_pf|) over rows p whose pre-activation
    |h_pf| is below 2^-7 of sum_c |Za_pc W1_cf| + 1e-4."""
    Za = cache["Za"].reshape(-1, cache["Za"].shape[-1])
    hpre = cache["hpre"].reshape(-1, cache["hpre"].shape[-1])
    W1, W2, g2 = (np.asarray(P[k], np.float64) for k in ("W1", "W2", "ln2_g"))
    dZz = OB.layer_norm_input_grad(np.asarray(dZo, np.float64), cache["xh2"], cache["r2"], g2)
    dh = dZz.reshape(-1, dZz.shape[-1]) @ W2.T
    band = np.abs(Za) @ np.abs(W1) * 2.0 ** -7 + 1e-4
    amb = (np.abs(hpre) < band).astype(np.float64)
    return np.abs(Za).T @ (amb * np.abs(dh)), (amb * np.abs(dh)).sum(axis=0)


@pytest.mark.parametrize("case", CASES[:3], ids=lambda c: f"B{c[0]}-n{c[1]}-{c[2]}")
def test_block_random_weights(case):
    """Random weights (gates near zero): what the gates cannot move at the
    tolerance; dW1, db1 within the tolerance plus the in-band gates' terms."""
    B, n, mask, seed = case
    p, d, W, Wb, dyo, buf = _run(B, n, mask, seed, margins=False)
    dims = dict(H=p.H, dh=p.dh)
    fwd = OB.block_forward(dims, d["X"], d["E"], d["y"], d["M"], W, Wb, storage=p.dtype)
    g = OB.block_backward(dims, d["X"], d["E"], d["y"], d["M"], W, Wb, d["dXout"], d["dEout"], dyo,
                          storage=p.dtype)
    pairs = {k: (getattr(buf, k), fwd[k]) for k in ("Xmid", "Emid", "Xout", "Eout", "yout")}
    for s in ("x", "e", "y"):
        for k in ("W2", "b2", "ln2_g", "ln2_s"):
            pairs[f"d{s}_{k}"] = (buf.dWb[f"{s}_{k}"], g[f"d{s}_{k}"])
    errs, bad = _errs(pairs)
    assert not bad, f"{bad} (all: {errs})"
    _, cache = OB.block_tail_forward(fwd["Xmid"], fwd["Emid"], d["y"], d["M"], Wb)
    M = d["M"].astype(np.float64)
    upstream = {"x": M[:, :, None] * d["dXout"], "e": (M[:, :, None] * M[:, None, :])[..., None] * d["dEout"],
                "y": dyo}
    for s in ("x", "e", "y"):
        P = {k: Wb[f"{s}_{k}"] for k in OB.SUB_PARAMS}
        bW, bb = _gate_bounds(None, P, upstream[s], cache[s])
        for k, bound in (("W1", bW), ("b1", bb)):
            ref = np.asarray(g[f"d{s}_{k}"], np.float64)
            gpu = buf.dWb[f"{s}_{k}"].float().cpu().numpy().astype(np.float64)
            slack = np.abs(gpu - ref) - TOL["bf16"] * np.abs(ref).max() - bound
            assert slack.max() <= 0, (s, k, float(slack.max()), float(np.abs(ref).max()))


def test_block_dx512():
    """The node sub-block at dx = 512 (FFN width 1024)."""
    p, d, W, Wb, dyo, buf = _run(2, 64, "random", 21, dx=512)
    dims = dict(H=p.H, dh=p.dh)
    fwd = OB.block_forward(dims, d["X"], d["E"], d["y"], d["M"], W, Wb, storage=p.dtype)
    g = OB.block_backward(dims, d["X"], d["E"], d["y"], d["M"], W, Wb, d["dXout"], d["dEout"], dyo,
                          storage=p.dtype)
    pairs = {"Xout": (buf.Xout, fwd["Xout"]), "yout": (buf.yout, fwd["yout"]), "dX": (buf.dX, g["dX"]),
             "dx_W1": (buf.dWb["x_W1"], g["dx_W1"]), "dx_W2": (buf.dWb["x_W2"], g["dx_W2"]),
             "dx_ln1_g": (buf.dWb["x_ln1_g"], g["dx_ln1_g"])}
    errs, bad = _errs(pairs)
    assert not bad, f"{bad} (all: {errs})"


def test_two_block_stack():
    """Two blocks, each with its own weights; the second block's input
    gradients are the first block's upstream gradients."""
    B, n = 3, 64
    p, d, Wl1 = custom_case(B, n, 256, 64, 64, 8, 32, "bf16", seed=31, mask="random")
    Wl2 = I.draw_weights(p, seed_offset=1500)
    Wb1 = _margin_block_weights(p, d, Wl1, I.draw_block_weights(p))
    dims = dict(H=p.H, dh=p.dh)
    o1 = OB.block_forward(dims, d["X"], d["E"], d["y"], d["M"], Wl1, Wb1, storage=p.dtype)
    Wb2 = _margin_block_weights(p, d, Wl2, I.draw_block_weights(p, seed_offset=2500),
                                X=o1["Xout"], E=o1["Eout"], y=o1["yout"])
    dyo = I.draw_block_upstream(p)
    b1 = BlockBuffers(B, n, 256, 64, 64, 8, 32, dtype="bf16", backward=True)
    b2 = BlockBuffers(B, n, 256, 64, 64, 8, 32, dtype="bf16", backward=True)
    b1.load_inputs(d, Wl1)
    b1.load_block(Wb1)
    b2.load_inputs(d, Wl2)
    b2.load_block(Wb2, dyo)
    b1.block_forward()
    b2.X.copy_(b1.Xout)
    b2.E.copy_(b1.Eout)
    b2.y.copy_(b1.yout)
    b2.block_forward()
    b2.block_backward()
    b1.dXout.copy_(b2.dX)
    b1.dEout.copy_(b2.dE)
    b1.dyout.copy_(b2.dy)
    b1.block_backward()
    torch.cuda.synchronize()

    o2 = OB.block_forward(dims, o1["Xout"], o1["Eout"], o1["yout"], d["M"], Wl2, Wb2, storage=p.dtype)
    g2 = OB.block_backward(dims, o1["Xout"], o1["Eout"], o1["yout"], d["M"], Wl2, Wb2, d["dXout"], d["dEout"], dyo,
                           storage=p.dtype)
    g1 = OB.block_backward(dims, d["X"], d["E"], d["y"], d["M"], Wl1, Wb1, g2["dX"], g2["dE"], g2["dy"],
                           storage=p.dtype)
    pairs = {"Xout2": (b2.Xout, o2["Xout"]), "Eout2": (b2.Eout, o2["Eout"]), "yout2": (b2.yout, o2["yout"]),
             "dX": (b1.dX, g1["dX"]), "dE": (b1.dE, g1["dE"]), "dy": (b1.dy, g1["dy"]),
             "dWq1": (b1.dW["Wq"], g1["dWq"]), "de_W1_1": (b1.dWb["e_W1"], g1["de_W1"]),
             "dWo2": (b2.dW["Wo"], g2["dWo"]), "dx_W2_2": (b2.dWb["x_W2"], g2["dx_W2"])}
    errs, bad = _errs(pairs)
    assert not bad, f"{bad} (all: {errs})"


def test_block_arguments_are_checked():
    d32 = eaga.dims(2, 16, 16, 8, 8, 2, 8, "fp32")
    assert eaga.block_workspace_size(d32, False) == 0
    assert eaga.block_saved_size(d32) == 0
    d_odd = eaga.dims(2, 64, 256, 64, 48, 8, 32, "bf16")      # dy not a multiple of 32
    assert eaga.block_workspace_size(d_odd, True) == 0
    p, d, W = custom_case(2, 64, 256, 64, 64, 8, 32, "bf16", seed=3, mask="random")
    buf = BlockBuffers(2, 64, 256, 64, 64, 8, 32, dtype="bf16", backward=True)
    buf.load_inputs(d, W)
    buf.load_block(I.draw_block_weights(p))
    small = buf.bws_fwd[: buf.bws_fwd.numel() - 256]
    with pytest.raises(eaga.EagaError) as ei:
        eaga.block_forward(buf.dims, buf.X, buf.E, buf.y, buf.M, buf.W, buf.Wb, buf.Xmid, buf.Emid, buf.Xout,
                           buf.Eout, buf.yout, buf.bsaved, small)
    assert ei.value.code == 4                           # EAGA_ERR_WORKSPACE
    with pytest.raises(eaga.EagaError) as ei:             # an output overlapping an input
        eaga.block_forward(buf.dims, buf.X, buf.E, buf.y, buf.M, buf.W, buf.Wb, buf.Xmid, buf.Emid, buf.Xout,
                           buf.E, buf.yout, buf.bsaved, buf.bws_fwd)
    assert ei.value.code == 1
