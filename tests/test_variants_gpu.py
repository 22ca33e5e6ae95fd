"""GPU parity of the layer's ablation variants (AI-summary page: the method
paragraph's ablation of unnormalised coefficients, and the "Light Edge"
bullet) against the fp64 oracle's variants, on the tcgen05 path and on the
CUDA-core path, with the error measures and bounds of the layer's parity
tests (including the residual increments on their own scale).

Light Edge: no per-edge FiLM map (Wfe is not read; its gradient is zero; on
the tcgen05 path the forward reads E once and the backward not at all).
Unnormalised: the edge update from the modulated scores s' on valid pairs.
"""
import numpy as np
import pytest
import torch

from edge_aware_graph_b200 import eaga
from edge_aware_graph_b200 import inputs as I
from edge_aware_graph_b200.buffers import LayerBuffers

from harness import TOL, custom_case, increment_err, rel_err

pytestmark = pytest.mark.gpu

GRAD_KEYS = ("dX", "dE", "dy") + tuple("d" + k for k in I.WEIGHT_NAMES)

CASES = [
    # B, n, dx, de, dy, H, dh, dtype, mask
    (3, 96, 256, 64, 64, 8, 32, "bf16", "random"),      # tcgen05 path
    (4, 30, 256, 64, 64, 8, 32, "bf16", "random"),      # tcgen05 path, one partial chunk
    (2, 250, 256, 64, 64, 8, 32, "bf16", "prefix"),     # tcgen05 path, S and dP reloaded
    (4, 160, 256, 64, 64, 8, 32, "bf16", "blocks"),     # tcgen05 path, chunks without a valid pair
    (2, 288, 256, 64, 64, 8, 32, "bf16", "blocks"),     # tcgen05 path, a row block over 2 CTAs
    (3, 37, 24, 24, 16, 3, 16, "fp32", "random"),       # CUDA-core path, fp32
    (2, 70, 64, 32, 8, 4, 16, "bf16", "prefix"),        # CUDA-core path, bf16
]


@pytest.mark.parametrize("variant", ["light_edge", "unnormalised"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:7])) + f"-{c[7]}")
def test_variant_parity(oracle_lib, variant, case):
    B, n, dx, de, dy, H, dh, dtype, mask = case
    p, d, W = custom_case(B, n, dx, de, dy, H, dh, dtype, seed=50 + n, mask=mask)
    buf = LayerBuffers(B, n, dx, de, dy, H, dh, dtype=dtype, backward=True)
    buf.load_inputs(d, W)
    buf.dW_flat.fill_(float("nan"))
    buf.forward(variant=variant)
    buf.backward(variant=variant)
    torch.cuda.synchronize()
    dims = dict(H=H, dh=dh)
    rf = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, variant=variant)
    rb = oracle_lib.backward(dims, d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"], variant=variant)
    tol = TOL[dtype]
    errs = {"Xout": rel_err(buf.Xout, rf["Xout"]), "Eout": rel_err(buf.Eout, rf["Eout"]),
            "O": rel_err(buf.saved_parts()["O"], rf["O"]),
            "Xinc": increment_err(buf.Xout, buf.X, rf["Xout"], dtype),
            "Einc": increment_err(buf.Eout, buf.E, rf["Eout"], dtype),
            "dXinc": increment_err(buf.dX, buf.dXout, rb["dX"], dtype),
            "dEinc": increment_err(buf.dE, buf.dEout, rb["dE"], dtype)}
    grads = {"dX": buf.dX, "dE": buf.dE, "dy": buf.dy}
    grads.update({"d" + k: buf.dW[k] for k in I.WEIGHT_NAMES})
    for k in GRAD_KEYS:
        errs[k] = rel_err(grads[k], rb[k])
    if variant == "light_edge":
        # with (1 + gamma) constant over j a key bias shifts a whole score row, so
        # dbk is exactly zero in exact arithmetic: checked against zero on the
        # scale of the query-bias gradient
        errs["dbk"] = float(np.abs(grads["dbk"].cpu().numpy()).max() / np.abs(rb["dbq"]).max())
    bad = {k: v for k, v in errs.items() if not v <= tol}      # NaN fails too
    assert not bad, f"{variant}: errors above {tol}: {bad} (all: {errs})"
    if variant == "light_edge":
        assert torch.all(buf.dW["Wfe"] == 0)                    # not a parameter of that layer
        assert torch.equal(buf.dE, buf.dEout)                   # no per-edge FiLM term


def test_light_edge_ignores_wfe():
    """The Light Edge variant does not read Wfe: two different Wfe give
    bitwise identical outputs and gradients."""
    p, d, W = custom_case(2, 64, 256, 64, 64, 8, 32, "bf16", seed=3, mask="random")
    outs = []
    for scale in (1.0, -7.0):
        W2 = dict(W)
        W2["Wfe"] = (W["Wfe"] * scale).astype(np.float32)
        buf = LayerBuffers(2, 64, 256, 64, 64, 8, 32, dtype="bf16", backward=True)
        buf.load_inputs(d, W2)
        buf.forward(variant="light_edge")
        buf.backward(variant="light_edge")
        torch.cuda.synchronize()
        outs.append([t.clone() for t in (buf.Xout, buf.Eout, buf.dE, buf.dy, buf.dX, buf.dW_flat)])
    # Xout, Eout, dE and dy do not depend on the dk, dv sums over row blocks
    # (fp32 additions in L2 in no fixed order): bitwise
    for a, b in zip(outs[0][:4], outs[1][:4]):
        assert torch.equal(a, b)
    # dX (bf16: one rounding step, at most 2^-7 of an element) and the flat fp32
    # weight gradients (dWk, dbk, dWv, dbv among them: 1e-3) do, far below what a
    # seven-fold Wfe would change
    for (a, b), bound in zip(zip(outs[0][4:], outs[1][4:]), (2.0 ** -7, 1e-3)):
        a, b = a.float(), b.float()
        assert float((a - b).abs().max()) <= bound * float(a.abs().max())
