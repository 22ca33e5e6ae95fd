"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Error measure: max|gpu - oracle| / max|oracle| per output tensor; bound 1e-4
in fp32 storage mode and 2e-2 in bf16 storage mode (fp32 accumulation in
both).  Cases: the tiny preset (fp32 and bf16), ragged shapes with
non-prefix masks (an empty graph, a single-node graph), the generic and the
specialised dims, and the full-size planar, tree, SBM and large presets.
"""
import numpy as np
import pytest
import torch

from edge_aware_graph_b200 import inputs as I
from edge_aware_graph_b200.buffers import LayerBuffers

from harness import TOL, custom_case, increment_err, oracle_backward, oracle_forward, rel_err

pytestmark = pytest.mark.gpu

GRAD_KEYS = ("dX", "dE", "dy") + tuple("d" + k for k in I.WEIGHT_NAMES)


def make(p, d, W, backward):
    buf = LayerBuffers(p.B, p.n, p.dx, p.de, p.dy, p.H, p.dh, dtype=p.dtype, backward=backward)
    buf.load_inputs(d, W)
    return buf


def gpu_grads(buf):
    out = {"dX": buf.dX, "dE": buf.dE, "dy": buf.dy}
    for k in I.WEIGHT_NAMES:
        out["d" + k] = buf.dW[k]
    return out


def check_forward(buf, ref, tol, rows=None):
    errs = {"Xout": rel_err(buf.Xout, ref["Xout"]), "Eout": rel_err(buf.Eout, ref["Eout"])}
    # the residual outputs' increments X' - X and E' - E on their own scale
    errs["dXinc"] = increment_err(buf.Xout, buf.X, ref["Xout"], buf.dtype)
    errs["dEinc"] = increment_err(buf.Eout, buf.E, ref["Eout"], buf.dtype)
    sv = buf.saved_parts()
    errs["O"] = rel_err(sv["O"], ref["O"])
    valid = np.isfinite(ref["LSE"])
    lse = sv["LSE"].cpu().numpy()
    errs["LSE"] = float(np.abs(lse[valid] - ref["LSE"][valid]).max() / np.abs(ref["LSE"][valid]).max()) if valid.any() else 0.0
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"forward errors above {tol}: {bad} (all: {errs})"
    return errs


def check_backward(buf, ref, tol, loose=None):
    """loose: {name: bound} for outputs whose exact value is zero in exact
    arithmetic (checked elsewhere against another scale)."""
    g = gpu_grads(buf)
    errs = {k: rel_err(g[k], ref[k]) for k in GRAD_KEYS}
    # the residual gradients' increments dX - dX' and dE - dE' on their own scale
    errs["dX-inc"] = increment_err(buf.dX, buf.dXout, ref["dX"], buf.dtype)
    errs["dE-inc"] = increment_err(buf.dE, buf.dEout, ref["dE"], buf.dtype)
    loose = loose or {}
    bad = {k: v for k, v in errs.items() if not v <= loose.get(k, tol)}
    assert not bad, f"backward errors above {tol}: {bad} (all: {errs})"
    return errs


def test_tiny_forward_backward(oracle_lib):
    """The tiny preset (fp32 storage, the CUDA-core path) at the fp32 bound,
    with the attention map the forward used."""
    p = I.preset("tiny")
    d = I.draw_inputs(p, with_grads=True)
    W = I.draw_weights(p)
    buf = make(p, d, W, backward=True)
    buf.forward()
    buf.backward()
    torch.cuda.synchronize()
    ref = oracle_forward(oracle_lib, p, d, W, want_attention=True)
    check_forward(buf, ref, TOL["fp32"])
    A = buf.attention_map()
    assert rel_err(A, ref["A"]) <= TOL["fp32"]
    check_backward(buf, oracle_backward(oracle_lib, p, d, W), TOL["fp32"])


CASES = [
    # B, n, dx, de, dy, H, dh, dtype, mask
    (3, 37, 24, 24, 16, 3, 16, "fp32", "random"),
    (4, 64, 256, 64, 64, 8, 32, "bf16", "random"),
    (3, 100, 256, 64, 64, 8, 32, "bf16", "prefix"),
    (2, 130, 256, 64, 64, 8, 32, "bf16", "random"),
    (2, 200, 64, 32, 8, 4, 16, "bf16", "prefix"),
    (5, 1, 16, 8, 8, 2, 8, "fp32", "full"),
    (2, 257, 256, 64, 64, 8, 32, "bf16", "random"),
    (2, 96, 576, 64, 64, 8, 32, "bf16", "random"),     # node GEMMs: N a multiple of 64 only
    (3, 64, 64, 64, 64, 8, 32, "bf16", "prefix"),      # narrowest node width of the fast path
    (2, 250, 256, 64, 64, 8, 32, "bf16", "random"),    # backward: S, dP reloaded instead of kept
    # edges of the tcgen05 path's domain (n even, dx a multiple of 64 up to 1024):
    # one partial 32-column chunk whose TMA boxes reach past the graph (out-of-
    # bounds fill on loads, clipped stores), an empty and a single-node graph
    (4, 2, 256, 64, 64, 8, 32, "bf16", "random"),
    (4, 16, 256, 64, 64, 8, 32, "bf16", "random"),
    (4, 30, 256, 64, 64, 8, 32, "bf16", "random"),
    (3, 64, 1024, 64, 64, 8, 32, "bf16", "random"),    # widest node features
    # block sparsity: chunks and row blocks without a valid pair between live
    # ones (copied, not computed), with S, dP kept and reloaded
    (4, 160, 256, 64, 64, 8, 32, "bf16", "blocks"),
    (4, 250, 256, 64, 64, 8, 32, "bf16", "blocks"),
    # a row block's columns over a cluster of CTAs (more than 8 chunks): 2 CTAs
    # of 5 and 4 chunks; 4 CTAs of 5, 5, 5 and 2 chunks; 4 CTAs of 8 chunks
    (2, 288, 256, 64, 64, 8, 32, "bf16", "blocks"),
    (2, 544, 256, 64, 64, 8, 32, "bf16", "random"),
    (1, 1024, 256, 64, 64, 8, 32, "bf16", "prefix"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:7])) + f"-{c[7]}-{c[8]}")
def test_ragged_shapes(oracle_lib, case):
    B, n, dx, de, dy, H, dh, dtype, mask = case
    p, d, W = custom_case(B, n, dx, de, dy, H, dh, dtype, seed=10 + n, mask=mask)
    buf = make(p, d, W, backward=True)
    buf.forward()
    buf.backward()
    torch.cuda.synchronize()
    check_forward(buf, oracle_forward(oracle_lib, p, d, W), TOL[dtype])
    check_backward(buf, oracle_backward(oracle_lib, p, d, W), TOL[dtype])


def test_light_edge_variant(oracle_lib):
    """Light Edge (no per-edge modulation) is the layer with Wfe = 0; the
    specialised path computes it like any other weights.  With (1 + gamma)
    constant over j, a key bias shifts a whole score row, so its gradient dbk
    is exactly zero: the GPU's value is checked against zero, to the parity
    tolerance taken on the scale of the query-bias gradient."""
    p, d, W = custom_case(3, 96, 256, 64, 64, 8, 32, "bf16", seed=21, mask="random")
    W = dict(W)
    W["Wfe"] = np.zeros_like(W["Wfe"])
    buf = make(p, d, W, backward=True)
    buf.forward()
    buf.backward()
    torch.cuda.synchronize()
    check_forward(buf, oracle_forward(oracle_lib, p, d, W), TOL["bf16"])
    ref = oracle_backward(oracle_lib, p, d, W)
    check_backward(buf, ref, TOL["bf16"], loose={"dbk": float("inf")})
    dbk = buf.dW["bk"].cpu().numpy().astype(np.float64)
    assert np.abs(ref["dbk"]).max() <= 1e-12 * np.abs(ref["dbq"]).max()
    assert np.abs(dbk).max() <= TOL["bf16"] * np.abs(ref["dbq"]).max()


@pytest.mark.parametrize("mask", ["random", "blocks"])
def test_masked_garbage_is_ignored(mask):
    """Large finite values in masked node rows and invalid pairs leave every
    valid output bitwise unchanged; masked outputs equal their inputs (also
    where whole chunks hold no valid pair and are copied)."""
    p, d, W = custom_case(4, 96, 256, 64, 64, 8, 32, "bf16", seed=3, mask=mask)
    buf = make(p, d, W, backward=True)
    buf.forward(); buf.backward()
    base = {k: getattr(buf, k).clone() for k in ("Xout", "Eout", "dX", "dE", "dy")}
    base_dw = {k: v.clone() for k, v in buf.dW.items()}
    rows = d["M"].astype(bool)
    valid = rows[:, :, None] & rows[:, None, :]
    rng = np.random.default_rng(1)
    d2 = dict(d)
    d2["X"] = d["X"].copy(); d2["X"][~rows] = I.to_storage(rng.standard_normal(d2["X"][~rows].shape) * 1e3, "bf16")
    d2["E"] = d["E"].copy(); d2["E"][~valid] = I.to_storage(rng.standard_normal(d2["E"][~valid].shape) * 1e3, "bf16")
    buf.load_inputs(d2, W)
    buf.forward(); buf.backward()
    torch.cuda.synchronize()
    vt = torch.from_numpy(valid).cuda()
    rt = torch.from_numpy(rows).cuda()
    assert torch.equal(buf.Xout[rt], base["Xout"][rt])
    assert torch.equal(buf.Eout[vt], base["Eout"][vt])
    assert torch.equal(buf.dE[vt], base["dE"][vt])
    assert torch.equal(buf.dy, base["dy"])
    # dk, dv are fp32 sums over row blocks that arrive in the order the CTAs run,
    # so what depends on them (dX, dWk, dbk, dWv, dbv) may differ in the last bits
    # between any two calls (fp32: 1e-3 of the scale; bf16 dX: such a difference
    # can move a rounding by one bf16 step, at most 2^-7 of the element); garbage
    # reaching them would show at its 1e3 scale
    for k in base_dw:
        if k in ("Wk", "bk", "Wv", "bv"):
            assert rel_err(buf.dW[k], base_dw[k].cpu().numpy()) <= 1e-3, k
        else:
            assert torch.equal(buf.dW[k], base_dw[k]), k
    assert rel_err(buf.dX[rt], base["dX"][rt].float().cpu().numpy()) <= 2.0 ** -7
    assert torch.equal(buf.Xout[~rt], buf.X[~rt])
    assert torch.equal(buf.Eout[~vt], buf.E[~vt])
    assert torch.equal(buf.dE[~vt], buf.dEout[~vt])


def test_permutation_equivariance_gpu():
    p, d, W = custom_case(2, 80, 256, 64, 64, 8, 32, "bf16", seed=8, mask="random", with_grads=False)
    buf = make(p, d, W, backward=False)
    buf.forward()
    X0, E0 = buf.Xout.float().cpu().numpy(), buf.Eout.float().cpu().numpy()
    perm = np.random.default_rng(2).permutation(p.n)
    d2 = dict(d)
    d2["X"], d2["E"], d2["M"] = d["X"][:, perm], d["E"][:, perm][:, :, perm], d["M"][:, perm]
    buf.load_inputs(d2, W)
    buf.forward()
    torch.cuda.synchronize()
    assert rel_err(buf.Xout, X0[:, perm]) <= TOL["bf16"]
    assert rel_err(buf.Eout, E0[:, perm][:, :, perm]) <= TOL["bf16"]


@pytest.mark.parametrize("name", ["planar", "tree"])
def test_forward_presets(oracle_lib, name):
    p = I.preset(name)
    d = I.draw_inputs(p, with_grads=False)
    W = I.draw_weights(p)
    buf = make(p, d, W, backward=False)
    buf.forward()
    torch.cuda.synchronize()
    check_forward(buf, oracle_forward(oracle_lib, p, d, W), TOL[p.dtype])


def test_sbm_training_step(oracle_lib):
    p = I.preset("sbm")
    d = I.draw_inputs(p)
    W = I.draw_weights(p)
    buf = make(p, d, W, backward=True)
    buf.forward()
    buf.backward()
    torch.cuda.synchronize()
    check_forward(buf, oracle_forward(oracle_lib, p, d, W), TOL[p.dtype])
    check_backward(buf, oracle_backward(oracle_lib, p, d, W), TOL[p.dtype])


@pytest.mark.slow
def test_large_training_step(oracle_lib):
    """Full-size large preset on the GPU; the oracle runs one graph at a time
    (graphs are independent; weight gradients are sums over graphs)."""
    p = I.preset("large")
    d = I.draw_inputs(p)
    W = I.draw_weights(p)
    buf = make(p, d, W, backward=True)
    buf.forward()
    buf.backward()
    torch.cuda.synchronize()
    tol = TOL[p.dtype]
    gw = {k: np.zeros(W[k].shape) for k in I.WEIGHT_NAMES}
    errs = {}
    sv = buf.saved_parts()
    for b in range(p.B):
        sl = {k: d[k][b:b + 1] for k in ("X", "E", "y", "M", "dXout", "dEout")}
        pb = I.preset("large", B=1)
        rf = oracle_forward(oracle_lib, pb, sl, W)
        errs[f"Xout{b}"] = rel_err(buf.Xout[b:b + 1], rf["Xout"])
        errs[f"Eout{b}"] = rel_err(buf.Eout[b:b + 1], rf["Eout"])
        errs[f"Xinc{b}"] = increment_err(buf.Xout[b:b + 1], buf.X[b:b + 1], rf["Xout"], p.dtype)
        errs[f"Einc{b}"] = increment_err(buf.Eout[b:b + 1], buf.E[b:b + 1], rf["Eout"], p.dtype)
        errs[f"O{b}"] = rel_err(sv["O"][b:b + 1], rf["O"])
        del rf
        rb = oracle_backward(oracle_lib, pb, sl, W)
        errs[f"dX{b}"] = rel_err(buf.dX[b:b + 1], rb["dX"])
        errs[f"dE{b}"] = rel_err(buf.dE[b:b + 1], rb["dE"])
        errs[f"dXinc{b}"] = increment_err(buf.dX[b:b + 1], buf.dXout[b:b + 1], rb["dX"], p.dtype)
        errs[f"dEinc{b}"] = increment_err(buf.dE[b:b + 1], buf.dEout[b:b + 1], rb["dE"], p.dtype)
        errs[f"dy{b}"] = rel_err(buf.dy[b:b + 1], rb["dy"])
        for k in I.WEIGHT_NAMES:
            gw[k] += rb["d" + k]
        del rb
    for k in I.WEIGHT_NAMES:
        errs["d" + k] = rel_err(buf.dW[k], gw[k])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"errors above {tol}: {bad}"


def test_device_status_ok():
    from edge_aware_graph_b200 import eaga
    p, d, W = custom_case(2, 16, 16, 8, 8, 2, 8, "fp32", seed=1, mask="full", with_grads=False)
    buf = make(p, d, W, backward=False)
    buf.forward()
    assert eaga.get_device_status(buf.ws_fwd) == 0


def test_bounded_wait_reports_timeout_and_context_survives(oracle_lib):
    """A device wait that can never complete gives up after its poll limit,
    the status word reports EAGA_ERR_TIMEOUT, and the next calls run normally."""
    from edge_aware_graph_b200 import eaga
    p, d, W = custom_case(2, 64, 256, 64, 64, 8, 32, "bf16", seed=5, mask="random", with_grads=False)
    buf = make(p, d, W, backward=False)
    eaga.debug_wait_probe(buf.ws_fwd, 2000)
    torch.cuda.synchronize()
    assert eaga.get_device_status(buf.ws_fwd) == 6            # EAGA_ERR_TIMEOUT
    assert eaga.get_device_status(buf.ws_fwd) == 0            # reading it cleared it
    buf.forward()
    torch.cuda.synchronize()
    assert eaga.get_device_status(buf.ws_fwd) == 0
    check_forward(buf, oracle_forward(oracle_lib, p, d, W), TOL["bf16"])


def test_calls_allocate_no_device_memory():
    """After the first calls (library load, streams), forward and backward
    leave the device's free memory and torch's allocations unchanged."""
    p = I.preset("sbm", B=4)
    d = I.draw_inputs(p, with_grads=True)
    W = I.draw_weights(p)
    buf = make(p, d, W, backward=True)
    for _ in range(2):
        buf.forward()
        buf.backward()
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(3):
        buf.forward()
        buf.backward()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
