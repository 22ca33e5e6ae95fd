"""Parity in the launch configuration the benchmark times: the training step's
kernels (one forward, one backward, with the backward's work on the library's
auxiliary streams) captured once into a CUDA graph and replayed.  Every output
(X', E', dX, dE, dy, the weight gradients) is poisoned with NaN before the
replay, so each value compared was written by the replay itself.  Full-size
SBM-shaped batch, against the fp64 oracle.
"""
import pytest
import torch

from edge_aware_graph_b200 import inputs as I
from edge_aware_graph_b200.buffers import LayerBuffers

from harness import TOL, increment_err, oracle_backward, oracle_forward, rel_err

pytestmark = pytest.mark.gpu


def test_sbm_training_step_replayed_from_a_cuda_graph(oracle_lib):
    p = I.preset("sbm")
    d = I.draw_inputs(p)
    W = I.draw_weights(p)
    buf = LayerBuffers(p.B, p.n, p.dx, p.de, p.dy, p.H, p.dh, dtype=p.dtype, backward=True)
    buf.load_inputs(d, W)

    # the capture the benchmark makes: warm the capture stream, then capture
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        buf.forward(cap)
        buf.backward(cap)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        buf.forward(cap)
        buf.backward(cap)
    torch.cuda.synchronize()

    for t in (buf.Xout, buf.Eout, buf.dX, buf.dE, buf.dy, buf.dW_flat):
        t.fill_(float("nan"))
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    del graph

    rf = oracle_forward(oracle_lib, p, d, W)
    rb = oracle_backward(oracle_lib, p, d, W)
    tol = TOL[p.dtype]
    errs = {"Xout": rel_err(buf.Xout, rf["Xout"]), "Eout": rel_err(buf.Eout, rf["Eout"]),
            "O": rel_err(buf.saved_parts()["O"], rf["O"]),
            "dX": rel_err(buf.dX, rb["dX"]), "dE": rel_err(buf.dE, rb["dE"]), "dy": rel_err(buf.dy, rb["dy"])}
    errs["Xinc"] = increment_err(buf.Xout, buf.X, rf["Xout"], p.dtype)
    errs["Einc"] = increment_err(buf.Eout, buf.E, rf["Eout"], p.dtype)
    errs["dXinc"] = increment_err(buf.dX, buf.dXout, rb["dX"], p.dtype)
    errs["dEinc"] = increment_err(buf.dE, buf.dEout, rb["dE"], p.dtype)
    for k in I.WEIGHT_NAMES:
        errs["d" + k] = rel_err(buf.dW[k], rb["d" + k])
    bad = {k: v for k, v in errs.items() if not v <= tol}       # NaN fails this test too
    assert not bad, f"errors above {tol}: {bad} (all: {errs})"
